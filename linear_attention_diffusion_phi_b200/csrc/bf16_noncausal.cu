// bf16_noncausal.cu -- tcgen05 tensor-core path for non-causal phi attention
// with bf16 storage and fp32 accumulation, F = 0 (phi acts on the D channels).
//
// Method (page "NNT Define Linear Attention", "How it works"): collapse the
// sequence into kv = phi(K)^T V and ksum = sum_j phi(k_j), then
// out_i = phi(q_i)^T kv / (phi(q_i) . ksum + eps).
//
// One kernel per forward.  Each head is served by a thread-block cluster of S
// CTAs (one per SM); CTA r owns the r-th run of 128-token tiles of the head.
// S is the largest cluster size (<= 8) whose clusters for all heads can be
// resident at once on this device.  Two kernels share that plan:
//
// fused_t_kernel (D = 128)
//   phase 1  TMA streams the CTA's K and V tiles into a ring of shared-memory
//            slots.  Eight warps read each K tile transposed (ldmatrix.trans),
//            apply phi and write phi(K)^T into tensor memory (lane = feature);
//            the K slot is free again at once.  One thread issues tcgen05.mma
//            kv = phi(K)^T V  (B = the V tile as TMA left it) and
//            ksum = phi(K)^T 1  into tensor memory (fp32).
//   combine  eight warps write the CTA's partial [kv | ksum], rounded to bf16,
//            into its own copy of the apply MMA's B operand (stmatrix.trans:
//            row = value, features contiguous).  The image rows are split
//            among the cluster's CTAs; bulk copies send every owner its rows
//            from every CTA, the owner sums them in ascending CTA order (no
//            atomics: bitwise reproducible) and bulk-copies the sums into the
//            image of every CTA.  No global round trip.
//   phase 2  the CTA's Q tiles (prefetched during the combine) get phi into
//            tensor memory (lane = token), one MMA per tile computes
//            [num | den] = phi(Q) [kv | ksum], and eight warps write
//            out = num / (den + eps) as bf16 into a staging buffer that TMA
//            stores to global memory.
//
// fused_kernel (D = 64): the same plan with phi(K) and phi(Q) applied in place
// in shared memory, kv^T = V^T phi(K) and ksum^T = 1^T phi(K), and a combine
// by 16-byte asynchronous remote stores.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>
#include <type_traits>

#include "bf16_common.cuh"
#include "la_internal.h"
#include "sm100.cuh"

namespace la {
namespace {

template <int D>
struct Cfg {
  static constexpr int kBoxes = D / 64;
  static constexpr uint32_t kSlotBytes = 128u * D * 2u;          // one 128-token tile
  static constexpr int kNB = D + 16;                               // apply MMA N: values + den
  // [kv | ksum | 0]^T as the apply MMA's B operand, K-major with the 128-byte
  // swizzle: row n < D holds kv[.][n], row D holds ksum, rows above are zero;
  // each row's D features are split in 64-feature k-atoms of kNB rows.
  static constexpr uint32_t kBlobAtomBytes = kNB * 128;
  static constexpr uint32_t kBlobBytes = (D / 64) * kBlobAtomBytes;
  // 16-byte chunks of image rows 0..D, the unit of the cluster combine.
  static constexpr int kChunks = (D + 1) * (D / 8);
  // Receive buffer of the combine: S slices of at most ceil(kChunks / S)
  // chunks, one per sending CTA; S * ceil(kChunks / S) <= kChunks + 7.
  static constexpr uint32_t kRecvBytes = kBlobBytes;
  static_assert((kChunks + 7) * 16 <= kRecvBytes, "receive buffer too small");
  static constexpr uint32_t kOnesBytes = 2048;                     // A of the ksum MMA (64 x 16)
  static constexpr int kSlots = D == 128 ? 4 : 8;                 // ring of tile slots
  // During phase 1 the image and receive regions are idle; where a tile fits
  // in them they serve as two more K/V slots.
  static constexpr int kExtra = (kBlobBytes >= kSlotBytes) ? 2 : 0;
  static constexpr int kRing1 = kSlots + kExtra;                   // phase-1 ring (K, V tiles)
  // Phase 2 adds the receive region once this CTA has summed its chunks.
  static constexpr int kRing2 = kSlots + kExtra / 2;
  static constexpr uint32_t kSmemBytes = kBlobBytes + kRecvBytes + kOnesBytes + kSlots * kSlotBytes + 1024;
  static constexpr uint32_t kAccStride = D == 128 ? 256 : 128;    // TMEM columns per accumulator
  static constexpr uint32_t kTmemCols = 2 * kAccStride;
  static constexpr int kPhiWarps = 8;
  static constexpr int kPhiThreads = 32 * kPhiWarps;
  static constexpr int kChunksPerRow = D / 8;                      // 16-byte chunks per token row
  static constexpr int kThreadsPerChunk = kPhiThreads / kChunksPerRow;
  static constexpr int kRowsPerThread = 128 / kThreadsPerChunk;
  static constexpr int kCombWarp0 = 2 + kPhiWarps;                 // 8 warps: combine, then outputs
  static constexpr int kThreads = 32 * (kCombWarp0 + 8);
};

__device__ __forceinline__ uint4 pack8(const float* v) {
  uint32_t w[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    __nv_bfloat162 b = __floats2bfloat162_rn(v[2 * e], v[2 * e + 1]);
    w[e] = *reinterpret_cast<uint32_t*>(&b);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

template <int D, int FMAP>
__global__ void __launch_bounds__(Cfg<D>::kThreads, 1)
    fused_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_out,
                 int* status, int N, int tiles, float eps) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  // full / ready: arrival of a K or Q tile / phi done on it (the phi warps
  // wait on every phase of full[] in order); vfull: arrival of a V tile
  // (waited on by the MMA issuer only); empty: every use of a slot.
  __shared__ __align__(8) uint64_t full[C::kRing1], ready[C::kRing1], vfull[C::kRing1], empty[C::kRing1];
  // Tensor-memory accumulators a = 0, 1: phase 1 uses accumulator 0 once
  // (p1full / p1empty, consumed by the combine warps); phase-2 tile u uses
  // accumulator u & 1 (accfull / accempty, consumed by the output warps).
  // Separate barriers keep each barrier's phases consumed in order by one
  // consumer, so parity waits cannot alias.
  __shared__ __align__(8) uint64_t p1full, p1empty, accfull[2], accempty[2];
  // Combine: peers_free gets one (relaxed) arrival from every CTA of the
  // cluster once its image and receive regions are out of phase-1 use;
  // recv_full completes when every CTA's share of this CTA's chunks has
  // arrived, blob_full when the whole image has (transaction counts of the
  // asynchronous stores); recv_drained once this CTA has summed its chunks.
  __shared__ __align__(8) uint64_t peers_free, recv_full, blob_full, recv_drained;
  __shared__ uint32_t tmem_slot;
  __shared__ int comb_flag, ep_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = static_cast<int>(gridDim.x);   // CTAs per head == cluster size
  const int rank = static_cast<int>(cluster_ctarank());
  const int bh = blockIdx.y;
  const int tile0 = rank * tiles / S;
  const int T = (rank + 1) * tiles / S - tile0;   // >= 1 because S <= tiles
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* blob = smem;
  uint8_t* recv = blob + C::kBlobBytes;
  uint8_t* ones = recv + C::kRecvBytes;
  uint8_t* slots = ones + C::kOnesBytes;
  // Physical slots 0..kSlots-1 are the ring, kSlots and kSlots+1 the image
  // and receive regions.  Phase-1 use i (K, V of tile i / 2) takes slot
  // i % kRing1; phase-2 use u (Q tile u) takes ring2(u % kRing2), the ring
  // plus the receive region.  Every use of a slot completes one phase of its
  // full / ready / empty barriers, so a use's phase parity is the number of
  // earlier uses of that slot.
  auto slot_ptr = [&](int phys) {
    return phys < C::kSlots ? slots + phys * C::kSlotBytes : (phys == C::kSlots ? blob : recv);
  };
  auto uses1 = [&](int phys) { return (2 * T + C::kRing1 - 1 - phys) / C::kRing1; };   // phase-1 uses
  auto ring2 = [&](int j) { return j < C::kSlots ? j : C::kSlots + 1; };
  auto q_slot = [&](int u) { return ring2(u % C::kRing2); };
  auto q_round = [&](int u) { return uses1(ring2(u % C::kRing2)) + u / C::kRing2; };
  // Phases of full[] / ready[] before Q tile u: the phase-1 K uses of its
  // slot (K tiles land in even slots, V tiles in odd ones) and the earlier Q
  // uses.
  auto q_kround = [&](int u) {
    const int s = ring2(u % C::kRing2);
    return ((s & 1) == 0 ? uses1(s) : 0) + u / C::kRing2;
  };

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kRing1; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&vfull[i], 1);
      mbar_init(&ready[i], C::kPhiWarps);
      mbar_init(&empty[i], 1);
    }
    mbar_init(&p1full, 1);
    mbar_init(&p1empty, 8);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&accfull[i], 1);
      mbar_init(&accempty[i], 8);
    }
    mbar_init(&peers_free, S);
    mbar_init(&recv_full, 1);
    mbar_init(&blob_full, 1);
    mbar_init(&recv_drained, 1);
    fence_mbarrier_init();
    // every CTA sends this CTA its share of the chunks [i0, i1) it owns; the
    // owners together send the whole image
    const int i0 = rank * C::kChunks / S, i1 = (rank + 1) * C::kChunks / S;
    mbar_arrive_expect_tx(&recv_full, static_cast<uint32_t>(S * (i1 - i0) * 16));
    mbar_arrive_expect_tx(&blob_full, static_cast<uint32_t>(C::kChunks * 16));
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    prefetch_tmap(&tm_out);
    comb_flag = 0;
    ep_flag = 0;
  }
  // A operand of the ksum MMA: 64 (m) x 16 (k) bf16, K-major without swizzle
  // (core matrices of 8 rows x 16 bytes; m-groups 128 B apart, k-groups
  // 1024 B apart); row m = 0 is all ones, the rest zero, so row 0 of the
  // product is 1^T phi(K) = ksum^T.
  for (int i = threadIdx.x; i < 128; i += blockDim.x) {
    const int off = 16 * i;
    const bool one = ((off % 1024) / 128 == 0) && ((off % 128) / 16 == 0);
    const uint32_t w = one ? 0x3F803F80u : 0u;
    *reinterpret_cast<uint4*>(ones + off) = make_uint4(w, w, w, w);
  }
  // Rows D+1..kNB-1 of the operand image (the MMA's N padding) only feed
  // accumulator columns D+1.. that nobody reads; they start at zero, and
  // where the image region serves as a phase-1 slot they keep whatever the
  // last tile left there.
  for (int i = threadIdx.x; i < (D / 64) * (C::kNB - D - 1) * 8; i += blockDim.x) {
    const int a = i / ((C::kNB - D - 1) * 8), rem = i % ((C::kNB - D - 1) * 8);
    const int n = D + 1 + rem / 8, c = rem % 8;
    *reinterpret_cast<uint4*>(blob + a * C::kBlobAtomBytes + n * 128 + c * 16) = make_uint4(0u, 0u, 0u, 0u);
  }
  fence_proxy_async_smem();
  if (warp == 1) {
    tmem_alloc(&tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;

  // ------------------------------------------------------------ producer
  // Slot sequence: K, V of each phase-1 tile, then the Q tiles.  The first
  // round of slots is issued before the cluster handshake.
  int seq = 0;
  bool recv_free = false;
  auto issue = [&](int upto) {
    while (seq < upto) {
      const bool p1 = seq < 2 * T;
      const int s = p1 ? seq % C::kRing1 : q_slot(seq - 2 * T);
      const int round = p1 ? seq / C::kRing1 : q_round(seq - 2 * T);
      if (round > 0 && !mbar_wait(&empty[s], (round - 1) & 1, status)) return;
      if (!p1 && s == C::kSlots + 1 && !recv_free) {
        // the receive region holds the cluster's partials until this CTA has summed them
        if (!mbar_wait(&recv_drained, 0, status)) return;
        recv_free = true;
      }
      const bool is_v = p1 && (seq & 1);
      const CUtensorMap* m = p1 ? (is_v ? &tm_v : &tm_k) : &tm_q;
      const int tile = p1 ? seq / 2 : seq - 2 * T;
      uint64_t* bar = is_v ? &vfull[s] : &full[s];
      uint8_t* dst = slot_ptr(s);
      mbar_arrive_expect_tx(bar, C::kSlotBytes);
#pragma unroll
      for (int b = 0; b < C::kBoxes; ++b)
        tma_load_3d(dst + b * kBoxBytes, m, bar, 64 * b, (tile0 + tile) * kTileTokens, bh);
      ++seq;
    }
  };
  // Programmatic dependent launch: this grid may have started while the
  // previous launch on the stream still ran.  Nothing above touched global
  // memory; wait for that launch to complete before the first load, and let
  // the next launch begin its own set-up as this grid's CTAs leave.
  pdl_wait();
  pdl_launch_dependents();
  // Every CTA's barriers exist (fence.mbarrier_init above) before any remote
  // arrival: relaxed arrive, first loads, then the acquiring wait.
  cluster_arrive_relaxed();
  if (warp == 0 && lane == 0) issue(min(C::kRing1, 2 * T));
  cluster_wait();

  if (warp == 0) {
    if (lane == 0) issue(3 * T);
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_kv = idesc_bf16_f32(D, D, 1, 1);     // kv^T: M = D values, N = D features
      constexpr uint32_t idesc_ks = idesc_bf16_f32(64, D, 0, 1);    // ksum^T: M = 64 (row 0 used)
      constexpr uint32_t idesc_ap = idesc_bf16_f32(128, C::kNB, 0, 0);
      const uint64_t ones_desc = smem_desc_noswz(smem_u32(ones), 1024, 128);
      bool ok = true;
      for (int t = 0; t < T; ++t) {
        const int qk = 2 * t, qv = 2 * t + 1;
        const int sk = qk % C::kRing1, sv = qv % C::kRing1;
        // phi(K) done; V as it arrived
        if (!mbar_wait(&ready[sk], (qk / C::kRing1) & 1, status) ||
            !mbar_wait(&vfull[sv], (qv / C::kRing1) & 1, status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t ka = smem_u32(slot_ptr(sk));
        const uint32_t va = smem_u32(slot_ptr(sv));
        // kv^T: A = V^T (MN-major: values contiguous), B = phi(K) (MN-major:
        // features contiguous); ksum^T: A = ones block, same B.  16 tokens
        // per MMA, 2048 bytes apart.
        const uint64_t vdesc = smem_desc_sw128(va, kBoxBytes, 1024);
        const uint64_t kdesc = smem_desc_sw128(ka, kBoxBytes, 1024);
        if (t == 0) {
          umma_ss<0>(tmem, vdesc, kdesc, idesc_kv);
          umma_ss<0>(tmem + D, ones_desc, kdesc, idesc_ks);
        } else {
          umma_ss<1>(tmem, vdesc, kdesc, idesc_kv);
          umma_ss<1>(tmem + D, ones_desc, kdesc, idesc_ks);
        }
#pragma unroll
        for (int k = 1; k < kTileTokens / 16; ++k) {
          umma_ss<1>(tmem, desc_add(vdesc, 2048 * k), desc_add(kdesc, 2048 * k), idesc_kv);
          umma_ss<1>(tmem + D, ones_desc, desc_add(kdesc, 2048 * k), idesc_ks);
        }
        umma_commit(&empty[sk]);
        umma_commit(&empty[sv]);
      }
      umma_commit(&p1full);
      if (ok && mbar_wait_cluster(&blob_full, 0, status)) {
        fence_proxy_async_smem();   // the cluster's stores into `blob` feed the tensor core
        const uint32_t ba = smem_u32(blob);
        for (int u = 0; u < T; ++u) {
          const int s = q_slot(u);
          const int a = u & 1, ar = u >> 1;
          bool got = mbar_wait(&ready[s], q_kround(u) & 1, status);
          if (got && ar == 0 && a == 0) got = mbar_wait(&p1empty, 0, status);   // freed by the combine warps
          if (got && ar > 0) got = mbar_wait(&accempty[a], (ar - 1) & 1, status);
          if (!got) break;
          tc_fence_after();
          const uint32_t qa = smem_u32(slot_ptr(s));
          // A = phi(Q) and B = [kv | ksum]^T, both K-major (features contiguous)
          const uint64_t adesc = smem_desc_sw128(qa, 16, 1024);
          const uint64_t bdesc = smem_desc_sw128(ba, 16, 1024);
          const uint32_t d = tmem + a * C::kAccStride;
          umma_ss<0>(d, adesc, bdesc, idesc_ap);
#pragma unroll
          for (int k = 1; k < D / 16; ++k)
            umma_ss<1>(d, desc_add(adesc, (k >> 2) * kBoxBytes + (k & 3) * 32),
                       desc_add(bdesc, (k >> 2) * C::kBlobAtomBytes + (k & 3) * 32), idesc_ap);
          umma_commit(&accfull[a]);
        }
      }
    }
  } else if (warp < C::kCombWarp0) {
    // ----------------- phi on the K tiles, then on the Q tiles, in place
    // Every K or Q use of a slot completes one phase of full[] and one of
    // ready[]; V tiles are not touched here.
    const int pt = threadIdx.x - 64;
    const int cc = pt / C::kThreadsPerChunk;
    const int r0 = pt % C::kThreadsPerChunk;
    for (int v = 0; v < 2 * T; ++v) {
      const bool is_k = v < T;
      const int u = v - T;
      const int s = is_k ? (2 * v) % C::kRing1 : q_slot(u);
      const int round = is_k ? (2 * v) / C::kRing1 : q_kround(u);
      if (!warp_wait(&full[s], round & 1, status)) break;
      // key rows past the sequence end must not reach kv or ksum
      const int valid = is_k ? min(kTileTokens, N - (tile0 + v) * kTileTokens) : kTileTokens;
      phi_rows<FMAP, C::kRowsPerThread, C::kThreadsPerChunk>(slot_ptr(s), cc, r0, valid);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ready[s]);
    }
  } else {
    // --------------------------------------- combine, then the outputs
    // Eight warps, two per tensor-memory lane quarter, each taking one half
    // of the columns: (1) copy the partial (kv | ksum)^T into the CTA's own
    // shared memory; (2) sum their share of the cluster's partials; (3) write
    // the phase-2 outputs.
    const int ct = threadIdx.x - 32 * C::kCombWarp0;   // 0..255
    const int half = ct >> 7;
    const bool leader = ct == 0;
    const int q = warp & 3;                             // TMEM lane quarter
    const uint32_t tq = static_cast<uint32_t>(32 * q) << 16;
    bool got = true;
    auto sync_ok = [&](bool mine) {   // every warp takes the leader's verdict
      if (leader && !mine) comb_flag = 1;
      named_bar_sync(3, 256);
      return comb_flag == 0;
    };
    if (leader) got = mbar_wait(&p1full, 0, status);
    bool ok = sync_ok(got);
    if (ok) {
      // (1) this CTA's image and receive regions are out of phase-1 use (the
      // MMAs that read them are complete): tell every CTA, then wait until
      // every CTA has said the same.  A signal only, so a relaxed arrive.
      if (ct < S) mbar_arrive_remote_relaxed(mapa_shared(smem_u32(&peers_free), ct));
      if (leader) got = mbar_wait_cluster(&peers_free, 0, status);
      ok = sync_ok(got);
    }
    // Chunk i (row i / (D/8), feature chunk i % (D/8)) of image rows 0..D is
    // owned by CTA o with i0(o) <= i < i0(o + 1), i0(o) = o * kChunks / S;
    // slice `r` of o's receive buffer holds CTA r's partial of those chunks.
    const int slice = (C::kChunks + S - 1) / S;
    if (ok) {
      // (2) the partial (kv | ksum)^T, rounded to bf16, chunk by chunk to
      // the owners
      tc_fence_after();
      const uint32_t recv_base = smem_u32(recv), recv_bar = smem_u32(&recv_full);
      auto push_row = [&](int n, const float* v, int c0) {   // 32 values of row n from column c0
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int i = n * (D / 8) + c0 / 8 + j;
          const int o = ((i + 1) * S - 1) / C::kChunks;
          const int js = i - o * C::kChunks / S;
          st_async_v4(mapa_shared(recv_base + (rank * slice + js) * 16, o), pack8(v + 8 * j),
                      mapa_shared(recv_bar, o));
        }
      };
      constexpr int kHalfCols = D / 2;
      // kv^T: M = 128 -> row = lane; M = 64 -> rows 16q..16q+15 in lanes 32q..32q+15
      const bool valid = (D == 128) || lane < 16;
      const int n = (D == 128) ? 32 * q + lane : 16 * q + lane;
      {
        float v[kHalfCols];
#pragma unroll
        for (int c0 = 0; c0 < kHalfCols; c0 += 32) tmem_ld32(tmem + tq + half * kHalfCols + c0, *reinterpret_cast<float(*)[32]>(v + c0));
        tmem_wait_ld();
        if (valid)
#pragma unroll
          for (int c0 = 0; c0 < kHalfCols; c0 += 32) push_row(n, v + c0, half * kHalfCols + c0);
      }
      // ksum^T is row 0 of the M = 64 product: lane 0 of quarter 0
      if (q == 0) {
        float v[kHalfCols];
#pragma unroll
        for (int c0 = 0; c0 < kHalfCols; c0 += 32) tmem_ld32(tmem + D + half * kHalfCols + c0, *reinterpret_cast<float(*)[32]>(v + c0));
        tmem_wait_ld();
        if (lane == 0)
#pragma unroll
          for (int c0 = 0; c0 < kHalfCols; c0 += 32) push_row(D, v + c0, half * kHalfCols + c0);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p1empty);
      if (leader) got = mbar_wait_cluster(&recv_full, 0, status);
      ok = sync_ok(got);
    }
    if (ok) {
      // (3) this CTA's chunks: the sum over the S partials in ascending CTA
      // order, rounded to bf16, sent into the image of every CTA
      const int i0 = rank * C::kChunks / S, i1 = (rank + 1) * C::kChunks / S;
      const uint32_t blob_base = smem_u32(blob), blob_bar = smem_u32(&blob_full);
      for (int js = ct; js < i1 - i0; js += 256) {
        float acc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = 0.f;
        for (int p = 0; p < S; ++p) {
          const uint4 w = *reinterpret_cast<const uint4*>(recv + (p * slice + js) * 16);
          const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wv[e]));
            acc[2 * e] += x.x;
            acc[2 * e + 1] += x.y;
          }
        }
        const uint4 val = pack8(acc);
        const int i = i0 + js, nn = i / (D / 8), c = i % (D / 8);
        const uint32_t off = (c >> 3) * C::kBlobAtomBytes + nn * 128 + (((c & 7) ^ (nn & 7)) << 4);
        for (int p = 0; p < S; ++p) st_async_v4(mapa_shared(blob_base + off, p), val, mapa_shared(blob_bar, p));
      }
      named_bar_sync(3, 256);
      if (leader) mbar_arrive(&recv_drained);   // the receive region may take a Q tile
    }
    if (ok) {
      // (3) outputs of the CTA's Q tiles: each warp its rows' half of the
      // value columns
      constexpr int kHalfCols = D / 2;
      int prev_slot = -1;
      for (int u = 0; u < T; ++u) {
        const int s = q_slot(u);
        const int a = u & 1, ar = u >> 1;
        got = true;
        if (leader) got = mbar_wait(&accfull[a], ar & 1, status);
        if (leader && !got) ep_flag = 1;
        named_bar_sync(2, 256);
        if (ep_flag) break;
        tc_fence_after();
        const uint32_t trow = tmem + a * C::kAccStride + tq;
        const int r = 32 * q + lane;   // token row within the tile
        float v[kHalfCols];
        const float den = tmem_ld1(trow + D);
#pragma unroll
        for (int c0 = 0; c0 < kHalfCols; c0 += 32) tmem_ld32(trow + half * kHalfCols + c0, *reinterpret_cast<float(*)[32]>(v + c0));
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&accempty[a]);   // the accumulator is free for tile u + 2
        const float inv = 1.0f / (den + eps);
#pragma unroll
        for (int e = 0; e < kHalfCols; ++e) v[e] *= inv;
        uint8_t* ob = slot_ptr(s);   // the MMA is done with this Q tile
#pragma unroll
        for (int jj = 0; jj < kHalfCols / 8; ++jj)
          *reinterpret_cast<uint4*>(ob + swz_off(r, half * (kHalfCols / 8) + jj)) = pack8(v + 8 * jj);
        fence_proxy_async_smem();
        named_bar_sync(2, 256);
        if (leader) {
#pragma unroll
          for (int b = 0; b < C::kBoxes; ++b)
            tma_store_3d(&tm_out, ob + b * kBoxBytes, 64 * b, (tile0 + u) * kTileTokens, bh);
          bulk_commit_group();
          if (prev_slot >= 0) {   // the previous tile's store has read its slot: hand it back
            bulk_wait_group_read<1>();
            mbar_arrive(&empty[prev_slot]);
          }
        }
        prev_slot = s;
      }
      if (leader) bulk_wait_group<0>();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, C::kTmemCols);
  cluster_sync_all();   // no CTA leaves while the cluster may still address its shared memory
}

// ---------------------------------------------------------------------------
// D = 128: phi(K)^T and phi(Q) in tensor memory.
//
// The phi warps read each K tile with ldmatrix.trans (16 tokens x 16 features
// per instruction, two tokens of one feature per register), apply phi and
// store the result with tcgen05.st into tensor memory, lane = feature and
// column = token pair: the A operand of  kv = phi(K)^T V  (M = 128 features,
// N = 128 values, B = the V tile as TMA left it) and of  ksum = phi(K)^T 1
// (N = 16, B = a block of ones).  The K slot is free as soon as it has been
// read, and the tensor core reads only V from shared memory.  Q tiles go the
// same way untransposed (lane = token), as the A operand of the apply MMA.
// The partial state [kv | ksum] (lane = feature, column = value) is written
// into the CTA's image with stmatrix.trans (row = value, features
// contiguous), and the cluster exchanges image rows with bulk copies:
// every CTA sends the rows that CTA o owns to o, o sums them in ascending
// CTA order and sends the sum back into every CTA's image.

struct CfgT {
  static constexpr int D = 128;
  static constexpr int kBoxes = 2;
  static constexpr uint32_t kSlotBytes = 128u * D * 2u;
  static constexpr int kNB = D + 16;                       // apply MMA N: values + den
  static constexpr uint32_t kBlobAtomBytes = kNB * 128;    // image: 2 k-atoms of kNB rows x 128 B
  static constexpr uint32_t kBlobBytes = 2 * kBlobAtomBytes;
  static constexpr int kRows = D + 1;                      // exchanged image rows: kv rows, ksum row
  static constexpr uint32_t kRecvBytes = kBlobBytes;       // >= 8 senders x 2 atoms x 17 rows x 128 B
  static_assert(8u * 2u * ((kRows + 7) / 8) * 128u <= kRecvBytes, "receive buffer too small");
  static constexpr uint32_t kOnesBytes = 2048;
  static constexpr int kSlots = 4;
  static constexpr int kRing1 = kSlots + 2;                // phase 1 also uses the image and receive regions
  static constexpr int kRing2 = kSlots - 1;                // phase-2 Q ring; slot kSlots-1 stages outputs
  static constexpr uint32_t kSmemBytes = kBlobBytes + kRecvBytes + kOnesBytes + kSlots * kSlotBytes + 1024;
  // tensor memory: [kv | ksum] of phase 1 at column 0 (lane = feature; ksum
  // in columns D..D+15); phase-2 accumulators at 0 and kNB (lane = token);
  // three A buffers of 64 columns above them.
  static constexpr uint32_t kAccStride = kNB;
  static constexpr int kABufs = 3;
  static constexpr uint32_t kABufCols = 64;
  static constexpr uint32_t kABuf0 = 2 * kNB;
  static constexpr uint32_t kTmemCols = 512;
  static_assert(kABuf0 + kABufs * kABufCols <= kTmemCols, "tensor memory");
  static constexpr int kPhiWarps = 8;
  static constexpr int kCombWarp0 = 2 + kPhiWarps;
  static constexpr int kThreads = 32 * (kCombWarp0 + 8);
  static constexpr int kMaxClusters = 4;                   // clusters per head
};

__device__ __forceinline__ uint32_t cluster_nctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t ld_relaxed_gpu(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release_gpu(uint32_t* p, uint32_t v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
// 16 bytes from global memory, cached in L2 only (written by another SM in
// this launch).
__device__ __forceinline__ uint4 ld_cg_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.cg.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p)
               : "memory");
  return v;
}

// XC: a head may span several clusters (the exchange through L2 is compiled
// in only then).
__device__ __forceinline__ void mbar_arrive_n(uint64_t* bar, uint32_t n) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(n) : "memory");
}

// 16 E4M3 codes (one 16-byte chunk, lowest feature in the lowest byte) times
// `scale`, rounded to bf16: features 0..7 into lo, 8..15 into hi.  The codes
// are widened exactly to f16 by the hardware conversion, the product is
// formed in fp32.
__device__ __forceinline__ void e4m3x16_to_bf16(uint4 raw, float scale, uint4& lo, uint4& hi) {
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
  uint32_t o[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t f16x2;
      const uint16_t two = static_cast<uint16_t>(w[i] >> (16 * h));
      asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(f16x2) : "h"(two));
      const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&f16x2));
      const __nv_bfloat162 b = __floats2bfloat162_rn(f.x * scale, f.y * scale);
      o[2 * i + h] = *reinterpret_cast<const uint32_t*>(&b);
    }
  }
  lo = make_uint4(o[0], o[1], o[2], o[3]);
  hi = make_uint4(o[4], o[5], o[6], o[7]);
}

// Softmax features of two tokens' values of one feature (bf16x2, lower token
// in the low half): exp(x - m) * rz with that token's row maximum m and
// reciprocal exponential sum rz, rounded to bf16.
__device__ __forceinline__ uint32_t softmax_pair(uint32_t w, float m0, float rz0, float m1, float rz1) {
  const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w));
  const __nv_bfloat162 r = __floats2bfloat162_rn(ex2_approx((x.x - m0) * kLog2e) * rz0,
                                                 ex2_approx((x.y - m1) * kLog2e) * rz1);
  return *reinterpret_cast<const uint32_t*>(&r);
}

// E8: q, k and v are E4M3 codes (tensor maps of bytes, 128 x 128 boxes) with
// one scale each; out is bf16 as for bf16 inputs.
// PRO: Flux's attention prologue on q and k (RMS norm times the scales pq /
// pk, then the rotation table rope [positions][64][2]).
template <int FMAP, bool XC, bool E8, bool PRO>
__global__ void __launch_bounds__(CfgT::kThreads, 1)
    fused_t_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_out,
                   int* status, uint32_t* sync, uint8_t* xchg, int N, int tiles, float eps, float sq, float sk,
                   float sv, const float* pq, const float* pk, const float* rope, float neps) {
  using C = CfgT;
  constexpr int D = C::D;
  // Warps that apply phi to the K tiles: with elu+1 (an exponential per
  // element) the combine warps, idle in phase 1, join the eight phi warps;
  // relu is cheap enough for eight.  With E4M3 inputs the combine warps
  // widen the K and V tiles to bf16 in phase 1 instead.
  // (with the prologue the combine warps normalise and rotate the K tiles
  // in phase 1, so eight warps apply phi)
  constexpr int kKWarps = FMAP == 0 && !E8 && !PRO ? 16 : 8;
  // Softmax (FMAP 2): the combine warps compute each K row's maximum and
  // reciprocal exponential sum in phase 1 (kst, a ring over K tiles; kstat
  // when a tile's rows are in), and read the K slot too.
  constexpr bool kSmx = FMAP == 2;
  constexpr int kStatRing = 6;
  constexpr uint32_t kCodeTileBytes = kTileTokens * C::D;   // one E4M3 tile
  extern __shared__ uint8_t smem_raw[];
  // full: a K or Q tile has arrived (waited on by the phi warps, every phase
  // in order); vfull: a V tile has arrived (MMA issuer); empty: a phase-1
  // slot is free again (a K slot once the phi warps have read it, a V slot
  // once its MMAs are done); qfree: a Q tile has been read by the phi warps.
  __shared__ __align__(8) uint64_t full[C::kRing1], vfull[C::kRing1], empty[C::kRing1], qfree[C::kRing1];
  // E8: an E4M3 tile has landed in the second half of its slot (landed), and
  // a K or V tile has been widened to bf16 over the whole slot by the eight
  // widening warps (wready; the phi warps and the MMA issuer wait on it in
  // place of full and vfull)
  __shared__ __align__(8) uint64_t landed[C::kRing1], wready[C::kRing1];
  __shared__ __align__(8) uint64_t kstat[kStatRing];
  __shared__ __align__(16) float2 kst[kSmx ? kStatRing * kTileTokens : 1];
  // PRO: the norm scales of q (0..127) and k (128..255)
  __shared__ __align__(16) float pscale[PRO ? 2 * D : 4];
  // A buffers in tensor memory, used in turn by the T key tiles and then the
  // T query tiles: written by the phi warps (aready), read by the MMAs (aempty).
  __shared__ __align__(8) uint64_t aready[C::kABufs], aempty[C::kABufs];
  __shared__ __align__(8) uint64_t p1full, p1empty, accfull[2], accempty[2];
  // combine: peers_free (one relaxed arrival per cluster CTA: its receive
  // region is out of phase-1 use); recv_full (the rows this CTA owns have
  // arrived from every other CTA); blob_full (the summed rows of every other
  // owner have arrived, and this CTA's own sum is written).
  __shared__ __align__(8) uint64_t peers_free, recv_full, blob_full;
  __shared__ uint32_t tmem_slot;
  __shared__ int comb_flag, ep_flag;

  // A head is served by P CTAs (blockIdx.x), NC clusters of S CTAs.
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int P = static_cast<int>(gridDim.x);
  const int S = static_cast<int>(cluster_nctarank());
  const int NC = XC ? P / S : 1;
  const int rank = static_cast<int>(cluster_ctarank());
  const int cl = static_cast<int>(blockIdx.x) / S;   // this CTA's cluster within the head
  const int bh = blockIdx.y;
  const int tile0 = static_cast<int>(blockIdx.x) * tiles / P;
  const int T = (static_cast<int>(blockIdx.x) + 1) * tiles / P - tile0;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* blob = smem;
  uint8_t* recv = blob + C::kBlobBytes;
  uint8_t* ones = recv + C::kRecvBytes;
  uint8_t* slots = ones + C::kOnesBytes;
  auto slot_ptr = [&](int phys) {
    return phys < C::kSlots ? slots + phys * C::kSlotBytes : (phys == C::kSlots ? blob : recv);
  };
  // Phase-1 use j (K, V of tile j / 2) takes slot j % kRing1: K tiles in even
  // slots, V tiles in odd ones.  Q tile u takes ring slot u % kRing2.
  auto uses1 = [&](int phys) { return (2 * T + C::kRing1 - 1 - phys) / C::kRing1; };
  auto q_full_round = [&](int u) {   // phases of full[] before Q tile u
    const int s = u % C::kRing2;
    // (E4M3 K tiles complete wready, not full)
    return ((s & 1) == 0 && !E8 ? uses1(s) : 0) + u / C::kRing2;
  };
  // image rows [row0(o), row0(o + 1)) are owned by cluster CTA o
  auto row0 = [&](int o) { return o * C::kRows / S; };
  const int rmax = (C::kRows + S - 1) / S;
  const uint32_t recv_slot = 2u * static_cast<uint32_t>(rmax) * 128u;   // receive bytes per sender

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kRing1; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&vfull[i], 1);
      mbar_init(&empty[i], (i & 1) == 0 ? kKWarps + (kSmx ? 8 : 0) : 1);
      mbar_init(&qfree[i], C::kPhiWarps);
      mbar_init(&landed[i], 1);
      mbar_init(&wready[i], 8);
    }
    for (int i = 0; i < kStatRing; ++i) mbar_init(&kstat[i], 8);
    for (int i = 0; i < C::kABufs; ++i) {
      mbar_init(&aready[i], kKWarps);
      mbar_init(&aempty[i], 1);
    }
    mbar_init(&p1full, 1);
    mbar_init(&p1empty, 8);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&accfull[i], 1);
      mbar_init(&accempty[i], 8);
    }
    mbar_init(&peers_free, S);
    mbar_init(&recv_full, 1);
    mbar_init(&blob_full, 2);
    fence_mbarrier_init();
    const uint32_t mine = static_cast<uint32_t>(row0(rank + 1) - row0(rank));
    mbar_arrive_expect_tx(&recv_full, static_cast<uint32_t>(S - 1) * mine * 256u);
    mbar_arrive_expect_tx(&blob_full, static_cast<uint32_t>(C::kRows - static_cast<int>(mine)) * 256u);
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    prefetch_tmap(&tm_out);
    comb_flag = 0;
    ep_flag = 0;
  }
  if constexpr (PRO) {
    for (int i = threadIdx.x; i < 2 * D; i += blockDim.x) pscale[i] = i < D ? pq[i] : pk[i - D];
  }
  // B operand of the ksum MMA: a block of bf16 ones (any layout reads 1.0)
  for (int i = threadIdx.x; i < static_cast<int>(C::kOnesBytes / 16); i += blockDim.x)
    *reinterpret_cast<uint4*>(ones + 16 * i) = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
  fence_proxy_async_smem();
  if (warp == 1) {
    tmem_alloc(&tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;

  // ------------------------------------------------------------ producer
  int seq = 0;
  auto issue = [&](int upto) {
    while (seq < upto) {
      const bool p1 = seq < 2 * T;
      const int u = seq - 2 * T;
      const int s = p1 ? seq % C::kRing1 : u % C::kRing2;
      if (p1) {
        const int round = seq / C::kRing1;
        if (round > 0 && !mbar_wait(&empty[s], (round - 1) & 1, status)) return;
      } else if (u >= C::kRing2) {
        if (!mbar_wait(&qfree[s], ((u / C::kRing2) - 1) & 1, status)) return;
      } else if (uses1(s) > 0) {
        if (!mbar_wait(&empty[s], (uses1(s) - 1) & 1, status)) return;
      }
      const bool is_v = p1 && (seq & 1);
      const CUtensorMap* m = p1 ? (is_v ? &tm_v : &tm_k) : &tm_q;
      const int tile = p1 ? seq / 2 : u;
      uint64_t* bar = is_v ? &vfull[s] : &full[s];
      uint8_t* dst = slot_ptr(s);
      if constexpr (E8) {
        // the codes fill the second 16 KB of the slot: K and V are widened
        // over the whole slot, Q is read as codes by the phi warps
        if (p1) bar = &landed[s];
        mbar_arrive_expect_tx(bar, kCodeTileBytes);
        tma_load_3d(dst + kCodeTileBytes, m, bar, 0, (tile0 + tile) * kTileTokens, bh);
      } else {
        mbar_arrive_expect_tx(bar, C::kSlotBytes);
#pragma unroll
        for (int b = 0; b < C::kBoxes; ++b)
          tma_load_3d(dst + b * kBoxBytes, m, bar, 64 * b, (tile0 + tile) * kTileTokens, bh);
      }
      ++seq;
    }
  };
  pdl_wait();
  pdl_launch_dependents();
  // Launch count of the exchange between clusters: stable until every CTA of
  // this launch has finished (the last one to finish advances it).
  const uint32_t gen = NC > 1 ? ld_relaxed_gpu(&sync[0]) : 0u;
  cluster_arrive_relaxed();
  if (warp == 0 && lane == 0) issue(min(C::kRing1, 2 * T));
  cluster_wait();

  // phi on the K tiles into tensor memory, by kKWarps warps (kKWarps / 4 per
  // lane quarter): warp (qd, kq) takes features 32 qd .. 32 qd + 31 (two
  // 16-lane halves) of tokens kq * kTok .. kq * kTok + kTok - 1 (16-token blocks).
  auto k_phase = [&]() {
    constexpr int kTok = 128 / (kKWarps / 4), kBlocks = kTok / 16;
    const int qd = warp & 3, kq = (warp - 2) >> 2;
    const int lm = lane >> 3, lr = lane & 7;
    for (int t = 0; t < T; ++t) {
      const int s = (2 * t) % C::kRing1, b = t % C::kABufs;
      if (!warp_wait(E8 || PRO ? &wready[s] : &full[s], ((2 * t) / C::kRing1) & 1, status)) return false;
      const uint32_t base = smem_u32(slot_ptr(s));
      uint32_t x[2][kBlocks][4];
#pragma unroll
      for (int fh = 0; fh < 2; ++fh)
#pragma unroll
        for (int tb = 0; tb < kBlocks; ++tb) {
          // matrix lm: tokens +8 (lm >> 1), features +8 (lm & 1); row lr
          const int tok = kTok * kq + 16 * tb + 8 * (lm >> 1) + lr;
          const int cc = 4 * qd + 2 * fh + (lm & 1);
          ldsm_x4_trans(base + swz_off(tok, cc), x[fh][tb]);
        }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);   // the K tile is in registers
      // softmax: this tile's row statistics (their ring entry is rewritten
      // only after this warp has read the K slot of three tiles later)
      const float2* st = kst + (t % kStatRing) * kTileTokens;
      if (kSmx && !warp_wait(&kstat[t % kStatRing], (t / kStatRing) & 1, status)) return false;
      // key rows past the sequence end must not reach kv or ksum
      const int valid = min(kTileTokens, N - (tile0 + t) * kTileTokens);
#pragma unroll
      for (int fh = 0; fh < 2; ++fh)
#pragma unroll
        for (int tb = 0; tb < kBlocks; ++tb)
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            uint32_t w;
            if constexpr (kSmx) {
              const int tk = kTok * kq + 16 * tb + 8 * (r >> 1) + 2 * (lane & 3);
              const float4 mz = *reinterpret_cast<const float4*>(st + tk);   // tokens tk, tk + 1
              w = softmax_pair(x[fh][tb][r], mz.x, mz.y, mz.z, mz.w);
            } else {
              w = phi_pair<FMAP>(x[fh][tb][r]);
            }
            if (valid < kTileTokens) {
              const int tok = kTok * kq + 16 * tb + 8 * (r >> 1) + 2 * (lane & 3);
              w &= (tok < valid ? 0x0000FFFFu : 0u) | (tok + 1 < valid ? 0xFFFF0000u : 0u);
            }
            x[fh][tb][r] = w;
          }
      if (t >= C::kABufs && !warp_wait(&aempty[b], ((t / C::kABufs) - 1) & 1, status)) return false;
      tc_fence_after();
#pragma unroll
      for (int fh = 0; fh < 2; ++fh)
#pragma unroll
        for (int tb = 0; tb < kBlocks; ++tb)
          tmem_st_16x128b_x2(tmem + (static_cast<uint32_t>(32 * qd + 16 * fh) << 16) + C::kABuf0 +
                                 b * C::kABufCols + kTok / 2 * kq + 8 * tb,
                             x[fh][tb]);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&aready[b]);
    }
    return true;
  };

  // PRO: one 16-byte chunk (features 8 c .. 8 c + 7) of the row at token
  // position pos, times the row's 1 / rms and the feature scales sc, then its
  // four feature pairs turned by the rotation table; rounded to bf16.
  auto prologue_chunk = [&](uint4 x, float rinv, const float* sc, int c, int pos) {
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
    const float4* rp = reinterpret_cast<const float4*>(rope + (static_cast<size_t>(pos) * (D / 2) + 4 * c) * 2);
    uint32_t o[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 v2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[e]));
      const float x0 = v2.x * rinv * sc[8 * c + 2 * e], x1 = v2.y * rinv * sc[8 * c + 2 * e + 1];
      const float4 cs = __ldg(rp + (e >> 1));   // (cos, sin) of pairs 2 (e >> 1) and 2 (e >> 1) + 1
      const float cn = (e & 1) ? cs.z : cs.x, sn = (e & 1) ? cs.w : cs.y;
      const __nv_bfloat162 r = __floats2bfloat162_rn(cn * x0 - sn * x1, sn * x0 + cn * x1);
      o[e] = *reinterpret_cast<const uint32_t*>(&r);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
  };
  // sum of squares of the 8 bf16 values of a chunk
  auto chunk_ss = [](uint4 x) {
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
    float ss = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 v2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[e]));
      ss = fmaf(v2.x, v2.x, fmaf(v2.y, v2.y, ss));
    }
    return ss;
  };

  if (warp == 0) {
    if (lane == 0) issue(3 * T);
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_kv = idesc_bf16_f32(128, D, 0, 1);        // A = phi(K)^T (TMEM), B = V (MN-major)
      constexpr uint32_t idesc_ks = idesc_bf16_f32(128, 16, 0, 0);       // B = ones (K-major)
      constexpr uint32_t idesc_ap = idesc_bf16_f32(128, C::kNB, 0, 0);   // A = phi(Q) (TMEM), B = image
      const uint64_t ones_desc = smem_desc_noswz(smem_u32(ones), 128, 256);
      bool ok = true;
      for (int t = 0; t < T; ++t) {
        const int sv = (2 * t + 1) % C::kRing1, b = t % C::kABufs;
        if (!mbar_wait(&aready[b], (t / C::kABufs) & 1, status) ||
            !mbar_wait(E8 ? &wready[sv] : &vfull[sv], ((2 * t + 1) / C::kRing1) & 1, status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t atm = tmem + C::kABuf0 + b * C::kABufCols;
        const uint64_t vdesc = smem_desc_sw128(smem_u32(slot_ptr(sv)), kBoxBytes, 1024);
        // 16 tokens per MMA: 8 A columns, 2048 bytes of V
        if (t == 0) {
          umma_ts<0>(tmem, atm, vdesc, idesc_kv);
          umma_ts<0>(tmem + D, atm, ones_desc, idesc_ks);
        } else {
          umma_ts<1>(tmem, atm, vdesc, idesc_kv);
          umma_ts<1>(tmem + D, atm, ones_desc, idesc_ks);
        }
#pragma unroll
        for (int k = 1; k < kTileTokens / 16; ++k) {
          umma_ts<1>(tmem, atm + 8 * k, desc_add(vdesc, 2048 * k), idesc_kv);
          umma_ts<1>(tmem + D, atm + 8 * k, ones_desc, idesc_ks);
        }
        umma_commit(&empty[sv]);
        umma_commit(&aempty[b]);
      }
      umma_commit(&p1full);
      if (ok && mbar_wait_cluster(&blob_full, 0, status)) {
        fence_proxy_async_smem();   // the cluster's copies into `blob` feed the tensor core
        const uint64_t bdesc = smem_desc_sw128(smem_u32(blob), 16, 1024);
        for (int u = 0; u < T; ++u) {
          const int j = T + u, b = j % C::kABufs;
          const int a = u & 1, ar = u >> 1;
          bool got = mbar_wait(&aready[b], (j / C::kABufs) & 1, status);
          if (got) got = ar == 0 ? mbar_wait(&p1empty, 0, status) : mbar_wait(&accempty[a], (ar - 1) & 1, status);
          if (!got) break;
          tc_fence_after();
          const uint32_t atm = tmem + C::kABuf0 + b * C::kABufCols;
          const uint32_t d = tmem + a * C::kAccStride;
          umma_ts<0>(d, atm, bdesc, idesc_ap);
#pragma unroll
          for (int k = 1; k < D / 16; ++k)
            umma_ts<1>(d, atm + 8 * k, desc_add(bdesc, (k >> 2) * C::kBlobAtomBytes + (k & 3) * 32), idesc_ap);
          umma_commit(&aempty[b]);
          umma_commit(&accfull[a]);
        }
      }
    }
  } else if (warp < C::kCombWarp0) {
    // ------------------------------------------------------- phi warps
    // Tensor-memory lane quarter qd (the warp's accessible lanes); half hf.
    const int qd = warp & 3, hf = (warp - 2) >> 2;
    bool ok = k_phase();
    // Q tiles: token row 32 qd + lane, features 64 hf .. 64 hf + 63
    const int i = 32 * qd + lane;
    const uint32_t lanes = static_cast<uint32_t>(32 * qd) << 16;
    for (int u = 0; u < T && ok; ++u) {
      const int s = u % C::kRing2, j = T + u, b = j % C::kABufs;
      if (!warp_wait(&full[s], q_full_round(u) & 1, status)) break;
      const uint8_t* src = slot_ptr(s);
      uint4 x[8];
      float rowmax = 0.f;
      if constexpr (E8) {
        // codes of features 64 hf .. 64 hf + 63: four 16-byte chunks of the
        // 128-byte row (128-byte swizzle), widened to bf16 times sq
        uint4 raw[4];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const int c = 4 * hf + m;
          raw[m] = *reinterpret_cast<const uint4*>(src + kCodeTileBytes + i * 128 + ((c ^ (i & 7)) << 4));
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&qfree[s]);   // the Q tile is in registers
#pragma unroll
        for (int m = 0; m < 4; ++m) e4m3x16_to_bf16(raw[m], sq, x[2 * m], x[2 * m + 1]);
      } else if constexpr (PRO) {
        // the row's sum of squares over all 128 features (the other half's
        // chunks are read for it, before the slot is released)
        float ss = 0.f;
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          x[m] = *reinterpret_cast<const uint4*>(src + swz_off(i, 8 * hf + m));
          ss += chunk_ss(x[m]) + chunk_ss(*reinterpret_cast<const uint4*>(src + swz_off(i, 8 * (1 - hf) + m)));
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&qfree[s]);   // the Q tile is in registers
        const int pos = (tile0 + u) * kTileTokens + i;
        if (pos < N) {   // rows past the sequence end are never stored
          const float rinv = 1.f / sqrtf(ss * (1.f / D) + neps);
#pragma unroll
          for (int m = 0; m < 8; ++m) x[m] = prologue_chunk(x[m], rinv, pscale, 8 * hf + m, pos);
        }
      } else {
#pragma unroll
        for (int m = 0; m < 8; ++m) x[m] = *reinterpret_cast<const uint4*>(src + swz_off(i, 8 * hf + m));
        if constexpr (kSmx) {
          // softmax: the row's maximum over all 128 features (the other
          // half's chunks are read for it, before the slot is released)
          __nv_bfloat162 mx = *reinterpret_cast<const __nv_bfloat162*>(&x[0].x);
#pragma unroll
          for (int m = 0; m < 8; ++m) {
            const uint32_t o[4] = {x[m].x, x[m].y, x[m].z, x[m].w};
            const uint4 y = *reinterpret_cast<const uint4*>(src + swz_off(i, 8 * (1 - hf) + m));
            const uint32_t p[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
            for (int e = 0; e < 4; ++e)
              mx = __hmax2(mx, __hmax2(*reinterpret_cast<const __nv_bfloat162*>(&o[e]),
                                       *reinterpret_cast<const __nv_bfloat162*>(&p[e])));
          }
          rowmax = fmaxf(__low2float(mx), __high2float(mx));
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&qfree[s]);   // the Q tile is in registers
      }
      uint32_t w[32];
      if constexpr (kSmx) {
        // exp(x - rowmax): the row's normaliser is not applied; with eps
        // folded into ksum it cancels exactly
        const float c = rowmax;
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          const uint32_t o[4] = {x[m].x, x[m].y, x[m].z, x[m].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) w[4 * m + e] = softmax_pair(o[e], c, 1.f, c, 1.f);
        }
      } else {
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          const uint4 y = phi_chunk<FMAP>(x[m]);
          w[4 * m] = y.x;
          w[4 * m + 1] = y.y;
          w[4 * m + 2] = y.z;
          w[4 * m + 3] = y.w;
        }
      }
      if (j >= C::kABufs && !warp_wait(&aempty[b], ((j / C::kABufs) - 1) & 1, status)) break;
      tc_fence_after();
      tmem_st32(tmem + C::kABuf0 + b * C::kABufCols + 32 * hf + lanes, w);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_n(&aready[b], kKWarps / 8);   // counted like the K-tile warps
    }
  } else {
    // ----------------------------------------- combine, then the outputs
    const int ct = threadIdx.x - 32 * C::kCombWarp0;   // 0..255
    const int half = ct >> 7;
    const bool leader = ct == 0;
    const int q = warp & 3;
    const uint32_t tq = static_cast<uint32_t>(32 * q) << 16;
    // E8: widen every K and V tile to bf16 (codes times sk or sv, rounded to
    // bf16, in the layout of a bf16 tile), in the order they were issued.
    // Warp w takes rows 16 w .. 16 w + 15, eight lanes per row.  The codes of
    // row r sit in the slot's second half exactly where the bf16 row r of
    // features 64..127 goes, and only the eight lanes of row r touch either,
    // so a __syncwarp between their reads and writes is all the ordering the
    // rewrite needs; each warp then arrives on wready.
    auto widen = [&]() {
      const int w8 = warp - C::kCombWarp0, c = lane & 7;
      for (int j = 0; j < 2 * T; ++j) {
        const int s = j % C::kRing1;
        uint8_t* slot = slot_ptr(s);
        if (!warp_wait(&landed[s], (j / C::kRing1) & 1, status)) return false;
        uint4 raw[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const int row = 16 * w8 + 4 * r + (lane >> 3);
          raw[r] = *reinterpret_cast<const uint4*>(slot + kCodeTileBytes + row * 128 + ((c ^ (row & 7)) << 4));
        }
        __syncwarp();
        const float sc = (j & 1) ? sv : sk;
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const int row = 16 * w8 + 4 * r + (lane >> 3);
          uint4 lo, hi;
          e4m3x16_to_bf16(raw[r], sc, lo, hi);
          *reinterpret_cast<uint4*>(slot + swz_off(row, 2 * c)) = lo;
          *reinterpret_cast<uint4*>(slot + swz_off(row, 2 * c + 1)) = hi;
        }
        fence_proxy_async_smem();   // V tiles feed the tensor core
        __syncwarp();
        if (lane == 0) mbar_arrive(&wready[s]);
      }
      return true;
    };
    // softmax: each K row's maximum and reciprocal exponential sum, two
    // threads per row (adjacent lanes, 64 features each), into kst
    auto kstats = [&]() {
      const int row = ct >> 1, hh = ct & 1;
      for (int t = 0; t < T; ++t) {
        const int s = (2 * t) % C::kRing1;
        if (!warp_wait(&full[s], ((2 * t) / C::kRing1) & 1, status)) return false;
        const uint8_t* slot = slot_ptr(s);
        uint4 x[8];
#pragma unroll
        for (int m = 0; m < 8; ++m) x[m] = *reinterpret_cast<const uint4*>(slot + swz_off(row, 8 * hh + m));
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);   // the K tile is in registers
        __nv_bfloat162 mx = *reinterpret_cast<const __nv_bfloat162*>(&x[0].x);
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          const uint32_t o[4] = {x[m].x, x[m].y, x[m].z, x[m].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) mx = __hmax2(mx, *reinterpret_cast<const __nv_bfloat162*>(&o[e]));
        }
        float m0 = fmaxf(__low2float(mx), __high2float(mx));
        m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, 1));
        float z = 0.f;
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          const uint32_t o[4] = {x[m].x, x[m].y, x[m].z, x[m].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 v2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&o[e]));
            z += ex2_approx((v2.x - m0) * kLog2e) + ex2_approx((v2.y - m0) * kLog2e);
          }
        }
        z += __shfl_xor_sync(0xffffffffu, z, 1);
        if (hh == 0) kst[(t % kStatRing) * kTileTokens + row] = make_float2(m0, 1.f / z);
        __syncwarp();
        if (lane == 0) mbar_arrive(&kstat[t % kStatRing]);
      }
      return true;
    };
    // PRO: every K tile normalised and rotated in place before the phi warps
    // read it: warp w takes rows 16 w .. 16 w + 15, eight lanes per row (two
    // chunks each, features 16 c .. 16 c + 15), the row's sum of squares over
    // the eight lanes by shuffles; each warp arrives on wready.
    auto kprologue = [&]() {
      const int w8 = warp - C::kCombWarp0, c = lane & 7;
      for (int t = 0; t < T; ++t) {
        const int s = (2 * t) % C::kRing1;
        if (!warp_wait(&full[s], ((2 * t) / C::kRing1) & 1, status)) return false;
        uint8_t* slot = slot_ptr(s);
#pragma unroll 1
        for (int r = 0; r < 4; ++r) {
          const int row = 16 * w8 + 4 * r + (lane >> 3);
          uint4 a = *reinterpret_cast<const uint4*>(slot + swz_off(row, 2 * c));
          uint4 b = *reinterpret_cast<const uint4*>(slot + swz_off(row, 2 * c + 1));
          float ss = chunk_ss(a) + chunk_ss(b);
          ss += __shfl_xor_sync(0xffffffffu, ss, 1);
          ss += __shfl_xor_sync(0xffffffffu, ss, 2);
          ss += __shfl_xor_sync(0xffffffffu, ss, 4);
          const int pos = (tile0 + t) * kTileTokens + row;
          if (pos < N) {   // rows past the sequence end are masked to zero later
            const float rinv = 1.f / sqrtf(ss * (1.f / D) + neps);
            a = prologue_chunk(a, rinv, pscale + D, 2 * c, pos);
            b = prologue_chunk(b, rinv, pscale + D, 2 * c + 1, pos);
            *reinterpret_cast<uint4*>(slot + swz_off(row, 2 * c)) = a;
            *reinterpret_cast<uint4*>(slot + swz_off(row, 2 * c + 1)) = b;
          }
        }
        fence_proxy_async_smem();   // TMA refills the slot later
        __syncwarp();
        if (lane == 0) mbar_arrive(&wready[s]);
      }
      return true;
    };
    bool got = E8 ? widen() : (kSmx ? kstats() : (PRO ? kprologue() : (kKWarps == 16 ? k_phase() : true)));
    auto sync_ok = [&](bool mine) {
      if (leader && !mine) comb_flag = 1;
      named_bar_sync(3, 256);
      return comb_flag == 0;
    };
    if (leader && got) got = mbar_wait(&p1full, 0, status);
    bool ok = sync_ok(got);
    if (ok) {
      // (1) the partial [kv | ksum] (lane = feature, column = value) into
      // this CTA's image, bf16, row = value with the features contiguous:
      // 16 features x 16 columns per tcgen05.ld / stmatrix.trans pair.
      // Columns D..D+15 all hold ksum: they fill rows D..D+15, whose copies
      // above row D only feed accumulator columns nobody reads.
      tc_fence_after();
      const uint32_t blob_base = smem_u32(blob);
      auto put = [&](int fh, int n0) {
        uint32_t r[8];
        tmem_ld_16x256b_x2(tmem + tq + (static_cast<uint32_t>(16 * fh) << 16) + n0, r);
        tmem_wait_ld();
        // matrix m: features +8 (m & 1), values +8 (m >> 1); row = value
        const int m = lane >> 3;
        const int n = n0 + 8 * (m >> 1) + (lane & 7);
        const int c = 4 * q + 2 * fh + (m & 1);   // 16-byte feature chunk
        const uint32_t addr =
            blob_base + (c >> 3) * C::kBlobAtomBytes + n * 128 + (((c & 7) ^ (n & 7)) << 4);
        stsm_x4_trans(addr, pack_bf16x2(r[0], r[1]), pack_bf16x2(r[2], r[3]), pack_bf16x2(r[4], r[5]),
                      pack_bf16x2(r[6], r[7]));
      };
#pragma unroll
      for (int fh = 0; fh < 2; ++fh)
#pragma unroll
        for (int nb = 0; nb < 4; ++nb) put(fh, 64 * half + 16 * nb);
      if (half == 1) {
        put(0, D);
        put(1, D);
      }
      fence_proxy_async_smem();   // read by the bulk copies and the tensor core
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p1empty);
      // (2) every CTA's receive region is out of phase-1 use: send each owner
      // its rows, one bulk copy per owner and k-atom
      named_bar_sync(3, 256);
      if (ct < S) mbar_arrive_remote_relaxed(mapa_shared(smem_u32(&peers_free), ct));
      if (ct < 32) {
        int g = 1;
        if (lane == 0) g = mbar_wait_cluster(&peers_free, 0, status) ? 1 : 0;
        g = __shfl_sync(0xffffffffu, g, 0);
        if (g && lane < 2 * (S - 1)) {
          const int o = (rank + 1 + (lane >> 1)) % S, a = lane & 1;
          const int n0 = row0(o), n1 = row0(o + 1);
          bulk_copy_to_cluster(mapa_shared(smem_u32(recv) + rank * recv_slot + a * rmax * 128, o),
                               blob + a * C::kBlobAtomBytes + n0 * 128, static_cast<uint32_t>(n1 - n0) * 128u,
                               mapa_shared(smem_u32(&recv_full), o));
        }
        if (leader) got = g != 0;
      }
      if (leader && got) got = mbar_wait_cluster(&recv_full, 0, status);
      ok = sync_ok(got);
    }
    if (ok) {
      // (3) this CTA's rows: the sum over the S partials in ascending CTA
      // order, rounded to bf16, into its own image, then into every other
      // CTA's image.  Positions within a row are the same in every copy.
      const int n0 = row0(rank), rows = row0(rank + 1) - n0;
      for (int js = ct; js < 2 * rows * 8; js += 256) {
        const int a = js / (rows * 8), rem = js % (rows * 8);
        const uint32_t off_img = a * C::kBlobAtomBytes + (n0 + rem / 8) * 128 + (rem % 8) * 16;
        const uint32_t off_rcv = a * rmax * 128 + rem * 16;
        float acc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = 0.f;
        for (int p = 0; p < S; ++p) {
          const uint8_t* src = p == rank ? blob + off_img : recv + p * recv_slot + off_rcv;
          const uint4 w = *reinterpret_cast<const uint4*>(src);
          const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wv[e]));
            acc[2 * e] += x.x;
            acc[2 * e + 1] += x.y;
          }
        }
        // softmax: eps joins every ksum entry once (after the last sum), so
        // the apply's denominator is sum_f u_f (ksum_f + eps) for the
        // unnormalised query features u
        if (kSmx && !(XC && NC > 1) && n0 + rem / 8 >= D) {
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[e] += eps;
        }
        *reinterpret_cast<uint4*>(blob + off_img) = pack8(acc);
      }
      if (XC && NC > 1) {
        // (3b) the head spans NC clusters: publish these rows (this cluster's
        // sums) in the exchange area, wait for the CTAs of the same rank in
        // the other clusters to publish theirs, and sum the NC copies in
        // ascending cluster order (every cluster gets the same bits).
        uint8_t* mine = xchg + (static_cast<size_t>(bh) * NC + cl) * C::kBlobBytes;
        named_bar_sync(3, 256);
        for (int js = ct; js < 2 * rows * 8; js += 256) {
          const int a = js / (rows * 8), rem = js % (rows * 8);
          const uint32_t off = a * C::kBlobAtomBytes + (n0 + rem / 8) * 128 + (rem % 8) * 16;
          *reinterpret_cast<uint4*>(mine + off) = *reinterpret_cast<const uint4*>(blob + off);
        }
        __threadfence();
        named_bar_sync(3, 256);
        uint32_t* flags = sync + 2;
        if (leader) st_release_gpu(&flags[bh * P + blockIdx.x], gen + 1);
        if (ct < 32) {
          int g = 1;
          if (lane < NC && lane != cl) {
            const uint32_t* f = &flags[bh * P + lane * S + rank];
            const uint64_t t0 = globaltimer_ns();
            while (ld_acquire_gpu(f) < gen + 1) {
              if (globaltimer_ns() - t0 > kWaitLimitNs) {
                record_error(status, kDeviceTimeout);
                g = 0;
                break;
              }
            }
          }
          g = __all_sync(0xffffffffu, g);
          if (leader && !g) comb_flag = 1;
        }
        named_bar_sync(3, 256);
        if (comb_flag == 0) {
          const uint8_t* base = xchg + static_cast<size_t>(bh) * NC * C::kBlobBytes;
          for (int js0 = ct; js0 < 2 * rows * 8; js0 += 256 * 4) {
            uint4 w[4][C::kMaxClusters];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int js = js0 + 256 * e;
              if (js < 2 * rows * 8) {
                const int a = js / (rows * 8), rem = js % (rows * 8);
                const uint32_t off = a * C::kBlobAtomBytes + (n0 + rem / 8) * 128 + (rem % 8) * 16;
#pragma unroll
                for (int c = 0; c < C::kMaxClusters; ++c)
                  if (c < NC)
                    w[e][c] = c == cl ? *reinterpret_cast<const uint4*>(blob + off)
                                      : ld_cg_v4(base + static_cast<size_t>(c) * C::kBlobBytes + off);
              }
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int js = js0 + 256 * e;
              if (js < 2 * rows * 8) {
                const int a = js / (rows * 8), rem = js % (rows * 8);
                const uint32_t off = a * C::kBlobAtomBytes + (n0 + rem / 8) * 128 + (rem % 8) * 16;
                float acc[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) acc[i] = 0.f;
#pragma unroll
                for (int c = 0; c < C::kMaxClusters; ++c)
                  if (c < NC) {
                    const uint32_t wv[4] = {w[e][c].x, w[e][c].y, w[e][c].z, w[e][c].w};
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                      const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wv[i]));
                      acc[2 * i] += x.x;
                      acc[2 * i + 1] += x.y;
                    }
                  }
                if (kSmx && n0 + rem / 8 >= D) {   // eps into ksum (see above)
#pragma unroll
                  for (int i = 0; i < 8; ++i) acc[i] += eps;
                }
                *reinterpret_cast<uint4*>(blob + off) = pack8(acc);
              }
            }
          }
        }
      }
      fence_proxy_async_smem();
      named_bar_sync(3, 256);
      if (comb_flag == 0 && ct < 2 * (S - 1)) {
        const int o = (rank + 1 + (ct >> 1)) % S, a = ct & 1;
        const uint32_t off = a * C::kBlobAtomBytes + n0 * 128;
        bulk_copy_to_cluster(mapa_shared(smem_u32(blob) + off, o), blob + off, static_cast<uint32_t>(rows) * 128u,
                             mapa_shared(smem_u32(&blob_full), o));
      }
      if (leader) mbar_arrive(&blob_full);   // this CTA's own rows are in place
      ok = comb_flag == 0;
    }
    if (ok) {
      // (4) outputs: each warp its rows' half of the value columns, staged
      // in buffer u & 1 (the receive region, then the last ring slot), one
      // TMA store per tile
      constexpr int kHalfCols = D / 2;
      for (int u = 0; u < T; ++u) {
        const int a = u & 1, ar = u >> 1;
        got = true;
        if (leader) {
          got = mbar_wait(&accfull[a], ar & 1, status);
          if (u >= 2) bulk_wait_group_read<1>();
        }
        if (leader && !got) ep_flag = 1;
        named_bar_sync(2, 256);
        if (ep_flag) break;
        tc_fence_after();
        const uint32_t trow = tmem + a * C::kAccStride + tq;
        const int r = 32 * q + lane;
        float v[kHalfCols];
        const float den = tmem_ld1(trow + D);
#pragma unroll
        for (int c0 = 0; c0 < kHalfCols; c0 += 32) tmem_ld32(trow + half * kHalfCols + c0, *reinterpret_cast<float(*)[32]>(v + c0));
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&accempty[a]);
        const float inv = 1.0f / (kSmx ? den : den + eps);   // softmax: eps is in den already
#pragma unroll
        for (int e = 0; e < kHalfCols; ++e) v[e] *= inv;
        uint8_t* ob = a == 0 ? recv : slots + (C::kSlots - 1) * C::kSlotBytes;
#pragma unroll
        for (int jj = 0; jj < kHalfCols / 8; ++jj)
          *reinterpret_cast<uint4*>(ob + swz_off(r, half * (kHalfCols / 8) + jj)) = pack8(v + 8 * jj);
        fence_proxy_async_smem();
        named_bar_sync(2, 256);
        if (leader) {
#pragma unroll
          for (int bb = 0; bb < C::kBoxes; ++bb)
            tma_store_3d(&tm_out, ob + bb * kBoxBytes, 64 * bb, (tile0 + u) * kTileTokens, bh);
          bulk_commit_group();
        }
      }
      if (leader) bulk_wait_group<0>();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, C::kTmemCols);
  if (XC && NC > 1 && threadIdx.x == 0) {
    // the last CTA of the launch to get here advances the launch count
    __threadfence();
    const uint32_t total = gridDim.x * gridDim.y;
    if (atomicAdd(&sync[1], 1u) == total - 1) {
      sync[1] = 0;
      __threadfence();
      st_release_gpu(&sync[0], gen + 1);
    }
  }
  cluster_sync_all();
}

// Clusters of `kern` (cluster size s, `smem` bytes, `threads` threads) that
// can be resident at once on the current device; cached per device, kernel
// and size.
int max_active_clusters(const void* kern, uint32_t smem, int threads, int s) {
  static std::mutex mu;
  static const void* key[16];
  static int cache[64][16][17];
  static bool have[64][16][17] = {};
  static int nkeys = 0;
  int dev = 0;
  if (s < 1 || s > 16 || cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return 0;
  }
  std::lock_guard<std::mutex> lock(mu);
  int k = 0;
  while (k < nkeys && key[k] != kern) ++k;
  if (k == nkeys) {
    if (nkeys == 16) return 0;
    key[nkeys++] = kern;
  }
  if (!have[dev][k][s]) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(s), 1);
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(s);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int m = 0;
    if (ensure_smem_attr(kern, smem) != cudaSuccess || cudaOccupancyMaxActiveClusters(&m, kern, &cfg) != cudaSuccess) {
      cudaGetLastError();
      m = 0;
    }
    cache[dev][k][s] = m;
    have[dev][k][s] = true;
  }
  return cache[dev][k][s];
}

// D = 64: one cluster per head, the largest size S <= min(8, tiles) for
// which B*H clusters fit on the device at once (one wave); 1 when none does.
int pick_cluster(const void* kern, uint32_t smem, int threads, long long BH, int tiles) {
  const int smax = tiles < 8 ? tiles : 8;
  for (int s = smax; s >= 2; --s)
    if (max_active_clusters(kern, smem, threads, s) >= BH) return s;
  return 1;
}

// D = 128: P CTAs per head in NC = P / S clusters of S.  One cluster per
// head (the largest S <= min(8, tiles) whose B*H clusters fit at once) unless
// that leaves more than half of the SMs idle; then heads are spread over up to
// four clusters (P <= 16, every CTA of the launch resident at once, since the
// clusters of a head wait for one another).  The exchange between clusters
// goes through L2 and costs several microseconds under full memory load, so
// it only pays where one cluster per head would use few SMs (few heads).
// Heads that outnumber the SMs run one CTA each, in waves.
void geometry_t(long long BH, int tiles, int num_sms, int* P_out, int* S_out) {
  const void* kern = reinterpret_cast<const void*>(fused_t_kernel<0, false, false, false>);
  const int s1 = pick_cluster(kern, CfgT::kSmemBytes, CfgT::kThreads, BH, tiles);
  *P_out = s1;
  *S_out = s1;
  if (BH * s1 * 2 >= num_sms) return;
  const long long pmax = std::min<long long>(std::min(tiles, 16), num_sms / std::max<long long>(BH, 1));
  for (long long P = pmax; P > s1; --P) {
    if (BH * P > kSyncFlags) continue;
    for (int S = static_cast<int>(std::min<long long>(P, 8)); S >= 1; --S) {
      if (P % S != 0 || P / S > CfgT::kMaxClusters) continue;
      if (max_active_clusters(kern, CfgT::kSmemBytes, CfgT::kThreads, S) >= BH * (P / S)) {
        *P_out = static_cast<int>(P);
        *S_out = S;
        return;
      }
    }
  }
}

template <class C, class Kern>
cudaError_t launch_fused(const LaunchArgs& a, Kern kern, int P, int S, uint32_t* sync, uint8_t* xchg) {
  const Plan& p = *a.p;
  cudaError_t err = ensure_smem_attr(reinterpret_cast<const void*>(kern), C::kSmemBytes);
  if (err != cudaSuccess) return err;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(S);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(P), static_cast<unsigned>(p.BH));
  cfg.blockDim = dim3(C::kThreads);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = a.stream;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  int* status = reinterpret_cast<int*>(a.ws + p.off_status);
  if constexpr (std::is_same<C, CfgT>::value)
    return cudaLaunchKernelEx(&cfg, kern, *a.tm_q, *a.tm_k, *a.tm_v, *a.tm_out, status, sync, xchg, p.N, p.tiles,
                              p.eps, a.scale_q, a.scale_k, a.scale_v, a.pro_q, a.pro_k, a.pro_rope, a.pro_eps);
  else
    return cudaLaunchKernelEx(&cfg, kern, *a.tm_q, *a.tm_k, *a.tm_v, *a.tm_out, status, p.N, p.tiles, p.eps);
}

}  // namespace

void noncausal_geometry(Plan* p, size_t* xchg_bytes) {
  *xchg_bytes = 0;
  if (p->D == 128) {
    geometry_t(p->BH, std::max(p->tiles, 1), p->num_sms, &p->ctas_per_head, &p->cluster);
    const int nc = p->ctas_per_head / p->cluster;
    if (nc > 1) *xchg_bytes = static_cast<size_t>(p->BH) * nc * CfgT::kBlobBytes;
  } else {
    const void* kern = reinterpret_cast<const void*>(fused_kernel<64, 0>);
    const int s = pick_cluster(kern, Cfg<64>::kSmemBytes, Cfg<64>::kThreads, p->BH, std::max(p->tiles, 1));
    p->ctas_per_head = s;
    p->cluster = s;
  }
}

cudaError_t launch_bf16_noncausal(const LaunchArgs& a) {
  const Plan& p = *a.p;
  if (p.F != 0 || p.ctas_per_head < 1 || p.cluster < 1) return cudaErrorNotSupported;
  uint32_t* sync = reinterpret_cast<uint32_t*>(a.ws + p.off_sync);
  uint8_t* xchg = reinterpret_cast<uint8_t*>(a.ws + p.off_xchg);
  const int P = p.ctas_per_head, S = p.cluster;
  if (p.D == 128) {
    if (a.prologue) {
      if (a.e4m3 || p.fmap == 2) return cudaErrorNotSupported;
      if (P > S)
        return p.fmap == 0 ? launch_fused<CfgT>(a, fused_t_kernel<0, true, false, true>, P, S, sync, xchg)
                           : launch_fused<CfgT>(a, fused_t_kernel<1, true, false, true>, P, S, sync, xchg);
      return p.fmap == 0 ? launch_fused<CfgT>(a, fused_t_kernel<0, false, false, true>, P, S, sync, xchg)
                         : launch_fused<CfgT>(a, fused_t_kernel<1, false, false, true>, P, S, sync, xchg);
    }
    if (p.fmap == 2) {
      if (a.e4m3) return cudaErrorNotSupported;
      return P > S ? launch_fused<CfgT>(a, fused_t_kernel<2, true, false, false>, P, S, sync, xchg)
                   : launch_fused<CfgT>(a, fused_t_kernel<2, false, false, false>, P, S, sync, xchg);
    }
    if (a.e4m3) {
      if (P > S)
        return p.fmap == 0 ? launch_fused<CfgT>(a, fused_t_kernel<0, true, true, false>, P, S, sync, xchg)
                           : launch_fused<CfgT>(a, fused_t_kernel<1, true, true, false>, P, S, sync, xchg);
      return p.fmap == 0 ? launch_fused<CfgT>(a, fused_t_kernel<0, false, true, false>, P, S, sync, xchg)
                         : launch_fused<CfgT>(a, fused_t_kernel<1, false, true, false>, P, S, sync, xchg);
    }
    if (P > S)
      return p.fmap == 0 ? launch_fused<CfgT>(a, fused_t_kernel<0, true, false, false>, P, S, sync, xchg)
                         : launch_fused<CfgT>(a, fused_t_kernel<1, true, false, false>, P, S, sync, xchg);
    return p.fmap == 0 ? launch_fused<CfgT>(a, fused_t_kernel<0, false, false, false>, P, S, sync, xchg)
                       : launch_fused<CfgT>(a, fused_t_kernel<1, false, false, false>, P, S, sync, xchg);
  }
  if (a.e4m3 || p.fmap == 2 || a.prologue) return cudaErrorNotSupported;
  if (p.D == 64)
    return p.fmap == 0 ? launch_fused<Cfg<64>>(a, fused_kernel<64, 0>, P, S, sync, xchg)
                       : launch_fused<Cfg<64>>(a, fused_kernel<64, 1>, P, S, sync, xchg);
  return cudaErrorNotSupported;
}

}  // namespace la
