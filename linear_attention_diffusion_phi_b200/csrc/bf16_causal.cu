// bf16_causal.cu -- tcgen05 tensor-core path for causal phi attention, bf16
// storage and fp32 accumulation, D = 64, F = 0.
//
// Method (page "NNT Define Linear Attention", "The inputs": with causal set,
// a token attends only to itself and earlier tokens; "How it works":
// kv = phi(K)^T V and the normaliser 1/(phi(Q) . sum phi(K) + eps)).  Query i
// sees keys j <= i:
//   out_i = phi(q_i)^T S_i / (phi(q_i) . z_i + eps),
//   S_i = sum_{j<=i} phi(k_j) v_j^T,  z_i = sum_{j<=i} phi(k_j).
// Each head's sequence is cut into `splits` segments of whole 128-token
// chunks, one CTA per (segment, head):
//   causal_state_kernel  the sum S_seg^T, z_seg^T of every segment but the
//                        last, as one MMA per 16 tokens: [V | 1]^T phi(K)
//                        (M = 128: 64 value rows, a row of ones, zeros);
//   causal_chunk_kernel  the segment's starting state is the sum of the
//                        earlier segments' states (ascending order, fp32);
//                        then chunk by chunk:
//                          P  = phi(Q_c) phi(K_c)^T           (128 x 128)
//                          Pm = P with j > i zeroed, bf16; r_i = sum_j Pm_ij
//                          O  = phi(Q_c) [S_c | z_c] + Pm [V_c | 1]
//                               (numerator; column 64: phi(q_i) . z_c + r_i)
//                          out_i = O_i[0:64] / (O_i[64] + eps)
//                          S_{c+1} = S_c + [V_c | 1]^T phi(K_c)
//                        with the running state in fp32 registers of four
//                        warps and each chunk's increment in tensor memory.
// The chunk length (128) is a performance choice; the result depends on it
// only through rounding.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "bf16_common.cuh"
#include "la_internal.h"
#include "sm100.cuh"

namespace la {
namespace {

constexpr int kD = 64;
constexpr uint32_t kTile = 128u * kD * 2u;     // one 128-token tile of Q, K or V: 16 KB (one TMA box)
constexpr int kStateRows = kD + 1;             // S^T rows, then z^T
constexpr int kStateFloats = kStateRows * kD;  // per segment, fp32, row-major [65][64]
constexpr int kImgRows = kD + 16;              // B operand [S | z | 0]^T: N = 80
constexpr uint32_t kImgBytes = kImgRows * 128;

// A-operand atom of ones: [128 tokens x 64] bf16 in the MN-major 128-byte
// swizzled layout; element 0 of every token row is 1, the rest 0.  Placed as
// the second M atom after a V tile, [V | ones]^T phi(K) has z^T in row 64.
__device__ __forceinline__ void fill_ones_atom(uint8_t* p) {
  for (int i = threadIdx.x; i < static_cast<int>(kTile / 16); i += blockDim.x) {
    const int t = i >> 3, stored = i & 7;      // token row, stored 16-byte chunk
    const uint32_t w = (stored == (t & 7)) ? 0x3F80u : 0u;   // logical chunk 0 lives at t & 7
    *reinterpret_cast<uint4*>(p + i * 16) = make_uint4(w, 0u, 0u, 0u);
  }
}

// phi on the 128 x 64 tile the 256 calling threads (8 warps, two per
// sub-partition) share: column chunk pt / 32, rows pt % 32 + 32 j.
template <int FMAP>
__device__ __forceinline__ void phi_tile(uint8_t* tile, int pt, int valid) {
  phi_rows<FMAP, 4, 32>(tile, pt >> 5, pt & 31, valid);
}

constexpr int kPhiWarps = 8;

// ================================================= kernel 1: segment states

constexpr int kStSlots = 8;
constexpr uint32_t kStSmem = kStSlots * kTile + kTile + 1024;

constexpr int kStThreads = 64 + 32 * kPhiWarps;   // producer, MMA, phi warps

template <int FMAP>
__global__ void __launch_bounds__(kStThreads, 1)
    causal_state_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                        float* __restrict__ state, int* status, int tps, int nseg) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full[kStSlots], ready[kStSlots], empty[kStSlots], accfull;
  __shared__ uint32_t tmem_slot;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int seg = blockIdx.x, bh = blockIdx.y;
  const int tile0 = seg * tps, T = tps;   // never the last segment: always whole and inside N
  uint8_t* slots = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ones = slots + kStSlots * kTile;   // above every slot: a positive atom stride

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStSlots; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&ready[i], kPhiWarps);
      mbar_init(&empty[i], 1);
    }
    mbar_init(&accfull, 1);
    fence_mbarrier_init();
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
  }
  fill_ones_atom(ones);
  fence_proxy_async_smem();
  if (warp == 1) {
    tmem_alloc(&tmem_slot, 64);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  // programmatic dependent launch: no global access before the previous
  // launch on the stream has completed; the chunk kernel may launch now
  pdl_wait();
  pdl_launch_dependents();

  if (warp == 0) {
    // producer: K_0, V_0, K_1, V_1, ...
    if (lane == 0) {
      for (int q = 0; q < 2 * T; ++q) {
        const int s = q % kStSlots, round = q / kStSlots;
        if (round > 0 && !mbar_wait(&empty[s], (round - 1) & 1, status)) break;
        mbar_arrive_expect_tx(&full[s], kTile);
        tma_load_3d(slots + s * kTile, (q & 1) ? &tm_v : &tm_k, &full[s], 0, (tile0 + q / 2) * kTileTokens, bh);
      }
    }
  } else if (warp == 1) {
    // S'^T (128 x 64) += [V | ones]^T phi(K): A MN-major (atoms V, ones), B MN-major
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, kD, 1, 1);
      const uint32_t ones_a = smem_u32(ones);
      for (int t = 0; t < T; ++t) {
        const int qk = 2 * t, qv = qk + 1, sk = qk % kStSlots, sv = qv % kStSlots;
        if (!mbar_wait(&ready[sk], (qk / kStSlots) & 1, status) ||
            !mbar_wait(&ready[sv], (qv / kStSlots) & 1, status))
          break;
        tc_fence_after();
        const uint32_t ka = smem_u32(slots + sk * kTile), va = smem_u32(slots + sv * kTile);
        const uint64_t a = smem_desc_sw128(va, ones_a - va, 1024), bk = smem_desc_sw128(ka, kTile, 1024);
        if (t == 0)
          umma_ss<0>(tmem, a, bk, idesc);
        else
          umma_ss<1>(tmem, a, bk, idesc);
#pragma unroll
        for (int k = 1; k < kTileTokens / 16; ++k)
          umma_ss<1>(tmem, desc_add(a, 2048 * k), desc_add(bk, 2048 * k), idesc);
        umma_commit(&empty[sk]);
        umma_commit(&empty[sv]);
      }
      umma_commit(&accfull);
    }
  } else {
    // phi on K, V passes through; then the readout of the state
    const int pt = threadIdx.x - 64;
    bool ok = true;
    for (int q = 0; q < 2 * T; ++q) {
      const int s = q % kStSlots;
      if (!warp_wait(&full[s], (q / kStSlots) & 1, status)) {
        ok = false;
        break;
      }
      if (!(q & 1)) {
        phi_tile<FMAP>(slots + s * kTile, pt, kTileTokens);
        fence_proxy_async_smem();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&ready[s]);
    }
    // warps 2..5 cover the four lane quarters of tensor memory
    if (ok && warp < 6 && warp_wait(&accfull, 0, status)) {
      tc_fence_after();
      const int qd = warp & 3, row = 32 * qd + lane;   // TMEM lane = row of S'^T
      float* dst = state + (static_cast<size_t>(bh) * nseg + seg) * kStateFloats + row * kD;
#pragma unroll 1
      for (int c0 = 0; c0 < kD; c0 += 32) {
        float v[32];
        tmem_ld32(tmem + (static_cast<uint32_t>(32 * qd) << 16) + c0, v);
        tmem_wait_ld();
        if (row < kStateRows) {
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            *reinterpret_cast<float4*>(dst + c0 + e) = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, 64);
}

// ====================================================== kernel 2: the chunks

// Shared memory: rings of Q, K and V tiles, state images (two of 10 KB), the
// ones atom.  phi(Q) goes straight to tensor memory, so a Q tile is free once
// phi has read it; a chunk's output is staged in its K tile, free once both
// MMAs that read phi(K) are done.
constexpr int kRQ = 3, kRK = 4, kRV = 4;
constexpr uint32_t kOffK = kRQ * kTile;
constexpr uint32_t kOffV = kOffK + kRK * kTile;
constexpr uint32_t kOffImg = kOffV + kRV * kTile;
constexpr uint32_t kOffOnes = kOffImg + 2 * kImgBytes;
constexpr uint32_t kChSmem = kOffOnes + kTile + 1024;
// Tensor-memory columns, two buffers each.  P (fp32, 128 columns) becomes, in
// place, masked P (bf16, columns 0..63); O then takes columns 64..143.
__device__ __forceinline__ constexpr uint32_t col_p(int b) { return 160u * b; }
__device__ __forceinline__ constexpr uint32_t col_q(int b) { return 320u + 32u * b; }   // phi(Q), bf16: 32 columns
constexpr uint32_t kColD = 384;             // increment [V | 1]^T phi(K): 64 columns
constexpr int kChThreads = 64 + 32 * kPhiWarps + 256;   // producer, MMA, phi, 4 P + output, 4 state warps

template <int FMAP>
__global__ void __launch_bounds__(kChThreads, 1)
    causal_chunk_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_out,
                        const float* __restrict__ state, int* status, int N, int tiles, int tps, int nseg,
                        float eps) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t qfull[kRQ], qempty[kRQ], kfull[kRK], kready[kRK], kempty[kRK];
  __shared__ __align__(8) uint64_t vfull[kRV], vempty[kRV];
  __shared__ __align__(8) uint64_t qready[2], qfree[2], pfull[2], pmready[2], ofull[2], oempty[2];
  __shared__ __align__(8) uint64_t imgready[2], imgfree[2], dfull, dfree;
  __shared__ uint32_t tmem_slot;
  __shared__ int flag_p, flag_s;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int seg = blockIdx.x, bh = blockIdx.y;
  const int tile0 = seg * tps;
  const int C = min(tiles, tile0 + tps) - tile0;   // chunks of this segment, >= 1
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* img = smem + kOffImg;
  uint8_t* ones = smem + kOffOnes;   // above every V tile: a positive atom stride
  auto q_tile = [&](int c) { return smem + (c % kRQ) * kTile; };
  auto k_tile = [&](int c) { return smem + kOffK + (c % kRK) * kTile; };
  auto v_tile = [&](int c) { return smem + kOffV + (c % kRV) * kTile; };

  if (threadIdx.x == 0) {
    for (int i = 0; i < kRQ; ++i) {
      mbar_init(&qfull[i], 1);
      mbar_init(&qempty[i], kPhiWarps);
    }
    for (int i = 0; i < kRK; ++i) {
      mbar_init(&kfull[i], 1);
      mbar_init(&kready[i], kPhiWarps);
      mbar_init(&kempty[i], 1);
    }
    for (int i = 0; i < kRV; ++i) {
      mbar_init(&vfull[i], 1);
      mbar_init(&vempty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&qready[i], kPhiWarps);
      mbar_init(&qfree[i], 1);
      mbar_init(&pfull[i], 1);
      mbar_init(&pmready[i], 4);
      mbar_init(&ofull[i], 1);
      mbar_init(&oempty[i], 4);
      mbar_init(&imgready[i], 4);
      mbar_init(&imgfree[i], 1);
    }
    mbar_init(&dfull, 1);
    mbar_init(&dfree, 4);
    fence_mbarrier_init();
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    prefetch_tmap(&tm_out);
    flag_p = flag_s = 0;
  }
  fill_ones_atom(ones);
  // image rows 65..79 are the MMA's zero padding, in both buffers
  constexpr int kPadChunks = (kImgRows - kStateRows) * 8;
  for (int i = threadIdx.x; i < 2 * kPadChunks; i += blockDim.x) {
    const int b = i / kPadChunks, rem = i % kPadChunks;
    *reinterpret_cast<uint4*>(img + b * kImgBytes + (kStateRows + rem / 8) * 128 + (rem % 8) * 16) =
        make_uint4(0u, 0u, 0u, 0u);
  }
  fence_proxy_async_smem();
  if (warp == 1) {
    tmem_alloc(&tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  // the segment states come from the previous launch: wait for it before any
  // global access; the next launch may begin its set-up
  pdl_wait();
  pdl_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      for (int c = 0; c < C; ++c) {
        const int row = (tile0 + c) * kTileTokens;
        if (c >= kRQ && !mbar_wait(&qempty[c % kRQ], ((c / kRQ) - 1) & 1, status)) break;
        mbar_arrive_expect_tx(&qfull[c % kRQ], kTile);
        tma_load_3d(q_tile(c), &tm_q, &qfull[c % kRQ], 0, row, bh);
        if (c >= kRK && !mbar_wait(&kempty[c % kRK], ((c / kRK) - 1) & 1, status)) break;
        mbar_arrive_expect_tx(&kfull[c % kRK], kTile);
        tma_load_3d(k_tile(c), &tm_k, &kfull[c % kRK], 0, row, bh);
        if (c >= kRV && !mbar_wait(&vempty[c % kRV], ((c / kRV) - 1) & 1, status)) break;
        mbar_arrive_expect_tx(&vfull[c % kRV], kTile);
        tma_load_3d(v_tile(c), &tm_v, &vfull[c % kRV], 0, row, bh);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t id_p = idesc_bf16_f32(128, 128, 0, 0);        // phi(Q) phi(K)^T
      constexpr uint32_t id_o = idesc_bf16_f32(128, kImgRows, 0, 0);   // phi(Q) [S | z | 0]
      constexpr uint32_t id_pv = idesc_bf16_f32(128, kImgRows, 0, 1);  // Pm [V | 1]
      constexpr uint32_t id_d = idesc_bf16_f32(128, kD, 1, 1);         // [V | 1]^T phi(K)
      const uint32_t ones_a = smem_u32(ones);
      auto kmajor = [&](const uint8_t* p) { return smem_desc_sw128(smem_u32(p), 16, 1024); };
      // [V | ones] as an MN-major operand: the ones atom is the second atom
      auto v_ones = [&](const uint8_t* p) { return smem_desc_sw128(smem_u32(p), ones_a - smem_u32(p), 1024); };
      // inputs of P for chunk c: phi(Q_c), phi(K_c), and buffer b read out by the epilogue of c - 2
      auto p_inputs = [&](int c, bool block) -> bool {
        const int b = c & 1, r2 = c >> 1;
        const uint32_t pq = r2 & 1, pk = (c / kRK) & 1, po = (r2 - 1) & 1;
        if (!block)
          return mbar_test(&qready[b], pq) && mbar_test(&kready[c % kRK], pk) && (r2 == 0 || mbar_test(&oempty[b], po));
        return mbar_wait(&qready[b], pq, status) && mbar_wait(&kready[c % kRK], pk, status) &&
               (r2 == 0 || mbar_wait(&oempty[b], po, status));
      };
      // (1) P_b = phi(Q_c) phi(K_c)^T
      auto issue_p = [&](int c) {
        const int b = c & 1;
        tc_fence_after();
        const uint64_t bk = kmajor(k_tile(c));
        const uint32_t d = tmem + col_p(b), a = tmem + col_q(b);
        umma_ts<0>(d, a, bk, id_p);
#pragma unroll
        for (int k = 1; k < kD / 16; ++k) umma_ts<1>(d, a + 8 * k, desc_add(bk, 32 * k), id_p);
        umma_commit(&pfull[b]);
      };
      // (3) the increment [V_c | 1]^T phi(K_c) for the next chunk's state
      auto issue_d = [&](int c) -> bool {
        if (!mbar_wait(&vfull[c % kRV], (c / kRV) & 1, status) || (c > 0 && !mbar_wait(&dfree, (c - 1) & 1, status)))
          return false;
        tc_fence_after();
        const uint64_t a = v_ones(v_tile(c)), bk = smem_desc_sw128(smem_u32(k_tile(c)), kTile, 1024);
        umma_ss<0>(tmem + kColD, a, bk, id_d);
#pragma unroll
        for (int k = 1; k < kTileTokens / 16; ++k)
          umma_ss<1>(tmem + kColD, desc_add(a, 2048 * k), desc_add(bk, 2048 * k), id_d);
        umma_commit(&dfull);
        return true;
      };
      // (2) O_b = phi(Q_c) [S_c | z_c | 0] + Pm_b [V_c | 1], columns 64.. of buffer b
      auto issue_o = [&](int c) -> bool {
        const int b = c & 1, r2 = c >> 1;
        if (!mbar_wait(&vfull[c % kRV], (c / kRV) & 1, status) || !mbar_wait(&pmready[b], r2 & 1, status) ||
            !mbar_wait(&imgready[b], r2 & 1, status))
          return false;
        tc_fence_after();
        const uint32_t d = tmem + col_p(b) + 64, aq = tmem + col_q(b), pm = tmem + col_p(b);
        const uint64_t bi = kmajor(img + b * kImgBytes), bv = v_ones(v_tile(c));
        umma_ts<0>(d, aq, bi, id_o);
#pragma unroll
        for (int k = 1; k < kD / 16; ++k) umma_ts<1>(d, aq + 8 * k, desc_add(bi, 32 * k), id_o);
#pragma unroll
        for (int k = 0; k < kTileTokens / 16; ++k) umma_ts<1>(d, pm + 8 * k, desc_add(bv, 2048 * k), id_pv);
        umma_commit(&qfree[b]);
        umma_commit(&imgfree[b]);
        umma_commit(&vempty[c % kRV]);
        umma_commit(&ofull[b]);   // last: its arrival implies every MMA of the CTA so far is done
        return true;
      };
      bool ok = p_inputs(0, true);
      if (ok) issue_p(0);
      for (int c = 0; c < C && ok; ++c) {
        const bool more = c + 1 < C;
        if (more && !issue_d(c)) break;
        // P of chunk c + 1 ahead of the output MMAs of chunk c when its inputs are there already
        bool early = false;
        if (more && p_inputs(c + 1, false)) {
          issue_p(c + 1);
          early = true;
        }
        if (!issue_o(c)) break;
        if (more && !early) {
          if (!p_inputs(c + 1, true)) break;
          issue_p(c + 1);
        }
      }
    }
  } else if (warp < 2 + kPhiWarps) {
    // -------- phi: Q rows into tensor memory, K in place; V needs nothing
    // Two warps per lane quarter: Q row i = tensor-memory lane, each warp one
    // half of the 64 features.
    const int qd = warp & 3, half = (warp - 2) >> 2, i = 32 * qd + lane;
    const int pt = threadIdx.x - 64;
    const uint32_t lanes = static_cast<uint32_t>(32 * qd) << 16;
    for (int c = 0; c < C; ++c) {
      const int b = c & 1, r2 = c >> 1;
      if (!warp_wait(&qfull[c % kRQ], (c / kRQ) & 1, status)) break;
      if (r2 > 0 && !warp_wait(&qfree[b], (r2 - 1) & 1, status)) break;
      {
        const uint8_t* src = q_tile(c) + i * 128;
        uint4 x[4];
#pragma unroll
        for (int m = 0; m < 4; ++m) x[m] = *reinterpret_cast<const uint4*>(src + (((4 * half + m) ^ (i & 7)) << 4));
        uint32_t w[16];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const uint4 y = phi_chunk<FMAP>(x[m]);
          w[4 * m] = y.x; w[4 * m + 1] = y.y; w[4 * m + 2] = y.z; w[4 * m + 3] = y.w;
        }
        tc_fence_after();
        tmem_st16(tmem + col_q(b) + 16 * half + lanes, w);
        tmem_wait_st();
        tc_fence_before();
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&qempty[c % kRQ]);
        mbar_arrive(&qready[b]);
      }
      if (!warp_wait(&kfull[c % kRK], (c / kRK) & 1, status)) break;
      // key rows past the sequence end must reach neither P nor the state
      phi_tile<FMAP>(k_tile(c), pt, min(kTileTokens, N - (tile0 + c) * kTileTokens));
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&kready[c % kRK]);
    }
  } else if (warp < 14) {
    // ---- P and output warps: masked P of chunk c, then the output of c - 1
    const int qd = warp & 3, i = 32 * qd + lane;
    const bool leader = threadIdx.x == 64 + 32 * kPhiWarps;
    const uint32_t lanes = static_cast<uint32_t>(32 * qd) << 16;
    int prev = -1;   // K ring slot whose store is still reading it
    for (int c = 0; c <= C; ++c) {
      if (c < C) {
        // mask j > i, masked P back to tensor memory as bf16
        const int b = c & 1, r2 = c >> 1;
        if (leader && !mbar_wait(&pfull[b], r2 & 1, status)) flag_p = 1;
        named_bar_sync(1, 128);
        if (flag_p) break;
        tc_fence_after();
        const uint32_t pcol = tmem + col_p(b) + lanes;
        // block j0 (32 keys) is read from columns j0.. and written, packed, to
        // columns j0 / 2..: always columns of blocks already read
#pragma unroll 1
        for (int j0 = 0; j0 < 128; j0 += 32) {
          uint32_t w[16];
          if (j0 > 32 * qd) {   // wholly above the diagonal for this warp's rows
#pragma unroll
            for (int e = 0; e < 16; ++e) w[e] = 0u;
          } else {
            float v[32];
            tmem_ld32(pcol + j0, v);
            tmem_wait_ld();
            if (j0 == 32 * qd) {   // the diagonal block: keys j <= i only
#pragma unroll
              for (int e = 0; e < 32; ++e) v[e] = (j0 + e <= i) ? v[e] : 0.f;
            }
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * e], v[2 * e + 1]);
              w[e] = *reinterpret_cast<uint32_t*>(&h);
            }
          }
          tmem_st16(pcol + j0 / 2, w);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&pmready[b]);
      }
      if (c > 0) {
        // output of chunk e = c - 1
        const int e = c - 1, b = e & 1, r2 = e >> 1;
        if (leader && !mbar_wait(&ofull[b], r2 & 1, status)) flag_p = 1;
        named_bar_sync(1, 128);
        if (flag_p) break;
        tc_fence_after();
        const uint32_t trow = tmem + col_p(b) + 64 + lanes;
        float v[2][32];
        tmem_ld32(trow, v[0]);
        tmem_ld32(trow + 32, v[1]);
        const float den = tmem_ld1(trow + kD);   // phi(q_i) . z_e + sum_j Pm_ij
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&oempty[b]);
        const float inv = 1.0f / (den + eps);
        uint8_t* ob = k_tile(e);   // every MMA reading this K tile is done
#pragma unroll
        for (int h = 0; h < 2; ++h) {
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) {
            uint32_t w[4];
#pragma unroll
            for (int t = 0; t < 4; ++t) {
              __nv_bfloat162 hv = __floats2bfloat162_rn(v[h][8 * jj + 2 * t] * inv, v[h][8 * jj + 2 * t + 1] * inv);
              w[t] = *reinterpret_cast<uint32_t*>(&hv);
            }
            *reinterpret_cast<uint4*>(ob + swz_off(i, 4 * h + jj)) = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
        fence_proxy_async_smem();
        named_bar_sync(1, 128);
        if (leader) {
          tma_store_3d(&tm_out, ob, 0, (tile0 + e) * kTileTokens, bh);
          bulk_commit_group();
          if (prev >= 0) {   // the previous chunk's store has read its K tile: hand it back
            bulk_wait_group_read<1>();
            mbar_arrive(&kempty[prev]);
          }
        }
        prev = e % kRK;
      }
    }
    if (leader) bulk_wait_group<0>();
  } else {
    // ------------- state warps: running S'^T row n in registers -> image
    const int qd = warp & 3, n = 32 * qd + lane;   // TMEM lane = row of S'^T
    const bool leader = threadIdx.x == 64 + 32 * kPhiWarps + 128;
    const uint32_t trow = tmem + kColD + (static_cast<uint32_t>(32 * qd) << 16);
    float S[kD];
    // starting state: the sum of the earlier segments' states, ascending
#pragma unroll
    for (int e = 0; e < kD; ++e) S[e] = 0.f;
    if (n < kStateRows) {
      for (int s = 0; s < seg; ++s) {
        const float* src = state + (static_cast<size_t>(bh) * nseg + s) * kStateFloats + n * kD;
#pragma unroll
        for (int e = 0; e < kD; e += 4) {
          const float4 x = *reinterpret_cast<const float4*>(src + e);
          S[e] += x.x; S[e + 1] += x.y; S[e + 2] += x.z; S[e + 3] += x.w;
        }
      }
    }
    for (int c = 0; c < C; ++c) {
      const int b = c & 1, r2 = c >> 1;
      if (leader) {
        if ((c > 0 && !mbar_wait(&dfull, (c - 1) & 1, status)) ||
            (r2 > 0 && !mbar_wait(&imgfree[b], (r2 - 1) & 1, status)))
          flag_s = 1;
      }
      named_bar_sync(2, 128);
      if (flag_s) break;
      if (c > 0) {
        tc_fence_after();
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          float v[32];
          tmem_ld32(trow + 32 * h, v);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) S[32 * h + e] += v[e];
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&dfree);
      }
      if (n < kStateRows) {
        uint8_t* dst = img + b * kImgBytes + n * 128;
#pragma unroll
        for (int c8 = 0; c8 < kD / 8; ++c8) {
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            __nv_bfloat162 h = __floats2bfloat162_rn(S[8 * c8 + 2 * e], S[8 * c8 + 2 * e + 1]);
            w[e] = *reinterpret_cast<uint32_t*>(&h);
          }
          *reinterpret_cast<uint4*>(dst + ((c8 ^ (n & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&imgready[b]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

template <int FMAP>
cudaError_t run(const LaunchArgs& a) {
  const Plan& p = *a.p;
  float* state = reinterpret_cast<float*>(a.ws + p.off_partial);
  int* status = reinterpret_cast<int*>(a.ws + p.off_status);
  const unsigned bh = static_cast<unsigned>(p.BH);
  cudaError_t err;
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.stream = a.stream;
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  if (p.splits > 1) {
    auto kern = causal_state_kernel<FMAP>;
    if ((err = ensure_smem_attr(reinterpret_cast<const void*>(kern), kStSmem)) != cudaSuccess) return err;
    cfg.gridDim = dim3(p.splits - 1, bh);
    cfg.blockDim = dim3(kStThreads);
    cfg.dynamicSmemBytes = kStSmem;
    if ((err = cudaLaunchKernelEx(&cfg, kern, *a.tm_k, *a.tm_v, state, status, p.tiles_per_split, p.splits)) !=
        cudaSuccess)
      return err;
  }
  auto kern = causal_chunk_kernel<FMAP>;
  if ((err = ensure_smem_attr(reinterpret_cast<const void*>(kern), kChSmem)) != cudaSuccess) return err;
  cfg.gridDim = dim3(p.splits, bh);
  cfg.blockDim = dim3(kChThreads);
  cfg.dynamicSmemBytes = kChSmem;
  return cudaLaunchKernelEx(&cfg, kern, *a.tm_q, *a.tm_k, *a.tm_v, *a.tm_out, static_cast<const float*>(state),
                            status, p.N, p.tiles, p.tiles_per_split, p.splits, p.eps);
}

}  // namespace

cudaError_t launch_bf16_causal(const LaunchArgs& a) {
  const Plan& p = *a.p;
  if (p.F != 0 || p.D != kD) return cudaErrorNotSupported;
  return p.fmap == 0 ? run<0>(a) : run<1>(a);
}

}  // namespace la
