// bf16_landmark.cu -- the exact-softmax landmark branch of the TTR layer and
// its bounded blend with the kernel branch, bf16 storage, D = 128.
//
// Page "Flux2TTRTrainer", "How the distillation works": the student layer
// fuses a linear-time kernel branch with a small exact-softmax branch over
// "landmark" tokens, blended by a bounded weight.  Readings (the page gives
// neither the rule nor the form): L landmarks at tokens floor(l N / L);
// scores q_i . k_l / sqrt(D); out = a_h * softmax branch + (1 - a_h) * kernel
// branch with a_h = sigmoid(g_h) for a per-head logit g_h.
//
// One launch after the kernel branch has written `out`: every CTA serves a
// run of 128-query tiles of one head.  The landmark keys and values (L <= 128
// rows, zero-padded to a multiple of 16) are gathered once per CTA into
// shared memory in the layout a TMA tile has (row = landmark, 128-byte
// swizzle): the B operand of  S = Q K_L^T  (K-major) and of  O = P V_L
// (MN-major).  Per tile: TMA brings the Q tile and the kernel branch's output
// tile; one thread issues the S MMA (tensor memory, fp32); eight warps turn
// each row of S into softmax weights (row max, exp2, rounded to bf16, summed)
// and write them back into the same tensor-memory columns as the A operand of
// the O MMA; the same warps read O, divide by the weight sum, blend with the
// kernel branch's row in shared memory and TMA-store the tile.  Two such
// groups of eight warps (two per row, one half of the columns each) take
// alternate tiles, each with its own tensor memory (S/P 128 columns, O 128
// columns), so one group's softmax overlaps the other's loads and MMAs.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "bf16_common.cuh"
#include "la_internal.h"
#include "sm100.cuh"

namespace la {
namespace {

constexpr int kD = 128;
constexpr int kMaxLandmarks = 128;
constexpr uint32_t kTileBytes = 128u * kD * 2u;                  // one 128-row bf16 tile
constexpr uint32_t kLmBytes = kMaxLandmarks * kD * 2u;           // landmark keys (or values)
constexpr uint32_t kSmemBytes = 2 * kLmBytes + 4 * kTileBytes + 1024;
constexpr int kThreads = 32 * 18;                                // producer, MMA, 2 x 8 softmax warps
constexpr uint32_t kTmemCols = 512;                              // per group: S/P 128, O 128

__global__ void __launch_bounds__(kThreads, 1)
    landmark_blend_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_out,
                          const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
                          const float* __restrict__ gate, int* status, int H, int N, int tiles, int L) {
  extern __shared__ uint8_t smem_raw[];
  // qfull / ofull: a Q tile / a kernel-branch output tile has arrived in slot
  // s; qempty: the S MMA has read the Q tile.  Group g (tiles u with
  // u % 2 == g) owns slot g; it reloads its output slot itself once the store
  // of its previous tile has read it.
  __shared__ __align__(8) uint64_t qfull[2], ofull[2], qempty[2];
  // sfull: S in tensor memory; pready: the weights P written over S;
  // ofull_acc: O in tensor memory; tfree: the group has read O (its tensor
  // memory may take the tile after next).
  __shared__ __align__(8) uint64_t sfull[2], pready[2], ofull_acc[2], tfree[2];
  // lm_ready: the landmark keys and values are in shared memory
  __shared__ __align__(8) uint64_t lm_ready;
  __shared__ uint32_t tmem_slot;
  // per group and column half: each row's partial max and weight sum
  __shared__ float row_max[2][2][128], row_sum[2][2][128];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.y;
  const int G = static_cast<int>(gridDim.x);
  const int tile0 = static_cast<int>(blockIdx.x) * tiles / G;
  const int T = (static_cast<int>(blockIdx.x) + 1) * tiles / G - tile0;
  const int Lp = (L + 15) & ~15;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* kl = smem;                      // [Lp x 128] landmark keys, two 64-feature atoms of Lp rows
  uint8_t* vl = kl + kLmBytes;             // [Lp x 128] landmark values, same layout
  uint8_t* qs = vl + kLmBytes;             // two Q slots
  uint8_t* os = qs + 2 * kTileBytes;       // two output slots
  const uint32_t lm_atom = static_cast<uint32_t>(Lp) * 128u;   // bytes of one 64-column atom
  auto lm_off = [&](int l, int c) {        // row l, 16-byte chunk c (0..15)
    return static_cast<uint32_t>((c >> 3) * lm_atom + l * 128 + (((c & 7) ^ (l & 7)) << 4));
  };

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&qfull[i], 1);
      mbar_init(&ofull[i], 1);
      mbar_init(&qempty[i], 1);
      mbar_init(&sfull[i], 1);
      mbar_init(&pready[i], 8);
      mbar_init(&ofull_acc[i], 1);
      mbar_init(&tfree[i], 8);
    }
    mbar_init(&lm_ready, 16);
    fence_mbarrier_init();
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_out);
  }
  if (warp == 1) {
    tmem_alloc(&tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  // The kernel branch (the previous launch on the stream) wrote `out`: wait for
  // it before any global access.
  pdl_wait();
  pdl_launch_dependents();

  if (warp == 0) {
    // -------------------------------------------------------- producer
    if (lane == 0) {
      for (int u = 0; u < T; ++u) {
        const int s = u & 1;
        if (u >= 2 && !mbar_wait(&qempty[s], ((u >> 1) - 1) & 1, status)) break;
        const int row = (tile0 + u) * kTileTokens;
        mbar_arrive_expect_tx(&qfull[s], kTileBytes);
        tma_load_3d(qs + s * kTileBytes, &tm_q, &qfull[s], 0, row, bh);
        tma_load_3d(qs + s * kTileBytes + kBoxBytes, &tm_q, &qfull[s], 64, row, bh);
      }
    }
  } else if (warp == 1) {
    // -------------------------------------------------- MMA issuers
    // Lane 0 issues the S MMAs, lane 1 the O MMAs, each tracking (commit) its
    // own: an O MMA waits only for its tile's weights, never behind the next
    // tile's S MMA and what that one waits for.
    const uint32_t idesc_s = idesc_bf16_f32(128, Lp, 0, 0);       // A = Q (K-major), B = K_L (K-major)
    constexpr uint32_t idesc_o = idesc_bf16_f32(128, kD, 0, 1);   // A = P (tensor memory), B = V_L (MN-major)
    if (lane == 0) {
      const uint64_t kdesc = smem_desc_sw128(smem_u32(kl), 16, 1024);
      bool ok = mbar_wait(&lm_ready, 0, status);
      for (int u = 0; u < T && ok; ++u) {
        const int g = u & 1;
        if (!mbar_wait(&qfull[g], (u >> 1) & 1, status) ||
            (u >= 2 && !mbar_wait(&tfree[g], ((u >> 1) - 1) & 1, status)))
          break;
        tc_fence_after();
        const uint64_t qdesc = smem_desc_sw128(smem_u32(qs + g * kTileBytes), 16, 1024);
        const uint32_t sacc = tmem + g * 256;
        umma_ss<0>(sacc, qdesc, kdesc, idesc_s);
#pragma unroll
        for (int kk = 1; kk < kD / 16; ++kk)
          umma_ss<1>(sacc, desc_add(qdesc, (kk >> 2) * kBoxBytes + (kk & 3) * 32),
                     desc_add(kdesc, (kk >> 2) * lm_atom + (kk & 3) * 32), idesc_s);
        umma_commit(&qempty[g]);
        umma_commit(&sfull[g]);
      }
    } else if (lane == 1) {
      const uint64_t vdesc = smem_desc_sw128(smem_u32(vl), lm_atom, 1024);
      for (int u = 0; u < T; ++u) {
        const int g = u & 1;
        if (!mbar_wait(&pready[g], (u >> 1) & 1, status)) break;
        tc_fence_after();
        const uint32_t p = tmem + g * 256, o = tmem + g * 256 + 128;
        // P: landmarks 0..63 at columns 0..31, 64..127 at columns 64..95
        umma_ts<0>(o, p, vdesc, idesc_o);
        for (int kk = 1; kk < Lp / 16; ++kk)
          umma_ts<1>(o, p + 8 * kk + (kk >= 4 ? 32 : 0), desc_add(vdesc, 2048 * kk), idesc_o);
        umma_commit(&ofull_acc[g]);
      }
    }
  } else {
    // Gather the landmark rows of this head (token floor(l N / L)) while the
    // first tiles load; rows L..Lp-1 are zero, so their scores are masked
    // below and their values add nothing.
    {
      // 512 threads, 2048 16-byte chunks of each at most: all of a thread's
      // loads are issued before its stores, so they overlap
      const size_t head = static_cast<size_t>(bh) * N * kD;
      constexpr int kPer = kMaxLandmarks * 16 / (kThreads - 64);
      uint4 kk[kPer], vv[kPer];
#pragma unroll
      for (int j = 0; j < kPer; ++j) {
        const int i = threadIdx.x - 64 + j * (kThreads - 64), l = i >> 4, c = i & 15;
        kk[j] = vv[j] = make_uint4(0u, 0u, 0u, 0u);
        if (l < L) {
          const size_t row = head + static_cast<size_t>((static_cast<long long>(l) * N) / L) * kD + c * 8;
          kk[j] = *reinterpret_cast<const uint4*>(k + row);
          vv[j] = *reinterpret_cast<const uint4*>(v + row);
        }
      }
#pragma unroll
      for (int j = 0; j < kPer; ++j) {
        const int i = threadIdx.x - 64 + j * (kThreads - 64), l = i >> 4, c = i & 15;
        if (l < Lp) {
          *reinterpret_cast<uint4*>(kl + lm_off(l, c)) = kk[j];
          *reinterpret_cast<uint4*>(vl + lm_off(l, c)) = vv[j];
        }
      }
      fence_proxy_async_smem();   // read by the tensor core
      __syncwarp();
      if (lane == 0) mbar_arrive(&lm_ready);
    }
    // -------------------------------------- softmax, blend and store
    // Group g (warps 2 + 8 g .. 9 + 8 g) takes tiles u with u % 2 == g; two
    // warps per tensor-memory lane quarter, each one half of a row's columns.
    const int g = (warp - 2) >> 3;
    const int ch = ((warp - 2) >> 2) & 1;  // column half
    const int q4 = warp & 3;               // tensor-memory lane quarter
    const int r = 32 * q4 + lane;          // row of the tile
    const bool leader = warp == 2 + 8 * g && lane == 0;   // lane 0 of the group's first warp
    const uint32_t lanes = static_cast<uint32_t>(32 * q4) << 16;
    const float a = 1.0f / (1.0f + expf(-gate[bh % H]));
    auto load_out = [&](int u) {   // the kernel branch's output tile u into slot g
      const int row = (tile0 + u) * kTileTokens;
      mbar_arrive_expect_tx(&ofull[g], kTileBytes);
      tma_load_3d(os + g * kTileBytes, &tm_out, &ofull[g], 0, row, bh);
      tma_load_3d(os + g * kTileBytes + kBoxBytes, &tm_out, &ofull[g], 64, row, bh);
    };
    if (leader && g < T) load_out(g);
    const float sl2 = 1.4426950408889634f / sqrtf(static_cast<float>(kD));   // log2(e) / sqrt(D)
    const int c_lo = 64 * ch;              // this warp's score columns c_lo .. c_lo + 63
    for (int u = g; u < T; u += 2) {
      const int it = u >> 1;
      if (!warp_wait(&sfull[g], it & 1, status)) break;
      tc_fence_after();
      const uint32_t srow = tmem + g * 256 + lanes;
      // Softmax of the row, columns from L on masked: each warp the maximum of
      // its half, exchanged; then its weights exp((s - m) / sqrt(D)) rounded
      // to bf16 and their sum, exchanged before the blend (the sum is over the
      // rounded weights, so numerator and denominator see the same ones).
      // The weights go over this warp's own scores, two per column: landmarks
      // 0..63 at columns 0..31, 64..127 at columns 64..95.
      float m = -INFINITY;
#pragma unroll
      for (int h0 = 0; h0 < 64; h0 += 32) {
        float x[32];
        tmem_ld32(srow + c_lo + h0, x);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e)
          if (c_lo + h0 + e < L) m = fmaxf(m, x[e]);
      }
      row_max[g][ch][r] = m;
      named_bar_sync(1 + g, 256);
      m = fmaxf(m, row_max[g][ch ^ 1][r]);
      float sum = 0.f;
#pragma unroll
      for (int h0 = 0; h0 < 64; h0 += 32) {
        float x[32];
        tmem_ld32(srow + c_lo + h0, x);
        tmem_wait_ld();
        uint32_t w[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int c = c_lo + h0 + 2 * e;
          const float p0 = c < L ? ex2_approx((x[2 * e] - m) * sl2) : 0.f;
          const float p1 = c + 1 < L ? ex2_approx((x[2 * e + 1] - m) * sl2) : 0.f;
          const __nv_bfloat162 b = __floats2bfloat162_rn(p0, p1);
          const float2 f = __bfloat1622float2(b);
          sum += f.x + f.y;
          w[e] = *reinterpret_cast<const uint32_t*>(&b);
        }
        tmem_st16(srow + c_lo + h0 / 2, w);
      }
      row_sum[g][ch][r] = sum;
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&pready[g]);
      // O, then the blend with the kernel branch's row: this warp's half of
      // the value columns, 32 at a time, each run blended into 4 chunks
      if (!warp_wait(&ofull_acc[g], it & 1, status) || !warp_wait(&ofull[g], it & 1, status)) break;
      tc_fence_after();
      named_bar_sync(1 + g, 256);          // both halves' sums are written
      sum += row_sum[g][ch ^ 1][r];
      const float scale = a / sum;
      uint8_t* ob = os + g * kTileBytes;
#pragma unroll 1
      for (int c0 = 64 * ch; c0 < 64 * ch + 64; c0 += 32) {
        float o[32];
        tmem_ld32(tmem + g * 256 + 128 + lanes + c0, o);
        tmem_wait_ld();
        if (c0 == 64 * ch + 32) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tfree[g]);   // S/P and O of this group are read
        }
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          uint4* p = reinterpret_cast<uint4*>(ob + swz_off(r, c0 / 8 + cc));
          const uint4 kb = *p;
          const uint32_t kw[4] = {kb.x, kb.y, kb.z, kb.w};
          uint32_t res[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 kf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&kw[e]));
            const float y0 = scale * o[8 * cc + 2 * e] + (1.0f - a) * kf.x;
            const float y1 = scale * o[8 * cc + 2 * e + 1] + (1.0f - a) * kf.y;
            const __nv_bfloat162 b = __floats2bfloat162_rn(y0, y1);
            res[e] = *reinterpret_cast<const uint32_t*>(&b);
          }
          *p = make_uint4(res[0], res[1], res[2], res[3]);
        }
      }
      fence_proxy_async_smem();
      named_bar_sync(1 + g, 256);
      if (leader) {
        const int row = (tile0 + u) * kTileTokens;
        tma_store_3d(&tm_out, ob, 0, row, bh);
        tma_store_3d(&tm_out, ob + kBoxBytes, 64, row, bh);
        bulk_commit_group();
        if (u + 2 < T) {
          bulk_wait_group_read<0>();   // the store has read the slot
          load_out(u + 2);
        }
      }
    }
    if (leader) bulk_wait_group<0>();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

cudaError_t launch_bf16_landmark(const LaunchArgs& a, const void* gate, int n_landmarks) {
  const Plan& p = *a.p;
  if (p.D != kD || n_landmarks < 1 || n_landmarks > kMaxLandmarks || n_landmarks > p.N) return cudaErrorNotSupported;
  auto kern = landmark_blend_kernel;
  cudaError_t err = ensure_smem_attr(reinterpret_cast<const void*>(kern), kSmemBytes);
  if (err != cudaSuccess) return err;
  const int tiles = p.tiles;
  long long per_head = std::max<long long>(1, p.num_sms / std::max<long long>(p.BH, 1));
  const int G = static_cast<int>(std::min<long long>(per_head, tiles));
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(G), static_cast<unsigned>(p.BH));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = a.stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int* status = reinterpret_cast<int*>(a.ws + p.off_status);
  return cudaLaunchKernelEx(&cfg, kern, *a.tm_q, *a.tm_out, static_cast<const __nv_bfloat16*>(a.k),
                            static_cast<const __nv_bfloat16*>(a.v), static_cast<const float*>(gate), status, p.H,
                            p.N, tiles, n_landmarks);
}

}  // namespace la
