// bf16_noncausal.cu -- tcgen05 tensor-core path for non-causal phi attention
// with bf16 storage and fp32 accumulation, F = 0 (phi acts on the D channels).
//
// Method (page "NNT Define Linear Attention", "How it works"): collapse the
// sequence into kv = phi(K)^T V and ksum = sum_j phi(k_j), then
// out_i = phi(q_i)^T kv / (phi(q_i) . ksum + eps).
//
// Three kernels, chained with programmatic dependent launch:
//   kv_partial  grid (S, B*H): TMA streams 128-token K/V tiles of one N-split
//               into shared memory, four warps apply phi to K in place and sum
//               ksum, one thread issues tcgen05.mma  kv += phi(K_tile)^T V_tile
//               into tensor memory; the fp32 partial is written to workspace.
//   kv_combine  grid (B*H, F/8): sums the S partials in ascending order (no
//               atomics, bitwise reproducible) and writes, per head, the bf16
//               image of [kv | ksum | 0] laid out as the MMA's B operand.
//   apply       persistent grid: per 128-query tile, TMA load, phi in place,
//               one MMA [num | den] = phi(Q) [kv | ksum], epilogue
//               out = num / (den + eps) rounded to bf16, TMA store.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "la_internal.h"
#include "sm100.cuh"

namespace la {
namespace {

constexpr uint32_t kBoxBytes = 128 * 128;   // one TMA box: 128 rows x 64 bf16 (128 B)

template <int D>
struct TileCfg {
  static constexpr int kBoxes = D / 64;
  static constexpr uint32_t kTileBytes = 128u * D * 2u;    // 128 tokens x D bf16
  static constexpr int kChunksPerRow = D / 8;               // 16-byte chunks per token row
  static constexpr int kThreadsPerChunk = 128 / kChunksPerRow;
  static constexpr int kRowsPerThread = 128 / kThreadsPerChunk;
};

// Byte offset of (row r, logical 16-byte chunk cc) inside a [128 x D] bf16 tile
// stored as D/64 TMA boxes with the 128-byte swizzle.
__device__ __forceinline__ uint32_t swz_off(int r, int cc) {
  return static_cast<uint32_t>((cc >> 3) * kBoxBytes + r * 128 + (((cc & 7) ^ (r & 7)) << 4));
}

// Apply phi to 8 bf16 values in place (one 16-byte chunk); returns the rounded
// values as floats in y[] so that sums use exactly what the MMA will read.
template <int FMAP>
__device__ __forceinline__ uint4 phi_chunk(uint4 x, float (&y)[8]) {
  uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162*>(&w[i]);
    float2 f = __bfloat1622float2(b);
    __nv_bfloat162 r = __floats2bfloat162_rn(phi_fast<FMAP>(f.x), phi_fast<FMAP>(f.y));
    float2 g = __bfloat1622float2(r);
    y[2 * i] = g.x;
    y[2 * i + 1] = g.y;
    w[i] = *reinterpret_cast<uint32_t*>(&r);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// Lane 0 waits on the barrier, the result is broadcast so the warp stays
// converged.  Returns false on timeout.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, int* status) {
  int ok = 1;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, status) ? 1 : 0;
  ok = __shfl_sync(0xffffffffu, ok, 0);
  __syncwarp();
  return ok != 0;
}

// =============================================================== kv_partial

template <int D>
struct PartialCfg : TileCfg<D> {
  static constexpr int kStages = D == 128 ? 3 : 4;
  static constexpr uint32_t kStageBytes = 2 * TileCfg<D>::kTileBytes;   // K then V
  static constexpr uint32_t kSmemBytes = kStages * kStageBytes + 1024;  // +1024 for alignment
  static constexpr uint32_t kTmemCols = D;                             // fp32 accumulator D x D
};

template <int D, int FMAP>
__global__ void __launch_bounds__(192, 1)
    kv_partial_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                      float* __restrict__ part, float* __restrict__ part_ksum, int* status, int N, int tiles,
                      int tiles_per_split, int S) {
  using C = PartialCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[C::kStages], phi_bar[C::kStages], empty_bar[C::kStages];
  __shared__ __align__(8) uint64_t acc_bar;
  __shared__ uint32_t tmem_slot;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int s = blockIdx.x;
  const int bh = blockIdx.y;
  const int tile0 = s * tiles_per_split;
  const int ntile = min(tiles, tile0 + tiles_per_split) - tile0;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  // Let the combine kernel's blocks get scheduled; they wait for this grid.
  pdl_launch_dependents();

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kStages; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&phi_bar[i], 4);
      mbar_init(&empty_bar[i], 1);
    }
    mbar_init(&acc_bar, 1);
    fence_mbarrier_init();
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
  }
  if (warp == 1) {
    tmem_alloc(&tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;

  if (warp == 0) {
    // ---------------------------------------------------------- TMA producer
    if (lane == 0) {
      for (int i = 0; i < ntile; ++i) {
        const int st = i % C::kStages, round = i / C::kStages;
        if (i >= C::kStages && !mbar_wait(&empty_bar[st], (round - 1) & 1, status)) break;
        uint8_t* ks = smem + st * C::kStageBytes;
        uint8_t* vs = ks + C::kTileBytes;
        mbar_arrive_expect_tx(&full_bar[st], C::kStageBytes);
        const int tok = (tile0 + i) * kTileTokens;
#pragma unroll
        for (int b = 0; b < C::kBoxes; ++b) tma_load_3d(ks + b * kBoxBytes, &tm_k, &full_bar[st], 64 * b, tok, bh);
#pragma unroll
        for (int b = 0; b < C::kBoxes; ++b) tma_load_3d(vs + b * kBoxBytes, &tm_v, &full_bar[st], 64 * b, tok, bh);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      // kv[f][n] += sum_t phi(K)[t][f] V[t][n]: A = phi(K)^T (M = D features,
      // MN-major), B = V (N = D, MN-major), K = 16 tokens per instruction.
      constexpr uint32_t idesc = idesc_bf16_f32(D, D, 1, 1);
      for (int i = 0; i < ntile; ++i) {
        const int st = i % C::kStages, round = i / C::kStages;
        if (!mbar_wait(&phi_bar[st], round & 1, status)) break;
        tc_fence_after();
        const uint32_t ka = smem_u32(smem + st * C::kStageBytes);
        const uint32_t va = ka + C::kTileBytes;
#pragma unroll
        for (int k = 0; k < kTileTokens / 16; ++k) {
          const uint64_t adesc = smem_desc_sw128(ka + k * 2048, kBoxBytes, 1024);
          const uint64_t bdesc = smem_desc_sw128(va + k * 2048, kBoxBytes, 1024);
          umma_bf16(tmem, adesc, bdesc, idesc, (i > 0 || k > 0) ? 1u : 0u);
        }
        umma_commit(&empty_bar[st]);
      }
      umma_commit(&acc_bar);
    }
  } else {
    // --------------------------------------------- phi on K, ksum, epilogue
    const int pt = threadIdx.x - 64;    // 0..127
    const int cc = pt / C::kThreadsPerChunk;
    const int r0 = pt % C::kThreadsPerChunk;
    float ks[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) ks[e] = 0.f;
    bool ok = true;
    for (int i = 0; i < ntile && ok; ++i) {
      const int st = i % C::kStages, round = i / C::kStages;
      if (!warp_wait(&full_bar[st], round & 1, status)) {
        ok = false;
        break;
      }
      uint8_t* kt = smem + st * C::kStageBytes;
      const int tok0 = (tile0 + i) * kTileTokens;
#pragma unroll 4
      for (int j = 0; j < C::kRowsPerThread; ++j) {
        const int r = r0 + j * C::kThreadsPerChunk;
        uint4* p = reinterpret_cast<uint4*>(kt + swz_off(r, cc));
        float y[8];
        uint4 x = phi_chunk<FMAP>(*p, y);
        if (tok0 + r >= N) {   // rows past the sequence end contribute nothing
          x = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
          for (int e = 0; e < 8; ++e) y[e] = 0.f;
        }
        *p = x;
#pragma unroll
        for (int e = 0; e < 8; ++e) ks[e] += y[e];
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&phi_bar[st]);
    }
    // ksum: reduce the threads that share chunk column cc (consecutive lanes).
#pragma unroll
    for (int o = 1; o < C::kThreadsPerChunk; o <<= 1)
#pragma unroll
      for (int e = 0; e < 8; ++e) ks[e] += __shfl_xor_sync(0xffffffffu, ks[e], o);
    float* ksd = part_ksum + (static_cast<size_t>(bh) * S + s) * D;
    if (r0 == 0) {
      reinterpret_cast<float4*>(ksd + cc * 8)[0] = make_float4(ks[0], ks[1], ks[2], ks[3]);
      reinterpret_cast<float4*>(ksd + cc * 8)[1] = make_float4(ks[4], ks[5], ks[6], ks[7]);
    }
    // Epilogue: TMEM lane = feature row (M = 128: row = lane; M = 64: rows
    // 16q..16q+15 sit in lanes 32q..32q+15).
    if (ok && warp_wait(&acc_bar, 0, status)) {
      tc_fence_after();
      const int q = warp & 3;
      const uint32_t trow = tmem + (static_cast<uint32_t>(32 * q) << 16);
      const bool valid = (D == 128) || lane < 16;
      const int f = (D == 128) ? 32 * q + lane : 16 * q + lane;
      float* dst = part + ((static_cast<size_t>(bh) * S + s) * D + f) * D;
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 32) {
        float v[32];
        tmem_ld32(trow + c0, v);
        tmem_wait_ld();
        if (valid) {
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            *reinterpret_cast<float4*>(dst + c0 + e) = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, C::kTmemCols);
}

// =============================================================== kv_combine

// Writes, for head bh and k-group g (features 8g..8g+7), the 128-byte-swizzled
// MN-major image of rows [kv[f][0..D) | ksum[f] | 0 ...] of the apply MMA's B
// operand.  One thread per 16-byte chunk.
__global__ void __launch_bounds__(256) kv_combine_kernel(const float* __restrict__ part,
                                                         const float* __restrict__ part_ksum,
                                                         uint8_t* __restrict__ blobs, int D, int Fe, int S,
                                                         size_t blob_bytes) {
  pdl_wait();
  pdl_launch_dependents();
  const int bh = blockIdx.x, g = blockIdx.y;
  const int atoms = blob_atoms(D);
  const int chunks_per_row = atoms * 8;
  const int t = threadIdx.x;
  if (t >= 8 * chunks_per_row) return;
  const int r = t / chunks_per_row, ch = t % chunks_per_row;
  const int a = ch >> 3, c = ch & 7;
  const int f = 8 * g + r;
  const int n0 = 64 * a + 8 * c;
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  if (n0 + 8 <= D) {
    for (int s = 0; s < S; ++s) {
      const float4* src =
          reinterpret_cast<const float4*>(part + ((static_cast<size_t>(bh) * S + s) * Fe + f) * D + n0);
      const float4 x0 = src[0], x1 = src[1];
      acc[0] += x0.x; acc[1] += x0.y; acc[2] += x0.z; acc[3] += x0.w;
      acc[4] += x1.x; acc[5] += x1.y; acc[6] += x1.z; acc[7] += x1.w;
    }
  } else if (n0 <= D && D < n0 + 8) {
    for (int s = 0; s < S; ++s) acc[D - n0] += part_ksum[(static_cast<size_t>(bh) * S + s) * Fe + f];
  }
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    __nv_bfloat162 b = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
    w[i] = *reinterpret_cast<uint32_t*>(&b);
  }
  uint8_t* dst = blobs + static_cast<size_t>(bh) * blob_bytes + static_cast<size_t>(a) * Fe * 128 + g * 1024 +
                 r * 128 + ((c ^ r) << 4);
  *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
}

// ==================================================================== apply

template <int D>
struct ApplyCfg : TileCfg<D> {
  static constexpr int kStages = D == 128 ? 3 : 4;
  static constexpr int kNB = D + 16;                       // MMA N: D value columns + den
  static constexpr uint32_t kAccCols = D == 128 ? 256 : 128;
  static constexpr uint32_t kTmemCols = 2 * kAccCols;
  static constexpr uint32_t kBlobBytes = blob_atoms(D) * D * 128;
  static constexpr uint32_t kSmemBytes = kStages * TileCfg<D>::kTileBytes + kBlobBytes +
                                         2 * TileCfg<D>::kTileBytes + 1024;
};

template <int D, int FMAP>
__global__ void __launch_bounds__(320, 1)
    apply_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_out,
                 const uint8_t* __restrict__ blobs, int* status, float eps, int tiles, long long total) {
  using C = ApplyCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t qfull[C::kStages], qphi[C::kStages], qempty[C::kStages];
  __shared__ __align__(8) uint64_t accfull[2], accempty[2], blobfull, blobempty;
  __shared__ uint32_t tmem_slot;
  __shared__ int ep_abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* qs = smem;
  uint8_t* blob = qs + C::kStages * C::kTileBytes;
  uint8_t* os = blob + C::kBlobBytes;

  const long long per = total / gridDim.x, rem = total % gridDim.x;
  const long long begin = blockIdx.x * per + min(static_cast<long long>(blockIdx.x), rem);
  const int count = static_cast<int>(per + (blockIdx.x < rem ? 1 : 0));

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kStages; ++i) {
      mbar_init(&qfull[i], 1);
      mbar_init(&qphi[i], 4);
      mbar_init(&qempty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&accfull[i], 1);
      mbar_init(&accempty[i], 4);
    }
    mbar_init(&blobfull, 1);
    mbar_init(&blobempty, 1);
    fence_mbarrier_init();
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_out);
    ep_abort = 0;
  }
  if (warp == 1) {
    tmem_alloc(&tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;

  if (warp == 0) {
    // ---------------------------------------------------------- TMA producer
    if (lane == 0) {
      pdl_wait();   // the state images come from the previous kernel
      long long cur = -1;
      int nblob = 0;
      for (int li = 0; li < count; ++li) {
        const long long item = begin + li;
        const int bh = static_cast<int>(item / tiles), tile = static_cast<int>(item % tiles);
        if (bh != cur) {
          if (nblob > 0 && !mbar_wait(&blobempty, (nblob - 1) & 1, status)) break;
          mbar_arrive_expect_tx(&blobfull, C::kBlobBytes);
          bulk_load(blob, blobs + static_cast<size_t>(bh) * C::kBlobBytes, C::kBlobBytes, &blobfull);
          cur = bh;
          ++nblob;
        }
        const int st = li % C::kStages, round = li / C::kStages;
        if (li >= C::kStages && !mbar_wait(&qempty[st], (round - 1) & 1, status)) break;
        mbar_arrive_expect_tx(&qfull[st], C::kTileBytes);
        uint8_t* dst = qs + st * C::kTileBytes;
#pragma unroll
        for (int b = 0; b < C::kBoxes; ++b)
          tma_load_3d(dst + b * kBoxBytes, &tm_q, &qfull[st], 64 * b, tile * kTileTokens, bh);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      // [num | den] (128 x (D+16)) = phi(Q) (128 x D, K-major) x [kv | ksum]
      // (D x (D+16), MN-major image from kv_combine).
      constexpr uint32_t idesc = idesc_bf16_f32(128, C::kNB, 0, 1);
      const uint32_t ba = smem_u32(blob);
      long long cur = -1;
      int nblob = 0;
      for (int li = 0; li < count; ++li) {
        const long long item = begin + li;
        const int bh = static_cast<int>(item / tiles);
        if (bh != cur) {
          if (nblob > 0) umma_commit(&blobempty);
          if (!mbar_wait(&blobfull, nblob & 1, status)) break;
          cur = bh;
          ++nblob;
        }
        const int st = li % C::kStages, round = li / C::kStages;
        const int a = li & 1, ar = li >> 1;
        if (!mbar_wait(&qphi[st], round & 1, status)) break;
        if (li >= 2 && !mbar_wait(&accempty[a], (ar - 1) & 1, status)) break;
        tc_fence_after();
        const uint32_t qa = smem_u32(qs + st * C::kTileBytes);
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint64_t adesc = smem_desc_sw128(qa + (k >> 2) * kBoxBytes + (k & 3) * 32, 16, 1024);
          const uint64_t bdesc = smem_desc_sw128(ba + k * 2048, D * 128, 1024);
          umma_bf16(tmem + a * C::kAccCols, adesc, bdesc, idesc, k > 0 ? 1u : 0u);
        }
        umma_commit(&qempty[st]);
        umma_commit(&accfull[a]);
      }
    }
  } else if (warp < 6) {
    // ----------------------------------------------------------- phi on Q
    const int pt = threadIdx.x - 64;
    const int cc = pt / C::kThreadsPerChunk;
    const int r0 = pt % C::kThreadsPerChunk;
    for (int li = 0; li < count; ++li) {
      const int st = li % C::kStages, round = li / C::kStages;
      if (!warp_wait(&qfull[st], round & 1, status)) break;
      uint8_t* qt = qs + st * C::kTileBytes;
#pragma unroll 4
      for (int j = 0; j < C::kRowsPerThread; ++j) {
        const int r = r0 + j * C::kThreadsPerChunk;
        uint4* p = reinterpret_cast<uint4*>(qt + swz_off(r, cc));
        float y[8];
        *p = phi_chunk<FMAP>(*p, y);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&qphi[st]);
    }
  } else {
    // --------------------------------------------------------------- epilogue
    const int q = warp & 3;
    const int r = 32 * q + lane;                    // token row in the tile
    const bool leader = threadIdx.x == 192;
    for (int li = 0; li < count; ++li) {
      const long long item = begin + li;
      const int bh = static_cast<int>(item / tiles), tile = static_cast<int>(item % tiles);
      const int a = li & 1, ar = li >> 1;
      if (leader) {
        if (!mbar_wait(&accfull[a], ar & 1, status)) ep_abort = 1;
        bulk_wait_group_read<1>();                  // staging buffer li&1 is free again
      }
      named_bar_sync(1, 128);
      if (ep_abort) break;
      tc_fence_after();
      const uint32_t trow = tmem + a * C::kAccCols + (static_cast<uint32_t>(32 * q) << 16);
      const float den = tmem_ld1(trow + D);
      tmem_wait_ld();
      const float inv = 1.0f / (den + eps);
      uint8_t* ob = os + a * C::kTileBytes;
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 32) {
        float v[32];
        tmem_ld32(trow + c0, v);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint32_t w[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            __nv_bfloat162 b = __floats2bfloat162_rn(v[8 * j + 2 * i] * inv, v[8 * j + 2 * i + 1] * inv);
            w[i] = *reinterpret_cast<uint32_t*>(&b);
          }
          *reinterpret_cast<uint4*>(ob + swz_off(r, c0 / 8 + j)) = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&accempty[a]);
      fence_proxy_async_smem();
      named_bar_sync(1, 128);
      if (leader) {
#pragma unroll
        for (int b = 0; b < C::kBoxes; ++b) tma_store_3d(&tm_out, ob + b * kBoxBytes, 64 * b, tile * kTileTokens, bh);
        bulk_commit_group();
      }
    }
    if (leader) bulk_wait_group<0>();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, C::kTmemCols);
}

template <typename K>
cudaError_t set_smem(K kernel, uint32_t bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
}

template <int D, int FMAP>
cudaError_t run(const LaunchArgs& a) {
  const Plan& p = *a.p;
  float* part = reinterpret_cast<float*>(a.ws + p.off_partial);
  float* part_ksum = reinterpret_cast<float*>(a.ws + p.off_ksum_partial);
  uint8_t* blobs = reinterpret_cast<uint8_t*>(a.ws + p.off_blob);
  int* status = reinterpret_cast<int*>(a.ws + p.off_status);
  cudaError_t err;

  {
    auto kern = kv_partial_kernel<D, FMAP>;
    if ((err = set_smem(kern, PartialCfg<D>::kSmemBytes)) != cudaSuccess) return err;
    dim3 grid(p.splits, static_cast<unsigned>(p.BH));
    kern<<<grid, 192, PartialCfg<D>::kSmemBytes, a.stream>>>(*a.tm_k, *a.tm_v, part, part_ksum, status, p.N,
                                                             p.tiles, p.tiles_per_split, p.splits);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
  }
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(p.BH), p.Fe / 8);
    cfg.blockDim = dim3(256);
    cfg.stream = a.stream;
    cfg.attrs = pdl;
    cfg.numAttrs = 1;
    err = cudaLaunchKernelEx(&cfg, kv_combine_kernel, static_cast<const float*>(part),
                             static_cast<const float*>(part_ksum), blobs, p.D, p.Fe, p.splits, p.blob_bytes);
    if (err != cudaSuccess) return err;
  }
  {
    auto kern = apply_kernel<D, FMAP>;
    if ((err = set_smem(kern, ApplyCfg<D>::kSmemBytes)) != cudaSuccess) return err;
    const long long total = p.BH * p.tiles;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(total < p.num_sms ? total : p.num_sms));
    cfg.blockDim = dim3(320);
    cfg.dynamicSmemBytes = ApplyCfg<D>::kSmemBytes;
    cfg.stream = a.stream;
    cfg.attrs = pdl;
    cfg.numAttrs = 1;
    err = cudaLaunchKernelEx(&cfg, kern, *a.tm_q, *a.tm_out, static_cast<const uint8_t*>(blobs), status, p.eps,
                             p.tiles, total);
  }
  return err;
}

}  // namespace

cudaError_t launch_bf16_noncausal(const LaunchArgs& a) {
  const Plan& p = *a.p;
  if (p.F != 0) return cudaErrorNotSupported;
  if (p.D == 128) return p.fmap == 0 ? run<128, 0>(a) : run<128, 1>(a);
  if (p.D == 64) return p.fmap == 0 ? run<64, 0>(a) : run<64, 1>(a);
  return cudaErrorNotSupported;
}

}  // namespace la
