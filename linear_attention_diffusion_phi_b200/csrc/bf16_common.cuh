// bf16_common.cuh -- tile layout and feature-map helpers shared by the bf16
// tensor-core kernels.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "sm100.cuh"

namespace la {

constexpr uint32_t kBoxBytes = 128 * 128;   // one TMA box: 128 rows x 64 bf16 (128 B)

// Byte offset of (row r, logical 16-byte chunk cc) in a [128 x D] bf16 tile
// held as D/64 TMA boxes with the 128-byte swizzle.
__device__ __forceinline__ uint32_t swz_off(int r, int cc) {
  return static_cast<uint32_t>((cc >> 3) * kBoxBytes + r * 128 + (((cc & 7) ^ (r & 7)) << 4));
}

// phi on 8 bf16 values (one 16-byte chunk), branch-free and rounded once to
// bf16.  elu(x)+1 = max(x, 0) + exp(min(x, 0)): for x > 0 the exponential is
// exactly 1 and the bf16 add rounds x + 1 once; for x <= 0 the max is 0 and
// the sum is the bf16-rounded exponential.  exp(y) = 2^(y log2 e) uses the
// hardware ex2 on fp32.  relu = max(x, 0) is exact in bf16.
template <int FMAP>
__device__ __forceinline__ uint32_t phi_pair(uint32_t w) {
  const __nv_bfloat162 x = *reinterpret_cast<__nv_bfloat162*>(&w);
  const __nv_bfloat162 zero = __float2bfloat162_rn(0.f);
  __nv_bfloat162 r = __hmax2(x, zero);
  if (FMAP == 0) {
    const float2 n = __bfloat1622float2(__hmin2(x, zero));
    const __nv_bfloat162 e = __floats2bfloat162_rn(ex2_approx(n.x * kLog2e), ex2_approx(n.y * kLog2e));
    r = __hadd2(r, e);
  }
  return *reinterpret_cast<uint32_t*>(&r);
}

template <int FMAP>
__device__ __forceinline__ uint4 phi_chunk(uint4 x) {
  return make_uint4(phi_pair<FMAP>(x.x), phi_pair<FMAP>(x.y), phi_pair<FMAP>(x.z), phi_pair<FMAP>(x.w));
}

// phi in place on NR 16-byte chunks of one swizzled tile: column chunk cc,
// rows r0, r0 + RS, ...; rows >= valid become 0.  Every load is issued first,
// then the arithmetic, then every store, so that the loads overlap instead of
// each waiting behind the previous row's store.
template <int FMAP, int NR, int RS>
__device__ __forceinline__ void phi_rows(uint8_t* tile, int cc, int r0, int valid) {
  uint4 x[NR];
#pragma unroll
  for (int j = 0; j < NR; ++j) x[j] = *reinterpret_cast<const uint4*>(tile + swz_off(r0 + RS * j, cc));
#pragma unroll
  for (int j = 0; j < NR; ++j)
    x[j] = (r0 + RS * j < valid) ? phi_chunk<FMAP>(x[j]) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
  for (int j = 0; j < NR; ++j) *reinterpret_cast<uint4*>(tile + swz_off(r0 + RS * j, cc)) = x[j];
}

// Lane 0 waits, the verdict is broadcast so the warp stays converged.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, int* status) {
  int ok = 1;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, status) ? 1 : 0;
  ok = __shfl_sync(0xffffffffu, ok, 0);
  return ok != 0;
}

// 16-byte load from a cluster CTA's shared memory.
__device__ __forceinline__ void ld_cluster_v4(uint32_t cluster_addr, uint32_t (&v)[4]) {
  asm volatile("ld.shared::cluster.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3])
               : "r"(cluster_addr)
               : "memory");
}

}  // namespace la
