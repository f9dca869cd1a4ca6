// bf16_image.cu -- the combine step shared by the bf16 paths that reduce
// per-split partial states in global memory (the projected path).
//
// Method (page "NNT Define Linear Attention", "How it works"): the state of a
// head is kv = phi(K)^T V and ksum = sum_j phi(k_j) over all its tokens; the
// token range of a head is split over CTAs, each leaving an fp32 partial.  The
// combine sums a head's partials in ascending split order (fp32) and writes
// the apply's B operand [kv | ksum | 0]^T: bf16, K-major, 128-byte swizzle,
// D + 16 rows, 64-feature atoms.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "la_internal.h"
#include "sm100.cuh"

namespace la {
namespace {

// image[n][f] (K-major, 64-feature atoms of D + 16 rows, 128-byte swizzle) =
// sum over the head's splits, ascending, of kv^T[n][f] (n < D), ksum[f]
// (n = D), 0 (n > D).  Partial p = (bh * nsplit + s) * parts + part holds
// kv^T[D][fpart] and ksum[fpart] for features part * fpart ...
__global__ void __launch_bounds__(256)
    image_combine_kernel(const float* __restrict__ part_kv, const float* __restrict__ part_ks,
                         uint8_t* __restrict__ image, int nsplit, int D, int fpart, int parts) {
  pdl_wait();                // the partials come from the previous launch
  pdl_launch_dependents();   // the apply may begin its set-up
  const int bh = blockIdx.x;
  const int F = fpart * parts, chunks_per_row = F / 8;
  const int rows = D + 16, atom = rows * 128;
  uint8_t* img = image + static_cast<size_t>(bh) * (F / 64) * atom;
  const int idx = blockIdx.y * blockDim.x + threadIdx.x;
  if (idx < rows * chunks_per_row) {
    const int n = idx / chunks_per_row, f0 = (idx % chunks_per_row) * 8;
    const int part = f0 / fpart, fl = f0 % fpart;
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
    if (n <= D) {
      // every split's loads in flight before the sum, which stays in split order
      constexpr int kMax = 8;
      for (int s0 = 0; s0 < nsplit; s0 += kMax) {
        float4 a[kMax], b[kMax];
#pragma unroll
        for (int j = 0; j < kMax; ++j) {
          if (s0 + j < nsplit) {
            const size_t p = (static_cast<size_t>(bh) * nsplit + s0 + j) * parts + part;
            const float* src = n < D ? part_kv + p * (static_cast<size_t>(D) * fpart) + static_cast<size_t>(n) * fpart + fl
                                     : part_ks + p * fpart + fl;
            a[j] = *reinterpret_cast<const float4*>(src);
            b[j] = *reinterpret_cast<const float4*>(src + 4);
          }
        }
#pragma unroll
        for (int j = 0; j < kMax; ++j) {
          if (s0 + j < nsplit) {
            acc[0] += a[j].x; acc[1] += a[j].y; acc[2] += a[j].z; acc[3] += a[j].w;
            acc[4] += b[j].x; acc[5] += b[j].y; acc[6] += b[j].z; acc[7] += b[j].w;
          }
        }
      }
    }
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      __nv_bfloat162 h = __floats2bfloat162_rn(acc[2 * e], acc[2 * e + 1]);
      w[e] = *reinterpret_cast<uint32_t*>(&h);
    }
    const int at = f0 >> 6, cc = (f0 & 63) >> 3;
    *reinterpret_cast<uint4*>(img + at * atom + n * 128 + ((cc ^ (n & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

}  // namespace

cudaError_t launch_image_combine(const float* part_kv, const float* part_ks, uint8_t* image, long long BH, int nsplit,
                                 int D, int fpart, int parts, cudaStream_t stream) {
  const int chunks = (D + 16) * fpart * parts / 8;
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(BH), static_cast<unsigned>((chunks + 255) / 256));
  cfg.blockDim = dim3(256);
  cfg.stream = stream;
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, image_combine_kernel, part_kv, part_ks, image, nsplit, D, fpart, parts);
}

}  // namespace la
