// f32_kernels.cu -- fp32 CUDA-core path for every mode (non-causal, causal,
// projected).  fp32 inputs are held to a 1e-5 relative bar, which the bf16 /
// tf32 tensor-core operand formats cannot meet, so this path uses FFMA with
// fp32 accumulation and the accurate expf.
//
// Method (page "NNT Define Linear Attention", "How it works"): the state
// kv = phi(K)^T V and ksum = sum_j phi(k_j) is reduced over the sequence, then
// out_i = phi(q_i)^T kv / (phi(q_i) . ksum + eps).  The causal variant carries
// the state over the sequence: each segment's state is reduced, an exclusive
// scan over segments gives every segment its starting state, and each segment
// then walks its tokens in order (update with token i, then read row i).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "la_internal.h"
#include "sm100.cuh"

namespace la {
namespace {

constexpr int kT = 16;      // tokens per chunk
constexpr int kFB = 32;     // features per state block
constexpr int kMaxD = 128;
constexpr int kMaxFe = 256;

// phi of token row `t` (already in shared memory) for feature f.  The softmax
// map (fmap 2, no projection) takes the row's maximum and the reciprocal of
// its exponential sum from `st` (softmax_stats).
__device__ __forceinline__ float feature(const float* xs, int D, const float* W, int F, int f, int fmap,
                                         const float* st) {
  float x;
  if (F) {
    x = 0.f;
    for (int d = 0; d < D; ++d) x = fmaf(xs[d], __ldg(W + static_cast<size_t>(d) * F + f), x);
  } else {
    x = xs[f];
  }
  if (fmap == 2) return expf(x - st[0]) * st[1];
  return phi_accurate(x, fmap);
}

// Softmax over each row of xs [kT][kMaxD]: st[2 t] = max_d x_td and
// st[2 t + 1] = 1 / sum_d exp(x_td - max), one warp per row, lanes over d,
// butterfly reductions (a fixed order: deterministic).  Zero-filled rows
// give finite values that nothing reads.
__device__ void softmax_stats(const float* xs, int D, float* st) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  for (int t = warp; t < kT; t += blockDim.x / 32) {
    float m = -INFINITY;
    for (int d = lane; d < D; d += 32) m = fmaxf(m, xs[t * kMaxD + d]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float z = 0.f;
    for (int d = lane; d < D; d += 32) z += expf(xs[t * kMaxD + d] - m);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
    if (lane == 0) {
      st[2 * t] = m;
      st[2 * t + 1] = 1.f / z;
    }
  }
}

// Flux's attention prologue on the first `rows` rows of xs [kT][kMaxD] (token
// positions t0 + t): x_d / sqrt(mean x^2 + neps) * scale_d, then each pair
// (2i, 2i + 1) turned by rope[t0 + t][i] = (cos, sin).  One warp per row.
struct Prologue {
  const float* scale;   // [D]; nullptr: no prologue
  const float* rope;    // [positions][D / 2][2]
  float eps;
};
__device__ void prologue_rows(float* xs, int rows, int D, int t0, Prologue pr) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  for (int t = warp; t < rows; t += blockDim.x / 32) {
    float* x = xs + t * kMaxD;
    float ss = 0.f;
    for (int d = lane; d < D; d += 32) ss = fmaf(x[d], x[d], ss);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float r = 1.f / sqrtf(ss / static_cast<float>(D) + pr.eps);
    const float* rp = pr.rope + static_cast<size_t>(t0 + t) * D;
    for (int i = lane; i < D / 2; i += 32) {
      const float x0 = x[2 * i] * r * __ldg(pr.scale + 2 * i), x1 = x[2 * i + 1] * r * __ldg(pr.scale + 2 * i + 1);
      const float c = __ldg(rp + 2 * i), sn = __ldg(rp + 2 * i + 1);
      x[2 * i] = c * x0 - sn * x1;
      x[2 * i + 1] = sn * x0 + c * x1;
    }
  }
}

__device__ __forceinline__ void load_rows(float* dst, const float* src, int rows_valid, int D) {
  // dst[kT][kMaxD]; rows >= rows_valid are zero-filled.  D % 4 == 0.
  const int d4 = D / 4;
  for (int e = threadIdx.x; e < kT * d4; e += blockDim.x) {
    const int t = e / d4, c = e % d4;
    float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
    if (t < rows_valid) x = *reinterpret_cast<const float4*>(src + static_cast<size_t>(t) * D + 4 * c);
    *reinterpret_cast<float4*>(dst + t * kMaxD + 4 * c) = x;
  }
}

// Partial state of tokens [s*seg, min(N, (s+1)*seg)) of head bh, features
// [32*blockIdx.z, +32): part[bh][s][f][d] and part_ksum[bh][s][f].
__global__ void __launch_bounds__(256) f32_state_partial(const float* __restrict__ k, const float* __restrict__ v,
                                                         const float* __restrict__ W, long long wstride,
                                                         float* __restrict__ part, float* __restrict__ part_ksum,
                                                         int H, int N, int D, int F, int Fe, int fmap, int seg,
                                                         int S, Prologue pk) {
  __shared__ __align__(16) float Ks[kT * kMaxD];
  __shared__ __align__(16) float Vs[kT * kMaxD];
  __shared__ float Ps[kT * kFB];
  __shared__ float Kst[2 * kT];
  const int s = blockIdx.x;
  const long long bh = blockIdx.y;
  const int fb = blockIdx.z * kFB;
  const float* Wh = F ? W + static_cast<size_t>(bh % H) * wstride : nullptr;
  const float* kh = k + static_cast<size_t>(bh) * N * D;
  const float* vh = v + static_cast<size_t>(bh) * N * D;
  const int t0 = s * seg, t1 = min(N, t0 + seg);
  const int fl = threadIdx.x / 8, dl = threadIdx.x % 8;
  float acc[kMaxD / 8];
#pragma unroll
  for (int j = 0; j < kMaxD / 8; ++j) acc[j] = 0.f;
  float ks = 0.f;
  for (int tc = t0; tc < t1; tc += kT) {
    const int rows = min(kT, t1 - tc);
    load_rows(Ks, kh + static_cast<size_t>(tc) * D, rows, D);
    load_rows(Vs, vh + static_cast<size_t>(tc) * D, rows, D);
    __syncthreads();
    if (pk.scale) {
      prologue_rows(Ks, rows, D, tc, pk);
      __syncthreads();
    }
    if (fmap == 2) {
      softmax_stats(Ks, D, Kst);
      __syncthreads();
    }
    for (int e = threadIdx.x; e < kT * kFB; e += blockDim.x) {
      const int t = e / kFB, f = fb + e % kFB;
      Ps[e] = (t < rows && f < Fe) ? feature(Ks + t * kMaxD, D, Wh, F, f, fmap, Kst + 2 * t) : 0.f;
    }
    __syncthreads();
    for (int t = 0; t < kT; ++t) {
      const float p = Ps[t * kFB + fl];
#pragma unroll
      for (int j = 0; j < kMaxD / 8; ++j) {
        const int d = dl + 8 * j;
        if (d < D) acc[j] = fmaf(p, Vs[t * kMaxD + d], acc[j]);
      }
      ks += p;
    }
    __syncthreads();
  }
  const int f = fb + fl;
  if (f < Fe) {
    float* dst = part + ((static_cast<size_t>(bh) * S + s) * Fe + f) * D;
#pragma unroll
    for (int j = 0; j < kMaxD / 8; ++j) {
      const int d = dl + 8 * j;
      if (d < D) dst[d] = acc[j];
    }
    if (dl == 0) part_ksum[(static_cast<size_t>(bh) * S + s) * Fe + f] = ks;
  }
}

// final[bh] = sum_{s=0..S-1} part[bh][s], summed in ascending s.
__global__ void f32_state_combine(const float* __restrict__ part, const float* __restrict__ part_ksum,
                                  float* __restrict__ fin, float* __restrict__ fin_ksum, int Fe, int D, int S) {
  const long long bh = blockIdx.x;
  const int n_kv = Fe * D;
  const int e = blockIdx.y * blockDim.x + threadIdx.x;
  if (e < n_kv) {
    float acc = 0.f;
    for (int s = 0; s < S; ++s) acc += part[(static_cast<size_t>(bh) * S + s) * n_kv + e];
    fin[static_cast<size_t>(bh) * n_kv + e] = acc;
  } else if (e < n_kv + Fe) {
    const int f = e - n_kv;
    float acc = 0.f;
    for (int s = 0; s < S; ++s) acc += part_ksum[(static_cast<size_t>(bh) * S + s) * Fe + f];
    fin_ksum[static_cast<size_t>(bh) * Fe + f] = acc;
  }
}

// In-place exclusive scan over segments (ascending s): part[s] <- sum_{s'<s}.
__global__ void f32_state_scan(float* __restrict__ part, float* __restrict__ part_ksum, int Fe, int D, int S) {
  const long long bh = blockIdx.x;
  const int n_kv = Fe * D;
  const int e = blockIdx.y * blockDim.x + threadIdx.x;
  float* base;
  int stride;
  if (e < n_kv) {
    base = part + static_cast<size_t>(bh) * S * n_kv + e;
    stride = n_kv;
  } else if (e < n_kv + Fe) {
    base = part_ksum + static_cast<size_t>(bh) * S * Fe + (e - n_kv);
    stride = Fe;
  } else {
    return;
  }
  float run = 0.f;
  for (int s = 0; s < S; ++s) {
    const float x = base[static_cast<size_t>(s) * stride];
    base[static_cast<size_t>(s) * stride] = run;
    run += x;
  }
}

// out rows [blockIdx.x*16, +16) of head bh from the final state, the
// features taken in groups of kMaxFe (ascending; one group when Fe <= 256).
__global__ void __launch_bounds__(256) f32_apply(const float* __restrict__ q, const float* __restrict__ W,
                                                 long long wstride, const float* __restrict__ fin,
                                                 const float* __restrict__ fin_ksum, float* __restrict__ out,
                                                 int H, int N, int D, int F, int Fe, int fmap, float eps,
                                                 Prologue pq) {
  __shared__ __align__(16) float Qs[kT * kMaxD];
  __shared__ float Ps[kT * kMaxFe];
  __shared__ float den[kT];
  __shared__ float Qst[2 * kT];
  const long long bh = blockIdx.y;
  const int t0 = blockIdx.x * kT;
  const int rows = min(kT, N - t0);
  const float* Wh = F ? W + static_cast<size_t>(bh % H) * wstride : nullptr;
  const float* kv = fin + static_cast<size_t>(bh) * Fe * D;
  const float* ksum = fin_ksum + static_cast<size_t>(bh) * Fe;
  load_rows(Qs, q + (static_cast<size_t>(bh) * N + t0) * D, rows, D);
  __syncthreads();
  if (pq.scale) {
    prologue_rows(Qs, rows, D, t0, pq);
    __syncthreads();
  }
  if (fmap == 2) {
    softmax_stats(Qs, D, Qst);
    __syncthreads();
  }
  // Thread j of the block owns output elements e = j + 256 i (i < 8) of the
  // kT x D tile; their numerators run over all feature groups in registers.
  constexpr int kPer = kT * kMaxD / 256;
  float num[kPer];
#pragma unroll
  for (int i = 0; i < kPer; ++i) num[i] = 0.f;
  if (threadIdx.x < kT) den[threadIdx.x] = 0.f;
  for (int f0 = 0; f0 < Fe; f0 += kMaxFe) {
    const int fe = min(kMaxFe, Fe - f0);
    for (int e = threadIdx.x; e < kT * fe; e += blockDim.x) {
      const int t = e / fe, f = e % fe;
      Ps[t * kMaxFe + f] = t < rows ? feature(Qs + t * kMaxD, D, Wh, F, f0 + f, fmap, Qst + 2 * t) : 0.f;
    }
    __syncthreads();
    // den[t] += phi(q_t) . ksum over the group: one warp per two rows, lanes split f.
    {
      const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
      for (int t = warp; t < kT; t += blockDim.x / 32) {
        float acc = 0.f;
        for (int f = lane; f < fe; f += 32) acc = fmaf(Ps[t * kMaxFe + f], ksum[f0 + f], acc);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (lane == 0) den[t] += acc;
      }
    }
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int e = threadIdx.x + 256 * i;
      if (e < rows * D) {
        const int t = e / D, d = e % D;
        const float* kvf = kv + static_cast<size_t>(f0) * D + d;
        float acc = num[i];
        for (int f = 0; f < fe; ++f) acc = fmaf(Ps[t * kMaxFe + f], kvf[static_cast<size_t>(f) * D], acc);
        num[i] = acc;
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int e = threadIdx.x + 256 * i;
    if (e < rows * D) {
      const int t = e / D, d = e % D;
      out[(static_cast<size_t>(bh) * N + t0 + t) * D + d] = num[i] / (den[t] + eps);
    }
  }
}

// Causal: segment s of head bh starts from the exclusive prefix state
// pre[bh][s] and walks its tokens in order.  Dynamic shared memory holds the
// state St[Fe][D] and z[Fe].
__global__ void __launch_bounds__(256) f32_causal_apply(const float* __restrict__ q, const float* __restrict__ k,
                                                        const float* __restrict__ v, const float* __restrict__ W,
                                                        long long wstride, const float* __restrict__ pre,
                                                        const float* __restrict__ pre_ksum,
                                                        float* __restrict__ out, int H, int N, int D, int F,
                                                        int Fe, int fmap, float eps, int seg, int S, Prologue pq,
                                                        Prologue pk) {
  extern __shared__ __align__(16) float dyn[];
  __shared__ float Qst[2 * kT], Kst[2 * kT];
  float* Qs = dyn;                 // kT * kMaxD
  float* Ks = Qs + kT * kMaxD;
  float* Vs = Ks + kT * kMaxD;
  float* Pq = Vs + kT * kMaxD;     // kT * kMaxFe
  float* Pk = Pq + kT * kMaxFe;
  float* St = Pk + kT * kMaxFe;    // Fe * D
  float* z = St + Fe * D;          // Fe
  const int s = blockIdx.x;
  const long long bh = blockIdx.y;
  const float* Wh = F ? W + static_cast<size_t>(bh % H) * wstride : nullptr;
  const size_t head = static_cast<size_t>(bh) * N * D;
  const int t0 = s * seg, t1 = min(N, t0 + seg);
  const float* p0 = pre + (static_cast<size_t>(bh) * S + s) * Fe * D;
  for (int e = threadIdx.x; e < Fe * D; e += blockDim.x) St[e] = p0[e];
  for (int f = threadIdx.x; f < Fe; f += blockDim.x) z[f] = pre_ksum[(static_cast<size_t>(bh) * S + s) * Fe + f];
  for (int tc = t0; tc < t1; tc += kT) {
    const int rows = min(kT, t1 - tc);
    __syncthreads();
    load_rows(Qs, q + head + static_cast<size_t>(tc) * D, rows, D);
    load_rows(Ks, k + head + static_cast<size_t>(tc) * D, rows, D);
    load_rows(Vs, v + head + static_cast<size_t>(tc) * D, rows, D);
    __syncthreads();
    if (pq.scale) {
      prologue_rows(Qs, rows, D, tc, pq);
      prologue_rows(Ks, rows, D, tc, pk);
      __syncthreads();
    }
    if (fmap == 2) {
      softmax_stats(Qs, D, Qst);
      softmax_stats(Ks, D, Kst);
      __syncthreads();
    }
    for (int e = threadIdx.x; e < kT * Fe; e += blockDim.x) {
      const int t = e / Fe, f = e % Fe;
      Pq[t * kMaxFe + f] = t < rows ? feature(Qs + t * kMaxD, D, Wh, F, f, fmap, Qst + 2 * t) : 0.f;
      Pk[t * kMaxFe + f] = t < rows ? feature(Ks + t * kMaxD, D, Wh, F, f, fmap, Kst + 2 * t) : 0.f;
    }
    __syncthreads();
    for (int t = 0; t < rows; ++t) {
      for (int e = threadIdx.x; e < Fe * D; e += blockDim.x) {
        const int f = e / D, d = e % D;
        St[e] = fmaf(Pk[t * kMaxFe + f], Vs[t * kMaxD + d], St[e]);
      }
      for (int f = threadIdx.x; f < Fe; f += blockDim.x) z[f] += Pk[t * kMaxFe + f];
      __syncthreads();
      for (int d = threadIdx.x; d < D; d += blockDim.x) {
        float num = 0.f, den = 0.f;
        for (int f = 0; f < Fe; ++f) {
          const float p = Pq[t * kMaxFe + f];
          num = fmaf(p, St[f * D + d], num);
          den = fmaf(p, z[f], den);
        }
        out[head + static_cast<size_t>(tc + t) * D + d] = num / (den + eps);
      }
      __syncthreads();
    }
  }
}

// ------------------------------------------------- storage conversions
__global__ void bf16_to_f32_kernel(const __nv_bfloat16* __restrict__ in, float* __restrict__ out, size_t n) {
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x)
    out[i] = __bfloat162float(in[i]);
}
__global__ void f32_to_bf16_kernel(const float* __restrict__ in, __nv_bfloat16* __restrict__ out, size_t n) {
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x)
    out[i] = __float2bfloat16_rn(in[i]);
}

// ------------------------------------------------------------ backward
// Gradients of sum(out * dout), non-causal, no projection (features = D), for
// a loss whose gradient with respect to out is dout (page "Flux2TTRTrainer",
// "How the distillation works": the student layer is trained).  With
// den_i = phi(q_i).z + eps, out_i = phi(q_i) kv / den_i, g_i = dout_i / den_i
// and h_i = -(dout_i . out_i) / den_i:
//   dq_i = (kv g_i + h_i z) * phi'(q_i),
//   dkv = sum_i phi(q_i) g_i^T,  dz = sum_i h_i phi(q_i),
//   dk_j = (dkv v_j + dz) * phi'(k_j),  dv_j = dkv^T phi(k_j).

__device__ __forceinline__ float phi_grad(float x, int fmap) {
  if (fmap == 0) return x > 0.f ? 1.f : expf(x);
  return x > 0.f ? 1.f : 0.f;
}

// Query rows of split s of head bh: dq, and the split's partials of dkv
// ([bh][s][D][D], row f = feature) and dz ([bh][s][D]).
__global__ void __launch_bounds__(256) f32_bwd_query(const float* __restrict__ q, const float* __restrict__ dout,
                                                     const float* __restrict__ fin, const float* __restrict__ fin_ksum,
                                                     float* __restrict__ dq, float* __restrict__ part_dkv,
                                                     float* __restrict__ part_dz, int N, int D, int fmap, float eps,
                                                     int seg, int S) {
  __shared__ __align__(16) float Qs[kT * kMaxD];
  __shared__ __align__(16) float Ps[kT * kMaxD];
  __shared__ __align__(16) float Gs[kT * kMaxD];
  __shared__ float dens[kT], hs[kT];
  // the head's kv, rows padded to D + 1 floats: conflict-free whether the
  // lanes run along a row or down a column
  extern __shared__ float kvs[];
  const int s = blockIdx.x;
  const long long bh = blockIdx.y;
  const float* kvg = fin + static_cast<size_t>(bh) * D * D;
  for (int e = threadIdx.x; e < D * D; e += blockDim.x) kvs[(e / D) * (D + 1) + e % D] = kvg[e];
  const float* z = fin_ksum + static_cast<size_t>(bh) * D;
  const float* qh = q + static_cast<size_t>(bh) * N * D;
  const float* oh = dout + static_cast<size_t>(bh) * N * D;
  const int t0 = s * seg, t1 = min(N, t0 + seg);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  constexpr int kAcc = kMaxD * kMaxD / 256;
  float acc[kAcc];
#pragma unroll
  for (int j = 0; j < kAcc; ++j) acc[j] = 0.f;
  float dzacc = 0.f;
  for (int tc = t0; tc < t1; tc += kT) {
    const int rows = min(kT, t1 - tc);
    load_rows(Qs, qh + static_cast<size_t>(tc) * D, rows, D);
    load_rows(Gs, oh + static_cast<size_t>(tc) * D, rows, D);
    __syncthreads();
    for (int e = threadIdx.x; e < kT * D; e += blockDim.x) {
      const int t = e / D, f = e % D;
      Ps[t * kMaxD + f] = t < rows ? phi_accurate(Qs[t * kMaxD + f], fmap) : 0.f;
    }
    __syncthreads();
    // den_t and h_t = -(dout_t . num_t) / den_t^2: one warp per two rows
    for (int t = warp; t < kT; t += blockDim.x / 32) {
      float den = 0.f, dot = 0.f;
      for (int f = lane; f < D; f += 32) den = fmaf(Ps[t * kMaxD + f], z[f], den);
      for (int d = lane; d < D; d += 32) {
        float num = 0.f;
        for (int f = 0; f < D; ++f) num = fmaf(Ps[t * kMaxD + f], kvs[f * (D + 1) + d], num);
        dot = fmaf(Gs[t * kMaxD + d], num, dot);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        den += __shfl_xor_sync(0xffffffffu, den, o);
        dot += __shfl_xor_sync(0xffffffffu, dot, o);
      }
      den += eps;
      if (lane == 0) {
        dens[t] = den;
        hs[t] = -dot / (den * den);
      }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < kT * D; e += blockDim.x) {   // g = dout / den
      const int t = e / D, d = e % D;
      Gs[t * kMaxD + d] /= dens[t];
    }
    __syncthreads();
    for (int e = threadIdx.x; e < rows * D; e += blockDim.x) {
      const int t = e / D, f = e % D;
      float g = hs[t] * z[f];
      for (int d = 0; d < D; ++d) g = fmaf(kvs[f * (D + 1) + d], Gs[t * kMaxD + d], g);
      dq[(static_cast<size_t>(bh) * N + tc + t) * D + f] = g * phi_grad(Qs[t * kMaxD + f], fmap);
    }
#pragma unroll
    for (int j = 0; j < kAcc; ++j) {
      const int e = threadIdx.x + 256 * j;
      if (e < D * D) {
        const int f = e / D, d = e % D;
        float a = acc[j];
        for (int t = 0; t < kT; ++t) a = fmaf(Ps[t * kMaxD + f], Gs[t * kMaxD + d], a);
        acc[j] = a;
      }
    }
    if (threadIdx.x < D)
      for (int t = 0; t < kT; ++t) dzacc = fmaf(hs[t], Ps[t * kMaxD + threadIdx.x], dzacc);
    __syncthreads();
  }
  float* dst = part_dkv + (static_cast<size_t>(bh) * S + s) * D * D;
#pragma unroll
  for (int j = 0; j < kAcc; ++j) {
    const int e = threadIdx.x + 256 * j;
    if (e < D * D) dst[e] = acc[j];
  }
  if (threadIdx.x < D) part_dz[(static_cast<size_t>(bh) * S + s) * D + threadIdx.x] = dzacc;
}

// Key rows [blockIdx.x * kBwdRows, +kBwdRows) of head bh, in chunks of kT:
// dk and dv from dkv and dz.
constexpr int kBwdRows = 64;
__global__ void __launch_bounds__(256) f32_bwd_key(const float* __restrict__ k, const float* __restrict__ v,
                                                   const float* __restrict__ fin_dkv,
                                                   const float* __restrict__ fin_dz, float* __restrict__ dk,
                                                   float* __restrict__ dv, int N, int D, int fmap) {
  __shared__ __align__(16) float Ks[kT * kMaxD];
  __shared__ __align__(16) float Vs[kT * kMaxD];
  __shared__ __align__(16) float Ps[kT * kMaxD];
  extern __shared__ float dkvs[];   // dkv, rows padded to D + 1 floats
  const long long bh = blockIdx.y;
  const float* dkvg = fin_dkv + static_cast<size_t>(bh) * D * D;
  for (int e = threadIdx.x; e < D * D; e += blockDim.x) dkvs[(e / D) * (D + 1) + e % D] = dkvg[e];
  const float* dz = fin_dz + static_cast<size_t>(bh) * D;
  for (int t0 = blockIdx.x * kBwdRows; t0 < min(N, (blockIdx.x + 1) * kBwdRows); t0 += kT) {
  const int rows = min(kT, N - t0);
  __syncthreads();
  load_rows(Ks, k + (static_cast<size_t>(bh) * N + t0) * D, rows, D);
  load_rows(Vs, v + (static_cast<size_t>(bh) * N + t0) * D, rows, D);
  __syncthreads();
  for (int e = threadIdx.x; e < kT * D; e += blockDim.x) {
    const int t = e / D, f = e % D;
    Ps[t * kMaxD + f] = t < rows ? phi_accurate(Ks[t * kMaxD + f], fmap) : 0.f;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < rows * D; e += blockDim.x) {
    const int t = e / D, c = e % D;
    float gk = dz[c], gv = 0.f;
    for (int x = 0; x < D; ++x) {
      gk = fmaf(dkvs[c * (D + 1) + x], Vs[t * kMaxD + x], gk);   // (dkv v_t)_c
      gv = fmaf(Ps[t * kMaxD + x], dkvs[x * (D + 1) + c], gv);   // (dkv^T phi(k_t))_c
    }
    const size_t o = (static_cast<size_t>(bh) * N + t0 + t) * D + c;
    dk[o] = gk * phi_grad(Ks[t * kMaxD + c], fmap);
    dv[o] = gv;
  }
  }
}

}  // namespace

cudaError_t launch_f32(const LaunchArgs& a) {
  const Plan& p = *a.p;
  const float* q = static_cast<const float*>(a.q);
  const float* k = static_cast<const float*>(a.k);
  const float* v = static_cast<const float*>(a.v);
  const float* W = static_cast<const float*>(a.W);
  float* out = static_cast<float*>(a.out);
  float* part = reinterpret_cast<float*>(a.ws + p.off_partial);
  float* part_ksum = reinterpret_cast<float*>(a.ws + p.off_ksum_partial);
  const int S = p.splits;
  const int n_state = p.Fe * p.D + p.Fe;

  dim3 g1(S, static_cast<unsigned>(p.BH), (p.Fe + kFB - 1) / kFB);
  const Prologue pq = {a.prologue ? a.pro_q : nullptr, a.pro_rope, a.pro_eps};
  const Prologue pk = {a.prologue ? a.pro_k : nullptr, a.pro_rope, a.pro_eps};
  f32_state_partial<<<g1, 256, 0, a.stream>>>(k, v, W, a.w_head_stride, part, part_ksum, p.H, p.N, p.D, p.F, p.Fe,
                                              p.fmap, p.seg_len, S, pk);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  dim3 g2(static_cast<unsigned>(p.BH), (n_state + 255) / 256);
  if (!p.causal) {
    float* fin = reinterpret_cast<float*>(a.ws + p.off_final);
    float* fin_ksum = reinterpret_cast<float*>(a.ws + p.off_final_ksum);
    f32_state_combine<<<g2, 256, 0, a.stream>>>(part, part_ksum, fin, fin_ksum, p.Fe, p.D, S);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    dim3 g3((p.N + kT - 1) / kT, static_cast<unsigned>(p.BH));
    f32_apply<<<g3, 256, 0, a.stream>>>(q, W, a.w_head_stride, fin, fin_ksum, out, p.H, p.N, p.D, p.F, p.Fe, p.fmap,
                                        p.eps, pq);
    return cudaGetLastError();
  }
  f32_state_scan<<<g2, 256, 0, a.stream>>>(part, part_ksum, p.Fe, p.D, S);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  const size_t dyn = (3 * kT * kMaxD + 2 * kT * kMaxFe) * sizeof(float) +
                     (static_cast<size_t>(p.Fe) * p.D + p.Fe) * sizeof(float);
  err = cudaFuncSetAttribute(f32_causal_apply, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(dyn));
  if (err != cudaSuccess) return err;
  dim3 g3(S, static_cast<unsigned>(p.BH));
  f32_causal_apply<<<g3, 256, dyn, a.stream>>>(q, k, v, W, a.w_head_stride, part, part_ksum, out, p.H, p.N, p.D, p.F,
                                               p.Fe, p.fmap, p.eps, p.seg_len, S, pq, pk);
  return cudaGetLastError();
}

// Backward of the fp32 non-causal layer without projection: the forward
// state (kv, z) into the plan's final region, then per-split partials of
// (dkv, dz) with dq, summed in ascending split order into bfin / bfin_z, then
// dk and dv.
cudaError_t launch_f32_backward(const LaunchArgs& a, const void* dout, void* dq, void* dk, void* dv, int splits,
                                int seg, float* bpart, float* bpart_z, float* bfin, float* bfin_z) {
  const Plan& p = *a.p;
  if (p.F != 0 || p.causal || p.fmap > 1 || a.prologue) return cudaErrorNotSupported;
  const float* q = static_cast<const float*>(a.q);
  const float* k = static_cast<const float*>(a.k);
  const float* v = static_cast<const float*>(a.v);
  float* part = reinterpret_cast<float*>(a.ws + p.off_partial);
  float* part_ksum = reinterpret_cast<float*>(a.ws + p.off_ksum_partial);
  float* fin = reinterpret_cast<float*>(a.ws + p.off_final);
  float* fin_ksum = reinterpret_cast<float*>(a.ws + p.off_final_ksum);
  const int S = p.splits;
  const int n_state = p.D * p.D + p.D;
  const Prologue none = {nullptr, nullptr, 0.f};
  dim3 g1(S, static_cast<unsigned>(p.BH), (p.D + kFB - 1) / kFB);
  f32_state_partial<<<g1, 256, 0, a.stream>>>(k, v, nullptr, 0, part, part_ksum, p.H, p.N, p.D, 0, p.D, p.fmap,
                                              p.seg_len, S, none);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  dim3 g2(static_cast<unsigned>(p.BH), (n_state + 255) / 256);
  f32_state_combine<<<g2, 256, 0, a.stream>>>(part, part_ksum, fin, fin_ksum, p.D, p.D, S);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  const size_t mat = static_cast<size_t>(p.D) * (p.D + 1) * sizeof(float);
  if ((err = cudaFuncSetAttribute(f32_bwd_query, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(mat))) !=
          cudaSuccess ||
      (err = cudaFuncSetAttribute(f32_bwd_key, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(mat))) !=
          cudaSuccess)
    return err;
  f32_bwd_query<<<dim3(splits, static_cast<unsigned>(p.BH)), 256, mat, a.stream>>>(
      q, static_cast<const float*>(dout), fin, fin_ksum, static_cast<float*>(dq), bpart, bpart_z, p.N, p.D, p.fmap,
      p.eps, seg, splits);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  f32_state_combine<<<g2, 256, 0, a.stream>>>(bpart, bpart_z, bfin, bfin_z, p.D, p.D, splits);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  dim3 g3((p.N + kBwdRows - 1) / kBwdRows, static_cast<unsigned>(p.BH));
  f32_bwd_key<<<g3, 256, mat, a.stream>>>(k, v, bfin, bfin_z, static_cast<float*>(dk), static_cast<float*>(dv), p.N,
                                        p.D, p.fmap);
  return cudaGetLastError();
}

cudaError_t launch_bf16_to_f32(const void* in, float* out, size_t n, cudaStream_t stream) {
  if (n == 0) return cudaSuccess;
  const unsigned blocks = static_cast<unsigned>(std::min<size_t>((n + 255) / 256, 4096));
  bf16_to_f32_kernel<<<blocks, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(in), out, n);
  return cudaGetLastError();
}

cudaError_t launch_f32_to_bf16(const float* in, void* out, size_t n, cudaStream_t stream) {
  if (n == 0) return cudaSuccess;
  const unsigned blocks = static_cast<unsigned>(std::min<size_t>((n + 255) / 256, 4096));
  f32_to_bf16_kernel<<<blocks, 256, 0, stream>>>(in, static_cast<__nv_bfloat16*>(out), n);
  return cudaGetLastError();
}

}  // namespace la
