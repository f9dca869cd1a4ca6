// bf16_proj.cu -- tcgen05 tensor-core path for projected-feature phi
// attention, non-causal, bf16 storage and fp32 accumulation, D = 128, F = 256.
//
// Method (page "Flux2TTRTrainer", "Inputs worth setting": the feature
// dimension is a multiple of 256; page "NNT Define Linear Attention", "How it
// works"): per head h, phi(x) = elu(x W_h) + 1 with W_h a D x F matrix shared
// by queries and keys (or relu(x W_h)), then
//   kv = phi(K)^T V (F x D),  ksum = sum_j phi(k_j) (F),
//   out_i = phi(q_i)^T kv / (phi(q_i) . ksum + eps).
// Three launches:
//   proj_state_kernel    grid (splits, B H, 2): one 128-feature half of F per
//                        CTA.  Per 128-token tile: K W_half on the tensor core
//                        (fp32 in tensor memory, two buffers), phi by eight
//                        warps into shared memory (bf16), then
//                        kv^T += V^T phi(K) (M = D, N = 128) and
//                        ksum += phi(K)^T 1 (M = 128 features, N = 16).
//   image_combine_kernel (bf16_image.cu) sums the splits in ascending order
//                        (fp32) into the apply's B operand [kv | ksum | 0]^T,
//                        bf16, K-major, 128-byte swizzle (144 rows x 256).
//   proj_apply_kernel    grid (ctas, B H): W_h and the image stay in shared
//                        memory; per tile, Q W one feature half at a time,
//                        phi packed to bf16 in tensor memory (the A operand),
//                        O = phi(Q) [kv | ksum] (N = 144), out = num / (den + eps).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "bf16_common.cuh"
#include "la_internal.h"
#include "sm100.cuh"

namespace la {
namespace {

constexpr int kD = 128, kF = 256, kFH = 128;   // head size, features, features per half
constexpr uint32_t kT32 = 128u * 128u * 2u;    // 128 x 128 bf16: two TMA boxes
constexpr int kNB = kD + 16;                    // apply N: kv rows, the ksum row, zero rows
constexpr uint32_t kImgAtom = kNB * 128;        // one 64-feature atom of the image
constexpr uint32_t kImgBytes = (kF / 64) * kImgAtom;   // 73728
constexpr int kPhiWarps = 8;

// phi on two fp32 values, packed to bf16x2 (one rounding each).
template <int FMAP>
__device__ __forceinline__ uint32_t phi2_f32(float a, float b) {
  float ra, rb;
  if (FMAP == 0) {
    ra = fmaxf(a, 0.f) + ex2_approx(fminf(a, 0.f) * kLog2e);
    rb = fmaxf(b, 0.f) + ex2_approx(fminf(b, 0.f) * kLog2e);
  } else {
    ra = fmaxf(a, 0.f);
    rb = fmaxf(b, 0.f);
  }
  __nv_bfloat162 h = __floats2bfloat162_rn(ra, rb);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Two 64-column boxes of a [.., 128] bf16 tensor: a 128 x 128 tile.
__device__ __forceinline__ void load_tile128(void* dst, const CUtensorMap* m, uint64_t* bar, int row, int z) {
  mbar_arrive_expect_tx(bar, kT32);
  tma_load_3d(dst, m, bar, 0, row, z);
  tma_load_3d(static_cast<uint8_t*>(dst) + kBoxBytes, m, bar, 64, row, z);
}

// ====================================================== kernel 1: the state

// K ring of three slots: a slot holds K_t until the K W MMA has read it, then
// phi(K_t) (written over it by the phi warps) until the state MMAs have read
// that; V ring of two.
constexpr int kS1RK = 3;
constexpr uint32_t kS1OffW = 0;                       // W half: two 64-feature atoms [128 d][64 f]
constexpr uint32_t kS1OffOnes = kS1OffW + kT32;       // ones: K-major [16 rows][128 t], 4 KB
constexpr uint32_t kS1OffK = kS1OffOnes + 4096;
constexpr uint32_t kS1OffV = kS1OffK + kS1RK * kT32;
constexpr uint32_t kS1Smem = kS1OffV + 2 * kT32 + 1024;
constexpr int kS1Threads = 64 + 32 * kPhiWarps;
constexpr uint32_t kS1ColKv = 256, kS1ColKs = 384;   // kv^T (128 columns), ksum (16)

template <int FMAP>
__global__ void __launch_bounds__(kS1Threads, 1)
    proj_state_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                      const __grid_constant__ CUtensorMap tm_w, float* __restrict__ part_kv,
                      float* __restrict__ part_ks, int* status, int N, int H, int w_per_head, int tiles,
                      int tps) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t wfull, kfull[kS1RK], kempty[kS1RK], vfull[2], vempty[2], kwfull[2], kwfree[2];
  // phiready[t & 1]: phi(K_t) written; two barriers, as phi may run one tile
  // ahead of the state MMAs that wait for it
  __shared__ __align__(8) uint64_t phiready[2], accfull;
  __shared__ uint32_t tmem_slot;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = blockIdx.x, bh = blockIdx.y, fh = blockIdx.z, nsplit = gridDim.x;
  const int tile0 = split * tps;
  const int T = min(tiles, tile0 + tps) - tile0;   // >= 1
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* wsm = smem + kS1OffW;
  uint8_t* ones = smem + kS1OffOnes;
  auto k_slot = [&](int t) { return smem + kS1OffK + (t % kS1RK) * kT32; };

  if (threadIdx.x == 0) {
    mbar_init(&wfull, 1);
    for (int i = 0; i < kS1RK; ++i) {
      mbar_init(&kfull[i], 1);
      mbar_init(&kempty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&vfull[i], 1);
      mbar_init(&vempty[i], 1);
      mbar_init(&kwfull[i], 1);
      mbar_init(&kwfree[i], kPhiWarps);
    }
    mbar_init(&phiready[0], kPhiWarps);
    mbar_init(&phiready[1], kPhiWarps);
    mbar_init(&accfull, 1);
    fence_mbarrier_init();
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    prefetch_tmap(&tm_w);
  }
  for (int i = threadIdx.x; i < 4096 / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(ones)[i] = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
  fence_proxy_async_smem();
  if (warp == 1) {
    tmem_alloc(&tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  // programmatic dependent launch: no global access before the previous
  // launch has completed; the combine may launch now
  pdl_wait();
  pdl_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const int wz = w_per_head ? bh % H : 0;
      mbar_arrive_expect_tx(&wfull, kT32);
      tma_load_3d(wsm, &tm_w, &wfull, fh * kFH, 0, wz);
      tma_load_3d(wsm + kBoxBytes, &tm_w, &wfull, fh * kFH + 64, 0, wz);
      for (int t = 0; t < T; ++t) {
        const int s = t & 1, sk = t % kS1RK, row = (tile0 + t) * kTileTokens;
        if (t >= kS1RK && !mbar_wait(&kempty[sk], ((t / kS1RK) - 1) & 1, status)) break;
        load_tile128(k_slot(t), &tm_k, &kfull[sk], row, bh);
        if (t >= 2 && !mbar_wait(&vempty[s], ((t >> 1) - 1) & 1, status)) break;
        load_tile128(smem + kS1OffV + s * kT32, &tm_v, &vfull[s], row, bh);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t id_kw = idesc_bf16_f32(128, kFH, 0, 1);   // K W: A K-major, B MN-major
      constexpr uint32_t id_kv = idesc_bf16_f32(kD, kFH, 1, 1);    // V^T phi(K): both MN-major
      constexpr uint32_t id_ks = idesc_bf16_f32(kFH, 16, 1, 0);    // phi(K)^T 1: A MN-major, B K-major
      const uint64_t wdesc = smem_desc_sw128(smem_u32(wsm), kBoxBytes, 1024);
      const uint64_t odesc = smem_desc_sw128(smem_u32(ones), 16, 1024);
      // kv^T and ksum of tile u from phi(K_u), in K_u's slot
      auto issue_kv = [&](int u) -> bool {
        const int s = u & 1;
        if (!mbar_wait(&phiready[s], (u >> 1) & 1, status) || !mbar_wait(&vfull[s], (u >> 1) & 1, status))
          return false;
        tc_fence_after();
        const uint64_t pdesc = smem_desc_sw128(smem_u32(k_slot(u)), kBoxBytes, 1024);
        const uint64_t vdesc = smem_desc_sw128(smem_u32(smem + kS1OffV + s * kT32), kBoxBytes, 1024);
        if (u == 0) {
          umma_ss<0>(tmem + kS1ColKv, vdesc, pdesc, id_kv);
          umma_ss<0>(tmem + kS1ColKs, pdesc, odesc, id_ks);
        } else {
          umma_ss<1>(tmem + kS1ColKv, vdesc, pdesc, id_kv);
          umma_ss<1>(tmem + kS1ColKs, pdesc, odesc, id_ks);
        }
#pragma unroll
        for (int k = 1; k < kTileTokens / 16; ++k) {
          umma_ss<1>(tmem + kS1ColKv, desc_add(vdesc, 2048 * k), desc_add(pdesc, 2048 * k), id_kv);
          umma_ss<1>(tmem + kS1ColKs, desc_add(pdesc, 2048 * k), desc_add(odesc, (k >> 2) * 2048 + (k & 3) * 32),
                     id_ks);
        }
        umma_commit(&vempty[s]);
        umma_commit(&kempty[u % kS1RK]);
        return true;
      };
      bool ok = mbar_wait(&wfull, 0, status);
      for (int t = 0; t < T && ok; ++t) {
        const int s = t & 1;
        // K W_half for tile t into buffer s, once the phi warps have read its previous use
        if (!mbar_wait(&kfull[t % kS1RK], (t / kS1RK) & 1, status) ||
            (t >= 2 && !mbar_wait(&kwfree[s], ((t >> 1) - 1) & 1, status))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t kdesc = smem_desc_sw128(smem_u32(k_slot(t)), 16, 1024);
        const uint32_t d = tmem + s * 128;
        umma_ss<0>(d, kdesc, wdesc, id_kw);
#pragma unroll
        for (int k = 1; k < kD / 16; ++k)
          umma_ss<1>(d, desc_add(kdesc, (k >> 2) * kBoxBytes + (k & 3) * 32), desc_add(wdesc, 2048 * k), id_kw);
        umma_commit(&kwfull[s]);   // also: the K tile has been read, phi may go over it
        // the state MMAs of the previous tile, while phi works on this one
        if (t >= 1 && !issue_kv(t - 1)) {
          ok = false;
          break;
        }
      }
      if (ok) issue_kv(T - 1);
      umma_commit(&accfull);
    }
  } else {
    // ------------------------------------------ phi warps: K W -> phi(K)
    // Two warps per lane quarter; each takes 64 of the 128 features.  phi(K_t)
    // goes over K_t in its slot (the K W MMA has read it once kwfull fires),
    // so phi of tile t runs while the state MMAs of tile t - 1 read theirs.
    const int qd = warp & 3, hw = (warp - 2) >> 2, r = 32 * qd + lane;
    const uint32_t lanes = static_cast<uint32_t>(32 * qd) << 16;
    bool ok = true;
    for (int t = 0; t < T; ++t) {
      const int s = t & 1;
      uint8_t* dst = k_slot(t) + hw * kBoxBytes + r * 128;
      if (!warp_wait(&kwfull[s], (t >> 1) & 1, status)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float v[64];
      tmem_ld32(tmem + s * 128 + 64 * hw + lanes, *reinterpret_cast<float(*)[32]>(v));
      tmem_ld32(tmem + s * 128 + 64 * hw + 32 + lanes, *reinterpret_cast<float(*)[32]>(v + 32));
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&kwfree[s]);
      // key rows past the sequence end must not reach ksum
      const bool valid = (tile0 + t) * kTileTokens + r < N;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        uint4 w;
        w.x = valid ? phi2_f32<FMAP>(v[8 * c], v[8 * c + 1]) : 0u;
        w.y = valid ? phi2_f32<FMAP>(v[8 * c + 2], v[8 * c + 3]) : 0u;
        w.z = valid ? phi2_f32<FMAP>(v[8 * c + 4], v[8 * c + 5]) : 0u;
        w.w = valid ? phi2_f32<FMAP>(v[8 * c + 6], v[8 * c + 7]) : 0u;
        *reinterpret_cast<uint4*>(dst + ((c ^ (r & 7)) << 4)) = w;
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&phiready[s]);
    }
    // read-out: warps 2..5 cover the four lane quarters
    if (ok && warp < 6 && warp_wait(&accfull, 0, status)) {
      tc_fence_after();
      const size_t part = (static_cast<size_t>(bh) * nsplit + split) * 2 + fh;
      float* kvrow = part_kv + part * (kD * kFH) + static_cast<size_t>(r) * kFH;   // row r = value index d
#pragma unroll 1
      for (int c0 = 0; c0 < kFH; c0 += 32) {
        float v[32];
        tmem_ld32(tmem + kS1ColKv + c0 + lanes, v);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; e += 4)
          *reinterpret_cast<float4*>(kvrow + c0 + e) = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
      }
      const float ks = tmem_ld1(tmem + kS1ColKs + lanes);   // row r = feature index
      tmem_wait_ld();
      part_ks[part * kFH + r] = ks;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

// ====================================================== kernel 3: the apply

constexpr uint32_t kS3OffW = 0;                          // W: four 64-feature atoms [128 d][64 f]
constexpr uint32_t kS3OffImg = kS3OffW + 2 * kT32;       // [kv | ksum | 0]^T image
constexpr uint32_t kS3OffQ = kS3OffImg + kImgBytes;      // two Q tiles
constexpr uint32_t kS3Smem = kS3OffQ + 2 * kT32 + 1024;
constexpr int kS3Threads = 64 + 32 * kPhiWarps + 128;   // producer, MMA, phi, 4 output warps
constexpr uint32_t kS3ColPhi = 128, kS3ColO = 256;       // Q W half: 0..127; phi(Q) packed: 128..255; O: 256..399

template <int FMAP>
__global__ void __launch_bounds__(kS3Threads, 1)
    proj_apply_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_w,
                      const uint8_t* __restrict__ image, __nv_bfloat16* __restrict__ out, int* status, int N,
                      int H, int w_per_head, int tiles, int tps, float eps) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t wfull, imgfull, qfull[2], qempty[2], qwfull, qwfree, phiqready, phiqfree;
  __shared__ __align__(8) uint64_t ofull, oempty;
  __shared__ uint32_t tmem_slot;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.y;
  const int tile0 = blockIdx.x * tps;
  const int T = min(tiles, tile0 + tps) - tile0;   // >= 1
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* wsm = smem + kS3OffW;
  uint8_t* img = smem + kS3OffImg;

  if (threadIdx.x == 0) {
    mbar_init(&wfull, 1);
    mbar_init(&imgfull, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&qfull[i], 1);
      mbar_init(&qempty[i], 1);
    }
    mbar_init(&qwfull, 1);
    mbar_init(&qwfree, kPhiWarps);
    mbar_init(&phiqready, 2 * kPhiWarps);   // both feature halves of a tile
    mbar_init(&phiqfree, 1);
    mbar_init(&ofull, 1);
    mbar_init(&oempty, 4);
    fence_mbarrier_init();
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_w);
  }
  if (warp == 1) {
    tmem_alloc(&tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  // the image comes from the previous launch: wait before any global access
  pdl_wait();
  pdl_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const int wz = w_per_head ? bh % H : 0;
      mbar_arrive_expect_tx(&wfull, 2 * kT32);
#pragma unroll
      for (int a = 0; a < 4; ++a) tma_load_3d(wsm + a * kBoxBytes, &tm_w, &wfull, 64 * a, 0, wz);
      mbar_arrive_expect_tx(&imgfull, kImgBytes);
      bulk_load(img, image + static_cast<size_t>(bh) * kImgBytes, kImgBytes, &imgfull);
      for (int t = 0; t < T; ++t) {
        const int s = t & 1;
        if (t >= 2 && !mbar_wait(&qempty[s], ((t >> 1) - 1) & 1, status)) break;
        load_tile128(smem + kS3OffQ + s * kT32, &tm_q, &qfull[s], (tile0 + t) * kTileTokens, bh);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t id_qw = idesc_bf16_f32(128, kFH, 0, 1);   // Q W half
      constexpr uint32_t id_ap = idesc_bf16_f32(128, kNB, 0, 0);   // phi(Q) [kv | ksum]
      const uint64_t wdesc = smem_desc_sw128(smem_u32(wsm), kBoxBytes, 1024);
      const uint64_t idesc_img = smem_desc_sw128(smem_u32(img), 16, 1024);
      // Q W for feature half h of tile t (use g = 2 t + h of the one Q W
      // buffer, once the phi warps have read use g - 1)
      auto issue_qw = [&](int t, int h) -> bool {
        const int g = 2 * t + h;
        if (g > 0 && !mbar_wait(&qwfree, (g - 1) & 1, status)) return false;
        tc_fence_after();
        const uint64_t qdesc = smem_desc_sw128(smem_u32(smem + kS3OffQ + (t & 1) * kT32), 16, 1024);
        const uint64_t wh = desc_add(wdesc, h * kT32);
        umma_ss<0>(tmem, qdesc, wh, id_qw);
#pragma unroll
        for (int k = 1; k < kD / 16; ++k)
          umma_ss<1>(tmem, desc_add(qdesc, (k >> 2) * kBoxBytes + (k & 3) * 32), desc_add(wh, 2048 * k), id_qw);
        umma_commit(&qwfull);
        return true;
      };
      // Order on the tensor pipe: Q W (t, 1), Q W (t + 1, 0), then O of tile
      // t, so phi of the next tile's first half runs during O.
      bool ok = mbar_wait(&wfull, 0, status) && mbar_wait(&imgfull, 0, status) && mbar_wait(&qfull[0], 0, status) &&
                issue_qw(0, 0);
      for (int t = 0; t < T && ok; ++t) {
        const int s = t & 1;
        if (!issue_qw(t, 1)) break;
        umma_commit(&qempty[s]);
        if (t + 1 < T && (!mbar_wait(&qfull[(t + 1) & 1], ((t + 1) >> 1) & 1, status) || !issue_qw(t + 1, 0))) break;
        // O = phi(Q) [kv | ksum | 0]: 16 feature steps, A from tensor memory
        if (!mbar_wait(&phiqready, t & 1, status) || (t > 0 && !mbar_wait(&oempty, (t - 1) & 1, status))) break;
        tc_fence_after();
        umma_ts<0>(tmem + kS3ColO, tmem + kS3ColPhi, idesc_img, id_ap);
#pragma unroll
        for (int k = 1; k < kF / 16; ++k)
          umma_ts<1>(tmem + kS3ColO, tmem + kS3ColPhi + 8 * k,
                     desc_add(idesc_img, (k >> 2) * kImgAtom + (k & 3) * 32), id_ap);
        umma_commit(&phiqfree);
        umma_commit(&ofull);
      }
    }
  } else if (warp < 2 + kPhiWarps) {
    // ------------------------------------ phi warps: Q W half -> phi(Q)
    const int qd = warp & 3, hw = (warp - 2) >> 2;
    const uint32_t lanes = static_cast<uint32_t>(32 * qd) << 16;
    for (int t = 0; t < T; ++t) {
      bool ok = true;
      for (int h = 0; h < 2; ++h) {
        const int g = 2 * t + h;
        if (!warp_wait(&qwfull, g & 1, status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        float v[64];
        tmem_ld32(tmem + 64 * hw + lanes, *reinterpret_cast<float(*)[32]>(v));
        tmem_ld32(tmem + 64 * hw + 32 + lanes, *reinterpret_cast<float(*)[32]>(v + 32));
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&qwfree);
        uint32_t w[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) w[e] = phi2_f32<FMAP>(v[2 * e], v[2 * e + 1]);
        // phi of the first half is computed while the previous tile's output
        // MMAs still read phi(Q); it is stored once they are done
        if (h == 0 && t > 0 && !warp_wait(&phiqfree, (t - 1) & 1, status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // features 128 h + 64 hw .. : packed columns 64 h + 32 hw ..
        tmem_st32(tmem + kS3ColPhi + 64 * h + 32 * hw + lanes, w);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&phiqready);
      }
      if (!ok) break;
    }
  } else {
    // ------------------------------------------------------------ outputs
    const int qd = warp & 3, i = 32 * qd + lane;
    const uint32_t trow = tmem + kS3ColO + (static_cast<uint32_t>(32 * qd) << 16);
    for (int t = 0; t < T; ++t) {
      if (!warp_wait(&ofull, t & 1, status)) break;
      tc_fence_after();
      const float den = tmem_ld1(trow + kD);   // phi(q_i) . ksum
      tmem_wait_ld();
      const float inv = 1.0f / (den + eps);
      // the whole row is packed to bf16 in registers first, so that O is
      // handed back to the next tile's apply before the global stores
      uint32_t w[kD / 2];
#pragma unroll
      for (int c0 = 0; c0 < kD; c0 += 32) {
        float v[32];
        tmem_ld32(trow + c0, v);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          __nv_bfloat162 hv = __floats2bfloat162_rn(v[2 * e] * inv, v[2 * e + 1] * inv);
          w[c0 / 2 + e] = *reinterpret_cast<uint32_t*>(&hv);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&oempty);
      const int row = (tile0 + t) * kTileTokens + i;
      if (row < N) {
        uint4* dst = reinterpret_cast<uint4*>(out + (static_cast<size_t>(bh) * N + row) * kD);
#pragma unroll
        for (int c = 0; c < kD / 8; ++c) dst[c] = make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

template <int FMAP>
cudaError_t run(const LaunchArgs& a) {
  const Plan& p = *a.p;
  float* part_kv = reinterpret_cast<float*>(a.ws + p.off_partial);
  float* part_ks = reinterpret_cast<float*>(a.ws + p.off_ksum_partial);
  uint8_t* image = reinterpret_cast<uint8_t*>(a.ws + p.off_blob);
  int* status = reinterpret_cast<int*>(a.ws + p.off_status);
  const unsigned bh = static_cast<unsigned>(p.BH);
  const int w_per_head = a.w_head_stride != 0;
  cudaError_t err;
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.stream = a.stream;
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  {
    auto kern = proj_state_kernel<FMAP>;
    if ((err = ensure_smem_attr(reinterpret_cast<const void*>(kern), kS1Smem)) != cudaSuccess) return err;
    cfg.gridDim = dim3(p.splits, bh, 2);
    cfg.blockDim = dim3(kS1Threads);
    cfg.dynamicSmemBytes = kS1Smem;
    if ((err = cudaLaunchKernelEx(&cfg, kern, *a.tm_k, *a.tm_v, *a.tm_w, part_kv, part_ks, status, p.N, p.H,
                                  w_per_head, p.tiles, p.tiles_per_split)) != cudaSuccess)
      return err;
  }
  if ((err = launch_image_combine(part_kv, part_ks, image, p.BH, p.splits, kD, kFH, 2, a.stream)) != cudaSuccess)
    return err;
  auto kern = proj_apply_kernel<FMAP>;
  if ((err = ensure_smem_attr(reinterpret_cast<const void*>(kern), kS3Smem)) != cudaSuccess) return err;
  cfg.gridDim = dim3(p.apply_ctas, bh);
  cfg.blockDim = dim3(kS3Threads);
  cfg.dynamicSmemBytes = kS3Smem;
  return cudaLaunchKernelEx(&cfg, kern, *a.tm_q, *a.tm_w, static_cast<const uint8_t*>(image),
                            static_cast<__nv_bfloat16*>(a.out), status, p.N, p.H, w_per_head, p.tiles, p.apply_tps,
                            p.eps);
}

}  // namespace

cudaError_t launch_bf16_projected(const LaunchArgs& a) {
  const Plan& p = *a.p;
  if (p.D != kD || p.F != kF || p.causal) return cudaErrorNotSupported;
  return p.fmap == 0 ? run<0>(a) : run<1>(a);
}

}  // namespace la
