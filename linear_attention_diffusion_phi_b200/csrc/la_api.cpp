// la_api.cpp -- the C ABI of include/la.h: argument validation, the launch
// plan (splits and workspace layout), TMA descriptor encoding and dispatch to
// the fp32 CUDA-core or bf16 tensor-core kernels.  No device memory is ever
// allocated here; the caller owns every buffer.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <algorithm>
#include <cmath>
#include <mutex>

#include "la.h"
#include "la_internal.h"

struct la_handle_s {
  int dtype;
  const void* W;
  int wH, wD, wF;
  long long w_head_stride;
  // attention prologue (la_set_prologue); pro_q == nullptr: none
  const float* pro_q;
  const float* pro_k;
  const float* pro_rope;
  int pro_D, pro_npos;
  float pro_eps;
  void* ws;
  size_t ws_bytes;
  // The status word of a newly bound workspace is cleared by the next call
  // that uses it, on that call's stream (no device-wide synchronisation).
  bool ws_clear_pending;
};

namespace {

using la::Plan;

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }
long long cdiv(long long a, long long b) { return (a + b - 1) / b; }

struct DeviceInfo {
  int sms = 0, major = 0, minor = 0;
};

// SM count and compute capability of the current device (cached per device).
bool device_info(DeviceInfo* out) {
  static std::mutex mu;
  static DeviceInfo cache[64];
  static bool have[64] = {};
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return false;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (!have[dev]) {
    DeviceInfo d;
    if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
      cudaGetLastError();
      return false;
    }
    cache[dev] = d;
    have[dev] = true;
  }
  *out = cache[dev];
  return true;
}

// Whether the bf16 tensor-core kernels cover a shape: non-causal D = 64 or
// 128 (projected only at D = 128, F = 256) and causal D = 64 without
// projection.  Other valid bf16 shapes run widened on the fp32 kernels, so
// the plan, and the workspace, depend on the shape alone.
bool bf16_native(int D, int F, int causal) {
  if (D != 64 && D != 128) return false;
  if (F != 0 && (F != 256 || D != 128)) return false;
  if (causal && (F != 0 || D != 64)) return false;
  return true;
}

// Shape/dtype validation shared by la_workspace_bytes and la_forward.
la_status_t check_shape(const la_handle_s* h, int B, int H, int N, int D, int F, int fmap, float eps,
                        int causal) {
  if (B < 0 || H < 0 || N < 0 || D <= 0 || F < 0) return LA_ERR_INVALID_ARG;
  if (fmap != LA_PHI_ELU1 && fmap != LA_PHI_RELU && fmap != LA_PHI_SOFTMAX) return LA_ERR_INVALID_ARG;
  if (!(eps >= 0.f) || eps != eps) return LA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return LA_ERR_INVALID_ARG;
  if (F % 256 != 0) return LA_ERR_INVALID_ARG;   // feature_dim: a multiple of 256
  if (static_cast<long long>(B) * H > 65535) return LA_ERR_UNSUPPORTED;
  // the fp32 kernels' range (bf16 shapes outside the bf16 kernels' run there,
  // widened)
  const bool native = h->dtype == LA_BF16 && bf16_native(D, F, causal);
  if (!native) {
    // fp32 kernels: features in groups of 256 (non-causal, up to 4096); the
    // causal state of 256 features x D fills the shared memory
    if (D > 128 || D % 4 != 0) return LA_ERR_UNSUPPORTED;
    if (F > 4096 || (causal && F > 256)) return LA_ERR_UNSUPPORTED;
  }
  // softmax over each row's features: no projection; among the bf16 kernels
  // only the non-causal D = 128 one
  if (fmap == LA_PHI_SOFTMAX && (F != 0 || (native && (causal || D != 128)))) return LA_ERR_UNSUPPORTED;
  return LA_OK;
}

void make_plan(const la_handle_s* h, int B, int H, int N, int D, int F, int fmap, float eps, int causal,
               int num_sms, Plan* p) {
  memset(p, 0, sizeof(*p));
  p->dtype = h->dtype;
  p->B = B; p->H = H; p->N = N; p->D = D; p->F = F;
  p->Fe = F ? F : D;
  p->fmap = fmap; p->causal = causal; p->eps = eps;
  p->BH = static_cast<long long>(B) * H;
  p->tiles = static_cast<int>(cdiv(N, la::kTileTokens));
  p->num_sms = num_sms > 0 ? num_sms : 148;
  const long long BH = std::max<long long>(p->BH, 1);
  size_t partial_floats = 0, ksum_floats = 0, final_bytes = 0, final_ksum_bytes = 0, blob_total = 0, xchg_bytes = 0;
  p->widened = h->dtype == LA_BF16 && !bf16_native(D, F, causal);
  if (h->dtype == LA_F32 || p->widened) {
    // Enough (head, split, feature-block) blocks for ~2 waves; splits of whole
    // 16-token chunks (non-causal) or >= 64 tokens (causal).
    const long long fblocks = cdiv(p->Fe, 32);
    long long want = std::max<long long>(1, cdiv(2LL * p->num_sms, BH * (causal ? 1 : fblocks)));
    const int quantum = causal ? 64 : 16;
    long long seg = std::max<long long>(quantum, cdiv(cdiv(std::max(N, 1), want), quantum) * quantum);
    p->seg_len = static_cast<int>(seg);
    p->splits = static_cast<int>(std::max<long long>(1, cdiv(std::max(N, 1), seg)));
    partial_floats = static_cast<size_t>(BH) * p->splits * p->Fe * D;
    ksum_floats = static_cast<size_t>(BH) * p->splits * p->Fe;
    if (!causal) {
      final_bytes = static_cast<size_t>(BH) * p->Fe * D * 4;
      final_ksum_bytes = static_cast<size_t>(BH) * p->Fe * 4;
    }
  } else if (!causal && F == 0) {
    // Each head is split over clusters of CTAs chosen from the device's
    // cluster occupancy; the combine runs through distributed shared memory
    // inside a cluster and, where a head spans several clusters, through an
    // exchange area in the workspace.
    la::noncausal_geometry(p, &xchg_bytes);
  } else if (causal) {
    // Segments of whole 128-token chunks, about one CTA per SM in all; every
    // segment but the last leaves its state sum, [D + 1][D] fp32.
    const int tiles = std::max(p->tiles, 1);
    const long long want = std::max<long long>(1, p->num_sms / BH);
    p->tiles_per_split = static_cast<int>(cdiv(tiles, std::min<long long>(want, tiles)));
    p->splits = static_cast<int>(cdiv(tiles, p->tiles_per_split));
    p->seg_len = p->tiles_per_split * la::kTileTokens;
    // with one segment per head no state is written or read
    if (p->splits > 1) partial_floats = static_cast<size_t>(BH) * p->splits * (D + 1) * D;
  } else {
    // Projected (D = 128, F = 256): state CTAs per (split, head, feature
    // half), about one per SM; apply CTAs about one per SM. Partials are fp32
    // kv^T [D][F/2] and ksum [F/2] per (head, split, half); the image is the
    // apply's bf16 [kv | ksum | 0]^T operand, [D + 16][F] per head.
    const int tiles = std::max(p->tiles, 1);
    const long long want = std::max<long long>(1, p->num_sms / (2 * BH));
    p->tiles_per_split = static_cast<int>(cdiv(tiles, std::min<long long>(want, tiles)));
    p->splits = static_cast<int>(cdiv(tiles, p->tiles_per_split));
    p->seg_len = p->tiles_per_split * la::kTileTokens;
    const long long want3 = std::max<long long>(1, p->num_sms / BH);
    p->apply_tps = static_cast<int>(cdiv(tiles, std::min<long long>(want3, tiles)));
    p->apply_ctas = static_cast<int>(cdiv(tiles, p->apply_tps));
    partial_floats = static_cast<size_t>(BH) * p->splits * p->Fe * D;
    ksum_floats = static_cast<size_t>(BH) * p->splits * p->Fe;
    p->blob_bytes = static_cast<size_t>(D + 16) * p->Fe * 2;
    blob_total = static_cast<size_t>(BH) * p->blob_bytes;
  }
  size_t off = 0;
  p->off_status = off;        off += la::kStatusBytes;
  p->off_sync = off;          off += la::kSyncBytes;
  p->off_partial = off;       off = align256(off + partial_floats * 4);
  p->off_ksum_partial = off;  off = align256(off + ksum_floats * 4);
  p->off_final = off;         off = align256(off + final_bytes);
  p->off_final_ksum = off;    off = align256(off + final_ksum_bytes);
  p->off_blob = off;          off = align256(off + blob_total);
  p->off_xchg = off;          off = align256(off + xchg_bytes);
  if (p->widened) {
    // fp32 copies of q, k, v, out and W (W with its head stride)
    const size_t n = static_cast<size_t>(BH) * std::max(N, 1) * D;
    p->w_elems = F == 0 ? 0
                        : (h->w_head_stride ? static_cast<size_t>(std::max(H, 1) - 1) * h->w_head_stride : 0) +
                              static_cast<size_t>(D) * F;
    p->off_wq = off;            off = align256(off + n * 4);
    p->off_wk = off;            off = align256(off + n * 4);
    p->off_wv = off;            off = align256(off + n * 4);
    p->off_wo = off;            off = align256(off + n * 4);
    p->off_wW = off;            off = align256(off + p->w_elems * 4);
  }
  p->bytes = off;
}

// ------------------------------------------------------------ tensor maps

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
    cudaGetLastError();
  });
  return fn;
}

// [outer, rows, cols] bf16 tensor, box [1, 128, 64] with the 128-byte swizzle.
bool encode_bf16_3d(CUtensorMap* m, const void* base, long long outer, long long rows, long long cols,
                    long long outer_stride_elems, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(outer)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(cols) * 2, static_cast<cuuint64_t>(outer_stride_elems) * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// [outer, rows, cols] tensor of bytes (E4M3 codes), box [1, 128, 128] with
// the 128-byte swizzle: one box is a whole 128 x 128 tile.
bool encode_u8_3d(CUtensorMap* m, const void* base, long long outer, long long rows, long long cols,
                  long long outer_stride_elems) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(outer)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(outer_stride_elems)};
  cuuint32_t box[3] = {128, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

namespace la {

// Whether `p` is device (or managed) memory of the current device.  A
// pointer the runtime does not know (plain host memory) or one of another
// device is refused before anything is launched: a kernel given it would
// fault or read the wrong memory.
bool on_current_device(const void* p) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  cudaPointerAttributes attr;
  if (cudaPointerGetAttributes(&attr, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  if (attr.type == cudaMemoryTypeManaged) return true;
  return attr.type == cudaMemoryTypeDevice && attr.device == dev;
}

}  // namespace la

namespace la {

// Plan of the fused kernel for la_forward_noalloc: the same geometry as
// la_forward's (so both give the same bits); the scratch holds the header and
// the exchange area between the clusters of a head.
void plan_bf16_noncausal(int B, int H, int N, int D, int fmap, float eps, int num_sms, Plan* p) {
  memset(p, 0, sizeof(*p));
  p->dtype = LA_BF16;
  p->B = B; p->H = H; p->N = N; p->D = D; p->F = 0; p->Fe = D;
  p->fmap = fmap; p->causal = 0; p->eps = eps;
  p->BH = static_cast<long long>(B) * H;
  p->tiles = static_cast<int>(cdiv(N, la::kTileTokens));
  p->num_sms = num_sms > 0 ? num_sms : 148;
  size_t xchg_bytes = 0;
  la::noncausal_geometry(p, &xchg_bytes);
  size_t off = 0;
  p->off_status = off;        off += la::kStatusBytes;
  p->off_sync = off;          off += la::kSyncBytes;
  p->off_partial = p->off_ksum_partial = p->off_final = p->off_final_ksum = p->off_blob = off;
  p->off_xchg = off;          off = align256(off + xchg_bytes);
  p->bytes = off;
}

bool encode_tile_map_bf16(CUtensorMap* m, const void* base, long long outer, long long rows, long long cols,
                          long long outer_stride_elems) {
  return encode_bf16_3d(m, base, outer, rows, cols, outer_stride_elems, 128);
}

cudaError_t ensure_smem_attr(const void* kernel, uint32_t bytes) {
  static std::mutex mu;
  static const void* done_fn[256];
  static int done_dev[256];
  static int n_done = 0;
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < n_done; ++i)
    if (done_fn[i] == kernel && done_dev[i] == dev) return cudaSuccess;
  err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
  if (err == cudaSuccess && n_done < 256) {
    done_fn[n_done] = kernel;
    done_dev[n_done] = dev;
    ++n_done;
  }
  return err;
}

bool overlap(const void* a, size_t an, const void* b, size_t bn) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return an != 0 && bn != 0 && x < y + bn && y < x + an;
}

bool current_sm100(int* num_sms) {
  DeviceInfo di;
  if (!device_info(&di) || di.major != 10 || di.minor != 0) return false;
  *num_sms = di.sms;
  return true;
}

}  // namespace la

extern "C" {

la_status_t la_create(la_handle_t* handle, int dtype) {
  if (!handle) return LA_ERR_INVALID_ARG;
  *handle = nullptr;
  if (dtype != LA_F32 && dtype != LA_BF16) return LA_ERR_INVALID_ARG;
  la_handle_s* h = new (std::nothrow) la_handle_s();
  if (!h) return LA_ERR_INVALID_ARG;
  h->dtype = dtype;
  *handle = h;
  return LA_OK;
}

la_status_t la_destroy(la_handle_t handle) {
  if (!handle) return LA_ERR_INVALID_ARG;
  delete handle;
  return LA_OK;
}

la_status_t la_set_prologue(la_handle_t h, const float* q_scale, const float* k_scale, const float* rope, int D,
                            int n_positions, float norm_eps) {
  if (!h) return LA_ERR_INVALID_ARG;
  if (!q_scale) {
    h->pro_q = h->pro_k = h->pro_rope = nullptr;
    h->pro_D = h->pro_npos = 0;
    return LA_OK;
  }
  if (!k_scale || !rope || D <= 0 || D % 2 != 0 || n_positions <= 0) return LA_ERR_INVALID_ARG;
  if (!(norm_eps >= 0.f) || !std::isfinite(norm_eps)) return LA_ERR_INVALID_ARG;
  if (!aligned16(q_scale) || !aligned16(k_scale) || !aligned16(rope)) return LA_ERR_MISALIGNED;
  h->pro_q = q_scale;
  h->pro_k = k_scale;
  h->pro_rope = rope;
  h->pro_D = D;
  h->pro_npos = n_positions;
  h->pro_eps = norm_eps;
  return LA_OK;
}

la_status_t la_set_projection(la_handle_t h, const void* W, int H, int D, int F, long long head_stride) {
  if (!h) return LA_ERR_INVALID_ARG;
  if (!W) {
    h->W = nullptr;
    h->wH = h->wD = h->wF = 0;
    h->w_head_stride = 0;
    return LA_OK;
  }
  if (H <= 0 || D <= 0 || F <= 0 || F % 256 != 0 || head_stride < 0) return LA_ERR_INVALID_ARG;
  if (head_stride != 0 && head_stride < static_cast<long long>(D) * F) return LA_ERR_INVALID_ARG;
  if (!aligned16(W) || head_stride % 8 != 0) return LA_ERR_MISALIGNED;
  h->W = W;
  h->wH = H;
  h->wD = D;
  h->wF = F;
  h->w_head_stride = head_stride;
  return LA_OK;
}

size_t la_workspace_bytes(la_handle_t h, int B, int H, int N, int D, int F, int causal) {
  if (!h) return 0;
  if (check_shape(h, B, H, N, D, F, LA_PHI_ELU1, 0.f, causal) != LA_OK) return 0;
  DeviceInfo di;
  const int sms = device_info(&di) ? di.sms : 148;
  Plan p;
  make_plan(h, B, H, N, D, F, LA_PHI_ELU1, 0.f, causal, sms, &p);
  return p.bytes;
}

la_status_t la_set_workspace(la_handle_t h, void* ptr, size_t bytes) {
  if (!h) return LA_ERR_INVALID_ARG;
  if (!ptr || bytes == 0) {
    h->ws = nullptr;
    h->ws_bytes = 0;
    return LA_OK;
  }
  if ((reinterpret_cast<uintptr_t>(ptr) & 255u) != 0) return LA_ERR_MISALIGNED;
  if (bytes < la::kHeaderBytes) return LA_ERR_WORKSPACE;
  // The status word is cleared by the next la_forward (or la_sync_status)
  // on its own stream, so later reads see only errors of calls made with
  // this workspace; nothing is enqueued here.
  h->ws = ptr;
  h->ws_bytes = bytes;
  h->ws_clear_pending = true;
  return LA_OK;
}

namespace {

// la_forward, and with `gate` the landmark branch of la_forward_ttr blended
// into out right after the kernel branch (same stream, same tensor maps);
// with `scales` (q, k, v scales) the inputs are E4M3 codes (la_forward_e4m3).
la_status_t forward_impl(la_handle_t h, const void* q, const void* k, const void* v, void* out, int B, int H,
                         int N, int D, int F, int fmap, float eps, int causal, void* stream, const void* gate,
                         int n_landmarks, const float* scales = nullptr) {
  if (!h) return LA_ERR_INVALID_ARG;
  la_status_t st = check_shape(h, B, H, N, D, F, fmap, eps, causal);
  if (st != LA_OK) return st;
  if (static_cast<long long>(B) * H * N == 0) return LA_OK;
  if (!q || !k || !v || !out) return LA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return LA_ERR_MISALIGNED;
  if (F > 0) {
    if (!h->W) return LA_ERR_INVALID_ARG;
    if (h->wD != D || h->wF != F || (h->w_head_stride != 0 && h->wH < H)) return LA_ERR_INVALID_ARG;
  }
  const bool pro = h->pro_q != nullptr;
  if (pro) {
    if (h->pro_D != D || N > h->pro_npos) return LA_ERR_INVALID_ARG;
    const bool fits = F == 0 && !gate && !scales &&
                      (h->dtype == LA_F32 || !bf16_native(D, F, causal) ||
                       (D == 128 && !causal && fmap != LA_PHI_SOFTMAX));
    if (!fits) return LA_ERR_UNSUPPORTED;
  }
  // The kernels write out and the workspace while q, k, v and W are still
  // being read, so neither may share a byte with them or with each other; q,
  // k and v are only read and may coincide.
  {
    const size_t es = h->dtype == LA_F32 ? 4 : 2;
    const size_t nb = static_cast<size_t>(B) * H * N * D * es;
    const size_t nin = static_cast<size_t>(B) * H * N * D * (scales ? 1 : es);   // bytes of q, k or v
    const size_t wb = F == 0 ? 0
                      : (h->w_head_stride ? static_cast<size_t>(H - 1) * h->w_head_stride : 0) * es +
                            static_cast<size_t>(D) * F * es;
    const void* ins[3] = {q, k, v};
    for (const void* x : ins) {
      if (la::overlap(out, nb, x, nin)) return LA_ERR_INVALID_ARG;
      if (h->ws && la::overlap(h->ws, h->ws_bytes, x, nin)) return LA_ERR_INVALID_ARG;
    }
    if (F > 0 && la::overlap(out, nb, h->W, wb)) return LA_ERR_INVALID_ARG;
    if (pro) {   // out is written while the prologue's scales and table are read
      const size_t sb = static_cast<size_t>(D) * 4, rb = static_cast<size_t>(h->pro_npos) * D * 4;
      if (la::overlap(out, nb, h->pro_q, sb) || la::overlap(out, nb, h->pro_k, sb) ||
          la::overlap(out, nb, h->pro_rope, rb))
        return LA_ERR_INVALID_ARG;
    }
    if (h->ws && (la::overlap(h->ws, h->ws_bytes, out, nb) || (F > 0 && la::overlap(h->ws, h->ws_bytes, h->W, wb))))
      return LA_ERR_INVALID_ARG;
  }
  DeviceInfo di;
  if (!device_info(&di)) return LA_ERR_NO_DEVICE;
  if (di.major != 10 || di.minor != 0) return LA_ERR_NO_DEVICE;   // kernels are built for sm_100a
  Plan p;
  make_plan(h, B, H, N, D, F, fmap, eps, causal, di.sms, &p);
  if (p.widened && (gate || scales)) return LA_ERR_UNSUPPORTED;
  if (!h->ws || h->ws_bytes < p.bytes) return LA_ERR_WORKSPACE;
  if (!la::on_current_device(q) || !la::on_current_device(k) || !la::on_current_device(v) ||
      !la::on_current_device(out) || !la::on_current_device(h->ws) || (F > 0 && !la::on_current_device(h->W)))
    return LA_ERR_INVALID_ARG;
  if (pro && (!la::on_current_device(h->pro_q) || !la::on_current_device(h->pro_k) ||
              !la::on_current_device(h->pro_rope)))
    return LA_ERR_INVALID_ARG;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  if (h->ws_clear_pending) {
    if (cudaMemsetAsync(h->ws, 0, la::kHeaderBytes, cs) != cudaSuccess) {
      cudaGetLastError();
      return LA_ERR_CUDA;
    }
    h->ws_clear_pending = false;
  }

  la::LaunchArgs a = {};
  a.p = &p;
  a.q = q; a.k = k; a.v = v; a.out = out;
  a.W = F ? h->W : nullptr;
  a.w_head_stride = h->w_head_stride;
  a.ws = static_cast<char*>(h->ws);
  a.stream = cs;
  a.prologue = pro;
  a.pro_q = h->pro_q;
  a.pro_k = h->pro_k;
  a.pro_rope = h->pro_rope;
  a.pro_eps = h->pro_eps;

  cudaError_t err;
  if (h->dtype == LA_F32) {
    err = la::launch_f32(a);
  } else if (p.widened) {
    // widen q, k, v (and W) into the workspace, run the fp32 kernels there
    // and round their output back to bf16
    const size_t n = static_cast<size_t>(B) * H * N * D;
    float* wq = reinterpret_cast<float*>(a.ws + p.off_wq);
    float* wk = reinterpret_cast<float*>(a.ws + p.off_wk);
    float* wv = reinterpret_cast<float*>(a.ws + p.off_wv);
    float* wo = reinterpret_cast<float*>(a.ws + p.off_wo);
    float* wW = reinterpret_cast<float*>(a.ws + p.off_wW);
    err = la::launch_bf16_to_f32(q, wq, n, cs);
    if (err == cudaSuccess) err = la::launch_bf16_to_f32(k, wk, n, cs);
    if (err == cudaSuccess) err = la::launch_bf16_to_f32(v, wv, n, cs);
    if (err == cudaSuccess && F > 0) err = la::launch_bf16_to_f32(h->W, wW, p.w_elems, cs);
    if (err == cudaSuccess) {
      a.q = wq; a.k = wk; a.v = wv; a.out = wo;
      a.W = F ? wW : nullptr;
      err = la::launch_f32(a);
    }
    if (err == cudaSuccess) err = la::launch_f32_to_bf16(wo, out, n, cs);
  } else {
    CUtensorMap tq, tk, tv, to, tw;
    const long long BH = p.BH;
    const long long hs = static_cast<long long>(N) * D;
    if (scales) {
      if (!encode_u8_3d(&tq, q, BH, N, D, hs) || !encode_u8_3d(&tk, k, BH, N, D, hs) ||
          !encode_u8_3d(&tv, v, BH, N, D, hs) || !encode_bf16_3d(&to, out, BH, N, D, hs, 128))
        return LA_ERR_CUDA;
      a.e4m3 = true;
      a.scale_q = scales[0]; a.scale_k = scales[1]; a.scale_v = scales[2];
    } else if (!encode_bf16_3d(&tq, q, BH, N, D, hs, 128) || !encode_bf16_3d(&tk, k, BH, N, D, hs, 128) ||
               !encode_bf16_3d(&tv, v, BH, N, D, hs, 128) || !encode_bf16_3d(&to, out, BH, N, D, hs, 128)) {
      return LA_ERR_CUDA;
    }
    a.tm_q = &tq; a.tm_k = &tk; a.tm_v = &tv; a.tm_out = &to;
    if (F > 0) {
      const long long nW = h->w_head_stride ? H : 1;
      const long long ws = h->w_head_stride ? h->w_head_stride : static_cast<long long>(D) * F;
      if (!encode_bf16_3d(&tw, h->W, nW, D, F, ws, 128)) return LA_ERR_CUDA;
      a.tm_w = &tw;
    }
    err = causal ? la::launch_bf16_causal(a) : (F > 0 ? la::launch_bf16_projected(a) : la::launch_bf16_noncausal(a));
    if (err == cudaSuccess && gate) err = la::launch_bf16_landmark(a, gate, n_landmarks);
  }
  if (err == cudaErrorNotSupported) return LA_ERR_UNSUPPORTED;
  if (err != cudaSuccess) {
    cudaGetLastError();
    return LA_ERR_CUDA;
  }
  return LA_OK;
}

}  // namespace

la_status_t la_forward(la_handle_t h, const void* q, const void* k, const void* v, void* out, int B, int H, int N,
                       int D, int F, int fmap, float eps, int causal, void* stream) {
  return forward_impl(h, q, k, v, out, B, H, N, D, F, fmap, eps, causal, stream, nullptr, 0);
}

la_status_t la_forward_e4m3(la_handle_t h, const void* q, const void* k, const void* v, float scale_q,
                            float scale_k, float scale_v, void* out, int B, int H, int N, int D, int fmap, float eps,
                            void* stream) {
  if (!h) return LA_ERR_INVALID_ARG;
  la_status_t st = check_shape(h, B, H, N, D, 0, fmap, eps, 0);
  if (st != LA_OK) return st;
  const float sc[3] = {scale_q, scale_k, scale_v};
  for (float x : sc)
    if (!(x > 0.f) || !std::isfinite(x)) return LA_ERR_INVALID_ARG;
  if (h->dtype != LA_BF16 || D != 128 || fmap == LA_PHI_SOFTMAX) return LA_ERR_UNSUPPORTED;
  return forward_impl(h, q, k, v, out, B, H, N, D, 0, fmap, eps, 0, stream, nullptr, 0, sc);
}

namespace {

// The backward's workspace: the forward plan of the same shape, then the
// query pass's per-split [D][D] dkv and [D] dz partials (splits of whole
// 16-token chunks, about two blocks per SM in all), then their sums.
struct BwdLayout {
  int splits, seg;
  size_t off_part, off_part_z, off_fin, off_fin_z, bytes;
};
size_t backward_plan(la_handle_t h, int B, int H, int N, int D, int fmap, float eps, int sms, Plan* p,
                     BwdLayout* b) {
  make_plan(h, B, H, N, D, 0, fmap, eps, 0, sms, p);
  const long long BH = std::max<long long>(p->BH, 1);
  const long long want = std::max<long long>(1, cdiv(2LL * sms, BH));
  b->seg = static_cast<int>(std::max<long long>(16, cdiv(cdiv(std::max(N, 1), want), 16) * 16));
  b->splits = static_cast<int>(std::max<long long>(1, cdiv(std::max(N, 1), b->seg)));
  b->off_part = align256(p->bytes);
  b->off_part_z = align256(b->off_part + static_cast<size_t>(BH) * b->splits * D * D * 4);
  b->off_fin = align256(b->off_part_z + static_cast<size_t>(BH) * b->splits * D * 4);
  b->off_fin_z = align256(b->off_fin + static_cast<size_t>(BH) * D * D * 4);
  b->bytes = align256(b->off_fin_z + static_cast<size_t>(BH) * D * 4);
  return b->bytes;
}

la_status_t check_backward(la_handle_t h, int B, int H, int N, int D, int fmap, float eps) {
  if (!h) return LA_ERR_INVALID_ARG;
  la_status_t st = check_shape(h, B, H, N, D, 0, fmap, eps, 0);
  if (st != LA_OK) return st;
  if (h->dtype != LA_F32 || fmap == LA_PHI_SOFTMAX || h->pro_q) return LA_ERR_UNSUPPORTED;
  return LA_OK;
}

}  // namespace

size_t la_backward_workspace_bytes(la_handle_t h, int B, int H, int N, int D) {
  if (check_backward(h, B, H, N, D, LA_PHI_ELU1, 0.f) != LA_OK) return 0;
  DeviceInfo di;
  const int sms = device_info(&di) ? di.sms : 148;
  Plan p;
  BwdLayout b;
  return backward_plan(h, B, H, N, D, LA_PHI_ELU1, 0.f, sms, &p, &b);
}

la_status_t la_backward(la_handle_t h, const void* q, const void* k, const void* v, const void* dout, void* dq,
                        void* dk, void* dv, int B, int H, int N, int D, int fmap, float eps, void* stream) {
  la_status_t st = check_backward(h, B, H, N, D, fmap, eps);
  if (st != LA_OK) return st;
  if (static_cast<long long>(B) * H * N == 0) return LA_OK;
  const void* ins[4] = {q, k, v, dout};
  void* outs[3] = {dq, dk, dv};
  for (const void* x : ins)
    if (!x) return LA_ERR_INVALID_ARG;
  for (void* x : outs)
    if (!x) return LA_ERR_INVALID_ARG;
  for (const void* x : ins)
    if (!aligned16(x)) return LA_ERR_MISALIGNED;
  for (void* x : outs)
    if (!aligned16(x)) return LA_ERR_MISALIGNED;
  const size_t nb = static_cast<size_t>(B) * H * N * D * 4;
  // the outputs are written while the inputs are read: no output shares a
  // byte with an input, another output or the workspace
  for (int i = 0; i < 3; ++i) {
    for (const void* x : ins)
      if (la::overlap(outs[i], nb, x, nb)) return LA_ERR_INVALID_ARG;
    for (int j = i + 1; j < 3; ++j)
      if (la::overlap(outs[i], nb, outs[j], nb)) return LA_ERR_INVALID_ARG;
    if (h->ws && la::overlap(h->ws, h->ws_bytes, outs[i], nb)) return LA_ERR_INVALID_ARG;
  }
  for (const void* x : ins)
    if (h->ws && la::overlap(h->ws, h->ws_bytes, x, nb)) return LA_ERR_INVALID_ARG;
  DeviceInfo di;
  if (!device_info(&di)) return LA_ERR_NO_DEVICE;
  if (di.major != 10 || di.minor != 0) return LA_ERR_NO_DEVICE;
  Plan p;
  BwdLayout bl;
  const size_t need = backward_plan(h, B, H, N, D, fmap, eps, di.sms, &p, &bl);
  if (!h->ws || h->ws_bytes < need) return LA_ERR_WORKSPACE;
  for (const void* x : ins)
    if (!la::on_current_device(x)) return LA_ERR_INVALID_ARG;
  for (void* x : outs)
    if (!la::on_current_device(x)) return LA_ERR_INVALID_ARG;
  if (!la::on_current_device(h->ws)) return LA_ERR_INVALID_ARG;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  if (h->ws_clear_pending) {
    if (cudaMemsetAsync(h->ws, 0, la::kHeaderBytes, cs) != cudaSuccess) {
      cudaGetLastError();
      return LA_ERR_CUDA;
    }
    h->ws_clear_pending = false;
  }
  la::LaunchArgs a = {};
  a.p = &p;
  a.q = q; a.k = k; a.v = v;
  a.ws = static_cast<char*>(h->ws);
  a.stream = cs;
  char* ws = static_cast<char*>(h->ws);
  const cudaError_t err = la::launch_f32_backward(
      a, dout, dq, dk, dv, bl.splits, bl.seg, reinterpret_cast<float*>(ws + bl.off_part),
      reinterpret_cast<float*>(ws + bl.off_part_z), reinterpret_cast<float*>(ws + bl.off_fin),
      reinterpret_cast<float*>(ws + bl.off_fin_z));
  if (err == cudaErrorNotSupported) return LA_ERR_UNSUPPORTED;
  if (err != cudaSuccess) {
    cudaGetLastError();
    return LA_ERR_CUDA;
  }
  return LA_OK;
}

int la_landmark_count(int N, float fraction, int min_count, int max_count) {
  if (N < 1 || !(fraction >= 0.f) || min_count < 0 || max_count < 1) return 0;
  const double want = std::floor(static_cast<double>(fraction) * N + 0.5);
  long long n = want > 2e9 ? 2000000000LL : static_cast<long long>(want);
  n = std::max<long long>(min_count, std::min<long long>(max_count, n));
  return static_cast<int>(std::max<long long>(1, std::min<long long>(N, n)));
}

la_status_t la_forward_ttr(la_handle_t h, const void* q, const void* k, const void* v, void* out, int B, int H,
                           int N, int D, int F, int fmap, float eps, int n_landmarks, const float* gate,
                           void* stream) {
  if (!h) return LA_ERR_INVALID_ARG;
  la_status_t st = check_shape(h, B, H, N, D, F, fmap, eps, 0);
  if (st != LA_OK) return st;
  if (h->dtype != LA_BF16 || D != 128) return LA_ERR_UNSUPPORTED;
  if (static_cast<long long>(B) * H * N == 0) return LA_OK;
  if (n_landmarks < 1 || n_landmarks > N) return LA_ERR_INVALID_ARG;
  if (n_landmarks > 128) return LA_ERR_UNSUPPORTED;
  if (!gate || (reinterpret_cast<uintptr_t>(gate) & 3u) != 0) return LA_ERR_INVALID_ARG;
  // out is rewritten by the blend while every CTA reads the gate logits
  const size_t nb = static_cast<size_t>(B) * H * N * D * 2;
  if (out && la::overlap(out, nb, gate, static_cast<size_t>(H) * 4)) return LA_ERR_INVALID_ARG;
  if (h->ws && la::overlap(h->ws, h->ws_bytes, gate, static_cast<size_t>(H) * 4)) return LA_ERR_INVALID_ARG;
  int sms = 0;
  if (la::current_sm100(&sms) && !la::on_current_device(gate)) return LA_ERR_INVALID_ARG;
  return forward_impl(h, q, k, v, out, B, H, N, D, F, fmap, eps, 0, stream, gate, n_landmarks);
}

la_status_t la_forward_host(la_handle_t h, const void* q_host, const void* k_host, const void* v_host,
                            void* out_host, void* dq, void* dk, void* dv, void* dout, int B, int H, int N, int D,
                            int F, int fmap, float eps, int causal, void* stream) {
  if (!h) return LA_ERR_INVALID_ARG;
  la_status_t st = check_shape(h, B, H, N, D, F, fmap, eps, causal);
  if (st != LA_OK) return st;
  const size_t n = static_cast<size_t>(B) * H * N * D * (h->dtype == LA_F32 ? 4 : 2);
  if (n == 0) return LA_OK;
  if (!q_host || !k_host || !v_host || !out_host) return LA_ERR_INVALID_ARG;
  if (!dq || !dk || !dv || !dout) return LA_ERR_INVALID_ARG;
  // dq, dk and dv are copy destinations and dout the output: all disjoint
  void* const dev[4] = {dq, dk, dv, dout};
  for (int i = 0; i < 4; ++i)
    for (int j = i + 1; j < 4; ++j)
      if (la::overlap(dev[i], n, dev[j], n)) return LA_ERR_INVALID_ARG;
  for (int i = 0; i < 4; ++i)
    if (!la::on_current_device(dev[i])) return LA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(dq, q_host, n, cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaMemcpyAsync(dk, k_host, n, cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaMemcpyAsync(dv, v_host, n, cudaMemcpyHostToDevice, s) != cudaSuccess) {
    cudaGetLastError();
    return LA_ERR_CUDA;
  }
  st = la_forward(h, dq, dk, dv, dout, B, H, N, D, F, fmap, eps, causal, stream);
  if (st != LA_OK) return st;
  if (cudaMemcpyAsync(out_host, dout, n, cudaMemcpyDeviceToHost, s) != cudaSuccess) {
    cudaGetLastError();
    return LA_ERR_CUDA;
  }
  return LA_OK;
}

la_status_t la_sync_status(la_handle_t h, void* stream) {
  if (!h) return LA_ERR_INVALID_ARG;
  if (!h->ws) return LA_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (h->ws_clear_pending) {   // no call has used this workspace yet
    if (cudaMemsetAsync(h->ws, 0, la::kHeaderBytes, s) != cudaSuccess || cudaStreamSynchronize(s) != cudaSuccess) {
      cudaGetLastError();
      return LA_ERR_CUDA;
    }
    h->ws_clear_pending = false;
    return LA_OK;
  }
  int word = 0;
  if (cudaMemcpyAsync(&word, h->ws, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess) {
    cudaGetLastError();
    return LA_ERR_CUDA;
  }
  if (word == 0) return LA_OK;
  // An abandoned wait can leave barrier counts mid-way: clear the header,
  // ordered on the same stream.
  if (cudaMemsetAsync(h->ws, 0, la::kHeaderBytes, s) != cudaSuccess || cudaStreamSynchronize(s) != cudaSuccess) {
    cudaGetLastError();
    return LA_ERR_CUDA;
  }
  return word == la::kDeviceTimeout ? LA_ERR_TIMEOUT : LA_ERR_CUDA;
}

const char* la_status_string(la_status_t s) {
  switch (s) {
    case LA_OK: return "ok";
    case LA_ERR_INVALID_ARG: return "invalid argument";
    case LA_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case LA_ERR_MISALIGNED: return "pointer not 16-byte aligned";
    case LA_ERR_WORKSPACE: return "workspace missing or too small";
    case LA_ERR_CUDA: return "CUDA error";
    case LA_ERR_TIMEOUT: return "device-side wait timed out";
    case LA_ERR_NO_DEVICE: return "no sm_100 device current";
  }
  return "unknown status";
}

int la_version(void) { return 100; }

}  // extern "C"
