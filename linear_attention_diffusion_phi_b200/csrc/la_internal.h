// la_internal.h -- plan and launcher declarations shared by the host code and
// the kernel translation units of the linear-attention library.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace la {

// Device-side wait limit: a kernel that waits this long on one barrier gives up.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s
constexpr int kDeviceTimeout = 6;                            // == LA_ERR_TIMEOUT

constexpr int kTileTokens = 128;   // tokens per tensor-core tile (MMA M or K)

// Workspace header, zeroed by the first call that uses a newly bound
// workspace: a 256-byte status area, then the synchronisation words of the
// bf16 non-causal kernel's exchange between clusters (a launch counter, a
// done counter and one flag per CTA; see bf16_noncausal.cu).
constexpr size_t kStatusBytes = 256;
constexpr size_t kSyncBytes = 4096;
constexpr size_t kHeaderBytes = kStatusBytes + kSyncBytes;
constexpr int kSyncFlags = static_cast<int>(kSyncBytes / 4) - 2;   // CTAs a cross-cluster launch may have

// Everything la_forward decides on the host, shared with la_workspace_bytes.
struct Plan {
  int dtype;       // 0 f32, 1 bf16
  int B, H, N, D, F, Fe;   // Fe = F ? F : D (features per head)
  int fmap, causal;
  float eps;
  long long BH;
  int tiles;       // ceil(N / 128)
  int splits;      // non-causal: N-splits per head; causal: segments per head
  int tiles_per_split;   // in 128-token tiles (bf16) or tokens per split (f32, see seg_len)
  int seg_len;     // tokens per split/segment
  int num_sms;
  int apply_ctas, apply_tps;   // bf16 projected: apply CTAs per head, 128-token tiles each
  // bf16 non-causal: CTAs per head, made of clusters of `cluster` CTAs
  int ctas_per_head, cluster;
  // workspace layout (byte offsets from the workspace base, 256-aligned)
  size_t off_status, off_sync, off_partial, off_ksum_partial, off_final, off_final_ksum, off_blob, off_xchg, bytes;
  size_t blob_bytes;   // bf16 [kv | ksum | 0]^T image per head (projected path)
  // bf16 storage of a shape the bf16 kernels do not cover: q, k, v (and W) are
  // widened to fp32 copies in the workspace, the fp32 kernels run on them, and
  // their output is rounded back to bf16 (the plan is the fp32 one)
  bool widened;
  size_t off_wq, off_wk, off_wv, off_wo, off_wW, w_elems;
};

struct LaunchArgs {
  const Plan* p;
  const void* q;
  const void* k;
  const void* v;
  void* out;
  const void* W;
  long long w_head_stride;   // elements
  char* ws;                  // workspace base
  cudaStream_t stream;
  // tensor maps (bf16 path); built on the host per call
  const CUtensorMap* tm_q;
  const CUtensorMap* tm_k;
  const CUtensorMap* tm_v;
  const CUtensorMap* tm_out;
  const CUtensorMap* tm_w;
  // q, k and v stored as E4M3 codes (tm_q, tm_k, tm_v are then maps of
  // bytes), dequantised as scale x code value; out stays bf16
  bool e4m3;
  float scale_q, scale_k, scale_v;
  // Flux's attention prologue on q and k (la_set_prologue): RMS norm with the
  // scales pro_q / pro_k (fp32 [D]), then the rotation table pro_rope (fp32
  // [positions][D / 2][2], cos and sin)
  bool prologue;
  const float* pro_q;
  const float* pro_k;
  const float* pro_rope;
  float pro_eps;
};

// Host helpers defined in la_api.cpp for other host translation units.
// Plan of a bf16 non-causal F = 0 problem (the caller validated the shape).
void plan_bf16_noncausal(int B, int H, int N, int D, int fmap, float eps, int num_sms, Plan* p);
// [outer, rows, cols] bf16 tensor map, 128-row x 64-column boxes, 128-byte swizzle.
bool encode_tile_map_bf16(CUtensorMap* m, const void* base, long long outer, long long rows, long long cols,
                          long long outer_stride_elems);
// SM count of the current device; false unless it is an sm_100 device.
bool current_sm100(int* num_sms);
// `p` is device (or managed) memory of the current device.
bool on_current_device(const void* p);
// The byte ranges [a, a + an) and [b, b + bn) share at least one byte.
bool overlap(const void* a, size_t an, const void* b, size_t bn);

// Raise a kernel's dynamic shared-memory limit once per device (thread-safe).
cudaError_t ensure_smem_attr(const void* kernel, uint32_t bytes);

// f32 CUDA-core path (all modes).
cudaError_t launch_f32(const LaunchArgs& a);
// Elementwise bf16 -> fp32 (exact) and fp32 -> bf16 (round to nearest even) of
// n elements, on `stream`.
cudaError_t launch_bf16_to_f32(const void* in, float* out, size_t n, cudaStream_t stream);
cudaError_t launch_f32_to_bf16(const float* in, void* out, size_t n, cudaStream_t stream);
// Backward of the fp32 non-causal layer (F = 0, elu+1 or relu): dq, dk, dv of
// sum(out * dout).  The query pass runs `splits` splits of `seg` tokens per
// head; bpart / bpart_z: their [BH][splits][D][D] and [BH][splits][D]
// partials, bfin / bfin_z: the [BH][D][D] and [BH][D] sums (workspace regions
// past the forward plan).
cudaError_t launch_f32_backward(const LaunchArgs& a, const void* dout, void* dq, void* dk, void* dv, int splits,
                                int seg, float* bpart, float* bpart_z, float* bfin, float* bfin_z);
// bf16 tensor-core paths.
// CTAs per head and cluster size of the bf16 non-causal kernel for p's shape
// on the current device (from its cluster occupancy), and the bytes of the
// exchange area between the clusters of a head (0 when a head is one cluster).
void noncausal_geometry(Plan* p, size_t* xchg_bytes);
cudaError_t launch_bf16_noncausal(const LaunchArgs& a);
cudaError_t launch_bf16_causal(const LaunchArgs& a);
// The landmark branch of the TTR layer blended in place into a.out (which
// holds the kernel branch); gate: device float[H] logits; 1 <= n <= 128.
cudaError_t launch_bf16_landmark(const LaunchArgs& a, const void* gate, int n_landmarks);
cudaError_t launch_bf16_projected(const LaunchArgs& a);
// Sums fp32 partials (kv^T [D][fpart] and ksum [fpart] per (head, split, part))
// into the apply's bf16 [kv | ksum | 0]^T image, K-major, D + 16 rows.
cudaError_t launch_image_combine(const float* part_kv, const float* part_ks, uint8_t* image, long long BH,
                                 int nsplit, int D, int fpart, int parts, cudaStream_t stream);

}  // namespace la
