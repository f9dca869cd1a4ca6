// noalloc.cu -- la_forward_noalloc: the bf16 non-causal forward for callers
// that cannot allocate device memory at all (no cudaMalloc, no caching
// allocator, no workspace of their own), for instance code running inside
// another framework's memory pool or a process whose allocations are fixed up
// front.  Its scratch space is a file-scope __device__ array of fixed size
// that every device which loads this library reserves until the process
// exits.  The kernels are the same as la_forward's bf16 non-causal path; only
// where their scratch lives differs.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "la.h"
#include "la_internal.h"

namespace {

constexpr size_t kScratchBytes = LA_NOALLOC_SCRATCH_BYTES;

// Scratch for la_forward_noalloc, laid out as la_forward's workspace of the
// same problem: the status word of its kernel (written on a device-side
// timeout, read by nobody), the synchronisation words of the exchange between
// clusters (zero at load) and the exchange area.  In host code this name is
// only a handle for cudaGetSymbolAddress, never a device address.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;

// Device address of g_noalloc_scratch on the current device, looked up once
// per device (with that device current) and cached for the life of the
// process: after a cudaDeviceReset the cached address would be stale, so
// this entry point must not be used across a reset.
bool scratch_address(void** out) {
  static std::mutex mu;
  static void* addr[kMaxDevices] = {};
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return false;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return false;
    }
    addr[dev] = p;
  }
  *out = addr[dev];
  return true;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" la_status_t la_forward_noalloc(const void* q, const void* k, const void* v, void* out, int B, int H,
                                          int N, int D, int feature_map, float eps, void* stream) {
  if (B < 0 || H < 0 || N < 0 || D <= 0) return LA_ERR_INVALID_ARG;
  if (feature_map != LA_PHI_ELU1 && feature_map != LA_PHI_RELU && feature_map != LA_PHI_SOFTMAX)
    return LA_ERR_INVALID_ARG;
  if (!(eps >= 0.f)) return LA_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return LA_ERR_UNSUPPORTED;
  if (feature_map == LA_PHI_SOFTMAX && D != 128) return LA_ERR_UNSUPPORTED;
  if (static_cast<long long>(B) * H > 65535) return LA_ERR_UNSUPPORTED;
  if (static_cast<long long>(B) * H * N == 0) return LA_OK;
  if (!q || !k || !v || !out) return LA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return LA_ERR_MISALIGNED;
  // out is written while q, k and v are still being read
  const size_t nb = static_cast<size_t>(B) * H * N * D * 2;
  if (la::overlap(out, nb, q, nb) || la::overlap(out, nb, k, nb) || la::overlap(out, nb, v, nb))
    return LA_ERR_INVALID_ARG;

  int sms = 0;
  if (!la::current_sm100(&sms)) return LA_ERR_NO_DEVICE;
  if (!la::on_current_device(q) || !la::on_current_device(k) || !la::on_current_device(v) ||
      !la::on_current_device(out))
    return LA_ERR_INVALID_ARG;
  la::Plan p;
  la::plan_bf16_noncausal(B, H, N, D, feature_map, eps, sms, &p);
  if (p.bytes > kScratchBytes) return LA_ERR_WORKSPACE;   // problem too large for the static scratch

  void* scratch = nullptr;
  if (!scratch_address(&scratch)) return LA_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // The array keeps the previous call's contents.  Nothing in it has to
  // start at zero: the kernel only ever writes the status word (first error
  // wins) and never reads it, and this entry point does not report it, so no
  // clearing operation is put between consecutive forwards on the stream.

  CUtensorMap tq, tk, tv, to;
  const long long BH = p.BH, hs = static_cast<long long>(N) * D;
  if (!la::encode_tile_map_bf16(&tq, q, BH, N, D, hs) || !la::encode_tile_map_bf16(&tk, k, BH, N, D, hs) ||
      !la::encode_tile_map_bf16(&tv, v, BH, N, D, hs) || !la::encode_tile_map_bf16(&to, out, BH, N, D, hs))
    return LA_ERR_CUDA;
  la::LaunchArgs a = {};
  a.p = &p;
  a.q = q; a.k = k; a.v = v; a.out = out;
  a.ws = static_cast<char*>(scratch);
  a.stream = s;
  a.tm_q = &tq; a.tm_k = &tk; a.tm_v = &tv; a.tm_out = &to;
  const cudaError_t err = la::launch_bf16_noncausal(a);
  if (err != cudaSuccess) {
    cudaGetLastError();
    return LA_ERR_CUDA;
  }
  return LA_OK;
}
