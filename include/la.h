/*
 * la.h -- C ABI of the B200 (sm_100a) linear-time kernelised attention library.
 *
 * The operation (page "NNT Define Linear Attention", sections "The inputs" and
 * "How it works"): per head, a non-negative feature map phi is applied to the
 * query and key rows, the sequence is collapsed into the state
 *     kv = sum_j phi(k_j) v_j^T   (F x D)      ksum = sum_j phi(k_j)   (F)
 * and every output row is
 *     out_i = phi(q_i)^T kv / (phi(q_i) . ksum + eps).
 * This equals the weighted sum  sum_j w_ij v_j / (sum_j w_ij + eps)  with
 * w_ij = phi(q_i) . phi(k_j); the N x N weight matrix is never formed.
 *   feature maps  LA_PHI_ELU1: elu(x)+1 (alpha = 1);  LA_PHI_RELU: max(x, 0);
 *                 LA_PHI_SOFTMAX: softmax over each row's feature vector,
 *                 exp(x_f - max x) / sum_f' exp(x_f' - max x) (the page lists
 *                 softmax without naming its axis; a feature map takes one
 *                 token's vector to its features, so it runs over that vector)
 *   causal        query i sees keys j <= i (itself included)
 *   projection    F > 0: phi(x) = fmap(x W_h) with a D x F matrix per head
 *                 (page "Flux2TTRTrainer", "Inputs worth setting": feature_dim
 *                 is a multiple of 256); F = 0: phi acts on x itself (F = D).
 *
 * Memory.  Every pointer passed to the library is owned by the caller.  The
 * library allocates no device memory and keeps only non-owning pointers in a
 * handle; scratch space ("workspace") is a caller-owned device buffer of
 * la_workspace_bytes() bytes.  Device pointers must address memory of the
 * device that is current when la_forward is called.
 *
 * Layout.  q, k, v and out are dense row-major [B, H, N, D] tensors (D
 * innermost), all of the handle's dtype.  q, k and v are only read and may
 * coincide; out shares no byte with q, k, v, the part of W the call reads or
 * the workspace, nor the workspace with q, k, v or W (la_forward checks the
 * address ranges and returns LA_ERR_INVALID_ARG otherwise).
 * W is [H, D, F] row-major (F innermost) with head stride head_stride
 * elements (0: one matrix shared by all heads).
 *
 * Asynchrony.  la_forward only enqueues kernels on the given stream (a
 * cudaStream_t passed as void*, NULL = legacy default stream) and returns.
 * The bf16 kernels are launched with programmatic dependent launch: they may
 * start their set-up while earlier work on the stream is finishing, but touch
 * no global memory before it has completed; they also let the next launch on
 * the stream start early, so a following kernel that is itself launched with
 * programmatic serialization must wait (griddepcontrol.wait) before it reads
 * out.  Ordinary launches are ordered as usual.
 *
 * Errors.  Argument errors are detected on the host before anything is
 * enqueued; out is then untouched.  A pointer that is not device memory of
 * the current device is such an error (LA_ERR_INVALID_ARG).  Launch failures
 * return LA_ERR_CUDA.  Errors detected on the device (a bounded wait that ran
 * out) are recorded in a status word inside the workspace and reported by
 * la_sync_status() only: la_forward enqueues and returns, and reading the
 * word there would need a synchronisation with the stream, so it never looks
 * at it.  The word of a newly bound workspace is cleared by the first
 * la_forward (or la_sync_status) that uses it, on that call's stream.
 *
 * Threading.  A handle may be used by one host thread at a time.  Calls that
 * share a workspace must be ordered on the device (same stream, or events).
 */
#ifndef LA_H_
#define LA_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct la_handle_s* la_handle_t;

typedef enum {
  LA_OK = 0,
  LA_ERR_INVALID_ARG = 1,   /* null pointer, negative size, eps < 0, bad enum,
                               an output overlapping an input                  */
  LA_ERR_UNSUPPORTED = 2,   /* valid, but not a shape/dtype this library runs */
  LA_ERR_MISALIGNED = 3,    /* a pointer is not 16-byte aligned               */
  LA_ERR_WORKSPACE = 4,     /* no workspace bound, or it is too small         */
  LA_ERR_CUDA = 5,          /* a CUDA runtime call or kernel launch failed    */
  LA_ERR_TIMEOUT = 6,       /* a kernel gave up on a bounded device-side wait */
  LA_ERR_NO_DEVICE = 7      /* no usable sm_100 device is current             */
} la_status_t;

typedef enum { LA_F32 = 0, LA_BF16 = 1 } la_dtype_t;
typedef enum { LA_PHI_ELU1 = 0, LA_PHI_RELU = 1, LA_PHI_SOFTMAX = 2 } la_feature_map_t;

/* Create a handle for one storage dtype (LA_F32 or LA_BF16).  Allocates host
 * memory only.  LA_F32 runs fp32 CUDA-core kernels with fp32 accumulation;
 * LA_BF16 runs tcgen05 tensor-core kernels with fp32 accumulation. */
la_status_t la_create(la_handle_t* handle, int dtype);

/* Destroy a handle.  Frees host memory only; pending work is not waited on. */
la_status_t la_destroy(la_handle_t handle);

/* Bind the projection used when la_forward is called with F > 0.
 * W: device pointer, [H, D, F] of the handle's dtype, 16-byte aligned, not
 * copied (it must stay valid while calls that use it are pending).
 * head_stride: elements between consecutive heads' matrices, D*F for one
 * matrix per head, 0 for one matrix shared by all heads.  F must be a positive
 * multiple of 256 (page "Flux2TTRTrainer", "Inputs worth setting").
 * W = NULL unbinds. */
/* Bind Flux's attention prologue (page "FLUXNATION", "What it does": the
 * block's QKV split and RoPE fused into its kernel), applied to q and k as
 * they are loaded by every later la_forward: the QK norm of Flux's block, an
 * RMS norm over the head dimension times a per-feature scale,
 *     x_d / sqrt(mean_d' x_d'^2 + norm_eps) * scale_d,
 * then the rotary embedding, which turns each feature pair (2i, 2i + 1) of the
 * token at position n by rope[n][i] = (cos, sin):
 *     (cos x_2i - sin x_2i+1,  sin x_2i + cos x_2i+1).
 * v is not transformed.  The page names RoPE; the norm is read from the block
 * it fuses (Flux's attention normalises q and k before the rotation).
 * q_scale, k_scale: device fp32 [D]; rope: device fp32 [n_positions][D / 2][2]
 * (cos, sin), positions 0 .. N - 1 used, shared by all batches and heads; all
 * 16-byte aligned, not copied (they must stay valid while calls that use them
 * are pending).  D even and > 0, n_positions > 0, norm_eps >= 0 and finite,
 * else LA_ERR_INVALID_ARG.  q_scale = NULL unbinds.
 * la_forward then requires the bound D and N <= n_positions
 * (LA_ERR_INVALID_ARG) and supports: LA_F32 with F = 0, causal or not;
 * LA_BF16 with F = 0 either at D = 128, non-causal, feature map elu+1 or relu
 * (the tensor-core kernel) or on a shape that runs widened (see la_forward).  Other
 * forwards with a prologue bound (other shapes, la_forward_ttr,
 * la_forward_e4m3) return LA_ERR_UNSUPPORTED. */
la_status_t la_set_prologue(la_handle_t handle, const float* q_scale, const float* k_scale, const float* rope,
                            int D, int n_positions, float norm_eps);

la_status_t la_set_projection(la_handle_t handle, const void* W, int H, int D, int F,
                              long long head_stride);

/* Workspace bytes la_forward needs for this problem (0 if the arguments are
 * invalid for the handle).  The size depends only on the arguments and the
 * device (its SM count and how many thread-block clusters of the kernels fit
 * on it at once).  Every workspace starts with a 4352-byte header (the status
 * word and the synchronisation words of the exchange below).  bf16 non-causal
 * problems with F = 0 need the header only, plus, when a head is spread over
 * several clusters (D = 128 with fewer heads than SMs), an exchange area of
 * 36 KB per head and cluster: 2.6 MB for [1, 24, 4608, 128] on 148 SMs, never
 * more than 36 KB per SM.  bf16 causal problems with at least as many heads
 * (B*H) as SMs need the header only.  Otherwise the workspace holds fp32
 * partial states and grows with B*H and the number of splits per head: on
 * 148 SMs about 2 MB for causal [4, 8, 32768, 64], 11 MB for
 * [1, 24, 4608, 128] with F = 256, and 13.5 GB for B*H = 65535 with F = 256.
 * A bf16 shape that runs widened (see la_forward) needs the fp32 plan plus
 * fp32 copies of q, k, v and out (16 * B*H*N*D bytes) and of W. */
size_t la_workspace_bytes(la_handle_t handle, int B, int H, int N, int D, int F, int causal);

/* Bind a caller-owned device workspace (256-byte aligned).  The library writes
 * partial states and its status word there.  Bytes = 0 or ptr = NULL unbinds.
 * Nothing is enqueued and nothing waits: the status word is cleared by the
 * next la_forward or la_sync_status, on that call's stream. */
la_status_t la_set_workspace(la_handle_t handle, void* dev_ptr, size_t bytes);

/* Enqueue out = phi-attention(q, k, v) on `stream` (see the top of this file).
 * B, H, N >= 0 (any of them 0: nothing is enqueued, LA_OK); D > 0; F = 0 or a
 * positive multiple of 256 with a projection bound; feature_map is a
 * la_feature_map_t; eps >= 0; causal is 0 or 1.
 * Supported: D <= 128, D % 4 == 0; F <= 4096 non-causal, F <= 256 causal;
 *            LA_PHI_SOFTMAX with F = 0 only.  Other combinations:
 *            LA_ERR_UNSUPPORTED.
 *            LA_BF16 runs on the tensor-core kernels for non-causal D = 64
 *            or 128 (F > 0: F = 256 with D = 128 only) and causal D = 64 with
 *            F = 0 (also the shapes of la_forward_ttr and
 *            la_forward_noalloc); of these, LA_PHI_SOFTMAX runs at
 *            non-causal D = 128 only.  Any other LA_BF16 shape runs
 *            widened: q, k, v (and W) are converted to fp32 copies
 *            in the workspace on `stream`, the fp32 kernels run on them and
 *            out is their result rounded to bf16 (four more launches, five
 *            with W).
 * The result is deterministic: the same arguments give bitwise the same out. */
la_status_t la_forward(la_handle_t handle, const void* q, const void* k, const void* v,
                       void* out, int B, int H, int N, int D, int F, int feature_map,
                       float eps, int causal, void* stream);

/* End-to-end variant over HOST buffers: copies q, k, v (host, pinned for
 * asynchrony) into the caller's device buffers dq, dk, dv, runs la_forward into
 * dout and copies dout back to out_host, all enqueued on `stream`.  dq, dk, dv
 * and dout are [B, H, N, D] device buffers that share no byte (else
 * LA_ERR_INVALID_ARG).  The host buffers must stay valid until the stream
 * reaches the end of the copies. */
la_status_t la_forward_host(la_handle_t handle, const void* q_host, const void* k_host,
                            const void* v_host, void* out_host, void* dq, void* dk, void* dv,
                            void* dout, int B, int H, int N, int D, int F, int feature_map,
                            float eps, int causal, void* stream);

/* Read the device status word of the bound workspace after the work queued
 * on `stream` (a copy on that stream, then a wait for the stream only), and
 * clear it on the same stream if it was set.  Returns LA_OK, LA_ERR_TIMEOUT
 * (a kernel abandoned a bounded wait; its output is undefined) or
 * LA_ERR_CUDA. */
la_status_t la_sync_status(la_handle_t handle, void* stream);

/* The TTR student layer (page "Flux2TTRTrainer", "How the distillation
 * works"): the kernel branch of la_forward (non-causal, F = 0 or a projection
 * bound as for la_forward) fused with an exact-softmax branch over landmark
 * tokens, blended by a bounded weight.  The page gives neither the landmark
 * rule nor the blend; this library reads them as: n_landmarks tokens evenly
 * spaced, token floor(l N / n_landmarks) for l = 0 .. n_landmarks - 1; scores
 * q_i . k_l / sqrt(D) (the scale of the attention the layer replaces),
 * softmax over the landmarks per query, weights applied to the landmark value
 * rows; out = a_h * softmax branch + (1 - a_h) * kernel branch with
 * a_h = 1 / (1 + exp(-gate[h])), gate a device array of H floats (one logit per
 * head, 4-byte aligned, sharing no byte with out or the workspace).
 * Supported: LA_BF16 handles, D = 128, 1 <= n_landmarks <= min(N, 128)
 * (n_landmarks outside [1, N] gives LA_ERR_INVALID_ARG, above 128
 * LA_ERR_UNSUPPORTED).  Two launches on `stream`: the kernel branch into out,
 * then the landmark branch, which reads q, the landmark rows of k and v and
 * out, and rewrites out blended.  Same workspace, errors and determinism as
 * la_forward. */
la_status_t la_forward_ttr(la_handle_t handle, const void* q, const void* k, const void* v, void* out, int B,
                           int H, int N, int D, int F, int feature_map, float eps, int n_landmarks,
                           const float* gate, void* stream);

/* FP8 storage (page "FLUXNATION", "What it does": an FP8 CUDA kernel): the
 * non-causal F = 0 forward of la_forward with q, k and v stored as E4M3 codes
 * and one fp32 scale per tensor; the layer runs on scale_q x q, scale_k x k
 * and scale_v x v.  The page names FP8 only; this library reads it as the
 * finite E4M3 of the OCP 8-bit floating-point format (sign, four exponent
 * bits with bias 7, three mantissa bits; largest value 448; S.1111.111 is NaN
 * and yields NaN wherever it reaches the output) with per-tensor scales.
 * q, k, v: device uint8 [B, H, N, D] codes, 16-byte aligned, read only (they
 * may coincide).  out: device bf16 [B, H, N, D], 16-byte aligned, sharing no
 * byte with q, k, v or the workspace (else LA_ERR_INVALID_ARG).  Scales
 * finite and > 0 (else LA_ERR_INVALID_ARG).  Supported: LA_BF16 handles,
 * D = 128 (else LA_ERR_UNSUPPORTED).  Each dequantised value is rounded to
 * bf16 before the feature map (exact for power-of-two scales, at most 2^-9
 * relative otherwise); accumulation is fp32 as for bf16 inputs.  Workspace:
 * la_workspace_bytes of the same B, H, N, D with F = 0 and causal = 0.
 * One launch on `stream`; errors and determinism as la_forward. */
la_status_t la_forward_e4m3(la_handle_t handle, const void* q, const void* k, const void* v, float scale_q,
                            float scale_k, float scale_v, void* out, int B, int H, int N, int D,
                            int feature_map, float eps, void* stream);

/* Backward pass (page "Flux2TTRTrainer", "How the distillation works": the
 * student layer is trained): given dout = dL/dout of a forward with the same
 * arguments, writes dq, dk, dv = dL/dq, dL/dk, dL/dv.  With
 * den_i = phi(q_i).z + eps, out_i = phi(q_i) kv / den_i, g_i = dout_i / den_i
 * and h_i = -(dout_i . out_i) / den_i:
 *     dq_i = (kv g_i + h_i z) * phi'(q_i),
 *     dk_j = (dkv v_j + dz) * phi'(k_j),   dv_j = dkv^T phi(k_j),
 * where dkv = sum_i phi(q_i) g_i^T and dz = sum_i h_i phi(q_i); phi' of elu+1
 * is 1 for x > 0 and exp(x) otherwise, of relu 1 for x > 0 and 0 otherwise.
 * Supported: LA_F32 handles, non-causal, no projection, elu+1 or relu, no
 * prologue bound, D <= 128 with D % 4 == 0 (else LA_ERR_UNSUPPORTED).
 * q, k, v, dout: device fp32 [B, H, N, D], read only (may coincide); dq, dk,
 * dv: device fp32 [B, H, N, D], pairwise disjoint and sharing no byte with
 * the inputs or the workspace (else LA_ERR_INVALID_ARG); all 16-byte aligned.
 * Workspace: la_backward_workspace_bytes of the same shape.  Five launches on
 * `stream`; deterministic. */
la_status_t la_backward(la_handle_t handle, const void* q, const void* k, const void* v, const void* dout,
                        void* dq, void* dk, void* dv, int B, int H, int N, int D, int feature_map, float eps,
                        void* stream);

/* Workspace bytes la_backward needs for this shape (0 for an unsupported or
 * invalid one). */
size_t la_backward_workspace_bytes(la_handle_t handle, int B, int H, int N, int D);

/* Landmark count of the page's knobs (landmark fraction, min, max; page
 * "Flux2TTRTrainer", "Inputs worth setting"): round(fraction * N) (half up)
 * clamped to [min_count, max_count], then to [1, N].  0 for invalid arguments
 * (N < 1, fraction < 0 or NaN, min_count < 0, max_count < 1). */
int la_landmark_count(int N, float fraction, int min_count, int max_count);

/* Size of the static scratch array behind la_forward_noalloc (8 MiB).  A
 * device holds it from the moment the library's code is loaded on it (at the
 * latest, the first la_forward_noalloc call there) until the process exits. */
#define LA_NOALLOC_SCRATCH_BYTES (8u * 1024u * 1024u)

/* For callers that cannot allocate device memory (no cudaMalloc, no pool of
 * their own, nothing to bind with la_set_workspace): the bf16, non-causal,
 * F = 0 forward of la_forward, with its scratch in a static device array of
 * LA_NOALLOC_SCRATCH_BYTES inside this library instead of a workspace.  The
 * pages have no counterpart; this entry point exists only for such callers.
 * q, k, v, out: device pointers, bf16 [B, H, N, D] as for la_forward (out
 * overlapping q, k or v gives LA_ERR_INVALID_ARG); D is 64 or 128.  No handle is used and nothing is allocated, on host or device.
 * The scratch this path needs (the la_forward workspace of the same problem:
 * the header, plus at most 36 KB per SM of exchange area) fits the array on
 * devices of up to 220 SMs; a plan that needed more than the array would
 * return LA_ERR_WORKSPACE before anything is enqueued.  The first call on a device looks up the array's device
 * address (cudaGetSymbolAddress) with that device current; make that first
 * call before any stream capture.  The address is cached for the life of the
 * process, so this entry point must not be used on a device after
 * cudaDeviceReset.  Every call on a device shares the one array and it keeps
 * the last call's contents: calls that overlap on the GPU (different streams
 * without ordering between them) race and give undefined results.  The
 * kernel writes the array's status word (on a device-side timeout), which
 * nothing reads: timeouts of this entry point are not reported.  Its
 * synchronisation words (a launch count and one flag per CTA, zero when the
 * array is loaded) carry over from call to call, and every launch leaves them
 * consistent for the next, so no clearing operation is enqueued between
 * calls. */
la_status_t la_forward_noalloc(const void* q, const void* k, const void* v, void* out, int B, int H, int N,
                               int D, int feature_map, float eps, void* stream);

/* Static description of a status code. */
const char* la_status_string(la_status_t status);

/* Library version, major * 10000 + minor * 100 + patch. */
int la_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LA_H_ */
