"""Python binding of the B200 linear-time phi-attention library (libla_phi.so).

The functions named ``la_*`` are one-to-one ctypes wrappers of the C ABI in
``include/la.h`` (argument marshalling only: pointers are plain integers and
every step of the computation runs in the library's CUDA kernels).
``LinearAttention`` is a convenience layer over them for torch tensors: torch
supplies device memory (the workspace) and the current stream, nothing else.
There is no fallback: without the built library every call raises.
"""

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libla_phi.so")

LA_F32, LA_BF16 = 0, 1
LA_PHI_ELU1, LA_PHI_RELU, LA_PHI_SOFTMAX = 0, 1, 2
FEATURE_MAPS = {"elu": LA_PHI_ELU1, "relu": LA_PHI_RELU, "softmax": LA_PHI_SOFTMAX}

LA_OK = 0
(LA_ERR_INVALID_ARG, LA_ERR_UNSUPPORTED, LA_ERR_MISALIGNED, LA_ERR_WORKSPACE, LA_ERR_CUDA, LA_ERR_TIMEOUT,
 LA_ERR_NO_DEVICE) = range(1, 8)
STATUS_NAMES = {
    0: "LA_OK", 1: "LA_ERR_INVALID_ARG", 2: "LA_ERR_UNSUPPORTED", 3: "LA_ERR_MISALIGNED",
    4: "LA_ERR_WORKSPACE", 5: "LA_ERR_CUDA", 6: "LA_ERR_TIMEOUT", 7: "LA_ERR_NO_DEVICE",
}

EXPORTED = ("la_create", "la_destroy", "la_set_projection", "la_workspace_bytes", "la_set_workspace",
            "la_forward", "la_forward_host", "la_sync_status", "la_status_string", "la_version",
            "la_forward_noalloc", "la_forward_ttr", "la_landmark_count", "la_forward_e4m3", "la_set_prologue",
            "la_backward", "la_backward_workspace_bytes")


class LAError(RuntimeError):
    def __init__(self, status, what=""):
        self.status = status
        super().__init__(f"{what}: {STATUS_NAMES.get(status, status)} ({la_status_string(status)})")


_lib = None


def lib():
    """Load libla_phi.so (built by ``build.build()``); raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"CUDA library not built: {LIB_PATH} is missing "
                           "(run linear_attention_diffusion_phi_b200.build.build())")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, i64, f32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong, ctypes.c_float, ctypes.c_size_t
    L.la_create.argtypes = [ctypes.POINTER(vp), i32]
    L.la_destroy.argtypes = [vp]
    L.la_set_projection.argtypes = [vp, vp, i32, i32, i32, i64]
    L.la_workspace_bytes.argtypes = [vp, i32, i32, i32, i32, i32, i32]
    L.la_workspace_bytes.restype = sz
    L.la_set_workspace.argtypes = [vp, vp, sz]
    L.la_forward.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, f32, i32, vp]
    L.la_forward_host.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, f32, i32, vp]
    L.la_sync_status.argtypes = [vp, vp]
    L.la_forward_noalloc.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, f32, vp]
    L.la_forward_ttr.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, f32, i32, vp, vp]
    L.la_forward_e4m3.argtypes = [vp, vp, vp, vp, f32, f32, f32, vp, i32, i32, i32, i32, i32, f32, vp]
    L.la_set_prologue.argtypes = [vp, vp, vp, vp, i32, i32, f32]
    L.la_backward.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, f32, vp]
    L.la_backward_workspace_bytes.argtypes = [vp, i32, i32, i32, i32]
    L.la_backward_workspace_bytes.restype = sz
    L.la_landmark_count.argtypes = [i32, f32, i32, i32]
    L.la_landmark_count.restype = i32
    L.la_status_string.argtypes = [i32]
    L.la_status_string.restype = ctypes.c_char_p
    L.la_version.argtypes = []
    for name in ("la_create", "la_destroy", "la_set_projection", "la_set_workspace", "la_forward",
                 "la_forward_host", "la_sync_status", "la_forward_noalloc", "la_forward_ttr", "la_forward_e4m3",
                 "la_set_prologue", "la_backward"):
        getattr(L, name).restype = i32
    _lib = L
    return L


# ------------------------------------------------------------ C-ABI wrappers

def la_create(dtype):
    h = ctypes.c_void_p()
    st = lib().la_create(ctypes.byref(h), dtype)
    if st != LA_OK:
        raise LAError(st, "la_create")
    return h.value


def la_destroy(handle):
    return lib().la_destroy(handle)


def la_set_projection(handle, W_ptr, H, D, F, head_stride):
    return lib().la_set_projection(handle, W_ptr, H, D, F, head_stride)


def la_workspace_bytes(handle, B, H, N, D, F, causal):
    return lib().la_workspace_bytes(handle, B, H, N, D, F, int(causal))


def la_set_workspace(handle, ptr, nbytes):
    return lib().la_set_workspace(handle, ptr, nbytes)


def la_forward(handle, q, k, v, out, B, H, N, D, F, feature_map, eps, causal, stream):
    return lib().la_forward(handle, q, k, v, out, B, H, N, D, F, feature_map, eps, int(causal), stream)


def la_forward_host(handle, q_host, k_host, v_host, out_host, dq, dk, dv, dout, B, H, N, D, F,
                    feature_map, eps, causal, stream):
    return lib().la_forward_host(handle, q_host, k_host, v_host, out_host, dq, dk, dv, dout, B, H, N, D, F,
                                 feature_map, eps, int(causal), stream)


def la_forward_noalloc(q, k, v, out, B, H, N, D, feature_map, eps, stream):
    """bf16 non-causal forward whose scratch is a static device array inside the
    library, for callers that cannot allocate device memory."""
    return lib().la_forward_noalloc(q, k, v, out, B, H, N, D, feature_map, eps, stream)


def la_forward_ttr(handle, q, k, v, out, B, H, N, D, F, feature_map, eps, n_landmarks, gate, stream):
    """The TTR layer: kernel branch blended with exact softmax over landmarks."""
    return lib().la_forward_ttr(handle, q, k, v, out, B, H, N, D, F, feature_map, eps, n_landmarks, gate, stream)


def la_forward_e4m3(handle, q, k, v, scale_q, scale_k, scale_v, out, B, H, N, D, feature_map, eps, stream):
    """Non-causal forward on E4M3-stored q, k, v with one scale per tensor; out bf16."""
    return lib().la_forward_e4m3(handle, q, k, v, scale_q, scale_k, scale_v, out, B, H, N, D, feature_map, eps,
                                 stream)


def la_set_prologue(handle, q_scale, k_scale, rope, D, n_positions, norm_eps):
    """Bind Flux's attention prologue (QK RMS norm, then the rotary embedding)."""
    return lib().la_set_prologue(handle, q_scale, k_scale, rope, D, n_positions, norm_eps)


def la_backward(handle, q, k, v, dout, dq, dk, dv, B, H, N, D, feature_map, eps, stream):
    """Gradients dq, dk, dv of sum(out * dout) (fp32, non-causal, no projection)."""
    return lib().la_backward(handle, q, k, v, dout, dq, dk, dv, B, H, N, D, feature_map, eps, stream)


def la_backward_workspace_bytes(handle, B, H, N, D):
    return lib().la_backward_workspace_bytes(handle, B, H, N, D)


def la_landmark_count(N, fraction, min_count, max_count):
    return lib().la_landmark_count(N, fraction, min_count, max_count)


def la_sync_status(handle, stream):
    return lib().la_sync_status(handle, stream)


def la_status_string(status):
    try:
        return lib().la_status_string(status).decode()
    except RuntimeError:
        return "library not loaded"


def la_version():
    return lib().la_version()


def check(status, what="la call"):
    if status != LA_OK:
        raise LAError(status, what)


# ------------------------------------------------------- torch convenience

class LinearAttention:
    """out = phi-attention(q, k, v) for torch CUDA tensors [B, H, N, D].

    dtype: torch.bfloat16 (tensor-core path) or torch.float32 (CUDA-core path).
    W: optional projection [H, D, F] (or [D, F], shared by all heads).
    """

    def __init__(self, dtype, feature_map="elu", eps=1e-6, causal=False, W=None):
        import torch
        self.torch = torch
        self.dtype = dtype
        self.code = LA_BF16 if dtype == torch.bfloat16 else LA_F32
        if dtype not in (torch.bfloat16, torch.float32):
            raise ValueError("dtype must be torch.bfloat16 or torch.float32")
        self.fmap = FEATURE_MAPS[feature_map]
        self.eps = float(eps)
        self.causal = bool(causal)
        self.handle = la_create(self.code)
        self.W = None
        self.F = 0
        self._ws = None
        if W is not None:
            self.set_projection(W)

    def set_projection(self, W):
        if W.dim() not in (2, 3):
            raise ValueError(f"W: expected [H, D, F] or [D, F], got shape {tuple(W.shape)}")
        if W.dtype != self.dtype:
            raise ValueError(f"W: dtype {W.dtype}, the operator's is {self.dtype}")
        if W.device.type != "cuda":
            raise ValueError(f"W: on {W.device}, expected a CUDA tensor")
        if W.dim() == 2:
            H, (D, F), stride = 1, W.shape, 0
        else:
            H, D, F = W.shape
            stride = D * F
        W = W.contiguous()
        check(la_set_projection(self.handle, W.data_ptr(), H, D, F, stride), "la_set_projection")
        self.W, self.F = W, F

    def workspace_bytes(self, B, H, N, D):
        return la_workspace_bytes(self.handle, B, H, N, D, self.F, self.causal)

    def _bind_workspace(self, B, H, N, D, device):
        need = self.workspace_bytes(B, H, N, D)
        if need == 0:
            raise LAError(1, "la_workspace_bytes")
        if self._ws is None or self._ws.numel() < need or self._ws.device != device:
            self._ws = self.torch.empty(need, dtype=self.torch.uint8, device=device)
            check(la_set_workspace(self.handle, self._ws.data_ptr(), self._ws.numel()), "la_set_workspace")

    def _check_tensors(self, q, k, v, out):
        # the library sees only base pointers: every tensor must be a dense
        # [B, H, N, D] array of the operator's dtype on one CUDA device
        if q.dim() != 4:
            raise ValueError(f"q: expected [B, H, N, D], got shape {tuple(q.shape)}")
        ts = (("q", q), ("k", k), ("v", v), ("out", out))
        for name, t in ts:
            if t.shape != q.shape:
                raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(q.shape)}")
        for name, t in ts:
            if t.dtype != self.dtype:
                raise ValueError(f"{name}: dtype {t.dtype}, the operator's is {self.dtype}")
        for name, t in ts:
            if not t.is_contiguous():
                raise ValueError(f"{name}: must be contiguous (row-major [B, H, N, D])")
        for name, t in ts:
            if t.device.type != "cuda" or t.device != q.device:
                raise ValueError(f"{name}: on {t.device}, expected one CUDA device for all tensors")
        if self.W is not None and self.W.device != q.device:
            raise ValueError(f"W: on {self.W.device}, the inputs on {q.device}")

    def __call__(self, q, k, v, out=None, stream=None):
        if out is None:
            out = self.torch.empty_like(q)
        self._check_tensors(q, k, v, out)
        B, H, N, D = q.shape
        # the library launches on the current device and expects every
        # pointer to belong to it: make the tensors' device current
        with self.torch.cuda.device(q.device):
            self._bind_workspace(B, H, N, D, q.device)
            s = stream if stream is not None else self.torch.cuda.current_stream(q.device).cuda_stream
            check(la_forward(self.handle, q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                             B, H, N, D, self.F, self.fmap, self.eps, self.causal, s), "la_forward")
        return out

    def ttr(self, q, k, v, n_landmarks, gate, out=None, stream=None):
        """The TTR layer (la_forward_ttr): ``gate`` is a float32 CUDA tensor of
        one logit per head; non-causal operators only."""
        if self.causal:
            raise ValueError("the TTR layer is non-causal")
        if out is None:
            out = self.torch.empty_like(q)
        self._check_tensors(q, k, v, out)
        B, H, N, D = q.shape
        if gate.dtype != self.torch.float32 or gate.numel() != H or not gate.is_contiguous() \
                or gate.device != q.device:
            raise ValueError(f"gate: expected {H} contiguous float32 values on {q.device}")
        with self.torch.cuda.device(q.device):
            self._bind_workspace(B, H, N, D, q.device)
            s = stream if stream is not None else self.torch.cuda.current_stream(q.device).cuda_stream
            check(la_forward_ttr(self.handle, q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                 B, H, N, D, self.F, self.fmap, self.eps, int(n_landmarks), gate.data_ptr(), s),
                  "la_forward_ttr")
        return out

    def e4m3(self, q, k, v, scales, out=None, stream=None):
        """Forward on E4M3-stored inputs (la_forward_e4m3): ``q``, ``k``, ``v``
        are uint8 (or float8_e4m3fn) CUDA tensors of codes, ``scales`` the
        three fp32 scales; ``out`` is bf16.  Non-causal, F = 0, bf16 operators."""
        if self.causal or self.F:
            raise ValueError("E4M3 storage: non-causal operators without a projection only")
        if q.dim() != 4:
            raise ValueError(f"q: expected [B, H, N, D], got shape {tuple(q.shape)}")
        codes = []
        for name, t in (("q", q), ("k", k), ("v", v)):
            if t.dtype == getattr(self.torch, "float8_e4m3fn", None):
                t = t.view(self.torch.uint8)
            if t.dtype != self.torch.uint8:
                raise ValueError(f"{name}: dtype {t.dtype}, expected uint8 E4M3 codes")
            if t.shape != q.shape or not t.is_contiguous() or t.device.type != "cuda" or t.device != q.device:
                raise ValueError(f"{name}: expected a contiguous {tuple(q.shape)} tensor on {q.device}")
            codes.append(t)
        if out is None:
            out = self.torch.empty(q.shape, dtype=self.torch.bfloat16, device=q.device)
        if out.dtype != self.torch.bfloat16 or out.shape != q.shape or not out.is_contiguous() \
                or out.device != q.device:
            raise ValueError(f"out: expected a contiguous bfloat16 {tuple(q.shape)} tensor on {q.device}")
        sq, sk, sv = (float(x) for x in scales)
        B, H, N, D = q.shape
        with self.torch.cuda.device(q.device):
            self._bind_workspace(B, H, N, D, q.device)
            s = stream if stream is not None else self.torch.cuda.current_stream(q.device).cuda_stream
            check(la_forward_e4m3(self.handle, codes[0].data_ptr(), codes[1].data_ptr(), codes[2].data_ptr(),
                                  sq, sk, sv, out.data_ptr(), B, H, N, D, self.fmap, self.eps, s),
                  "la_forward_e4m3")
        return out

    def set_prologue(self, q_scale, k_scale, rope, norm_eps=1e-6):
        """Bind Flux's attention prologue for the following forwards: RMS norm
        of q and k over the head dimension times ``q_scale`` / ``k_scale``
        (float32 CUDA tensors [D]), then the rotation of feature pairs by
        ``rope`` (float32 CUDA tensor [positions, D/2, 2] of cos, sin).
        ``q_scale=None`` unbinds."""
        if q_scale is None:
            check(la_set_prologue(self.handle, None, None, None, 0, 0, 0.0), "la_set_prologue")
            self._prologue = None
            return
        D = q_scale.numel()
        for name, t in (("q_scale", q_scale), ("k_scale", k_scale), ("rope", rope)):
            if t.dtype != self.torch.float32 or not t.is_contiguous() or t.device.type != "cuda":
                raise ValueError(f"{name}: expected a contiguous float32 CUDA tensor")
        if k_scale.numel() != D or rope.dim() != 3 or rope.shape[1:] != (D // 2, 2):
            raise ValueError("expected q_scale, k_scale [D] and rope [positions, D/2, 2]")
        check(la_set_prologue(self.handle, q_scale.data_ptr(), k_scale.data_ptr(), rope.data_ptr(), D,
                              rope.shape[0], float(norm_eps)), "la_set_prologue")
        self._prologue = (q_scale, k_scale, rope)   # kept alive while bound

    def backward(self, q, k, v, dout, outs=None, stream=None):
        """dq, dk, dv of sum(out * dout) for this operator's forward (la_backward:
        fp32, non-causal, no projection, elu+1 or relu); ``outs`` = (dq, dk, dv)
        to write into."""
        self._check_tensors(q, k, v, dout)
        B, H, N, D = q.shape
        dq, dk, dv = outs if outs is not None else (self.torch.empty_like(q) for _ in range(3))
        for name, t in (("dq", dq), ("dk", dk), ("dv", dv)):
            if t.shape != q.shape or t.dtype != q.dtype or not t.is_contiguous() or t.device != q.device:
                raise ValueError(f"{name}: expected a contiguous tensor like q")
        with self.torch.cuda.device(q.device):
            need = la_backward_workspace_bytes(self.handle, B, H, N, D)
            if need == 0:
                raise LAError(2, "la_backward_workspace_bytes")
            if self._ws is None or self._ws.numel() < need or self._ws.device != q.device:
                self._ws = self.torch.empty(need, dtype=self.torch.uint8, device=q.device)
                check(la_set_workspace(self.handle, self._ws.data_ptr(), self._ws.numel()), "la_set_workspace")
            s = stream if stream is not None else self.torch.cuda.current_stream(q.device).cuda_stream
            check(la_backward(self.handle, q.data_ptr(), k.data_ptr(), v.data_ptr(), dout.data_ptr(), dq.data_ptr(),
                              dk.data_ptr(), dv.data_ptr(), B, H, N, D, self.fmap, self.eps, s), "la_backward")
        return dq, dk, dv

    def sync_status(self, stream=None):
        dev = self._ws.device if self._ws is not None else self.torch.cuda.current_device()
        with self.torch.cuda.device(dev):
            s = stream if stream is not None else self.torch.cuda.current_stream(dev).cuda_stream
            return la_sync_status(self.handle, s)

    def close(self):
        if self.handle:
            la_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
