"""Seeded synthetic inputs for the linear-attention workloads.

This module only draws random numbers and shapes them; it holds none of the
method's arithmetic.  The same arrays feed the CUDA library and the float64
oracle: values are drawn in float32 with numpy's PCG64, the workload's
transform is applied in float32, and the result is cast once (round to nearest
even) to the storage dtype.  Both sides then read exactly those stored values.

Workloads stand in for Flux's attention at 1024x1024 and 2048x2048 (4096 or
16384 image tokens plus 512 text tokens, 24 heads of 128 channels), for the
projected-feature student layer (feature_dim 256) and for a long causal
sequence at the NNT layer's default embed 512 / 8 heads.
"""

from dataclasses import dataclass, replace

import numpy as np


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    D: int
    F: int = 0              # 0: no projection (features = D)
    fmap: str = "elu"       # "elu" (elu(x)+1) or "relu"
    eps: float = 1e-6
    causal: bool = False
    dtype: str = "bf16"     # "bf16" or "f32"
    qk_unit_sqrtd: bool = False   # q, k rows L2-normalised then scaled by sqrt(D)
    seed: int = 0

    @property
    def tokens(self):
        return self.B * self.H * self.N

    @property
    def features(self):
        return self.F if self.F else self.D

    def with_(self, **kw):
        return replace(self, **kw)


WORKLOADS = {
    "tiny_f32": Workload("tiny_f32", 1, 2, 256, 64, dtype="f32", seed=1001),
    "flux1024": Workload("flux1024", 1, 24, 4608, 128, qk_unit_sqrtd=True, seed=1002),
    "flux2048_cfg": Workload("flux2048_cfg", 2, 24, 16896, 128, fmap="relu", seed=1003),
    "proj256": Workload("proj256", 1, 24, 4608, 128, F=256, seed=1004),
    "causal32k": Workload("causal32k", 4, 8, 32768, 64, causal=True, seed=1005),
}


def _draw(w: Workload, seed=None):
    rng = np.random.default_rng(w.seed if seed is None else seed)
    shape = (w.B, w.H, w.N, w.D)
    q = rng.standard_normal(shape, dtype=np.float32)
    k = rng.standard_normal(shape, dtype=np.float32)
    v = rng.standard_normal(shape, dtype=np.float32)
    W = None
    if w.F:
        W = rng.standard_normal((w.H, w.D, w.F), dtype=np.float32) * np.float32(1.0 / np.sqrt(w.D))
    if w.qk_unit_sqrtd:
        s = np.float32(np.sqrt(w.D))
        q = q / np.linalg.norm(q, axis=-1, keepdims=True) * s
        k = k / np.linalg.norm(k, axis=-1, keepdims=True) * s
    return q, k, v, W


def make_inputs(w: Workload, seed=None):
    """Return (q, k, v, W) as CPU torch tensors of the workload's dtype.

    q, k, v: [B, H, N, D]; W: [H, D, F] or None.
    """
    import torch
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    q, k, v, W = _draw(w, seed)
    cvt = lambda a: None if a is None else torch.from_numpy(np.ascontiguousarray(a)).to(dt)
    return cvt(q), cvt(k), cvt(v), cvt(W)


def as_float64(t):
    """The stored values of a torch tensor as a float64 numpy array."""
    if t is None:
        return None
    import torch
    return t.detach().to("cpu", torch.float64).numpy()


def e4m3_scale(a):
    """Power-of-two scale that keeps the largest |a| / scale at or below 448,
    the largest finite E4M3 value (1.0 for an all-zero array)."""
    amax = float(np.abs(a).max()) if a.size else 0.0
    if amax == 0.0:
        return 1.0
    return float(2.0 ** np.ceil(np.log2(amax / 448.0)))


def make_e4m3_inputs(w: Workload, seed=None):
    """E4M3 storage of the workload's q, k, v: (q8, k8, v8, scales).

    The values are drawn as for ``make_inputs``, divided by a per-tensor
    power-of-two scale (``e4m3_scale``) and rounded to the nearest code by
    torch's float8_e4m3fn conversion; q8, k8, v8 are uint8 CPU tensors of the
    codes and ``scales`` the three scales, so that the stored tensors are
    scale x code value.
    """
    import torch
    q, k, v, _ = _draw(w, seed)
    codes, scales = [], []
    for a in (q, k, v):
        s = e4m3_scale(a)
        t = torch.from_numpy(np.ascontiguousarray(a / np.float32(s)))
        codes.append(t.to(torch.float8_e4m3fn).view(torch.uint8).contiguous())
        scales.append(s)
    return codes[0], codes[1], codes[2], tuple(scales)


def make_prologue_params(w: Workload, seed=None, base=10000.0):
    """Parameters of Flux's attention prologue for workload w, as float32 CPU
    torch tensors: (q_scale [D], k_scale [D], rope [N, D/2, 2]).

    The norm scales are 1 + 0.1 N(0, 1) draws; the rotation table holds
    (cos, sin) of the angles n base^(-2 i / D) of the usual rotary frequencies,
    evaluated in float64 and stored as float32.
    """
    import torch
    rng = np.random.default_rng((w.seed if seed is None else seed) + 40009)
    qs = (1.0 + 0.1 * rng.standard_normal(w.D)).astype(np.float32)
    ks = (1.0 + 0.1 * rng.standard_normal(w.D)).astype(np.float32)
    ang = np.arange(w.N, dtype=np.float64)[:, None] * base ** (-2.0 * np.arange(w.D // 2) / w.D)[None, :]
    rope = np.stack([np.cos(ang), np.sin(ang)], axis=-1).astype(np.float32)
    return torch.from_numpy(qs), torch.from_numpy(ks), torch.from_numpy(np.ascontiguousarray(rope))

