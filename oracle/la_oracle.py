"""Float64 CPU oracle for linear-time kernelised ("phi") attention.

TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT. Only ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import
this module. The CUDA library never calls it and shares no code with it.

What it computes (page "NNT Define Linear Attention", sections "The inputs" and
"How it works"): a non-negative feature map phi is applied to queries and keys;
the similarity of query i and key j is phi(q_i).phi(k_j); every output row is
the similarity-weighted sum of value rows, divided by the sum of the weights
plus ``eps``.  The page's "How it works" section states the fast form that
groups the product as phi(Q) (phi(K)^T V) and normalises by
1 / (phi(Q) . sum_j phi(k_j) + eps); the definition below is the ungrouped
weighted sum, and the grouped form is implemented separately so that each can
be checked against the other.

Readings taken here where the pages leave a step open:
  * elu is the standard ELU with alpha = 1, so elu(x)+1 is x+1 for x > 0 and
    exp(x) for x <= 0 (page "NNT Define Linear Attention", "The inputs").
  * eps is added once per query row to the summed weights (same page, "How it
    works": normalise by 1 / (Q . sum(K) + eps)).
  * causal means each query sees keys j <= i, itself included (same page,
    "The inputs": tokens attend only to earlier tokens; the diagonal is kept so
    that row 0 is defined).
  * no 1/sqrt(D) temperature is applied (the page names none).
  * the optional projection (page "Flux2TTRTrainer", "Inputs worth setting":
    feature_dim is a multiple of 256) is one D x F matrix per head, shared by
    queries and keys, applied before the feature map: phi(x) = fmap(x W_h).

Everything is float64 with numpy; ``@`` (a library matmul) is the only
primitive used beyond elementwise numpy.  Arrays are [B, H, N, D] with the
feature axis last; W is [H, D, F] (one matrix per head) or [D, F] (shared).
"""

import numpy as np

FEATURE_MAPS = ("elu", "relu", "softmax")


# --------------------------------------------------------------------------
# Feature maps (page "NNT Define Linear Attention", "The inputs": feature_map
# is elu, mapped as elu(x)+1, relu or softmax; all are non-negative).
# --------------------------------------------------------------------------

def phi_elu1(x):
    """elu(x) + 1 with alpha = 1: x + 1 where x > 0, exp(x) where x <= 0."""
    x = np.asarray(x, dtype=np.float64)
    return np.where(x > 0.0, x + 1.0, np.exp(np.minimum(x, 0.0)))


def phi_relu(x):
    """relu(x) = max(x, 0)."""
    x = np.asarray(x, dtype=np.float64)
    return np.maximum(x, 0.0)


def phi_softmax(x):
    """softmax over the feature axis (the last): exp(x_f - max) / sum_f' exp(x_f' - max).

    Reading: the page lists softmax as a third feature map without naming its
    axis; a feature map takes one token's vector to a non-negative vector of
    features, so the softmax runs over that vector.
    """
    x = np.asarray(x, dtype=np.float64)
    e = np.exp(x - x.max(axis=-1, keepdims=True))
    return e / e.sum(axis=-1, keepdims=True)


def feature_map(x, fmap, W=None):
    """phi(x) for rows x[..., D].

    With ``W`` (D x F) the map is fmap(x W) (the projected-feature form, page
    "Flux2TTRTrainer", "Inputs worth setting"); without it, fmap acts on x
    directly and F = D.
    """
    x = np.asarray(x, dtype=np.float64)
    if W is not None:
        x = x @ np.asarray(W, dtype=np.float64)
    if fmap == "elu":
        return phi_elu1(x)
    if fmap == "relu":
        return phi_relu(x)
    if fmap == "softmax":
        return phi_softmax(x)
    raise ValueError(f"unknown feature map {fmap!r}")


def _head_W(W, h):
    if W is None:
        return None
    W = np.asarray(W, dtype=np.float64)
    return W if W.ndim == 2 else W[h]


# --------------------------------------------------------------------------
# The definition: explicit weights, O(N^2) per head.
# --------------------------------------------------------------------------

def brute_force_head(q, k, v, fmap, eps, causal, W=None):
    """One head by the definition.

    out_i = sum_j w_ij v_j / (sum_j w_ij + eps),  w_ij = phi(q_i) . phi(k_j),
    with j over all keys (non-causal) or over j <= i (causal).
    q, k: [N, D]; v: [N, Dv]. Returns [N, Dv] float64.
    """
    pq = feature_map(q, fmap, W)
    pk = feature_map(k, fmap, W)
    v = np.asarray(v, dtype=np.float64)
    w = pq @ pk.T                      # w[i, j] = phi(q_i) . phi(k_j)
    if causal:
        w = np.tril(w)                 # keep j <= i
    num = w @ v
    den = w.sum(axis=1) + eps
    return num / den[:, None]


def brute_force_rows(q, k, v, rows, fmap, eps, causal, W=None):
    """Selected query rows of one head by the definition, one row at a time.

    Costs O(len(rows) * N * (F + D)); used to check single outputs of large
    problems.  Returns [len(rows), Dv] float64.
    """
    pk = feature_map(k, fmap, W)
    v = np.asarray(v, dtype=np.float64)
    out = np.empty((len(rows), v.shape[1]), dtype=np.float64)
    for r, i in enumerate(rows):
        pqi = feature_map(q[i:i + 1], fmap, W)[0]
        jend = i + 1 if causal else pk.shape[0]
        w = pk[:jend] @ pqi            # w_j = phi(q_i) . phi(k_j)
        out[r] = (w @ v[:jend]) / (w.sum() + eps)
    return out


# --------------------------------------------------------------------------
# The grouped (linear-time) forms the method uses.
# --------------------------------------------------------------------------

def linear_noncausal_head(q, k, v, fmap, eps, W=None):
    """Grouped form of page "NNT Define Linear Attention", "How it works".

    kv = phi(K)^T V (F x Dv), ksum = sum_j phi(k_j) (F),
    out_i = phi(q_i)^T kv / (phi(q_i) . ksum + eps).
    """
    pq = feature_map(q, fmap, W)
    pk = feature_map(k, fmap, W)
    v = np.asarray(v, dtype=np.float64)
    kv = pk.T @ v
    ksum = pk.sum(axis=0)
    num = pq @ kv
    den = pq @ ksum + eps
    return num / den[:, None]


def linear_causal_head(q, k, v, fmap, eps, W=None):
    """Causal grouped form as a token-by-token recurrence.

    The state S = sum_{j<=i} phi(k_j) v_j^T and z = sum_{j<=i} phi(k_j) are
    updated with token i first, then row i is read out from them, so query i
    sees keys 0..i (the inclusive reading of "earlier tokens").
    """
    pq = feature_map(q, fmap, W)
    pk = feature_map(k, fmap, W)
    v = np.asarray(v, dtype=np.float64)
    n, f = pk.shape
    S = np.zeros((f, v.shape[1]), dtype=np.float64)
    z = np.zeros(f, dtype=np.float64)
    out = np.empty((n, v.shape[1]), dtype=np.float64)
    for i in range(n):
        S += np.outer(pk[i], v[i])
        z += pk[i]
        out[i] = (pq[i] @ S) / (pq[i] @ z + eps)
    return out


# --------------------------------------------------------------------------
# Whole [B, H, N, D] problems.
# --------------------------------------------------------------------------

def _check(q, k, v, fmap, eps):
    if fmap not in FEATURE_MAPS:
        raise ValueError(f"unknown feature map {fmap!r}")
    if eps < 0:
        raise ValueError("eps must be >= 0")
    if q.ndim != 4 or k.shape != q.shape or v.shape[:3] != q.shape[:3]:
        raise ValueError("q, k, v must be [B, H, N, D] with matching B, H, N")


def forward(q, k, v, fmap="elu", eps=1e-6, causal=False, W=None):
    """Grouped form over all heads; returns float64 [B, H, N, Dv]."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    _check(q, k, v, fmap, eps)
    B, H, N, _ = q.shape
    out = np.empty(q.shape[:3] + (v.shape[3],), dtype=np.float64)
    for b in range(B):
        for h in range(H):
            Wh = _head_W(W, h)
            if causal:
                out[b, h] = linear_causal_head(q[b, h], k[b, h], v[b, h], fmap, eps, Wh)
            else:
                out[b, h] = linear_noncausal_head(q[b, h], k[b, h], v[b, h], fmap, eps, Wh)
    return out


def brute_force(q, k, v, fmap="elu", eps=1e-6, causal=False, W=None):
    """The definition over all heads; returns float64 [B, H, N, Dv]."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    _check(q, k, v, fmap, eps)
    B, H, N, _ = q.shape
    out = np.empty(q.shape[:3] + (v.shape[3],), dtype=np.float64)
    for b in range(B):
        for h in range(H):
            out[b, h] = brute_force_head(q[b, h], k[b, h], v[b, h], fmap, eps, causal,
                                         _head_W(W, h))
    return out


def rows(q, k, v, b, h, idx, fmap="elu", eps=1e-6, causal=False, W=None):
    """Rows ``idx`` of head (b, h) by the definition; float64 [len(idx), Dv]."""
    return brute_force_rows(np.asarray(q[b, h], dtype=np.float64),
                            np.asarray(k[b, h], dtype=np.float64),
                            np.asarray(v[b, h], dtype=np.float64),
                            list(idx), fmap, eps, causal, _head_W(W, h))


# --------------------------------------------------------------------------
# The TTR student layer (page "Flux2TTRTrainer", "How the distillation works"):
# a linear-time kernel branch (the grouped form above) and a small
# exact-softmax branch over "landmark" tokens, blended by a bounded weight.
# The page names the landmark knobs (fraction, min, max; "Inputs worth
# setting") but gives neither the selection rule nor the blend form.
# Readings taken here:
#   * L landmarks, evenly spaced over the sequence: token floor(l N / L) for
#     l = 0..L-1, with L = clamp(round(fraction N), min, max), then clamped to
#     [1, N] (round half up);
#   * the landmark branch is exact softmax attention of every query over the
#     landmark keys and values, scores q_i . k_j / sqrt(D) (the scale of the
#     attention the layer replaces), no feature map and no projection;
#   * the bounded weight is alpha_h = sigmoid(g_h) for a per-head logit g_h,
#     out = alpha_h * landmark branch + (1 - alpha_h) * kernel branch;
#   * non-causal only (the layer replaces Flux's bidirectional attention).
# --------------------------------------------------------------------------

def landmark_count(n, fraction, lo, hi):
    """Number of landmarks: round(fraction * n) clamped to [lo, hi], then to [1, n]."""
    want = int(np.floor(fraction * n + 0.5))
    return max(1, min(n, max(lo, min(hi, want))))


def landmark_positions(n, count):
    """Token indices of ``count`` evenly spaced landmarks among ``n`` tokens."""
    return [(l * n) // count for l in range(count)]


def sigmoid(g):
    """1 / (1 + exp(-g)), evaluated without overflow for large |g|."""
    g = float(g)
    if g >= 0.0:
        return 1.0 / (1.0 + np.exp(-g))
    e = np.exp(g)
    return e / (1.0 + e)


def landmark_head(q, k, v, positions):
    """Exact softmax attention of every query row over the landmark rows.

    scores s_il = q_i . k_{p_l} / sqrt(D); weights softmax_l(s_il) (per query,
    over the landmarks); returns weights @ v[positions], [N, Dv] float64.
    """
    q = np.asarray(q, dtype=np.float64)
    kl = np.asarray(k, dtype=np.float64)[positions]
    vl = np.asarray(v, dtype=np.float64)[positions]
    s = (q @ kl.T) / np.sqrt(q.shape[1])
    s = s - s.max(axis=1, keepdims=True)
    e = np.exp(s)
    return (e / e.sum(axis=1, keepdims=True)) @ vl


def ttr_forward(q, k, v, gate, n_landmarks, fmap="elu", eps=1e-6, W=None):
    """The blended layer over all heads; ``gate`` holds one logit per head.

    Returns float64 [B, H, N, Dv]: alpha_h landmark + (1 - alpha_h) kernel.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    _check(q, k, v, fmap, eps)
    B, H, N, _ = q.shape
    gate = np.asarray(gate, dtype=np.float64).reshape(-1)
    if gate.shape[0] != H:
        raise ValueError("one gate logit per head")
    if not 1 <= n_landmarks <= N:
        raise ValueError("n_landmarks must be in [1, N]")
    pos = landmark_positions(N, n_landmarks)
    out = np.empty(q.shape[:3] + (v.shape[3],), dtype=np.float64)
    for b in range(B):
        for h in range(H):
            a = sigmoid(gate[h])
            lin = linear_noncausal_head(q[b, h], k[b, h], v[b, h], fmap, eps, _head_W(W, h))
            lm = landmark_head(q[b, h], k[b, h], v[b, h], pos)
            out[b, h] = a * lm + (1.0 - a) * lin
    return out


# --------------------------------------------------------------------------
# FP8 storage of Q, K and V (page "FLUXNATION", section "What it does": an
# FP8 CUDA kernel).  Readings: FP8 is the E4M3 format of the OCP 8-bit
# floating-point specification in its finite form (sign bit, four exponent
# bits with bias 7, three mantissa bits; no infinities; exponent 1111 with
# mantissa 111 is NaN; largest finite value 448), and each tensor carries one
# fp32 scale, its stored values being scale x code value.  The layer itself is
# unchanged: it runs on the dequantised tensors.
# --------------------------------------------------------------------------

def e4m3_decode(codes):
    """Float64 values of E4M3 codes (uint8 array of any shape).

    Exponent field e and mantissa field m: (1 + m/8) 2^(e-7) for e >= 1,
    (m/8) 2^-6 for e = 0 (subnormals); the sign bit negates; e = 15 with
    m = 7 is NaN.
    """
    c = np.asarray(codes).astype(np.int64)
    if np.any((c < 0) | (c > 255)):
        raise ValueError("E4M3 codes are bytes")
    e = (c >> 3) & 0xF
    m = c & 0x7
    mag = np.where(e == 0, (m / 8.0) * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    val = np.where((c & 0x80) != 0, -mag, mag)
    return np.where((e == 15) & (m == 7), np.nan, val)


def forward_e4m3(q8, k8, v8, scales, fmap="elu", eps=1e-6):
    """The non-causal layer on E4M3-stored Q, K, V (uint8 [B, H, N, D] codes).

    ``scales`` = (scale_q, scale_k, scale_v): each tensor is dequantised as
    scale x e4m3_decode(codes) before ``forward``.  Returns float64.
    """
    sq, sk, sv = (float(x) for x in scales)
    return forward(sq * e4m3_decode(q8), sk * e4m3_decode(k8), sv * e4m3_decode(v8), fmap, eps, causal=False)


# --------------------------------------------------------------------------
# The attention prologue of Flux's block (page "FLUXNATION", section "What it
# does": QKV split and RoPE fused into the block's kernel).  Readings: the
# split q and k of a head pass through Flux's QK norm, an RMS norm over the
# head dimension times a learned per-feature scale, and then the rotary
# position embedding, which rotates each feature pair (2i, 2i + 1) of the
# token at position n by the angle whose (cos, sin) is rope[n, i]; v is left
# as it is.  The layer then runs on the transformed q and k.
# --------------------------------------------------------------------------

def rms_norm(x, scale, norm_eps):
    """x / sqrt(mean_d x_d^2 + norm_eps) * scale over the last axis."""
    x = np.asarray(x, dtype=np.float64)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + norm_eps) * np.asarray(scale, dtype=np.float64)


def rope(x, table):
    """Rotate pairs (x_2i, x_2i+1) of token n by rope[n, i] = (cos, sin):
    (c x_2i - s x_2i+1, s x_2i + c x_2i+1).  x [..., N, D], table [N, D/2, 2]."""
    x = np.asarray(x, dtype=np.float64)
    t = np.asarray(table, dtype=np.float64)
    n = x.shape[-2]
    c, s = t[:n, :, 0], t[:n, :, 1]
    x0, x1 = x[..., 0::2], x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = c * x0 - s * x1
    out[..., 1::2] = s * x0 + c * x1
    return out


def forward_prologue(q, k, v, q_scale, k_scale, table, norm_eps=1e-6, fmap="elu", eps=1e-6, causal=False):
    """The layer on rope(rms_norm(q)), rope(rms_norm(k)), v.  Returns float64."""
    qn = rope(rms_norm(q, q_scale, norm_eps), table)
    kn = rope(rms_norm(k, k_scale, norm_eps), table)
    return forward(qn, kn, v, fmap, eps, causal)


# --------------------------------------------------------------------------
# Backward pass of the non-causal layer (page "Flux2TTRTrainer", "How the
# distillation works": the student layer is trained by distillation, which
# needs the gradients of the loss with respect to q, k and v).  For a loss L
# with dL/dout = dout, per head with F = D features:
#   den_i = phi(q_i).z + eps, out_i = phi(q_i) kv / den_i,
#   g_i = dout_i / den_i,  h_i = -(dout_i . out_i) / den_i,
#   dphi(q_i) = kv g_i + h_i z,   dkv = sum_i phi(q_i) g_i^T,   dz = sum_i h_i phi(q_i),
#   dphi(k_j) = dkv v_j + dz,     dv_j = dkv^T phi(k_j),
# and dq = dphi(q) * phi'(q), dk = dphi(k) * phi'(k) elementwise.
# --------------------------------------------------------------------------

def feature_map_grad(x, fmap):
    """phi'(x) elementwise: elu(x)+1 -> 1 for x > 0, exp(x) otherwise; relu ->
    1 for x > 0, 0 otherwise (0 at x = 0)."""
    x = np.asarray(x, dtype=np.float64)
    if fmap == "elu":
        return np.where(x > 0.0, 1.0, np.exp(np.minimum(x, 0.0)))
    if fmap == "relu":
        return np.where(x > 0.0, 1.0, 0.0)
    raise ValueError(f"no gradient for feature map {fmap!r}")


def backward_head(q, k, v, dout, fmap, eps):
    """(dq, dk, dv) of one non-causal head without projection, float64."""
    q, k, v, dout = (np.asarray(a, dtype=np.float64) for a in (q, k, v, dout))
    pq, pk = feature_map(q, fmap), feature_map(k, fmap)
    kv = pk.T @ v
    z = pk.sum(axis=0)
    den = pq @ z + eps
    out = (pq @ kv) / den[:, None]
    g = dout / den[:, None]
    h = -(dout * out).sum(axis=1) / den
    dpq = g @ kv.T + h[:, None] * z[None, :]
    dkv = pq.T @ g
    dz = pq.T @ h
    dpk = v @ dkv.T + dz[None, :]
    dv = pk @ dkv
    return dpq * feature_map_grad(q, fmap), dpk * feature_map_grad(k, fmap), dv


def backward(q, k, v, dout, fmap="elu", eps=1e-6):
    """Gradients (dq, dk, dv) of sum(out * dout) over all heads, non-causal,
    no projection; float64 [B, H, N, D] each."""
    q, k, v = (np.asarray(a, dtype=np.float64) for a in (q, k, v))
    _check(q, k, v, fmap, eps)
    if fmap not in ("elu", "relu"):
        raise ValueError("backward: elu or relu feature maps")
    dout = np.asarray(dout, dtype=np.float64)
    dq, dk, dv = np.empty_like(q), np.empty_like(k), np.empty_like(v)
    for b in range(q.shape[0]):
        for h in range(q.shape[1]):
            dq[b, h], dk[b, h], dv[b, h] = backward_head(q[b, h], k[b, h], v[b, h], dout[b, h], fmap, eps)
    return dq, dk, dv

