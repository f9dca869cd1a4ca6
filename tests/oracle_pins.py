"""Pins that tie the float64 oracle to facts fixed outside the oracle itself.

Each pin takes an oracle namespace ``ora`` (the real ``oracle.la_oracle`` or a
copy with a planted mistake) and raises AssertionError when ``ora`` disagrees
with a hand-derived worked example, a closed form, an invariant of the method
or a library routine.  The definition they check is the one on page "NNT Define
Linear Attention" ("The inputs", "How it works"):

    out_i = sum_j w_ij v_j / (sum_j w_ij + eps),   w_ij = phi(q_i) . phi(k_j)

with j <= i for the causal variant, phi = elu(x)+1 or relu, optionally after a
per-head D x F projection (page "Flux2TTRTrainer", "Inputs worth setting").
"""

import math
import os
from fractions import Fraction

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
SCALAR_KEYS = ("fmap", "eps", "landmarks", "gate0", "gate1")


# ---------------------------------------------------------------- fixtures --

def load_golden(name):
    """Parse a tests/golden text fixture into float64 arrays."""
    sections = {}
    cur = None
    with open(os.path.join(GOLDEN, name)) as fh:
        for raw in fh:
            line = raw.split("#", 1)[0].strip()
            if not line:
                continue
            parts = line.split()
            if parts[0] in SCALAR_KEYS:
                sections[parts[0]] = parts[1]
                cur = None
            elif len(parts) == 1 and not _is_number(parts[0]):
                cur = parts[0]
                sections[cur] = []
            else:
                sections[cur].append([float(Fraction(p)) for p in parts])
    out = {"fmap": sections["fmap"], "eps": float(Fraction(sections["eps"]))}
    for key in ("landmarks", "gate0", "gate1"):
        if key in sections:
            out[key] = sections[key]
    for key in ("q", "k", "v", "W", "out_noncausal", "out_causal", "out_head0", "out_head1"):
        if key in sections:
            out[key] = np.array(sections[key], dtype=np.float64)
    return out


def _is_number(tok):
    try:
        Fraction(tok)
        return True
    except ValueError:
        return False


def _as4(x):
    return np.asarray(x, dtype=np.float64)[None, None]


def _rng(seed):
    return np.random.default_rng(seed)


def _close(a, b, rtol=1e-12, atol=1e-13):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, (a.shape, b.shape)
    assert np.all(np.isfinite(a)), "non-finite values"
    err = np.max(np.abs(a - b)) if a.size else 0.0
    scale = max(np.max(np.abs(b)) if b.size else 0.0, 1.0)
    assert err <= atol + rtol * scale, f"max |diff| = {err:.3e}"


# -------------------------------------------------------------------- pins --

def pin_feature_maps(ora):
    """phi values fixed by the definitions of elu(x)+1 and relu."""
    x = np.array([-3.0, -1.0, -0.25, 0.0, 0.5, 2.0], dtype=np.float64)
    expect_elu = np.array([math.exp(-3.0), math.exp(-1.0), math.exp(-0.25), 1.0, 1.5, 3.0])
    _close(ora.phi_elu1(x), expect_elu, rtol=1e-15, atol=0)
    _close(ora.feature_map(x[None], "elu")[0], expect_elu, rtol=1e-15, atol=0)
    _close(ora.phi_relu(x), np.array([0, 0, 0, 0, 0.5, 2.0]), rtol=0, atol=0)
    _close(ora.feature_map(x[None], "relu")[0], np.array([0, 0, 0, 0, 0.5, 2.0]), rtol=0, atol=0)


def pin_feature_map_vs_torch(ora):
    """elu(x)+1 against the library ELU (alpha = 1) on a wide range."""
    import torch
    x = np.linspace(-30.0, 30.0, 2001)
    ref = torch.nn.functional.elu(torch.from_numpy(x), alpha=1.0).numpy() + 1.0
    _close(ora.phi_elu1(x), ref, rtol=1e-14, atol=1e-300)
    ref_relu = torch.relu(torch.from_numpy(x)).numpy()
    _close(ora.phi_relu(x), ref_relu, rtol=0, atol=0)


def pin_golden(ora):
    """Hand-derived worked examples (tests/golden/*.txt), every oracle entry."""
    for name in ("tiny_elu_rational.txt", "tiny_relu_rational.txt",
                 "tiny_projected_rational.txt"):
        g = load_golden(name)
        q, k, v, W = _as4(g["q"]), _as4(g["k"]), _as4(g["v"]), g.get("W")
        Wf = None if W is None else W[None]  # [H=1, D, F]
        for causal, key in ((False, "out_noncausal"), (True, "out_causal")):
            exp = g[key]
            _close(ora.forward(q, k, v, g["fmap"], g["eps"], causal, Wf)[0, 0], exp,
                   rtol=1e-14, atol=1e-15)
            _close(ora.brute_force(q, k, v, g["fmap"], g["eps"], causal, Wf)[0, 0], exp,
                   rtol=1e-14, atol=1e-15)
            _close(ora.rows(q, k, v, 0, 0, range(exp.shape[0]), g["fmap"], g["eps"],
                            causal, Wf), exp, rtol=1e-14, atol=1e-15)


def pin_negative_elu_closed_form(ora):
    """One query, keys on both elu branches, worked out with math.exp.

    q = [-1], k = [1, -2], v = [3, 5]:  phi(q) = e^-1, phi(k) = [2, e^-2],
    out = (3*2 + 5 e^-2) e^-1 / ((2 + e^-2) e^-1 + eps).
    """
    eps = 1e-3
    q = _as4([[-1.0], [-1.0]])
    k = _as4([[1.0], [-2.0]])
    v = _as4([[3.0], [5.0]])
    e1, e2 = math.exp(-1.0), math.exp(-2.0)
    full = (6.0 + 5.0 * e2) * e1 / ((2.0 + e2) * e1 + eps)
    first = 6.0 * e1 / (2.0 * e1 + eps)
    for f in (ora.forward, ora.brute_force):
        _close(f(q, k, v, "elu", eps, False)[0, 0, :, 0], [full, full], rtol=1e-14)
        _close(f(q, k, v, "elu", eps, True)[0, 0, :, 0], [first, full], rtol=1e-14)


def pin_constant_values(ora):
    """v_j = c for all j gives out_i = c * s_i / (s_i + eps) (s_i: row weight sum)."""
    rng = _rng(11)
    B, H, N, D = 1, 2, 37, 8
    q = rng.standard_normal((B, H, N, D))
    k = rng.standard_normal((B, H, N, D))
    c = rng.standard_normal(D)
    v = np.broadcast_to(c, (B, H, N, D)).copy()
    for fmap in ("elu", "relu"):
        for causal in (False, True):
            for f in (ora.forward, ora.brute_force):
                o0 = f(q, k, v, fmap, 0.0, causal)
                _close(o0, v, rtol=1e-12, atol=1e-12)     # eps = 0: exactly c
            # eps > 0: every row is c scaled by the same factor in (0, 1]
            o = ora.forward(q, k, v, fmap, 0.5, causal)
            ratio = o / c
            assert np.all(ratio <= 1.0 + 1e-12) and np.all(ratio > 0.0)
            _close(ratio, np.repeat(ratio[..., :1], D, axis=-1), rtol=1e-12)


def pin_zero_qk_closed_form(ora):
    """Q = K = 0 under elu+1: phi = 1, every weight is D.

    Non-causal out_i = mean_j v_j * N D / (N D + eps);
    causal    out_i = mean_{j<=i} v_j * (i+1) D / ((i+1) D + eps).
    """
    rng = _rng(12)
    B, H, N, D = 1, 1, 23, 5
    z = np.zeros((B, H, N, D))
    v = rng.standard_normal((B, H, N, 3))
    eps = 0.75
    mean = v[0, 0].mean(axis=0)
    exp_nc = np.tile(mean * (N * D) / (N * D + eps), (N, 1))
    cnt = np.arange(1, N + 1)[:, None]
    exp_c = np.cumsum(v[0, 0], axis=0) / cnt * (cnt * D) / (cnt * D + eps)
    for f in (ora.forward, ora.brute_force):
        _close(f(z, z, v, "elu", eps, False)[0, 0], exp_nc, rtol=1e-13)
        _close(f(z, z, v, "elu", eps, True)[0, 0], exp_c, rtol=1e-13)


def pin_identity_values_give_weights(ora):
    """With N <= Dv and V = I, row i of the output is the normalised weight row.

    Weights are non-negative; each row sums to s_i / (s_i + eps) <= 1; entries
    are proportional to phi(q_i).phi(k_j) computed here by explicit loops.
    """
    rng = _rng(13)
    N, D = 9, 6
    q = rng.standard_normal((1, 1, N, D))
    k = rng.standard_normal((1, 1, N, D))
    v = np.eye(N)[None, None]
    for fmap in ("elu", "relu"):
        for causal in (False, True):
            for f in (ora.forward, ora.brute_force):
                w = f(q, k, v, fmap, 1e-6, causal)[0, 0]
                assert np.all(w >= -1e-15)
                assert np.all(w.sum(axis=1) <= 1.0 + 1e-12)
                if fmap == "elu":     # elu+1 > 0: rows sum to 1 up to eps
                    _close(w.sum(axis=1), np.ones(N), rtol=0, atol=1e-5)
                if causal:
                    assert np.all(np.triu(w, 1) == 0.0)
                # proportionality to explicit dot products of the feature map
                for i in range(N):
                    pq = [(x + 1.0 if x > 0 else math.exp(x)) if fmap == "elu" else max(x, 0.0)
                          for x in q[0, 0, i]]
                    raw = []
                    for j in range(N):
                        pk = [(x + 1.0 if x > 0 else math.exp(x)) if fmap == "elu" else max(x, 0.0)
                              for x in k[0, 0, j]]
                        raw.append(sum(a * b for a, b in zip(pq, pk)) if (not causal or j <= i) else 0.0)
                    s = sum(raw)
                    exp = [r / (s + 1e-6) for r in raw]
                    _close(w[i], exp, rtol=1e-12, atol=1e-14)


def pin_linear_equals_definition(ora):
    """The grouped form phi(Q)(phi(K)^T V) equals the weighted-sum definition."""
    rng = _rng(14)
    B, H, N, D = 2, 3, 41, 7
    q = rng.standard_normal((B, H, N, D))
    k = rng.standard_normal((B, H, N, D))
    v = rng.standard_normal((B, H, N, D))
    W = rng.standard_normal((H, D, 16)) / math.sqrt(D)
    for fmap in ("elu", "relu"):
        for causal in (False, True):
            for Wx in (None, W, W[1]):
                a = ora.forward(q, k, v, fmap, 1e-6, causal, Wx)
                b = ora.brute_force(q, k, v, fmap, 1e-6, causal, Wx)
                _close(a, b, rtol=1e-12, atol=1e-13)
                r = ora.rows(q, k, v, 1, 2, [0, 5, N - 1], fmap, 1e-6, causal, Wx)
                _close(r, b[1, 2, [0, 5, N - 1]], rtol=1e-12, atol=1e-13)


def pin_causal_structure(ora):
    """Row 0 sees only key 0; the last causal row equals the last non-causal row;
    row i of a causal problem equals the non-causal answer on the first i+1 tokens."""
    rng = _rng(15)
    N, D = 17, 4
    q = rng.standard_normal((1, 1, N, D))
    k = rng.standard_normal((1, 1, N, D))
    v = rng.standard_normal((1, 1, N, D))
    for fmap in ("elu", "relu"):
        c = ora.forward(q, k, v, fmap, 1e-6, True)
        nc = ora.forward(q, k, v, fmap, 1e-6, False)
        _close(c[0, 0, -1], nc[0, 0, -1], rtol=1e-12)
        for i in (0, 3, 9):
            pre = ora.forward(q[:, :, :i + 1], k[:, :, :i + 1], v[:, :, :i + 1], fmap, 1e-6, False)
            _close(c[0, 0, i], pre[0, 0, i], rtol=1e-12)
        # row 0: s = phi(q_0).phi(k_0), out = v_0 s/(s+eps)
        pq = ora.feature_map(q[0, 0, :1], fmap)[0]
        pk = ora.feature_map(k[0, 0, :1], fmap)[0]
        s = float(sum(a * b for a, b in zip(pq, pk)))
        _close(c[0, 0, 0], v[0, 0, 0] * s / (s + 1e-6), rtol=1e-12)


def pin_invariances(ora):
    """Linear in V; non-causal output invariant to a joint permutation of the
    key/value rows; relu with eps = 0 invariant to scaling a query by c > 0."""
    rng = _rng(16)
    B, H, N, D = 1, 2, 29, 6
    q = rng.standard_normal((B, H, N, D))
    k = rng.standard_normal((B, H, N, D))
    v1 = rng.standard_normal((B, H, N, D))
    v2 = rng.standard_normal((B, H, N, D))
    for causal in (False, True):
        lhs = ora.forward(q, k, 2.0 * v1 - 3.0 * v2, "elu", 1e-6, causal)
        rhs = 2.0 * ora.forward(q, k, v1, "elu", 1e-6, causal) - 3.0 * ora.forward(q, k, v2, "elu", 1e-6, causal)
        _close(lhs, rhs, rtol=1e-11)
    perm = rng.permutation(N)
    _close(ora.forward(q, k[:, :, perm], v1[:, :, perm], "elu", 1e-6, False),
           ora.forward(q, k, v1, "elu", 1e-6, False), rtol=1e-12)
    # permuting the queries permutes the rows
    _close(ora.forward(q[:, :, perm], k, v1, "relu", 1e-6, False),
           ora.forward(q, k, v1, "relu", 1e-6, False)[:, :, perm], rtol=1e-12)
    qpos = np.abs(q) + 0.1
    _close(ora.forward(3.5 * qpos, k, v1, "relu", 0.0, False),
           ora.forward(qpos, k, v1, "relu", 0.0, False), rtol=1e-12)


def pin_relu_zero_denominator(ora):
    """relu with a query row <= 0: every weight is 0 and the row is 0/eps = 0."""
    rng = _rng(17)
    N, D = 8, 4
    q = rng.standard_normal((1, 1, N, D))
    q[0, 0, 3] = -np.abs(q[0, 0, 3])
    k = rng.standard_normal((1, 1, N, D))
    v = rng.standard_normal((1, 1, N, D))
    for causal in (False, True):
        for f in (ora.forward, ora.brute_force):
            o = f(q, k, v, "relu", 1e-6, causal)
            assert np.all(o[0, 0, 3] == 0.0)
            assert np.all(np.isfinite(o))


def pin_projection_reduction(ora):
    """W = [I_D | 0] (D x F): phi(xW) = [elu(x)+1, 1, ..., 1], so
    w_ij = (elu(q_i)+1).(elu(k_j)+1) + (F - D); checked against weights built
    here from the unprojected feature map.  A per-head W is indexed by head."""
    rng = _rng(18)
    B, H, N, D, F = 1, 2, 13, 4, 12
    q = rng.standard_normal((B, H, N, D))
    k = rng.standard_normal((B, H, N, D))
    v = rng.standard_normal((B, H, N, D))
    W = np.zeros((D, F))
    W[:, :D] = np.eye(D)
    for causal in (False, True):
        got = ora.forward(q, k, v, "elu", 1e-6, causal, W)
        for h in range(H):
            pq = ora.phi_elu1(q[0, h])
            pk = ora.phi_elu1(k[0, h])
            w = pq @ pk.T + (F - D)
            if causal:
                w = np.tril(w)
            exp = (w @ v[0, h]) / (w.sum(axis=1) + 1e-6)[:, None]
            _close(got[0, h], exp, rtol=1e-12)
    # per-head matrices: head 1 gets a permuted identity, which must not change
    # the result, while head 0 gets a scaled one, which must
    Wh = np.stack([2.0 * W, W[:, rng.permutation(F)]])
    got = ora.forward(q, k, v, "elu", 1e-6, False, Wh)
    _close(got[0, 1], ora.forward(q, k, v, "elu", 1e-6, False, W)[0, 1], rtol=1e-12)
    pq = ora.phi_elu1(2.0 * q[0, 0])
    pk = ora.phi_elu1(2.0 * k[0, 0])
    w = pq @ pk.T + (F - D)
    _close(got[0, 0], (w @ v[0, 0]) / (w.sum(axis=1) + 1e-6)[:, None], rtol=1e-12)


# ------------------------------------------------------ the TTR layer pins --
# Page "Flux2TTRTrainer", "How the distillation works": a kernel branch and an
# exact-softmax branch over landmark tokens blended by a bounded weight; the
# landmark rule, the softmax scale and the blend form are the readings stated
# in the oracle (evenly spaced landmarks, q.k/sqrt(D), sigmoid(g) on the
# landmark branch).

def _gate(tok):
    return math.log(3.0) if tok == "ln3" else float(Fraction(tok))


def pin_ttr_golden(ora):
    """Hand-derived worked example (tests/golden/ttr_blend_rational.txt): two
    heads with the same inputs and gates 0 and ln 3 (alpha = 1/2 and 3/4)."""
    g = load_golden("ttr_blend_rational.txt")
    q = np.stack([g["q"], g["q"]])[None]
    k = np.stack([g["k"], g["k"]])[None]
    v = np.stack([g["v"], g["v"]])[None]
    gate = [_gate(g["gate0"]), _gate(g["gate1"])]
    got = ora.ttr_forward(q, k, v, gate, int(g["landmarks"]), g["fmap"], g["eps"])
    _close(got[0, 0], g["out_head0"], rtol=1e-14, atol=1e-15)
    _close(got[0, 1], g["out_head1"], rtol=1e-14, atol=1e-15)


def pin_landmark_rule(ora):
    """Evenly spaced landmark tokens and the clamped count, by hand."""
    assert list(ora.landmark_positions(10, 4)) == [0, 2, 5, 7]
    assert list(ora.landmark_positions(4, 2)) == [0, 2]
    assert list(ora.landmark_positions(5, 5)) == [0, 1, 2, 3, 4]
    assert list(ora.landmark_positions(4608, 128))[:3] == [0, 36, 72]
    assert ora.landmark_count(4608, 1 / 32, 16, 128) == 128     # 144 capped at the max
    assert ora.landmark_count(100, 1 / 32, 16, 128) == 16       # 3 raised to the min
    assert ora.landmark_count(10, 0.5, 16, 128) == 10           # the min capped at N
    assert ora.landmark_count(1000, 0.1, 16, 128) == 100
    assert ora.landmark_count(3, 0.0, 0, 5) == 1                # at least one landmark
    assert ora.landmark_count(30, 0.05, 0, 64) == 2             # 1.5 rounds half up


def pin_sigmoid_values(ora):
    """The bounded weight: sigmoid(0) = 1/2, sigmoid(+-ln 3) = 3/4, 1/4,
    and finite, in (0, 1) or at its limits, for huge logits."""
    _close(ora.sigmoid(0.0), 0.5, rtol=0, atol=1e-16)
    _close(ora.sigmoid(math.log(3.0)), 0.75, rtol=1e-15, atol=0)
    _close(ora.sigmoid(-math.log(3.0)), 0.25, rtol=1e-15, atol=0)
    assert ora.sigmoid(800.0) == 1.0 and ora.sigmoid(-800.0) == 0.0
    for g in (-30.0, -2.5, 0.3, 7.0):
        assert 0.0 < ora.sigmoid(g) < 1.0


def pin_landmark_all_tokens_is_attention(ora):
    """With every token a landmark the softmax branch is plain scaled
    dot-product attention: the library routine (default scale 1/sqrt(D))."""
    import torch
    rng = _rng(41)
    for n, d in ((37, 8), (5, 3)):
        q, k, v = rng.standard_normal((3, n, d))
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q)[None], torch.from_numpy(k)[None], torch.from_numpy(v)[None])[0].numpy()
        _close(ora.landmark_head(q, k, v, list(range(n))), ref, rtol=1e-12)
        pos = ora.landmark_positions(n, n)
        _close(ora.landmark_head(q, k, v, pos), ref, rtol=1e-12)


def pin_landmark_invariances(ora):
    """Shifting every landmark key by one vector u shifts each query's scores
    by a constant (q.u / sqrt(D)): the softmax, and so the branch, is
    unchanged.  Scaling V scales the branch; weights are convex, so every
    output lies between the smallest and largest landmark value."""
    rng = _rng(43)
    q, k, v = rng.standard_normal((3, 40, 6))
    pos = ora.landmark_positions(40, 7)
    base = ora.landmark_head(q, k, v, pos)
    _close(ora.landmark_head(q, k + rng.standard_normal(6), v, pos), base, rtol=1e-11)
    _close(ora.landmark_head(q, k, 3.0 * v, pos), 3.0 * base, rtol=1e-12)
    vl = v[pos]
    assert np.all(base <= vl.max(axis=0) + 1e-12) and np.all(base >= vl.min(axis=0) - 1e-12)


def pin_ttr_blend_limits(ora):
    """A logit far above zero leaves the landmark branch alone, far below it
    the kernel branch alone; in between every output lies between the two
    branches (a convex blend)."""
    rng = _rng(47)
    q, k, v = rng.standard_normal((3, 2, 3, 50, 8))
    q, k, v = q[None, 0], k[None, 0], v[None, 0]
    n_l = 9
    pos = ora.landmark_positions(50, n_l)
    lin = ora.forward(q, k, v, "elu", 1e-6)
    lm = np.stack([ora.landmark_head(q[0, h], k[0, h], v[0, h], pos) for h in range(3)])[None]
    _close(ora.ttr_forward(q, k, v, [60.0, 60.0, 60.0], n_l, "elu", 1e-6), lm, rtol=1e-12)
    _close(ora.ttr_forward(q, k, v, [-60.0, -60.0, -60.0], n_l, "elu", 1e-6), lin, rtol=1e-12)
    mid = ora.ttr_forward(q, k, v, [0.4, -1.3, 2.2], n_l, "elu", 1e-6)
    lo, hi = np.minimum(lin, lm), np.maximum(lin, lm)
    assert np.all(mid >= lo - 1e-12) and np.all(mid <= hi + 1e-12)




# ------------------------------------------------------ softmax feature map --

def pin_softmax_vs_scipy(ora):
    """phi_softmax is scipy's softmax over the last axis (a library routine),
    including rows whose entries are far beyond exp's range."""
    from scipy.special import softmax
    rng = _rng(51)
    for scale in (1.0, 30.0, 800.0):
        x = rng.standard_normal((3, 5, 17)) * scale
        _close(ora.phi_softmax(x), softmax(x, axis=-1), rtol=1e-12, atol=1e-300)
        _close(ora.feature_map(x, "softmax"), softmax(x, axis=-1), rtol=1e-12, atol=1e-300)


def pin_softmax_closed_forms(ora):
    """[0, ln 2, ln 3] -> [1/6, 2/6, 3/6]; a constant row -> 1/D; adding a
    constant to a row changes nothing; the features of a row sum to 1."""
    _close(ora.phi_softmax(np.log([1.0, 2.0, 3.0])), np.array([1.0, 2.0, 3.0]) / 6.0, rtol=1e-14)
    _close(ora.phi_softmax(np.full((2, 8), 3.7)), np.full((2, 8), 1.0 / 8.0), rtol=1e-14)
    x = _rng(52).standard_normal((4, 9))
    _close(ora.phi_softmax(x + 11.0), ora.phi_softmax(x), rtol=1e-12)
    _close(ora.phi_softmax(x).sum(axis=-1), np.ones(4), rtol=1e-14)


def pin_softmax_equal_keys(ora):
    """With every key row equal, every weight is s = phi(q_i).phi(k), so
    out_i = s sum_j v_j / (N s + eps), for the grouped form and the definition."""
    rng = _rng(53)
    N, D = 7, 5
    q = rng.standard_normal((1, 1, N, D))
    k = np.broadcast_to(rng.standard_normal(D), (1, 1, N, D)).copy()
    v = rng.standard_normal((1, 1, N, 3))
    eps = 0.25
    s = ora.phi_softmax(q[0, 0]) @ ora.phi_softmax(k[0, 0, 0])
    want = (s[:, None] * v[0, 0].sum(axis=0)[None, :]) / (N * s[:, None] + eps)
    _close(ora.forward(q, k, v, "softmax", eps)[0, 0], want, rtol=1e-12)
    _close(ora.brute_force(q, k, v, "softmax", eps)[0, 0], want, rtol=1e-12)

# ------------------------------------------------------- FP8 (E4M3) storage --

def _torch_e4m3(codes):
    """Values of E4M3 codes by torch's float8_e4m3fn conversion (a library routine)."""
    import torch
    c = torch.from_numpy(np.ascontiguousarray(np.asarray(codes, dtype=np.uint8)))
    return c.view(torch.float8_e4m3fn).to(torch.float64).numpy()


def pin_e4m3_vs_torch(ora):
    """All 256 codes decode as torch's float8_e4m3fn does (NaN where it has NaN)."""
    c = np.arange(256, dtype=np.uint8)
    got, want = ora.e4m3_decode(c), _torch_e4m3(c)
    assert np.array_equal(np.isnan(got), np.isnan(want))
    ok = ~np.isnan(want)
    assert np.array_equal(got[ok], want[ok])


def pin_e4m3_format_facts(ora):
    """Landmarks of the E4M3 format: 448 the largest finite value, 2^-9 the
    smallest subnormal, 2^-6 the smallest normal, 1.0 at exponent field 7,
    signed zeros, NaN only at S.1111.111, magnitudes increasing with the code,
    and the sign bit negating."""
    d = ora.e4m3_decode
    c = np.arange(256, dtype=np.uint8)
    v = d(c)
    assert d(np.uint8(0x7E)) == 448.0 and d(np.uint8(0xFE)) == -448.0
    assert d(np.uint8(0x01)) == 2.0 ** -9 and d(np.uint8(0x07)) == 7 * 2.0 ** -9
    assert d(np.uint8(0x08)) == 2.0 ** -6 and d(np.uint8(0x38)) == 1.0 and d(np.uint8(0xB8)) == -1.0
    assert d(np.uint8(0x00)) == 0.0 and np.signbit(d(np.uint8(0x80)))
    assert list(np.flatnonzero(np.isnan(v))) == [0x7F, 0xFF]
    assert np.all(np.diff(v[:0x7F]) > 0)
    assert np.array_equal(v[0x80:0xFF], -v[:0x7F])


def pin_e4m3_forward(ora):
    """The layer on E4M3 storage is the layer on scale x decoded codes (decoded
    here by the library routine), and V's scale scales the output."""
    rng = _rng(41)
    shape = (1, 2, 37, 8)
    codes = [rng.integers(0, 256, size=shape).astype(np.uint8) for _ in range(3)]
    for cc in codes:
        cc[(cc & 0x7F) == 0x7F] = 0x3A   # no NaN codes
        cc[(cc & 0x78) >= 0x50] &= 0xC7  # keep magnitudes below about 8
    scales = (0.75, 0.125, 1.5)
    for fmap in ("elu", "relu"):
        want = ora.forward(*(s * _torch_e4m3(cc) for s, cc in zip(scales, codes)), fmap, 1e-6)
        got = ora.forward_e4m3(*codes, scales, fmap, 1e-6)
        _close(got, want, rtol=1e-12)
    twice = ora.forward_e4m3(*codes, (0.75, 0.125, 3.0), "elu", 1e-6)
    _close(twice, 2.0 * ora.forward_e4m3(*codes, scales, "elu", 1e-6), rtol=1e-12)



# ------------------------------------------------ Flux attention prologue --

def _torch_prologue(x, scale, table, norm_eps):
    """RMS norm by torch's rms_norm and the rotation by complex multiplication
    (x_2i + i x_2i+1) (cos + i sin): library routines, independent of the oracle."""
    import torch
    xt = torch.from_numpy(np.asarray(x, dtype=np.float64))
    y = torch.nn.functional.rms_norm(xt, (xt.shape[-1],), torch.from_numpy(np.asarray(scale, np.float64)),
                                     norm_eps).numpy()
    n = y.shape[-2]
    z = (y[..., 0::2] + 1j * y[..., 1::2]) * (table[:n, :, 0] + 1j * table[:n, :, 1])
    out = np.empty_like(y)
    out[..., 0::2], out[..., 1::2] = z.real, z.imag
    return out


def _rope_table(n, d, rng):
    ang = rng.uniform(-np.pi, np.pi, size=(n, d // 2))
    return np.stack([np.cos(ang), np.sin(ang)], axis=-1)


def pin_prologue_vs_library(ora):
    """rms_norm is torch's rms_norm, rope is complex multiplication, and the
    prologue layer is the layer on inputs transformed that way (norm first)."""
    rng = _rng(61)
    B, H, N, D = 1, 2, 11, 8
    q, k, v = (rng.standard_normal((B, H, N, D)) * 2.0 for _ in range(3))
    qs, ks = 1.0 + 0.3 * rng.standard_normal(D), 1.0 + 0.3 * rng.standard_normal(D)
    table = _rope_table(N + 3, D, rng)
    for norm_eps in (1e-6, 0.5):
        _close(ora.rms_norm(q, qs, norm_eps), _torch_prologue(q, qs, np.stack([np.ones((N, D // 2)),
                                                                                np.zeros((N, D // 2))], -1),
                                                             norm_eps), rtol=1e-12)
        want = ora.forward(_torch_prologue(q, qs, table, norm_eps), _torch_prologue(k, ks, table, norm_eps), v,
                           "elu", 1e-6)
        _close(ora.forward_prologue(q, k, v, qs, ks, table, norm_eps, "elu", 1e-6), want, rtol=1e-12)
    _close(ora.rope(q, table), _torch_prologue(q / np.sqrt(np.mean(q * q, -1, keepdims=True)), np.ones(D),
                                               table, 0.0) * np.sqrt(np.mean(q * q, -1, keepdims=True)),
           rtol=1e-10)


def pin_rope_invariants(ora):
    """A zero angle changes nothing, every pair keeps its length, and rotating
    by the angle then by its negative gives the input back."""
    rng = _rng(62)
    x = rng.standard_normal((2, 9, 6))
    ident = np.stack([np.ones((9, 3)), np.zeros((9, 3))], -1)
    _close(ora.rope(x, ident), x, rtol=1e-15)
    t = _rope_table(9, 6, rng)
    y = ora.rope(x, t)
    _close(y[..., 0::2] ** 2 + y[..., 1::2] ** 2, x[..., 0::2] ** 2 + x[..., 1::2] ** 2, rtol=1e-12)
    back = t.copy()
    back[..., 1] = -back[..., 1]
    _close(ora.rope(y, back), x, rtol=1e-12, atol=1e-14)


# ------------------------------------------------------------ backward pass --

def pin_backward_finite_differences(ora):
    """Each gradient entry equals the central difference of sum(out * dout)
    computed with the definition (brute force), for elu and relu, at points
    away from relu's kink."""
    rng = _rng(71)
    B, H, N, D = 1, 2, 5, 3
    q, k, v, dout = (rng.standard_normal((B, H, N, D)) for _ in range(4))
    for fmap in ("elu", "relu"):
        if fmap == "relu":   # keep every entry away from 0
            q = np.where(np.abs(q) < 0.2, q + np.sign(q + 1e-9) * 0.3, q)
            k = np.where(np.abs(k) < 0.2, k + np.sign(k + 1e-9) * 0.3, k)
        eps = 0.3
        grads = ora.backward(q, k, v, dout, fmap, eps)
        loss = lambda qq, kk, vv: float((ora.brute_force(qq, kk, vv, fmap, eps) * dout).sum())
        step = 1e-6
        for which, g in enumerate(grads):
            for idx in [(0, 0, 0, 0), (0, 1, 3, 2), (0, 0, 4, 1), (0, 1, 2, 0)]:
                args = [q.copy(), k.copy(), v.copy()]
                args[which][idx] += step
                up = loss(*args)
                args[which][idx] -= 2 * step
                dn = loss(*args)
                fd = (up - dn) / (2 * step)
                assert abs(g[idx] - fd) <= 1e-6 * max(1.0, abs(fd)), (fmap, which, idx, g[idx], fd)


def pin_backward_linear_in_dout(ora):
    """The gradients are linear in dout, and dv of a ones-weighted loss with
    eps = 0 has the closed form sum_i w_ij / den_i (phi(q_i).phi(k_j) = w_ij)."""
    rng = _rng(72)
    q, k, v = (rng.standard_normal((1, 1, 6, 4)) for _ in range(3))
    d1, d2 = rng.standard_normal((2, 1, 1, 6, 4))
    a = ora.backward(q, k, v, d1, "elu", 1e-3)
    b = ora.backward(q, k, v, d2, "elu", 1e-3)
    c = ora.backward(q, k, v, 2.0 * d1 - d2, "elu", 1e-3)
    for x, y, w in zip(a, b, c):
        _close(w, 2.0 * x - y, rtol=1e-10, atol=1e-12)
    ones = np.ones((1, 1, 6, 4))
    dv = ora.backward(q, k, v, ones, "elu", 0.0)[2][0, 0]
    pq, pk = ora.phi_elu1(q[0, 0]), ora.phi_elu1(k[0, 0])
    w = pq @ pk.T
    want = (w / w.sum(axis=1, keepdims=True)).sum(axis=0)
    _close(dv, np.repeat(want[:, None], 4, axis=1), rtol=1e-12)

ALL_PINS = [
    pin_feature_maps,
    pin_feature_map_vs_torch,
    pin_golden,
    pin_negative_elu_closed_form,
    pin_constant_values,
    pin_zero_qk_closed_form,
    pin_identity_values_give_weights,
    pin_linear_equals_definition,
    pin_causal_structure,
    pin_invariances,
    pin_relu_zero_denominator,
    pin_projection_reduction,
    pin_ttr_golden,
    pin_landmark_rule,
    pin_sigmoid_values,
    pin_landmark_all_tokens_is_attention,
    pin_landmark_invariances,
    pin_ttr_blend_limits,
    pin_e4m3_vs_torch,
    pin_e4m3_format_facts,
    pin_e4m3_forward,
    pin_softmax_vs_scipy,
    pin_softmax_closed_forms,
    pin_softmax_equal_keys,
    pin_prologue_vs_library,
    pin_rope_invariants,
    pin_backward_finite_differences,
    pin_backward_linear_in_dout,
]
