"""The float64 oracle against facts fixed outside it (CPU only).

Every pin in ``oracle_pins`` must pass on the oracle, and each mistake planted
below in a copy of the oracle's source must make at least one pin fail, so that
the pins are known to see a dropped term, a wrong sign or index, a transposed
operand or a shifted causal mask.
"""

import importlib.util
import os
import types

import pytest

import oracle_pins
from oracle import la_oracle

ORACLE_SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                          "oracle", "la_oracle.py")


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda p: p.__name__)
def test_pin(pin):
    pin(la_oracle)


# (name, text in the oracle, planted replacement)
MUTANTS = [
    ("elu_drops_plus_one", "x > 0.0, x + 1.0, np.exp", "x > 0.0, x, np.exp"),
    ("elu_wrong_sign", "np.exp(np.minimum(x, 0.0))", "np.exp(-np.minimum(x, 0.0))"),
    ("elu_branch_at_wrong_point", "np.where(x > 0.0,", "np.where(x > 1.0,"),
    ("relu_is_abs", "np.maximum(x, 0.0)", "np.abs(x)"),
    ("definition_transposed", "w = pq @ pk.T ", "w = pk @ pq.T "),
    ("definition_drops_eps", "den = w.sum(axis=1) + eps", "den = w.sum(axis=1)"),
    ("definition_eps_inside", "den = w.sum(axis=1) + eps", "den = (w + eps).sum(axis=1)"),
    ("definition_exclusive_causal", "w = np.tril(w) ", "w = np.tril(w, -1) "),
    ("definition_key_normaliser", "den = w.sum(axis=1) + eps", "den = w.sum(axis=0) + eps"),
    ("grouped_drops_eps", "den = pq @ ksum + eps", "den = pq @ ksum"),
    ("grouped_ksum_wrong_axis", "ksum = pk.sum(axis=0)", "ksum = pq.sum(axis=0)"),
    ("grouped_kv_uses_queries", "kv = pk.T @ v", "kv = pq.T @ v"),
    ("recurrence_reads_before_update",
     "        S += np.outer(pk[i], v[i])\n        z += pk[i]\n        out[i] = (pq[i] @ S) / (pq[i] @ z + eps)",
     "        out[i] = (pq[i] @ S) / (pq[i] @ z + eps)\n        S += np.outer(pk[i], v[i])\n        z += pk[i]"),
    ("recurrence_transposed_state", "S += np.outer(pk[i], v[i])", "S += np.outer(pk[i], v[i]) if pk.shape[1] != v.shape[1] else np.outer(v[i], pk[i])"),
    ("rows_exclusive_causal", "jend = i + 1 if causal", "jend = i if causal"),
    ("projection_after_map", "        x = x @ np.asarray(W, dtype=np.float64)\n    if fmap == \"elu\":\n        return phi_elu1(x)",
     "        pass\n    if fmap == \"elu\":\n        return phi_elu1(x) if W is None else phi_elu1(x) @ np.asarray(W, dtype=np.float64)"),
    ("projection_head_zero", "return W if W.ndim == 2 else W[h]", "return W if W.ndim == 2 else W[0]"),
    ("ttr_alpha_on_kernel_branch", "out[b, h] = a * lm + (1.0 - a) * lin", "out[b, h] = a * lin + (1.0 - a) * lm"),
    ("landmark_no_scale", "s = (q @ kl.T) / np.sqrt(q.shape[1])", "s = q @ kl.T"),
    ("landmark_softmax_over_queries", "s = s - s.max(axis=1, keepdims=True)\n    e = np.exp(s)\n    return (e / e.sum(axis=1, keepdims=True)) @ vl",
     "s = s - s.max(axis=0, keepdims=True)\n    e = np.exp(s)\n    return (e / e.sum(axis=0, keepdims=True)) @ vl"),
    ("landmark_positions_shifted", "return [(l * n) // count for l in range(count)]",
     "return [min(n - 1, (l * n) // count + 1) for l in range(count)]"),
    ("landmark_count_no_clamp", "return max(1, min(n, max(lo, min(hi, want))))", "return max(1, min(n, want))"),
    ("landmark_count_rounds_down", "want = int(np.floor(fraction * n + 0.5))", "want = int(np.floor(fraction * n))"),
    ("sigmoid_wrong_sign", "return 1.0 / (1.0 + np.exp(-g))", "return 1.0 / (1.0 + np.exp(g))"),
    ("softmax_wrong_axis", "e = np.exp(x - x.max(axis=-1, keepdims=True))\n    return e / e.sum(axis=-1, keepdims=True)",
     "e = np.exp(x - x.max(axis=0, keepdims=True))\n    return e / e.sum(axis=0, keepdims=True)"),
    ("softmax_not_normalised", "return e / e.sum(axis=-1, keepdims=True)", "return e"),
    ("softmax_wrong_sign", "e = np.exp(x - x.max(axis=-1, keepdims=True))", "e = np.exp(x.max(axis=-1, keepdims=True) - x)"),
    ("softmax_is_elu", "    if fmap == \"softmax\":\n        return phi_softmax(x)", "    if fmap == \"softmax\":\n        return phi_elu1(x)"),
    ("rms_no_eps", "x / np.sqrt(ms + norm_eps)", "x / np.sqrt(ms)"),
    ("rms_sum_not_mean", "ms = np.mean(x * x, axis=-1, keepdims=True)", "ms = np.sum(x * x, axis=-1, keepdims=True)"),
    ("rope_wrong_sign", "out[..., 0::2] = c * x0 - s * x1", "out[..., 0::2] = c * x0 + s * x1"),
    ("rope_half_split_pairs", "x0, x1 = x[..., 0::2], x[..., 1::2]",
     "x0, x1 = x[..., : x.shape[-1] // 2], x[..., x.shape[-1] // 2:]"),
    ("prologue_scales_swapped", "qn = rope(rms_norm(q, q_scale, norm_eps), table)", "qn = rope(rms_norm(q, k_scale, norm_eps), table)"),
    ("prologue_rope_before_norm", "qn = rope(rms_norm(q, q_scale, norm_eps), table)", "qn = rms_norm(rope(q, table), q_scale, norm_eps)"),
    ("backward_drops_h", "dpq = g @ kv.T + h[:, None] * z[None, :]", "dpq = g @ kv.T"),
    ("backward_h_sign", "h = -(dout * out).sum(axis=1) / den", "h = (dout * out).sum(axis=1) / den"),
    ("backward_dkv_uses_keys", "dkv = pq.T @ g", "dkv = pk.T @ g"),
    ("backward_dz_missing", "dpk = v @ dkv.T + dz[None, :]", "dpk = v @ dkv.T"),
    ("backward_dv_transposed", "dv = pk @ dkv", "dv = pq @ dkv"),
    ("backward_elu_grad_one", "return np.where(x > 0.0, 1.0, np.exp(np.minimum(x, 0.0)))", "return np.ones_like(x)"),
    ("e4m3_bias_eight", "np.exp2(e - 7.0)", "np.exp2(e - 8.0)"),
    ("e4m3_no_subnormals", "np.where(e == 0, (m / 8.0) * 2.0 ** -6,", "np.where(e < 0, (m / 8.0) * 2.0 ** -6,"),
    ("e4m3_subnormal_scale", "(m / 8.0) * 2.0 ** -6", "(m / 8.0) * 2.0 ** -7"),
    ("e4m3_sign_ignored", "val = np.where((c & 0x80) != 0, -mag, mag)", "val = mag"),
    ("e4m3_no_nan", "return np.where((e == 15) & (m == 7), np.nan, val)", "return val"),
    ("e4m3_scales_swapped", "forward(sq * e4m3_decode(q8), sk * e4m3_decode(k8)", "forward(sk * e4m3_decode(q8), sq * e4m3_decode(k8)"),
    ("e4m3_value_scale_dropped", "sv * e4m3_decode(v8)", "e4m3_decode(v8)"),
    ("landmark_values_from_keys", "vl = np.asarray(v, dtype=np.float64)[positions]",
     "vl = np.asarray(k, dtype=np.float64)[positions]"),
]


def _load_mutant(old, new):
    with open(ORACLE_SRC) as fh:
        src = fh.read()
    assert src.count(old) >= 1, f"mutation anchor not found: {old!r}"
    src = src.replace(old, new)
    mod = types.ModuleType("la_oracle_mutant")
    exec(compile(src, "la_oracle_mutant", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_is_caught(name, old, new):
    mod = _load_mutant(old, new)
    failed = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(mod)
        except Exception as exc:  # AssertionError or a shape error
            failed.append((pin.__name__, type(exc).__name__))
    assert failed, f"planted mistake {name!r} passed every pin"


def test_oracle_rejects_bad_arguments():
    import numpy as np
    x = np.zeros((1, 1, 4, 2))
    with pytest.raises(ValueError):
        la_oracle.forward(x, x, x, "tanh")
    with pytest.raises(ValueError):
        la_oracle.forward(x, x, x, "elu", eps=-1.0)
    with pytest.raises(ValueError):
        la_oracle.forward(x[0], x[0], x[0])


def test_oracle_module_spec_is_standalone():
    """The oracle imports nothing from the CUDA package."""
    spec = importlib.util.spec_from_file_location("o", ORACLE_SRC)
    with open(ORACLE_SRC) as fh:
        src = fh.read()
    assert "linear_attention_diffusion_phi_b200" not in src
    assert spec is not None


def test_grouped_form_equals_definition_on_random_shapes():
    """The identity the fast path rests on, sum_j (phi(q).phi(k_j)) v_j =
    phi(q)^T (sum_j phi(k_j) v_j^T), over random shapes the fixed pins do not
    reach: one token, value width unlike the key width, odd feature counts,
    eps from 0 to large (eps = 0 only under elu+1, whose weights are > 0)."""
    import numpy as np
    from hypothesis import given, settings, strategies as st

    @settings(max_examples=80, deadline=None, database=None, derandomize=True)
    @given(N=st.integers(1, 24), D=st.integers(1, 8), Dv=st.integers(1, 8), F=st.sampled_from([0, 3, 16]),
           fmap=st.sampled_from(["elu", "relu"]), causal=st.booleans(), eps=st.sampled_from([0.0, 1e-6, 0.5]),
           shared_w=st.booleans(), seed=st.integers(0, 2 ** 31 - 1))
    def check(N, D, Dv, F, fmap, causal, eps, shared_w, seed):
        if eps == 0.0 and fmap == "relu":
            eps = 1e-6
        rng = np.random.default_rng(seed)
        q = rng.standard_normal((1, 2, N, D))
        k = rng.standard_normal((1, 2, N, D))
        v = rng.standard_normal((1, 2, N, Dv))
        W = None
        if F:
            W = rng.standard_normal((D, F) if shared_w else (2, D, F)) / np.sqrt(D)
        a = la_oracle.forward(q, k, v, fmap, eps, causal, W)
        b = la_oracle.brute_force(q, k, v, fmap, eps, causal, W)
        assert a.shape == (1, 2, N, Dv)
        np.testing.assert_allclose(a, b, rtol=1e-10, atol=1e-12)

    check()
