"""The C-ABI library: it loads, exports every symbol include/la.h declares, and
rejects bad arguments on the host before touching a device (CPU only)."""

import ctypes
import os
import re

import pytest

import linear_attention_diffusion_phi_b200 as la
from linear_attention_diffusion_phi_b200 import build as la_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", f) for f in sorted(os.listdir(os.path.join(ROOT, "include")))
           if f.endswith(".h")]


@pytest.fixture(scope="module", autouse=True)
def built():
    la_build.build()
    yield


def declared_functions():
    names = []
    for path in HEADERS:
        with open(path) as fh:
            src = fh.read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        names += re.findall(r"^[A-Za-z_][\w \*]*?\b(la_\w+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_abi():
    names = declared_functions()
    for n in la.EXPORTED:
        assert n in names, n


def test_library_exports_every_declared_symbol():
    L = la.lib()
    for name in declared_functions():
        assert hasattr(L, name), f"{name} declared in include/ but not exported"


def test_version_and_status_strings():
    assert la.la_version() >= 100
    for code in range(8):
        s = la.la_status_string(code)
        assert s and s != "unknown status"
    assert la.la_status_string(99) == "unknown status"


def test_create_destroy_and_bad_dtype():
    h = la.la_create(la.LA_BF16)
    assert h
    assert la.la_destroy(h) == la.LA_OK
    with pytest.raises(la.LAError):
        la.la_create(7)
    L = la.lib()
    assert L.la_create(None, 0) == 1
    assert L.la_destroy(None) == 1


@pytest.fixture
def handles():
    hs = {"f32": la.la_create(la.LA_F32), "bf16": la.la_create(la.LA_BF16)}
    yield hs
    for h in hs.values():
        la.la_destroy(h)


def fwd(h, B=1, H=2, N=256, D=64, F=0, fmap=0, eps=1e-6, causal=0, ptr=0x1000, out=0x4000_0000):
    return la.la_forward(h, ptr, ptr, ptr, out, B, H, N, D, F, fmap, eps, causal, None)


# A call that passed every host check stops at the device: no sm_100 device
# here, or no workspace bound on a B200.
PAST_CHECKS = (7, 4)


def test_forward_argument_validation(handles):
    f32, b16 = handles["f32"], handles["bf16"]
    # bad values
    assert fwd(f32, B=-1) == 1
    assert fwd(f32, D=0) == 1
    assert fwd(f32, fmap=3) == 1
    assert fwd(f32, eps=-1.0) == 1
    assert fwd(f32, eps=float("nan")) == 1
    assert fwd(f32, causal=2) == 1
    assert fwd(f32, F=100) == 1            # feature_dim must be a multiple of 256
    assert fwd(b16, F=128, D=128) == 1
    # valid but not run by this build
    assert fwd(f32, D=130) == 2
    assert fwd(f32, D=6) == 2
    assert fwd(b16, D=130) == 2
    assert fwd(b16, D=6) == 2
    assert fwd(b16, D=128, F=512) == 1      # no projection bound (widened when bound)
    assert fwd(f32, D=64, F=512, causal=1) == 2   # causal: F <= 256
    assert fwd(b16, D=128, F=512, causal=1) == 2
    assert fwd(f32, D=64, F=4352) == 2      # non-causal: F <= 4096
    assert fwd(b16, D=64, F=256) == 1       # no projection bound
    assert fwd(b16, D=128, F=256, causal=1) == 1
    # bf16 shapes outside the tensor-core kernels run widened on the fp32 ones
    assert fwd(b16, D=96) in PAST_CHECKS
    assert fwd(b16, D=32, causal=1) in PAST_CHECKS
    assert fwd(b16, D=128, causal=1) in PAST_CHECKS
    assert fwd(f32, B=300, H=300) == 2      # B*H beyond the grid limit
    # empty problems are a no-op
    assert fwd(f32, N=0, ptr=0, out=0) == 0
    assert fwd(b16, B=0, D=128, ptr=0, out=0) == 0
    # null and misaligned pointers
    assert fwd(f32, ptr=0) == 1
    assert fwd(f32, ptr=0x1004) == 3
    assert fwd(b16, D=128, out=0x2008) == 3
    # projection requested but none bound
    assert fwd(b16, D=128, F=256) == 1


def test_outputs_may_not_overlap_inputs(handles):
    """Checked on the host before anything is enqueued (the addresses here
    are never dereferenced).  The default problem is 131072 bytes per tensor
    in fp32, 65536 in bf16."""
    f32, b16 = handles["f32"], handles["bf16"]
    nb = 1 * 2 * 256 * 64 * 4
    assert fwd(f32, ptr=0x1000, out=0x1000) == 1                 # in place
    assert fwd(f32, ptr=0x1000, out=0x1000 + nb - 16) == 1       # last 16 bytes shared
    assert fwd(f32, ptr=0x1000 + nb - 16, out=0x1000) == 1
    assert fwd(f32, ptr=0x1000, out=0x1000 + nb) not in (1, 0)    # adjacent: accepted, then no device / workspace
    assert fwd(f32, ptr=0x1000 + nb, out=0x1000) not in (1, 0)
    assert fwd(b16, ptr=0x1000, out=0x1000 + nb // 2 - 16) == 1
    # q, k and v are only read and may coincide: fwd passes one pointer for all three
    # la_forward_host: the four device buffers are pairwise disjoint
    h = 0x9000_0000
    host = lambda dq, dk, dv, do: la.la_forward_host(f32, h, h, h, h, dq, dk, dv, do, 1, 2, 256, 64, 0, 0, 1e-6, 0,
                                                    None)
    assert host(0x1000, 0x1000, 0x100000, 0x200000) == 1
    assert host(0x1000, 0x100000, 0x200000, 0x200000 + nb - 16) == 1
    assert host(0, 0x100000, 0x200000, 0x300000) == 1
    # la_forward_noalloc: out vs q, k, v
    nbb = 1 * 2 * 256 * 128 * 2
    call = lambda q, k, v, o: la.la_forward_noalloc(q, k, v, o, 1, 2, 256, 128, 0, 1e-6, None)
    assert call(0x1000, 0x100000, 0x200000, 0x1000) == 1
    assert call(0x1000, 0x100000, 0x200000, 0x200000 + nbb - 16) == 1


def test_projection_validation(handles):
    h = handles["bf16"]
    assert la.la_set_projection(h, 0x1000, 24, 128, 255, 0) == 1
    assert la.la_set_projection(h, 0x1000, 24, 128, 256, -1) == 1
    assert la.la_set_projection(h, 0x1000, 24, 128, 256, 100) == 1   # stride < D*F
    assert la.la_set_projection(h, 0x1008, 24, 128, 256, 0) == 3
    assert la.la_set_projection(h, 0x1000, 24, 128, 256, 128 * 256) == 0
    assert fwd(h, D=64, F=256) == 1       # the bound W is 128 x 256
    # out may not overlap the part of W the call reads: heads 0..H-1 at the
    # bound stride, bf16 (two heads here: 2 * 128 * 256 * 2 bytes from 0x1000)
    wend = 0x1000 + 2 * 128 * 256 * 2
    assert fwd(h, D=128, F=256, ptr=0x8000_0000, out=wend - 16) == 1
    assert fwd(h, D=128, F=256, ptr=0x8000_0000, out=wend) not in (1, 0)
    assert la.la_set_projection(h, None, 0, 0, 0, 0) == 0
    assert fwd(h, D=128, F=256) == 1


def test_workspace_bytes_and_binding(handles):
    for name, h in handles.items():
        n = la.la_workspace_bytes(h, 1, 24, 4608, 128 if name == "bf16" else 64, 0, 0)
        assert n >= 256 and n % 256 == 0
        assert n < 64 << 20
        assert la.la_workspace_bytes(h, 1, 24, 4608, 130, 0, 0) == 0
    h = handles["bf16"]
    header = 256 + 4096   # status word, synchronisation words
    # the bf16 non-causal F = 0 path reduces states in distributed shared
    # memory; a head spread over nc > 1 clusters adds a 36 KB exchange image
    # per (head, cluster).  Without a device the plan keeps one cluster.
    n = la.la_workspace_bytes(h, 1, 24, 4608, 128, 0, 0)
    assert n in [header] + [header + 24 * nc * 36864 for nc in (2, 3, 4)]
    assert la.la_workspace_bytes(h, 1, 24, 4608, 128, 256, 0) >= n
    # D = 64 keeps one cluster per head: the header only
    assert la.la_workspace_bytes(h, 1, 24, 4608, 64, 0, 0) == header
    # bf16 causal: the header plus one [D + 1][D] fp32 state per (segment, head)
    nc = la.la_workspace_bytes(h, 4, 8, 32768, 64, 0, 1)
    assert nc >= header + 32 * 3 * 65 * 64 * 4 and nc < 64 << 20
    # one segment per head (at least as many heads as SMs): no state at all
    assert la.la_workspace_bytes(h, 3, 21845, 3, 64, 0, 1) == header
    assert la.la_workspace_bytes(h, 2, 100, 700, 64, 0, 1) == header
    assert la.la_set_workspace(h, 0x1010, 4096) == 3          # not 256-aligned
    assert la.la_set_workspace(h, None, 0) == 0
    assert la.la_sync_status(h, None) == 4                    # no workspace bound


def test_widened_workspace_holds_the_fp32_plan_and_copies(handles):
    """A bf16 shape outside the tensor-core kernels runs on the fp32 kernels:
    its workspace is the fp32 plan of the same shape plus fp32 copies of q, k,
    v and out and of the part of W the call reads, each 256-byte aligned."""
    f32, b16 = handles["f32"], handles["bf16"]
    a256 = lambda x: (x + 255) // 256 * 256
    shapes = [(1, 2, 1000, 128, 0, 1), (2, 3, 77, 96, 0, 0), (1, 2, 300, 32, 0, 1), (1, 24, 4608, 64, 256, 0),
              (1, 2, 1000, 128, 512, 0), (1, 3, 5, 4, 256, 1)]
    for B, H, N, D, F, causal in shapes:
        n = B * H * N * D
        got = la.la_workspace_bytes(b16, B, H, N, D, F, causal)
        assert got == la.la_workspace_bytes(f32, B, H, N, D, F, causal) + 4 * a256(4 * n) + a256(4 * D * F), \
            (B, H, N, D, F, causal)
    # W bound with a head stride: heads 0 .. H - 1 are copied
    assert la.la_set_projection(b16, 0x1000, 24, 64, 256, 64 * 256 + 64) == 0
    n = 24 * 4608 * 64
    assert la.la_workspace_bytes(b16, 1, 24, 4608, 64, 256, 0) == (
        la.la_workspace_bytes(f32, 1, 24, 4608, 64, 256, 0) + 4 * a256(4 * n) + a256(4 * (23 * (64 * 256 + 64) + 64 * 256)))
    assert la.la_set_projection(b16, None, 0, 0, 0, 0) == 0
    # shapes the tensor-core kernels run keep their own plans, without copies
    assert la.la_workspace_bytes(b16, 1, 24, 4608, 128, 256, 0) < 4 * 24 * 4608 * 128


def test_no_device_is_reported_not_faked(handles):
    torch = pytest.importorskip("torch")
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    assert fwd(handles["f32"]) == 7


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(la, "_lib", None)
    monkeypatch.setattr(la, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="not built"):
        la.la_version()


def test_binding_checks_tensors_before_calling():
    """The binding hands the library base pointers only, so it refuses
    tensors that are not dense [B, H, N, D] arrays of its dtype on one CUDA
    device (all checks on the host; nothing reaches the library)."""
    torch = pytest.importorskip("torch")
    op = la.LinearAttention(torch.bfloat16)
    x = torch.zeros(1, 2, 8, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="expected \\[B, H, N, D\\]"):
        op(x[0], x[0], x[0])
    with pytest.raises(ValueError, match="k: shape"):
        op(x, x[:, :1], x)
    with pytest.raises(ValueError, match="v: dtype"):
        op(x, x, x.float())
    with pytest.raises(ValueError, match="q: must be contiguous"):
        t = torch.zeros(1, 8, 2, 64, dtype=torch.bfloat16).transpose(1, 2)
        op(t, x, x, out=x.clone())
    with pytest.raises(ValueError, match="CUDA device"):
        op(x, x, x)
    op.close()
    # the projection: its dtype must be the operator's, and it must be on a device
    with pytest.raises(ValueError, match="W: dtype"):
        la.LinearAttention(torch.bfloat16, W=torch.zeros(2, 128, 256))
    with pytest.raises(ValueError, match="W: on cpu"):
        la.LinearAttention(torch.bfloat16, W=torch.zeros(2, 128, 256, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="W: expected"):
        la.LinearAttention(torch.float32, W=torch.zeros(256))


def test_landmark_count_matches_the_rule():
    """la_landmark_count (host logic) against the oracle's landmark rule:
    round(fraction N) half up, clamped to [min, max], then to [1, N]."""
    from oracle import la_oracle as ora
    import numpy as np
    rng = np.random.default_rng(5)
    cases = [(4608, 1 / 32, 16, 128), (100, 1 / 32, 16, 128), (10, 0.5, 16, 128), (30, 0.05, 0, 64),
             (3, 0.0, 0, 5), (1, 0.9, 0, 1), (65536, 0.001, 8, 128)]
    for _ in range(200):
        cases.append((int(rng.integers(1, 20000)), float(rng.choice([0.25, 0.125, 1 / 32, 0.01, 0.0625])),
                      int(rng.integers(0, 40)), int(rng.integers(1, 300))))
    for n, f, lo, hi in cases:
        assert la.la_landmark_count(n, f, lo, hi) == ora.landmark_count(n, float(np.float32(f)), lo, hi), (n, f, lo, hi)
    assert la.la_landmark_count(0, 0.1, 1, 8) == 0
    assert la.la_landmark_count(10, -0.1, 1, 8) == 0
    assert la.la_landmark_count(10, float("nan"), 1, 8) == 0
    assert la.la_landmark_count(10, 0.1, -1, 8) == 0
    assert la.la_landmark_count(10, 0.1, 1, 0) == 0


def test_ttr_argument_checks_on_the_host(handles):
    """la_forward_ttr refuses what it does not support before touching a
    device: fp32 handles, D != 128, causal-free checks of the landmark count
    and of the gate pointer."""
    f = lambda h, D, L, gate: la.la_forward_ttr(h, 0x1000, 0x1000, 0x1000, 0x2000, 1, 2, 256, D, 0,
                                               la.LA_PHI_ELU1, 1e-6, L, gate, None)
    assert f(handles["f32"], 128, 8, 0x3000) == la.LA_ERR_UNSUPPORTED
    assert f(handles["bf16"], 64, 8, 0x3000) == la.LA_ERR_UNSUPPORTED
    assert f(handles["bf16"], 128, 0, 0x3000) == la.LA_ERR_INVALID_ARG       # no landmark
    assert f(handles["bf16"], 128, 257, 0x3000) == la.LA_ERR_INVALID_ARG     # more than N
    assert f(handles["bf16"], 128, 200, 0x3000) == la.LA_ERR_UNSUPPORTED     # more than 128
    assert f(handles["bf16"], 128, 8, None) == la.LA_ERR_INVALID_ARG         # no gate
    assert f(handles["bf16"], 128, 8, 0x3002) == la.LA_ERR_INVALID_ARG       # misaligned gate
    assert la.la_forward_ttr(handles["bf16"], 0, 0, 0, 0, 0, 2, 256, 128, 0, la.LA_PHI_ELU1, 1e-6, 8,
                             0x3000, None) == la.LA_OK                       # empty problem


def test_e4m3_argument_checks_on_the_host(handles):
    """la_forward_e4m3 refuses what it does not support before touching a
    device: scales that are not finite and positive, fp32 handles, D != 128,
    bad shapes; an empty problem is a no-op."""
    nan, inf = float("nan"), float("inf")
    f = lambda h, D, sq, sk, sv, fmap=la.LA_PHI_ELU1: la.la_forward_e4m3(
        h, 0x1000, 0x1000, 0x1000, sq, sk, sv, 0x2000, 1, 2, 256, D, fmap, 1e-6, None)
    for bad in ((0.0, 1.0, 1.0), (1.0, -1.0, 1.0), (1.0, 1.0, nan), (inf, 1.0, 1.0)):
        assert f(handles["bf16"], 128, *bad) == la.LA_ERR_INVALID_ARG, bad
    assert f(handles["f32"], 128, 1.0, 1.0, 1.0) == la.LA_ERR_UNSUPPORTED
    assert f(handles["bf16"], 64, 1.0, 1.0, 1.0) == la.LA_ERR_UNSUPPORTED
    assert f(handles["bf16"], 128, 1.0, 1.0, 1.0, fmap=7) == la.LA_ERR_INVALID_ARG
    assert la.la_forward_e4m3(handles["bf16"], 0, 0, 0, 1.0, 1.0, 1.0, 0, 0, 2, 256, 128, la.LA_PHI_ELU1,
                              1e-6, None) == la.LA_OK                        # empty problem



def test_softmax_support_is_checked_on_the_host(handles):
    """The softmax feature map runs without a projection: on the bf16
    non-causal D = 128 kernel and on the fp32 kernels (bf16 shapes outside
    the tensor-core kernels widened); the other bf16 kernel shapes, a
    projection and E4M3 inputs are refused before anything is enqueued."""
    SMX = la.LA_PHI_SOFTMAX
    f = lambda h, D, F, causal: la.la_forward(h, 0x1000, 0x1000, 0x1000, 0x4000_0000, 1, 2, 256, D, F, SMX, 1e-6,
                                              causal, None)
    assert f(handles["f32"], 64, 256, 0) == la.LA_ERR_UNSUPPORTED
    assert f(handles["bf16"], 64, 0, 0) == la.LA_ERR_UNSUPPORTED     # the bf16 D = 64 kernels
    assert f(handles["bf16"], 64, 0, 1) == la.LA_ERR_UNSUPPORTED
    assert f(handles["bf16"], 128, 0, 1) in PAST_CHECKS               # widened
    assert f(handles["bf16"], 96, 0, 0) in PAST_CHECKS
    assert f(handles["bf16"], 128, 256, 0) == la.LA_ERR_UNSUPPORTED
    assert la.la_forward_e4m3(handles["bf16"], 0x1000, 0x1000, 0x1000, 1.0, 1.0, 1.0, 0x2000, 1, 2, 256, 128,
                              SMX, 1e-6, None) == la.LA_ERR_UNSUPPORTED
    assert la.la_forward_noalloc(0x1000, 0x1000, 0x1000, 0x2000, 1, 2, 256, 64, SMX, 1e-6,
                                 None) == la.LA_ERR_UNSUPPORTED
    assert la.la_forward(handles["bf16"], 0x1000, 0x1000, 0x1000, 0x2000, 1, 2, 256, 128, 0, 3, 1e-6, 0,
                         None) == la.LA_ERR_INVALID_ARG


def test_prologue_binding_and_support_checks(handles):
    """la_set_prologue checks its arguments; la_forward with a prologue bound
    refuses other shapes and paths before anything is enqueued."""
    f = lambda h, D=128, npos=256, eps=1e-6, qs=0x1000, ks=0x2000, rope=0x3000: la.la_set_prologue(
        h, qs, ks, rope, D, npos, eps)
    bf = handles["bf16"]
    assert f(bf, D=127) == la.LA_ERR_INVALID_ARG
    assert f(bf, npos=0) == la.LA_ERR_INVALID_ARG
    assert f(bf, eps=-1.0) == la.LA_ERR_INVALID_ARG
    assert f(bf, ks=None) == la.LA_ERR_INVALID_ARG
    assert f(bf, rope=0x3004) == la.LA_ERR_MISALIGNED
    assert f(bf) == la.LA_OK
    fwd = lambda h, D=128, N=256, causal=0, fmap=la.LA_PHI_ELU1: la.la_forward(
        h, 0x10000, 0x10000, 0x10000, 0x4000_0000, 1, 2, N, D, 0, fmap, 1e-6, causal, None)
    assert fwd(bf, N=257) == la.LA_ERR_INVALID_ARG                 # more positions than the table
    assert fwd(bf, causal=1, D=128) in PAST_CHECKS                # widened onto the fp32 kernels
    assert fwd(bf, fmap=la.LA_PHI_SOFTMAX) == la.LA_ERR_UNSUPPORTED
    assert la.la_forward_e4m3(bf, 0x10000, 0x10000, 0x10000, 1.0, 1.0, 1.0, 0x20000, 1, 2, 256, 128,
                              la.LA_PHI_ELU1, 1e-6, None) == la.LA_ERR_UNSUPPORTED
    assert la.la_forward_ttr(bf, 0x10000, 0x10000, 0x10000, 0x20000, 1, 2, 256, 128, 0, la.LA_PHI_ELU1, 1e-6, 8,
                             0x80000, None) == la.LA_ERR_UNSUPPORTED
    assert f(bf, D=64) == la.LA_OK
    assert fwd(bf, D=128) == la.LA_ERR_INVALID_ARG                 # the bound D differs
    assert fwd(bf, D=64) == la.LA_ERR_UNSUPPORTED                  # bf16 prologue needs D = 128
    assert la.la_set_prologue(bf, None, None, None, 0, 0, 0.0) == la.LA_OK


def test_backward_checks_on_the_host(handles):
    """la_backward runs on fp32 handles without projection or prologue, elu+1
    or relu; it refuses overlapping outputs before anything is enqueued."""
    f32, bf = handles["f32"], handles["bf16"]
    assert la.la_backward_workspace_bytes(f32, 1, 2, 256, 64) > 0
    assert la.la_backward_workspace_bytes(bf, 1, 2, 256, 128) == 0
    nb = 1 * 2 * 256 * 64 * 4
    base = 0x100000
    ins = [base, base, base, base + nb]
    outs = [base + 4 * nb, base + 6 * nb, base + 8 * nb]
    b = lambda h, o=outs, fmap=la.LA_PHI_ELU1, D=64: la.la_backward(h, *ins, *o, 1, 2, 256, D, fmap, 1e-6, None)
    assert b(bf, D=128) == la.LA_ERR_UNSUPPORTED
    assert b(f32, fmap=la.LA_PHI_SOFTMAX) == la.LA_ERR_UNSUPPORTED
    assert b(f32, o=[outs[0], outs[0], outs[2]]) == la.LA_ERR_INVALID_ARG     # dq and dk coincide
    assert b(f32, o=[base + nb // 2, outs[1], outs[2]]) == la.LA_ERR_INVALID_ARG   # dq over the inputs
    assert b(f32, o=[outs[0] + 4, outs[1], outs[2]]) == la.LA_ERR_MISALIGNED
    assert la.la_backward(f32, 0, 0, 0, 0, 0, 0, 0, 1, 0, 256, 64, la.LA_PHI_ELU1, 1e-6, None) == la.LA_OK

