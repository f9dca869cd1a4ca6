"""la_forward_noalloc, the entry point for callers that cannot allocate device
memory: its scratch is a static array inside the library.  It must give the
same result as la_forward with a caller-owned workspace, call after call, even
though every call reuses the same array.  (This file is collected last.)"""

import numpy as np
import pytest

import linear_attention_diffusion_phi_b200 as la
from linear_attention_diffusion_phi_b200 import build as la_build
from linear_attention_diffusion_phi_b200.inputs import WORKLOADS, Workload, as_float64, make_inputs

pytestmark = pytest.mark.gpu

BF16_MAX, BF16_MEAN = 2e-2, 2e-3


def _close(a, b):
    d = np.abs(as_float64(a) - as_float64(b))
    assert d.max() <= BF16_MAX and d.mean() <= BF16_MEAN, (d.max(), d.mean())


def test_noalloc_matches_workspace_entry_point_twice_in_a_row():
    import torch
    la_build.build()
    dev = torch.device("cuda:0")
    s = torch.cuda.current_stream().cuda_stream
    cases = [WORKLOADS["flux1024"], Workload("noalloc_relu64", B=2, H=3, N=1001, D=64, fmap="relu", seed=21),
             Workload("noalloc_softmax", B=1, H=4, N=3000, D=128, fmap="softmax", seed=22),
             Workload("noalloc_heads", B=3, H=21845, N=3, D=64, seed=22)]   # B*H = 65535
    for w in cases:
        q, k, v, _ = make_inputs(w)
        qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
        op = la.LinearAttention(torch.bfloat16, w.fmap, w.eps)
        ref = op(qd, kd, vd).clone()
        for _ in range(2):
            out = torch.full_like(qd, float("nan"))
            st = la.la_forward_noalloc(qd.data_ptr(), kd.data_ptr(), vd.data_ptr(), out.data_ptr(),
                                       w.B, w.H, w.N, w.D, la.FEATURE_MAPS[w.fmap], w.eps, s)
            assert st == la.LA_OK, la.la_status_string(st)
            torch.cuda.synchronize()
            # same kernel, same cluster size: bitwise equal (la.h promises
            # deterministic results), and within the bf16 bar in any case
            assert torch.equal(out, ref)
            _close(out.cpu(), ref.cpu())
        op.close()


def test_noalloc_rejects_bad_arguments_before_launching():
    """Every rejection here happens on the host, before anything is enqueued,
    so the (deliberately tiny) buffer is never read."""
    import torch
    la_build.build()
    dev = torch.device("cuda:0")
    x = torch.empty(64, dtype=torch.bfloat16, device=dev)
    p = x.data_ptr()
    s = torch.cuda.current_stream().cuda_stream
    call = la.la_forward_noalloc
    assert call(0, p, p, p, 1, 2, 128, 128, la.LA_PHI_ELU1, 1e-6, s) == 1         # null pointer
    assert call(p + 2, p, p, p, 1, 2, 128, 128, la.LA_PHI_ELU1, 1e-6, s) == 3     # misaligned
    assert call(p, p, p, p, 1, 2, 128, 96, la.LA_PHI_ELU1, 1e-6, s) == 2          # D not 64 / 128
    assert call(p, p, p, p, 1, 2, 128, 128, 5, 1e-6, s) == 1                      # feature map
    assert call(p, p, p, p, 1, 2, 128, 128, la.LA_PHI_ELU1, -1.0, s) == 1        # eps < 0
    assert call(p, p, p, p, 300, 300, 128, 128, la.LA_PHI_ELU1, 1e-6, s) == 2    # B*H over the grid limit
    assert call(p, p, p, p, 1, 2, 0, 128, la.LA_PHI_ELU1, 1e-6, s) == 0          # empty: nothing to do
    torch.cuda.synchronize()
