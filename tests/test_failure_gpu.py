"""Device-side failure detection, without faulting the GPU.

Every wait in the library's kernels is bounded: after the limit it records
LA_ERR_TIMEOUT in the workspace status word and the kernel winds down.  Here a
test kernel waits on a phase that nothing completes (the same wait code), and
the host path that reports a recorded timeout is checked.
"""

import ctypes
import os
import subprocess

import pytest

import linear_attention_diffusion_phi_b200 as la
from linear_attention_diffusion_phi_b200 import build as la_build

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(os.path.dirname(HERE), "linear_attention_diffusion_phi_b200", "csrc")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")


@pytest.fixture(scope="module")
def waitlib(tmp_path_factory):
    out = str(tmp_path_factory.mktemp("bw") / "libbounded_wait.so")
    subprocess.check_call(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17",
                           "-Xcompiler", "-fPIC", "-shared", f"-I{CSRC}", f"-I{INCLUDE}",
                           os.path.join(HERE, "cuda", "bounded_wait.cu"), "-o", out])
    lib = ctypes.CDLL(out)
    lib.run_bounded_wait.argtypes = [ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_ulonglong)]
    lib.run_bounded_wait.restype = ctypes.c_int
    return lib


def test_unfinished_wait_gives_up_and_reports(waitlib):
    import torch
    status = ctypes.c_int(-1)
    out = (ctypes.c_ulonglong * 2)()
    assert waitlib.run_bounded_wait(ctypes.byref(status), out) == 0   # cudaSuccess: no fault
    assert status.value == la.LA_ERR_TIMEOUT
    assert out[1] == 0                                   # the wait reported failure
    assert 1.5e9 <= out[0] <= 20e9                       # after the bounded limit, not at once
    # the context is still usable
    x = torch.arange(4, device="cuda:0", dtype=torch.float32)
    assert float((x * 2).sum()) == 12.0


def test_sync_status_reports_and_clears_a_recorded_timeout():
    import torch
    la_build.build()
    from linear_attention_diffusion_phi_b200.inputs import Workload, make_inputs
    w = make_inputs(Workload("status", B=1, H=2, N=256, D=64, seed=31))[0].to("cuda:0")
    op = la.LinearAttention(torch.bfloat16, "elu", 1e-6)
    op(w, w, w)
    torch.cuda.synchronize()
    assert op.sync_status() == la.LA_OK
    op._ws[:4].view(torch.int32)[0] = la.LA_ERR_TIMEOUT   # what a timed-out kernel leaves
    torch.cuda.synchronize()
    assert op.sync_status() == la.LA_ERR_TIMEOUT
    assert op.sync_status() == la.LA_OK                    # reported once, then cleared
    op(w, w, w)                                            # the handle keeps working
    torch.cuda.synchronize()
    assert op.sync_status() == la.LA_OK
    op.close()
