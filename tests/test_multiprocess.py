"""The multi-process host logic of bench.py on CPU: two gloo ranks.

With N GPUs every rank runs its own replica of the workload (heads are
independent; no collective on the data path), the job's time is the slowest
rank's, and the whole-job throughput counts every rank's tokens.  The
reference arm runs on rank 0 only.
"""

import json
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, outdir):
    import contextlib
    import datetime
    import io
    import types
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    from linear_attention_diffusion_phi_b200.inputs import WORKLOADS
    w = WORKLOADS["tiny_f32"]
    res = {
        "env": list(bench.dist_env()),
        "max": bench.max_over_ranks([1.0 + 10 * rank, 5.0 - rank]),
        "seeds": [bench.input_seed(w, i, rank) for i in range(3)],
        "value": bench.job_throughput(1000, world, 10, 20.0),
    }
    buf = io.StringIO()
    args = types.SimpleNamespace(gpus=world, steps=1, warmup=0)
    with contextlib.redirect_stdout(buf):
        res["ref_rc"] = bench.run_reference(args, w)
    res["ref_out"] = buf.getvalue()
    dist.barrier()
    dist.destroy_process_group()
    with open(os.path.join(outdir, f"rank{rank}.json"), "w") as fh:
        json.dump(res, fh)


def test_two_gloo_ranks(tmp_path):
    import torch.multiprocessing as mp
    mp.start_processes(_rank_main, args=(2, _free_port(), str(tmp_path)), nprocs=2, join=True,
                       start_method="spawn")
    r = [json.load(open(tmp_path / f"rank{i}.json")) for i in range(2)]
    assert r[0]["env"] == [2, 0, 0] and r[1]["env"] == [2, 1, 1]
    # the job's time is the slowest rank's, element by element, on every rank
    assert r[0]["max"] == r[1]["max"] == [11.0, 5.0]
    # each rank streams its own replica: no input set is shared between ranks
    assert not set(r[0]["seeds"]) & set(r[1]["seeds"])
    assert len(set(r[0]["seeds"])) == 3
    # whole-job throughput: 2 ranks x 1000 tokens per 2 ms step
    assert r[0]["value"] == pytest.approx(1e6)
    # the reference arm prints one line on rank 0 and nothing elsewhere
    assert r[0]["ref_rc"] == 0 and r[1]["ref_rc"] == 0
    assert r[1]["ref_out"] == ""
    line = json.loads(r[0]["ref_out"].strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0


def test_per_call_percentiles_and_event_pairing(monkeypatch):
    """bench.py's per-call figure: one event pair around each single step, read
    after one synchronize, then p10 / p50 / p90 (CUDA events faked on the CPU,
    each 'step' advancing a fake device clock by its own duration)."""
    import sys
    import types
    import bench

    clock = [0.0]

    class Ev:
        def __init__(self, enable_timing=False):
            self.t = None

        def record(self, stream=None):
            self.t = clock[0]

        def elapsed_time(self, other):
            return other.t - self.t

    fake = types.SimpleNamespace(cuda=types.SimpleNamespace(Event=Ev, synchronize=lambda: None))
    monkeypatch.setitem(sys.modules, "torch", fake)
    durations = [0.5 + 0.1 * (i % 10) for i in range(20)]

    def run_one(i):
        clock[0] += durations[i]

    times = bench.per_call_ms(run_one, 20, stream=None)
    assert times == [pytest.approx(d) for d in durations]
    p = bench.percentiles_ms(times)
    assert p["calls"] == 20 and p["p10"] <= p["p50"] <= p["p90"]
    assert p["p50"] == pytest.approx(0.95)
