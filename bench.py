"""Throughput of the linear-time phi-attention path on B200.

One step = one full forward (feature map on K, state reduction, feature map on
Q, apply and normalise) over one batch of synthetic inputs already resident in
HBM.  The default workload is the Flux-1024 attention shape: B=1, H=24,
N=4608 (4096 image + 512 text tokens), D=128, bf16, elu(x)+1, eps=1e-6.

Prints one JSON line (rank 0).  Under torchrun every rank runs its own copy of
the workload (heads are independent, no collective on the data path: weak
scaling) and the time is the max over ranks.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference   # the float64 CPU oracle on host cores
"""

import argparse
import json
import os
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "linear-attn tokens/s (B*H*N), HBM GB/s vs B200 peak"
UNIT = "tokens/s"
L2_BYTES = 126 * 1024 * 1024


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="flux1024")
    ap.add_argument("--soak-s", type=float, default=1.5, help="untimed load before timing (clock ramp)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="launch each step from the host")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the other workloads timed after the headline (1 GPU only)")
    ap.add_argument("--no-parity", action="store_true", help="skip the oracle comparison of sampled heads")
    ap.add_argument("--extra-only", default=None, choices=list(EXTRA_WORKLOADS),
                    help="time only this extra configuration and print its entry (for profiling runs)")
    return ap.parse_args()


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as fh:
            d = json.load(fh)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


def algorithmic_bytes(w, e4m3=False):
    elem = 2 if w.dtype == "bf16" else 4
    t = w.B * w.H * w.N * w.D * elem
    if e4m3:   # q, k, v one byte per element, out bf16
        return 3 * w.B * w.H * w.N * w.D + t
    wbytes = (w.H * w.D * w.F * elem) if w.F else 0
    return 4 * t + wbytes    # read q, k, v once, write out once (+ W)


def algorithmic_flops(w):
    per_head = 2 * 2 * w.N * w.features * w.D
    if w.F:
        per_head += 2 * 2 * w.N * w.D * w.F
    return per_head * w.B * w.H


# DRAM traffic per step (dram__bytes_read.sum + dram__bytes_write.sum summed
# over the step's launches, from one ncu capture per workload; the summaries
# and their commands are in profiles/).  Reported only while the device code (the kernel file and the
# device headers it includes) still hashes to what was captured; else null.
DEVICE_HEADERS = ("bf16_common.cuh", "sm100.cuh")
NCU_TRAFFIC = {
    "flux1024": (85_913_536, ("bf16_noncausal.cu",), "4cacf1a734292776"),
    "flux2048_cfg": (780_845_568, ("bf16_noncausal.cu",), "4cacf1a734292776"),
    "causal32k": (716_144_384, ("bf16_causal.cu",), "3e37cbf7e846ccac"),
    "proj256": (99_814_016, ("bf16_proj.cu", "bf16_image.cu"), "4d91d4572082bf07"),
    "flux1024_ttr": (144_333_888, ("bf16_noncausal.cu", "bf16_landmark.cu"), "149eae33d416bf3b"),
    "flux1024_e4m3": (42_611_328, ("bf16_noncausal.cu",), "4cacf1a734292776"),
    "flux2048_cfg_e4m3": (460_977_920, ("bf16_noncausal.cu",), "4cacf1a734292776"),
    "flux1024_softmax": (85_996_800, ("bf16_noncausal.cu",), "4cacf1a734292776"),
    "flux1024_prologue": (88_411_392, ("bf16_noncausal.cu",), "4cacf1a734292776"),
}


def source_hash(kernel_files):
    import hashlib
    h = hashlib.sha256()
    for f in tuple(kernel_files) + DEVICE_HEADERS:
        with open(os.path.join(ROOT, "linear_attention_diffusion_phi_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def captured_traffic(w, name=None):
    entry = NCU_TRAFFIC.get(name or w.name)
    if entry is None:
        return None
    nbytes, kernel_files, digest = entry
    return nbytes if source_hash(kernel_files) == digest else None


def kernels_per_step(w, sms):
    """(description, launches) of the library's kernels for one forward."""
    if w.dtype == "bf16" and not w.F and not w.causal:
        return "fused_t_kernel (one cluster launch per step)" if w.D == 128 else "fused_kernel (one cluster launch per step)", 1
    if w.dtype == "bf16" and w.F:
        return "proj_state_kernel + image_combine_kernel + proj_apply_kernel (three launches per step)", 3
    if w.dtype == "bf16" and w.causal:
        tiles = max(1, -(-w.N // 128))
        want = max(1, sms // (w.B * w.H))
        tps = -(-tiles // min(want, tiles))
        splits = -(-tiles // tps)
        if splits > 1:
            return "causal_state_kernel + causal_chunk_kernel (two launches per step)", 2
        return "causal_chunk_kernel (one launch per step)", 1
    return "library kernels", None


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 200 ms."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        rows = []
        with open(self.path) as fh:
            for line in fh:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = np.array([float(r[1]) for r in rows])
        mx = float(rows[0][2])
        power = np.array([float(r[3]) if r[3].replace(".", "").isdigit() else 0.0 for r in rows])
        loaded = sm[power >= np.median(power)] if len(sm) > 2 else sm
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": float(np.median(loaded)), "sm_max_mhz": mx, "reasons": reasons,
                "samples": len(rows)}


def percentiles_ms(times_ms):
    """p10 / p50 / p90 of per-call device times (ms)."""
    t = np.asarray(times_ms, dtype=np.float64)
    p10, p50, p90 = np.percentile(t, [10, 50, 90])
    return {"p10": float(p10), "p50": float(p50), "p90": float(p90), "calls": int(t.size)}


def per_call_ms(run_one, n, stream):
    """Device time of each of n single steps, each between its own pair of
    CUDA events on the launching stream (outside the timed region)."""
    import torch
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    for i, (a, b) in enumerate(evs):
        a.record(stream)
        run_one(i)
        b.record(stream)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in evs]


def _limit_blas_threads():
    """Pool initializer: one BLAS thread per worker process, so that the
    pool's size is the number of cores the oracle uses."""
    try:
        from threadpoolctl import threadpool_limits
        threadpool_limits(1)
    except Exception:
        pass


def _oracle_head(task):
    """One head of the workload through the float64 oracle, as it stands."""
    from oracle import la_oracle as ora
    q, k, v, W, fmap, eps, causal = task
    ora.forward(q[None, None], k[None, None], v[None, None], fmap, eps, causal, W)
    return q.shape[0]


def oracle_pool():
    """A pool of host processes (spawn: safe after CUDA is initialised), one
    per core this process may run on."""
    import multiprocessing as mp
    try:
        cores = len(os.sched_getaffinity(0))
    except Exception:
        cores = os.cpu_count() or 1
    return mp.get_context("spawn").Pool(cores, initializer=_limit_blas_threads), cores


def head_tasks(w, q, k, v, W):
    """Per-head oracle tasks in (b, h) order, from the stored values (float32
    holds bf16 values exactly; the oracle upcasts to float64)."""
    from linear_attention_diffusion_phi_b200.inputs import as_float64
    qf, kf, vf = (as_float64(x).astype(np.float32) for x in (q, k, v))
    Wf = None if W is None else as_float64(W).astype(np.float32)
    tasks = []
    for b in range(w.B):
        for h in range(w.H):
            tasks.append((qf[b, h], kf[b, h], vf[b, h], None if Wf is None else Wf[h], w.fmap, w.eps, w.causal))
    return tasks


def cpu_baseline(w, budget_s=10.0, inputs=None):
    """The float64 oracle, as it stands, on the host cores: whole heads of the
    same workload, one head per worker process at a time, until ~budget_s of
    wall time has passed."""
    from linear_attention_diffusion_phi_b200.inputs import make_inputs
    q, k, v, W = inputs if inputs is not None else make_inputs(w)
    tasks = head_tasks(w, q, k, v, W)
    pool, cores = oracle_pool()
    try:
        pool.map(_oracle_head, tasks[:cores])    # workers started and warm
        done_tokens, heads = 0, 0
        t0 = time.perf_counter()
        while time.perf_counter() - t0 < budget_s:
            batch = [tasks[(heads + j) % len(tasks)] for j in range(cores)]
            done_tokens += sum(pool.map(_oracle_head, batch, chunksize=1))
            heads += len(batch)
        dt = time.perf_counter() - t0
    finally:
        pool.close()
        pool.join()
    return {"value": done_tokens / dt, "unit": UNIT, "cores": int(cores), "kind": "oracle",
            "sample": f"{heads} heads of {w.name} (N={w.N}, D={w.D}, F={w.F}, causal={int(w.causal)}), "
                      f"one head per process on {cores} processes with one BLAS thread each, {dt:.1f} s",
            "cores_meaning": "host processes running the oracle at once, one BLAS thread each"}


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def input_seed(w, i, rank):
    """Seed of input set i on `rank`: every rank streams its own replica."""
    return w.seed + 7919 * i + 104729 * rank


def max_over_ranks(values, device=None):
    """Element-wise max of per-rank float values over the process group (the
    job's time is its slowest rank's); identity without a process group."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.cpu()]


def job_throughput(tokens_per_rank, world_size, steps, ms_total):
    """Whole-job tokens/s: every rank's tokens over the slowest rank's time."""
    return tokens_per_rank * world_size / (ms_total / 1e3 / steps)


def run_reference(args, w):
    """The float64 oracle as the reference arm: each step is a bounded sample
    of the workload, one whole head per host process (every core busy)."""
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    from linear_attention_diffusion_phi_b200.inputs import make_inputs
    tasks = head_tasks(w, *make_inputs(w))
    pool, cores = oracle_pool()
    try:
        def step(i):
            batch = [tasks[(i * cores + j) % len(tasks)] for j in range(cores)]
            return sum(pool.map(_oracle_head, batch, chunksize=1))
        for i in range(getattr(args, "warmup", 0)):
            step(i)
        t0 = time.perf_counter()
        tokens = 0
        for i in range(args.steps):
            tokens += step(i)
        dt = time.perf_counter() - t0
    finally:
        pool.close()
        pool.join()
    value = tokens / dt
    sample = f"{cores} of {w.B * w.H} heads per step, one per host process, float64 oracle"
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": getattr(args, "warmup", 0), "ms_per_step": dt / max(args.steps, 1) * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "D": w.D, "F": w.F,
                       "feature_map": w.fmap, "causal": w.causal, "sample": sample},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": int(cores), "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# bf16 bar (fp32 accumulation), with the self-imposed relative L2 bound; fp32 bar
BF16_MAX_ABS, BF16_MEAN_ABS, BF16_REL_L2, F32_REL_INF = 2e-2, 2e-3, 1e-2, 1e-5


def parity_samples(w):
    """(b, h, rows) picked for the oracle comparison of a timed workload:
    whole heads when the oracle's grouped form is cheap (non-causal), else
    512-row slices (start, a middle stretch, the end) checked row by row
    against the prefix-masked definition."""
    heads = [(0, 0), (w.B - 1, w.H - 1), (w.B // 2, w.H // 2)]
    heads = list(dict.fromkeys(heads))
    if not w.causal:
        return [(b, h, None) for b, h in heads]
    n = w.N
    sl = sorted(set(range(0, min(512, n))) | set(range(max(0, n // 4 - 256), min(n, n // 4 + 256))) |
                set(range(max(0, n - 512), n)))
    return [(b, h, sl) for b, h in heads[:2]]


def parity_block(w, q, k, v, W, got, ttr=None, e4m3=False, prologue=None):
    """Error figures of the GPU output `got` against the float64 oracle on
    the sampled heads / rows (CPU torch tensors of the stored values); with
    `ttr` = (landmark count, logits), against the oracle's TTR layer; with
    `e4m3`, q, k, v are E4M3 codes and W holds their three scales."""
    from linear_attention_diffusion_phi_b200.inputs import as_float64
    from oracle import la_oracle as ora
    if e4m3:
        qf, kf, vf = (s * ora.e4m3_decode(c.numpy()) for s, c in zip(W, (q, k, v)))
        Wf = None
    else:
        qf, kf, vf, Wf = as_float64(q), as_float64(k), as_float64(v), as_float64(W)
    diffs, refs, n_rows = [], [], 0
    for b, h, rows in parity_samples(w):
        g = as_float64(got[b, h])
        Wh = None if Wf is None else Wf[h:h + 1]
        if ttr is not None:
            ref = ora.ttr_forward(qf[b:b + 1, h:h + 1], kf[b:b + 1, h:h + 1], vf[b:b + 1, h:h + 1],
                                  [ttr[1][h]], ttr[0], w.fmap, w.eps, Wh)[0, 0]
        elif prologue is not None:
            qs, ks, rope = (t.numpy() for t in prologue)
            ref = ora.forward_prologue(qf[b:b + 1, h:h + 1], kf[b:b + 1, h:h + 1], vf[b:b + 1, h:h + 1], qs, ks, rope,
                                       1e-6, w.fmap, w.eps, w.causal)[0, 0]
        elif rows is None:
            ref = ora.forward(qf[b:b + 1, h:h + 1], kf[b:b + 1, h:h + 1], vf[b:b + 1, h:h + 1], w.fmap, w.eps,
                              w.causal, Wh)[0, 0]
        else:
            ref = ora.rows(qf, kf, vf, b, h, rows, w.fmap, w.eps, w.causal, None if Wf is None else Wf)
            g = g[rows]
        diffs.append(np.abs(g - ref).ravel())
        refs.append(ref.ravel())
        n_rows += ref.shape[0]
    d, r = np.concatenate(diffs), np.concatenate(refs)
    out = {"max_abs": float(d.max()), "mean_abs": float(d.mean()),
           "rel_l2": float(np.linalg.norm(d) / max(np.linalg.norm(r), 1e-300)),
           "rel_inf": float(d.max() / max(np.abs(r).max(), 1e-300)),
           "ref_rms": float(np.sqrt(np.mean(r * r))),
           "heads_checked": len(parity_samples(w)), "rows_checked": n_rows}
    if w.dtype == "bf16":
        out["bar"] = {"max_abs": BF16_MAX_ABS, "mean_abs": BF16_MEAN_ABS, "rel_l2": BF16_REL_L2}
        out["pass"] = bool(out["max_abs"] <= BF16_MAX_ABS and out["mean_abs"] <= BF16_MEAN_ABS and
                           out["rel_l2"] <= BF16_REL_L2)
        out["margin"] = float(min(BF16_MAX_ABS / max(out["max_abs"], 1e-300),
                                  BF16_MEAN_ABS / max(out["mean_abs"], 1e-300),
                                  BF16_REL_L2 / max(out["rel_l2"], 1e-300)))
    else:
        out["bar"] = {"rel_inf": F32_REL_INF}
        out["pass"] = bool(out["rel_inf"] <= F32_REL_INF)
        out["margin"] = float(F32_REL_INF / max(out["rel_inf"], 1e-300))
    return out


class Timed:
    """One workload resident on the device: rotating input sets whose total
    exceeds 3x L2 (set 0 holds the seeded inputs; the others are copies of it
    shifted along the sequence, so every step reads memory the previous steps
    did not touch), the operator, and CUDA graphs of its steps."""

    def __init__(self, w, dev, rank, graphs=True, ttr=None, e4m3=False, prologue=False, backward=False):
        import torch
        import linear_attention_diffusion_phi_b200 as la
        from linear_attention_diffusion_phi_b200.inputs import make_e4m3_inputs, make_inputs
        self.w = w
        # (landmark count, logits): time the TTR layer instead of la_forward
        self.ttr = ttr
        self.gate = None if ttr is None else torch.tensor(ttr[1], dtype=torch.float32, device=dev)
        # e4m3: q, k, v stored as E4M3 codes with per-tensor scales (la_forward_e4m3)
        self.e4m3 = e4m3
        dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
        self.set_bytes = algorithmic_bytes(w, e4m3) - (w.H * w.D * w.F * (2 if w.dtype == "bf16" else 4) if w.F else 0)
        self.nsets = max(2, -(-3 * L2_BYTES // self.set_bytes))
        if e4m3:
            q, k, v, self.scales = make_e4m3_inputs(w, seed=input_seed(w, 0, rank))
            W = None
            self.host = (q, k, v, self.scales)
            out_like = lambda: torch.empty(q.shape, dtype=torch.bfloat16, device=dev)
        else:
            self.host = make_inputs(w, seed=input_seed(w, 0, rank))
            q, k, v, W = self.host
            out_like = None
        base = (q.to(dev), k.to(dev), v.to(dev))
        # backward: each step computes dq, dk, dv of sum(out * dout) (la_backward)
        self.bwd = None
        if backward:
            dout = make_inputs(w, seed=input_seed(w, 0, rank) + 1)[0]
            self.bwd = (dout.to(dev), [torch.empty_like(base[0]) for _ in range(3)])
            self.host = (q, k, v, dout)
            self.set_bytes += 3 * w.B * w.H * w.N * w.D * 4
        new_out = out_like or (lambda: torch.empty_like(base[0]))
        self.sets = [base + (new_out(),)]
        for i in range(1, self.nsets):
            sh = (97 * i) % max(w.N, 1)
            self.sets.append(tuple(torch.roll(x, shifts=sh, dims=2) for x in base) + (new_out(),))
        self.op = la.LinearAttention(dt, w.fmap, w.eps, w.causal, None if W is None else W.to(dev))
        # prologue: Flux's QK norm and rotary embedding ahead of the layer
        self.pro_host = None
        if prologue:
            from linear_attention_diffusion_phi_b200.inputs import make_prologue_params
            self.pro_host = make_prologue_params(w)
            self.op.set_prologue(*(t.to(dev) for t in self.pro_host))
        self.graphs = graphs
        self.g_all = None
        self.g_all_steps = 0
        self.g_one = []
        # steps the timed region will run: the big graph holds as many whole
        # rounds of the input sets as fit in it (at most 64 steps), so a timed
        # region of K steps pays few graph launches
        self.steps_hint = 64

    def step(self, i):
        q, k, v, o = self.sets[i % self.nsets]
        if self.bwd is not None:
            self.op.backward(q, k, v, self.bwd[0], outs=self.bwd[1])
        elif self.e4m3:
            self.op.e4m3(q, k, v, self.scales, out=o)
        elif self.ttr is None:
            self.op(q, k, v, out=o)
        else:
            self.op.ttr(q, k, v, self.ttr[0], self.gate, out=o)

    def capture(self):
        import torch
        if not self.graphs:
            return
        rounds = max(1, min(self.steps_hint, 64) // self.nsets)
        self.g_all_steps = rounds * self.nsets
        self.g_all = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.g_all):
            for j in range(self.g_all_steps):
                self.step(j)
        for j in range(self.nsets):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                self.step(j)
            self.g_one.append(g)
        self.g_all.replay()
        torch.cuda.synchronize()

    def run_steps(self, k):
        if not self.graphs:
            for i in range(k):
                self.step(i)
            return
        i = 0
        while i + self.g_all_steps <= k:
            self.g_all.replay()
            i += self.g_all_steps
        while i < k:
            self.g_one[i % self.nsets].replay()
            i += 1

    def run_one(self, i):
        if self.graphs:
            self.g_one[i % self.nsets].replay()
        else:
            self.step(i)

    def warm(self, warmup, soak_s):
        import torch
        for i in range(max(3, warmup)):
            self.step(i)
        torch.cuda.synchronize()
        t_end = time.perf_counter() + soak_s
        i = 0
        while time.perf_counter() < t_end:   # untimed load so clocks settle
            for _ in range(50):
                self.step(i)
                i += 1
            torch.cuda.synchronize()
        self.capture()

    def timed_ms(self, steps, stream, ws):
        """Device time (ms) of `steps` steps between CUDA events on the
        launching stream, bracketed by a barrier and a synchronize."""
        import torch
        import torch.distributed as dist
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if ws > 1:
            dist.barrier()
        torch.cuda.synchronize()
        ev0.record(stream)
        self.run_steps(steps)
        ev1.record(stream)
        torch.cuda.synchronize()
        if ws > 1:
            dist.barrier()
        return ev0.elapsed_time(ev1)

    def output0(self):
        """The output of input set 0 (the seeded inputs), on the host."""
        import torch
        self.step(0)
        torch.cuda.synchronize()
        return self.sets[0][3].cpu()

    def close(self):
        self.g_all = None
        self.g_one = []
        self.sets = []
        self.op.close()


def roofline(w, per_step_s, hbm, tflops, src, sms):
    abytes = algorithmic_bytes(w)
    achieved = abytes / per_step_s / 1e9
    kdesc, launches = kernels_per_step(w, sms)
    roof = {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
            "traffic": captured_traffic(w), "peak_source": f"{src} hbm_gbs", "frac_of": src, "kernel": kdesc,
            "algorithmic_bytes_per_step": abytes}
    if w.F:
        # the projected workload is reported against the tensor roofline (dense
        # bf16, the burst figure: a step lasts tens of microseconds); its HBM
        # fraction is kept alongside
        af = algorithmic_flops(w)
        hbm_part = {k: roof[k] for k in ("achieved", "peak", "unit", "frac")}
        roof.update({"bound": "tensor", "achieved": af / per_step_s / 1e12, "peak": tflops, "unit": "TFLOP/s",
                     "frac": af / per_step_s / 1e12 / tflops, "peak_source": f"{src} bf16_tflops",
                     "algorithmic_flops_per_step": af, "hbm": hbm_part})
    return roof, launches


def backward_parity(w, tx):
    """Largest error of dq, dk, dv on two sampled heads against the oracle's
    backward, relative to each gradient's largest magnitude."""
    import torch
    from linear_attention_diffusion_phi_b200.inputs import as_float64
    from oracle import la_oracle as ora
    tx.step(0)
    torch.cuda.synchronize()
    q, k, v, dout = tx.host
    got = [g.cpu() for g in tx.bwd[1]]
    worst = 0.0
    for b, h in ((0, 0), (w.B - 1, w.H - 1)):
        ref = ora.backward_head(*(as_float64(t[b, h]) for t in (q, k, v, dout)), w.fmap, w.eps)
        for g, r in zip(got, ref):
            worst = max(worst, float(np.abs(as_float64(g[b, h]) - r).max() / max(np.abs(r).max(), 1e-300)))
    return {"rel_inf": worst, "bar": {"rel_inf": F32_REL_INF}, "pass": bool(worst <= F32_REL_INF),
            "heads_checked": 2}


def roofline_e4m3(w, per_step_s, hbm, src, name):
    """HBM roofline of the E4M3-input forward (one launch per step): q, k, v
    read once at one byte per element, out written once in bf16."""
    abytes = algorithmic_bytes(w, e4m3=True)
    achieved = abytes / per_step_s / 1e9
    return {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
            "traffic": captured_traffic(w, name), "peak_source": f"{src} hbm_gbs", "frac_of": src,
            "kernel": "fused_t_kernel, E4M3 inputs (one cluster launch per step)",
            "algorithmic_bytes_per_step": abytes}


EXTRA_WORKLOADS = ("flux2048_cfg", "proj256", "causal32k", "flux1024_ttr", "flux1024_e4m3", "flux2048_cfg_e4m3",
                   "flux1024_softmax", "flux1024_prologue", "flux1024_f32_backward")
# The TTR layer on the flux1024 shape: 128 landmarks (the page's knobs at
# fraction 1/32, min 16, max 128) and one logit per head, spread over [-2, 2].
TTR_LANDMARKS = (1 / 32, 16, 128)


def ttr_params(w):
    """(landmark count, per-head logits) of the TTR layer on workload w."""
    import linear_attention_diffusion_phi_b200 as la
    return la.la_landmark_count(w.N, *TTR_LANDMARKS), [float(x) for x in np.linspace(-2.0, 2.0, w.H)]


def run_extra(name, args, dev, rank, local, stream, ws, hbm, tflops, src, sms):
    """Time one of EXTRA_WORKLOADS the way the headline is timed (at least 100
    steps) and return its entry for the line's extra_configs."""
    import torch
    import linear_attention_diffusion_phi_b200 as la
    from linear_attention_diffusion_phi_b200.inputs import WORKLOADS
    ttr = name.endswith("_ttr")
    e8 = name.endswith("_e4m3")
    smx = name.endswith("_softmax")   # the same shapes with the softmax feature map
    pro = name.endswith("_prologue")  # the same shapes behind Flux's attention prologue
    bwd = name.endswith("_backward")  # the fp32 backward pass on the same shapes
    base = name[:-4] if ttr else (name[:-5] if e8 else (name[:-8] if smx else (name[:-9] if pro else name)))
    if bwd:
        base = name[:-len("_f32_backward")]
    x = WORKLOADS[base]
    if bwd:
        x = x.with_(dtype="f32")
    if smx:
        x = x.with_(fmap="softmax")
    try:
        tx = Timed(x, dev, rank, graphs=not args.no_graph, ttr=ttr_params(x) if ttr else None, e4m3=e8,
                   prologue=pro, backward=bwd)
        xsteps = max(args.steps, 100)
        tx.steps_hint = xsteps
        smp = ClockSampler(local)
        smp.start()
        tx.warm(args.warmup, 0.3)
        xms = tx.timed_ms(xsteps, stream, ws)
        xclk = smp.stop()
        assert tx.op.sync_status() == la.LA_OK, "device-side error during the timed region"
        xroof, xl = roofline(x, xms / 1e3 / xsteps, hbm, tflops, src, sms)
        if ttr:
            # two launches; the roofline is the layer's: q, k, v read
            # once and out written once (the landmark pass adds a read
            # of q and a read and write of out on top)
            xl = 2
            xroof["kernel"] = "fused_t_kernel + landmark_blend_kernel (two launches per step)"
            xroof["traffic"] = captured_traffic(x, name)
            xroof["landmarks"], xroof["gates"] = tx.ttr[0], "linspace(-2, 2, H)"
        if e8:
            xroof = roofline_e4m3(x, xms / 1e3 / xsteps, hbm, src, name)
        if smx or pro:
            xroof["traffic"] = captured_traffic(x, name)
        if pro:
            xroof["kernel"] = "fused_t_kernel with the prologue (one cluster launch per step)"
        if bwd:
            # q, k, v, dout read and dq, dk, dv written once, fp32
            abytes = 7 * x.B * x.H * x.N * x.D * 4
            xroof = {"bound": "hbm", "achieved": abytes / (xms / 1e3 / xsteps) / 1e9, "peak": hbm, "unit": "GB/s",
                     "frac": abytes / (xms / 1e3 / xsteps) / 1e9 / hbm, "traffic": None,
                     "peak_source": f"{src} hbm_gbs", "frac_of": src, "algorithmic_bytes_per_step": abytes,
                     "kernel": "f32_state_partial, f32_state_combine, f32_bwd_query, f32_state_combine, f32_bwd_key "
                               "(five launches per step)"}
            xl = 5
        ent = {"workload": name, "B": x.B, "H": x.H, "N": x.N, "D": x.D, "F": x.F, "feature_map": x.fmap,
               "causal": x.causal, "dtype": "e4m3 in, bf16 out" if e8 else x.dtype, "steps": xsteps,
               "ms_per_step": xms / xsteps,
               "value": x.tokens / (xms / 1e3 / xsteps), "unit": UNIT, "roofline": xroof,
               "gpu_launches": None if xl is None else xl * xsteps, "clocks": xclk,
               "l2": f"{tx.nsets} rotating input sets, {tx.nsets * tx.set_bytes / 2**20:.0f} MiB > 3x L2"}
        if bwd:
            ent["dtype"] = "f32"
        if not args.no_parity and not bwd:
            ent["parity"] = parity_block(x, *tx.host, tx.output0(), ttr=tx.ttr, e4m3=e8, prologue=tx.pro_host)
        if not args.no_parity and bwd:
            ent["parity"] = backward_parity(x, tx)
        tx.close()
        del tx
    except Exception as e:   # an extra figure never costs the headline line
        ent = {"workload": name, "error": f"{type(e).__name__}: {e}"[:300]}
    torch.cuda.empty_cache()
    return ent


def main():
    args = parse()
    from linear_attention_diffusion_phi_b200.inputs import WORKLOADS
    w = WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, w)

    import torch
    import torch.distributed as dist
    import linear_attention_diffusion_phi_b200 as la
    from linear_attention_diffusion_phi_b200 import build as la_build

    ws, rank, local = dist_env()
    if ws > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if not os.path.exists(la.LIB_PATH):
        if rank == 0:
            la_build.build()
        if ws > 1:
            dist.barrier()
    stream = torch.cuda.current_stream(dev)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    hbm, tflops, src = peaks()

    if args.extra_only:
        ent = run_extra(args.extra_only, args, dev, rank, local, stream, ws, hbm, tflops, src, sms)
        if rank == 0:
            print(json.dumps(ent))
        return 0 if "error" not in ent else 1

    tw = Timed(w, dev, rank, graphs=not args.no_graph)
    tw.steps_hint = args.steps
    sampler = ClockSampler(local)
    sampler.start()
    tw.warm(args.warmup, args.soak_s)
    ms = tw.timed_ms(args.steps, stream, ws)
    clocks = sampler.stop()
    assert tw.op.sync_status() == la.LA_OK, "device-side error during the timed region"

    # distribution of single calls (this rank's), informational: the value
    # above is the mean over the bracketed steps
    try:
        per_call = percentiles_ms(per_call_ms(tw.run_one, max(10, min(args.steps, 100)), stream))
    except Exception as e:   # never let the extra figure cost the bench line
        per_call = {"error": f"{type(e).__name__}: {e}"[:200]}

    # end to end through the host-buffer entry point: pinned host inputs,
    # H2D copies, forward, D2H copy of the result, every step.  Two lanes
    # (a handle, its workspace, device buffers and a stream each) take the
    # steps in turn, so one step's result copy and the next step's input
    # copies share the full-duplex link and the kernels overlap the copies;
    # every copy of every step is inside the timed region.
    qh = [s[0].cpu().pin_memory() for s in tw.sets[:2]]
    kh = [s[1].cpu().pin_memory() for s in tw.sets[:2]]
    vh = [s[2].cpu().pin_memory() for s in tw.sets[:2]]
    oh = [torch.empty_like(x).pin_memory() for x in qh]
    dt = tw.sets[0][0].dtype
    lanes = []
    for j in range(2):
        op_j = tw.op if j == 0 else la.LinearAttention(dt, w.fmap, w.eps, w.causal,
                                                       None if tw.host[3] is None else tw.host[3].to(dev))
        bufs = tuple(torch.empty_like(tw.sets[0][0]) for _ in range(4))
        if j > 0:
            op_j(*bufs[:3], out=bufs[3])   # binds its workspace
        lanes.append((op_j, bufs, torch.cuda.Stream(device=dev)))
    torch.cuda.synchronize()
    e2e_steps = max(4, min(args.steps, 50))

    def e2e_step(i):
        op_j, (dq, dk, dv, do), st_j = lanes[i % 2]
        h = i % 2
        st = la.la_forward_host(op_j.handle, qh[h].data_ptr(), kh[h].data_ptr(), vh[h].data_ptr(),
                                oh[h].data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), do.data_ptr(),
                                w.B, w.H, w.N, w.D, w.F, la.FEATURE_MAPS[w.fmap], w.eps, int(w.causal),
                                st_j.cuda_stream)
        la.check(st, "la_forward_host")
    for i in range(4):
        e2e_step(i)
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if ws > 1:
        dist.barrier()
    ev0.record(stream)
    for _, _, st_j in lanes:
        st_j.wait_event(ev0)
    for i in range(e2e_steps):
        e2e_step(i)
    for _, _, st_j in lanes:
        done = torch.cuda.Event()
        done.record(st_j)
        stream.wait_event(done)
    ev1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = ev0.elapsed_time(ev1)
    for op_j, _, _ in lanes[1:]:
        assert op_j.sync_status() == la.LA_OK
        op_j.close()
    del qh, kh, vh, oh, lanes

    ms, e2e_ms = max_over_ranks([ms, e2e_ms], device=dev)
    got0 = tw.output0() if (rank == 0 and not args.no_parity) else None
    tw.close()

    # the other workloads, timed the same way after the headline (one GPU:
    # their figures are reported beside it, the headline value is unchanged)
    extras = []
    if ws == 1 and not args.no_extra and w.name == "flux1024":
        for name in EXTRA_WORKLOADS:
            extras.append(run_extra(name, args, dev, rank, local, stream, ws, hbm, tflops, src, sms))

    if ws > 1:
        dist.destroy_process_group()
    if rank != 0:
        return 0

    tokens = w.tokens * ws
    per_step_s = ms / 1e3 / args.steps
    value = job_throughput(w.tokens, ws, args.steps, ms)
    roof, launches = roofline(w, per_step_s, hbm, tflops, src, sms)
    elem = 2 if w.dtype == "bf16" else 4
    io = w.B * w.H * w.N * w.D * elem
    e2e = {"value": tokens / (e2e_ms / 1e3 / e2e_steps), "unit": UNIT, "h2d_bytes_per_step": 3 * io,
           "d2h_bytes_per_step": io, "steps": e2e_steps,
           "pipelining": "2 lanes (handle, workspace, device buffers, stream) take steps in turn"}
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "D": w.D, "F": w.F,
                       "feature_map": w.fmap, "eps": w.eps, "causal": w.causal,
                       "global_batch": w.B * ws, "seq_len": w.N, "parallelism": f"replicas{ws}",
                       "l2": f"{tw.nsets} rotating input sets, {tw.nsets * tw.set_bytes / 2**20:.0f} MiB > 3x L2"},
            "hbm_gbs": roof["achieved"] if roof["bound"] == "hbm" else roof["hbm"]["achieved"],
            "roofline": roof, "clocks": clocks, "e2e": e2e, "per_call_ms": per_call,
            "gpu_launches": None if launches is None else launches * args.steps,
            "launch": "cuda-graph" if not args.no_graph else "host"}
    if got0 is not None:
        line["parity"] = parity_block(w, *tw.host, got0)
    if extras:
        line["extra_configs"] = extras
    if not args.no_cpu_baseline and ws == 1:
        line["cpu_baseline"] = cpu_baseline(w, inputs=tw.host)
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
