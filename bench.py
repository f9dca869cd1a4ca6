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
    return ap.parse_args()


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as fh:
            d = json.load(fh)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


def algorithmic_bytes(w):
    elem = 2 if w.dtype == "bf16" else 4
    t = w.B * w.H * w.N * w.D * elem
    wbytes = (w.H * w.D * w.F * elem) if w.F else 0
    return 4 * t + wbytes    # read q, k, v once, write out once (+ W)


def algorithmic_flops(w):
    per_head = 2 * 2 * w.N * w.features * w.D
    if w.F:
        per_head += 2 * 2 * w.N * w.D * w.F
    return per_head * w.B * w.H


# DRAM traffic per step (dram__bytes_read.sum + dram__bytes_write.sum summed
# over the step's launches, one ncu --set full capture each; the summaries are
# in profiles/).  Reported only while the device code (the kernel file and the
# device headers it includes) still hashes to what was captured; else null.
DEVICE_HEADERS = ("bf16_common.cuh", "sm100.cuh")
NCU_TRAFFIC = {
    "flux1024": (89_287_168, ("bf16_noncausal.cu",), "09cb7e3d60d8e95f"),
    "causal32k": (722_496_256, ("bf16_causal.cu",), "0827122f020f8286"),
    "proj256": (102_777_344, ("bf16_proj.cu", "bf16_image.cu"), "af511b8a7d19cef5"),
}


def source_hash(kernel_files):
    import hashlib
    h = hashlib.sha256()
    for f in tuple(kernel_files) + DEVICE_HEADERS:
        with open(os.path.join(ROOT, "linear_attention_diffusion_phi_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def captured_traffic(w):
    entry = NCU_TRAFFIC.get(w.name)
    if entry is None:
        return None
    nbytes, kernel_files, digest = entry
    return nbytes if source_hash(kernel_files) == digest else None


def kernels_per_step(w, sms):
    """(description, launches) of the library's kernels for one forward."""
    if w.dtype == "bf16" and not w.F and not w.causal:
        return "fused_kernel (one cluster launch per step)", 1
    if w.dtype == "bf16" and w.F:
        return "proj_state_kernel + proj_combine_kernel + proj_apply_kernel (three launches per step)", 3
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


def cpu_baseline(w, budget_s=10.0):
    """The float64 oracle, as it stands, on the host cores: whole-problem
    forwards of the same workload until ~budget_s of CPU time has passed."""
    from linear_attention_diffusion_phi_b200.inputs import as_float64, make_inputs
    from oracle import la_oracle as ora
    q, k, v, W = make_inputs(w)
    q, k, v, W = as_float64(q), as_float64(k), as_float64(v), as_float64(W)
    heads = w.B * w.H
    per_call = max(1, heads)
    done_tokens = 0
    t0 = time.perf_counter()
    hs = 0
    while True:
        b, h = divmod(hs % heads, w.H)
        sl = (slice(b, b + 1), slice(h, h + 1))
        Wh = None if W is None else W[h:h + 1]
        ora.forward(q[sl], k[sl], v[sl], w.fmap, w.eps, w.causal, Wh)
        done_tokens += w.N
        hs += 1
        if time.perf_counter() - t0 >= budget_s and hs >= 1:
            break
    dt = time.perf_counter() - t0
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        cores = 1
    return {"value": done_tokens / dt, "unit": UNIT, "cores": int(cores), "kind": "oracle",
            "sample": f"{hs} heads of {w.name} (N={w.N}, D={w.D}, F={w.F}, causal={int(w.causal)}) "
                      f"through oracle.forward in {dt:.1f} s", "per_call_heads": per_call}


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
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    from linear_attention_diffusion_phi_b200.inputs import as_float64, make_inputs
    from oracle import la_oracle as ora
    q, k, v, W = make_inputs(w)
    q, k, v, W = as_float64(q), as_float64(k), as_float64(v), as_float64(W)
    heads_per_step = 2   # bounded sample of the workload per step
    def step(i):
        for j in range(heads_per_step):
            hs = (i * heads_per_step + j) % (w.B * w.H)
            b, h = divmod(hs, w.H)
            ora.forward(q[b:b + 1, h:h + 1], k[b:b + 1, h:h + 1], v[b:b + 1, h:h + 1], w.fmap, w.eps,
                        w.causal, None if W is None else W[h:h + 1])
    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(i)
    dt = time.perf_counter() - t0
    tokens = args.steps * heads_per_step * w.N
    value = tokens / dt
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        cores = 1
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "D": w.D, "F": w.F,
                       "feature_map": w.fmap, "causal": w.causal,
                       "sample": f"{heads_per_step} heads per step"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": int(cores), "kind": "oracle",
                             "sample": f"{heads_per_step} of {w.B * w.H} heads per step, float64 oracle"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse()
    from linear_attention_diffusion_phi_b200.inputs import WORKLOADS, make_inputs
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
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32

    # input sets rotated step to step so that consecutive steps never find
    # their inputs in L2 (total > 3x L2)
    set_bytes = 4 * w.B * w.H * w.N * w.D * (2 if w.dtype == "bf16" else 4)
    nsets = max(2, -(-3 * L2_BYTES // set_bytes))
    sets = []
    for i in range(nsets):
        q, k, v, W = make_inputs(w, seed=input_seed(w, i, rank))
        sets.append((q.to(dev), k.to(dev), v.to(dev), torch.empty_like(q, device=dev)))
    Wd = None if W is None else W.to(dev)
    op = la.LinearAttention(dt, w.fmap, w.eps, w.causal, Wd)
    stream = torch.cuda.current_stream(dev)

    def step(i):
        q, k, v, o = sets[i % nsets]
        op(q, k, v, out=o)

    sampler = ClockSampler(local)
    sampler.start()
    for i in range(max(3, args.warmup)):
        step(i)
    torch.cuda.synchronize()
    t_end = time.perf_counter() + args.soak_s
    i = 0
    while time.perf_counter() < t_end:   # untimed load so clocks settle
        for _ in range(200):
            step(i)
            i += 1
        torch.cuda.synchronize()

    # CUDA graphs remove host launch overhead: one graph runs one step over
    # every input set in turn, single-step graphs cover a remainder.

    if not args.no_graph:
        g_all = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_all):
            for j in range(nsets):
                step(j)
        g_one = []
        for j in range(nsets):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                step(j)
            g_one.append(g)
        g_all.replay()
        torch.cuda.synchronize()

    def run_steps(k):
        if args.no_graph:
            for i in range(k):
                step(i)
            return
        i = 0
        while i + nsets <= k:
            g_all.replay()
            i += nsets
        while i < k:
            g_one[i % nsets].replay()
            i += 1

    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize()
    ev0.record(stream)
    run_steps(args.steps)
    ev1.record(stream)
    torch.cuda.synchronize()
    if ws > 1:
        dist.barrier()
    ms = ev0.elapsed_time(ev1)
    clocks = sampler.stop()
    assert op.sync_status() == la.LA_OK, "device-side error during the timed region"

    # distribution of single calls (this rank's), informational: the value
    # above is the mean over the bracketed steps
    try:
        one = (lambda i: step(i)) if args.no_graph else (lambda i: g_one[i % nsets].replay())
        per_call = percentiles_ms(per_call_ms(one, max(10, min(args.steps, 100)), stream))
    except Exception as e:   # never let the extra figure cost the bench line
        per_call = {"error": f"{type(e).__name__}: {e}"[:200]}

    # end to end through the host-buffer entry point: pinned host inputs,
    # H2D copies, forward, D2H copy of the result, every step
    qh = [s[0].cpu().pin_memory() for s in sets[:2]]
    kh = [s[1].cpu().pin_memory() for s in sets[:2]]
    vh = [s[2].cpu().pin_memory() for s in sets[:2]]
    oh = [torch.empty_like(x).pin_memory() for x in qh]
    dq, dk, dv, do = (torch.empty_like(sets[0][0]) for _ in range(4))
    e2e_steps = max(3, min(args.steps, 50))
    s_ptr = stream.cuda_stream

    def e2e_step(i):
        j = i % 2
        st = la.la_forward_host(op.handle, qh[j].data_ptr(), kh[j].data_ptr(), vh[j].data_ptr(),
                                oh[j].data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), do.data_ptr(),
                                w.B, w.H, w.N, w.D, w.F, la.FEATURE_MAPS[w.fmap], w.eps, int(w.causal), s_ptr)
        la.check(st, "la_forward_host")
    for i in range(3):
        e2e_step(i)
    torch.cuda.synchronize()
    if ws > 1:
        dist.barrier()
    ev0.record(stream)
    for i in range(e2e_steps):
        e2e_step(i)
    ev1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = ev0.elapsed_time(ev1)

    ms, e2e_ms = max_over_ranks([ms, e2e_ms], device=dev)
    if ws > 1:
        dist.destroy_process_group()
    if rank != 0:
        return 0

    tokens = w.tokens * ws
    per_step_s = ms / 1e3 / args.steps
    value = job_throughput(w.tokens, ws, args.steps, ms)
    hbm, tflops, src = peaks()
    abytes = algorithmic_bytes(w)
    achieved = abytes / per_step_s / 1e9
    kdesc, launches = kernels_per_step(w, torch.cuda.get_device_properties(dev).multi_processor_count)
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
    elem = 2 if w.dtype == "bf16" else 4
    io = w.B * w.H * w.N * w.D * elem
    e2e = {"value": tokens / (e2e_ms / 1e3 / e2e_steps), "unit": UNIT, "h2d_bytes_per_step": 3 * io,
           "d2h_bytes_per_step": io, "steps": e2e_steps}
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "D": w.D, "F": w.F,
                       "feature_map": w.fmap, "eps": w.eps, "causal": w.causal,
                       "global_batch": w.B * ws, "seq_len": w.N, "parallelism": f"replicas{ws}",
                       "l2": f"{nsets} rotating input sets, {nsets * set_bytes / 2**20:.0f} MiB > 3x L2"},
            "hbm_gbs": achieved, "roofline": roof, "clocks": clocks, "e2e": e2e, "per_call_ms": per_call,
            "gpu_launches": None if launches is None else launches * args.steps, "launch": "cuda-graph" if not args.no_graph else "host"}
    if not args.no_cpu_baseline and ws == 1:
        line["cpu_baseline"] = cpu_baseline(w)
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
