"""Benchmark: RoPE/LeRoPE attention fwd + loss + bwd (incl. dalpha) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--config C]
    python bench.py --profile --shape B,H,n,d [--causal] [--steps K] [--warmup W] [--d-model M]

One step = the whole path on one batch: rope_attn_fwd (table, rotation, tcgen05
forward), rope_attn_loss, rope_attn_bwd_saved (Delta, dK/dV, dQ, dalpha from the table and
rotated Q~, K~ the forward left in the workspace, as a training step saves them).
Workload: 2 x 32 x 8192 x 128 bf16 causal, base 1e4, alpha ~ N(0, 0.3^2) -- the
headline configuration.  Metric: fwd+bwd TFLOP/s with the standard count
14 n^2 d per (batch, head), halved for causal masking.  Inputs (4 x 134 MB) exceed
the 126 MB L2, so no flush is needed between steps.

With --gpus N > 1 (under torchrun) every rank runs the same workload on its own
batch (seeded by rank): per-GPU work is fixed (weak scaling) and the one exchange the
method has -- the dalpha of the shared LeRoPE frequencies, summed over every head of
every rank -- is an NCCL all-reduce of d/2 floats per step.

--impl reference times the float64 CPU oracle (the only other implementation of the
method; the pages ship no code) on a bounded sample of the same workload.
"""
import argparse
import atexit
import datetime
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

NOMINAL_BF16_TFLOPS = 2250.0
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK), "fallback"


def workload(cfg):
    from rope_attention_fwd_b200.configs import WORKLOADS
    return WORKLOADS[cfg]


def config_dict(wl, cfg, world):
    return {"workload": f"config {cfg}: {wl.name}", "B": wl.B, "H": wl.H, "n": wl.n, "d": wl.d,
            "causal": wl.causal, "base": wl.base, "global_batch": wl.B * world,
            "seq_len": wl.n, "parallelism": f"dp{world}" if world > 1 else "single-gpu",
            "l2": "inputs larger than L2 (4 x %.0f MB > 126 MB), no flush" %
                  (wl.B * wl.H * wl.n * wl.d * 2 / 1e6)}


# ----------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples (every 50 ms, timestamped) from before the warm-up to the end of
    the timed passes; summary() keeps the samples inside the windows mark() recorded."""
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    PERIOD_MS = 50

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None
        self.windows = []

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader", "-lms", str(self.PERIOD_MS)],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        atexit.register(self.stop)   # never left running if the bench fails in between
        return self

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.proc = None

    def __exit__(self, *a):
        self.stop()

    def window(self):
        """Context manager marking a timed region (wall clock, as nvidia-smi stamps it)."""
        sampler = self

        class _Window:
            def __enter__(self):
                self.t0 = datetime.datetime.now()
                return self

            def __exit__(self, *a):
                sampler.windows.append((self.t0, datetime.datetime.now()))
        return _Window()

    @staticmethod
    def parse(lines, windows):
        """(sm MHz, max MHz, [hw_slowdown, hw_thermal, sw_thermal, sw_power_cap]) of the
        samples stamped inside any window."""
        rows = []
        for line in lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f")
                sm = float(parts[2].split()[0])
                mx = float(parts[3].split()[0])
            except ValueError:
                continue
            if any(a <= ts <= b for a, b in windows):
                rows.append((sm, mx, parts[6:10]))
        return rows

    def summary(self):
        rows = []
        if self.path and os.path.exists(self.path):
            with open(self.path) as f:
                rows = self.parse(f, self.windows)
            os.remove(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, r in rows for i in range(4)
                          if r[i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(r[0] for r in rows),
                "sm_max_mhz": max(r[1] for r in rows), "reasons": reasons,
                "samples": len(rows)}


# ----------------------------------------------------------------- oracle timing
def time_oracle(wl, max_seconds=30.0):
    """Oracle fwd+loss+bwd of one (batch, head) of the workload; FLOPs by the metric's
    count for that one head.  Returns (TFLOP/s, seconds, sample description, threads)."""
    import numpy as np
    import torch
    from oracle import rope_attn_ref as ref
    from rope_attention_fwd_b200.inputs import make_inputs
    one = wl.with_(B=1, H=1)
    inp = make_inputs(one)
    q, k, v, e, al = (inp.f64(x) for x in ("q", "k", "v", "e", "alpha"))
    t0 = time.perf_counter()
    ref.forward_backward(q, k, v, e, al, one.base, one.causal)
    dt = time.perf_counter() - t0
    flops = one.flops_fwd() + one.flops_bwd()
    try:
        threads = len(os.sched_getaffinity(0))
    except AttributeError:
        threads = os.cpu_count()
    sample = (f"1 of {wl.B * wl.H} (batch, head) slices of the workload "
              f"(n={wl.n}, d={wl.d}), full fwd+loss+bwd, float64 numpy")
    return flops / dt / 1e12, dt, sample, threads


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    wl = workload(args.config)
    vals = []
    for _ in range(max(0, args.warmup_ref)):
        time_oracle(wl)
    total = 0.0
    for _ in range(args.steps_ref):
        v, dt, sample, threads = time_oracle(wl)
        vals.append(v)
        total += dt
    value = statistics.mean(vals)
    line = {"impl": "reference", "metric": "RoPE-attn fwd+bwd TFLOP/s (bf16, incl. dalpha)",
            "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps_ref,
            "steps_requested": args.steps,
            "warmup": args.warmup_ref, "ms_per_step": 1e3 * total / max(1, args.steps_ref),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config_dict(wl, args.config, world),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------- our arm
def run_ours(args):
    import torch
    import torch.distributed as dist
    from rope_attention_fwd_b200 import binding as rb
    from rope_attention_fwd_b200.dist import allreduce_sum, rank_seed
    from rope_attention_fwd_b200.inputs import make_inputs

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=dev)
    wl = workload(args.config)
    inp = make_inputs(wl, seed=rank_seed(wl.seed, rank))
    flops_fwd, flops_bwd = wl.flops_fwd(), wl.flops_bwd()
    flops = flops_fwd + flops_bwd

    host = {x: getattr(inp, x).pin_memory() for x in ("q", "k", "v", "e", "alpha")}
    dv_in = {x: host[x].to(dev) for x in host}
    prob = rb.problem(wl.B, wl.H, wl.n, wl.d, dv_in["q"].dtype, wl.causal, wl.base)
    ws = rb.workspace(prob, dev)
    def outputs():
        o = torch.empty_like(dv_in["q"])
        return {"o": o, "lse": torch.empty((wl.B, wl.H, wl.n), dtype=torch.float32, device=dev),
                "L": torch.empty((), dtype=torch.float32, device=dev), "dO": torch.empty_like(o),
                "dq": torch.empty_like(o), "dk": torch.empty_like(o), "dv": torch.empty_like(o),
                "dalpha": torch.empty(wl.d // 2, dtype=torch.float32, device=dev)}

    out0 = outputs()

    def step(t, r):
        rb.rope_attn_fwd(t["q"], t["k"], t["v"], t["alpha"], wl.base, wl.causal, ws=ws,
                         o=r["o"], lse=r["lse"])
        rb.rope_attn_loss(r["o"], t["e"], ws=ws, L=r["L"], dO=r["dO"])
        # the backward takes the table and rotated Q~, K~ the forward just wrote into ws
        rb.rope_attn_bwd_saved(t["v"], r["o"], r["lse"], r["dO"], t["alpha"], wl.base,
                               wl.causal, ws, dq=r["dq"], dk=r["dk"], dv=r["dv"],
                               dalpha=r["dalpha"])
        # L and dalpha are sums over every head of every rank (no-ops on one GPU)
        allreduce_sum(r["L"])
        allreduce_sum(r["dalpha"])

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    def max_over_ranks(x):
        if world == 1:
            return x
        t = torch.tensor([x], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    stream = torch.cuda.current_stream(dev)
    # ---------------- device-resident timing
    clk = ClockSampler(local).__enter__()   # running before the timed passes begin
    for _ in range(args.warmup):
        step(dv_in, out0)
    barrier()
    code, info = rb.rope_attn_device_status(ws)
    if code != 0:
        raise RuntimeError(f"device status {rb.STATUS.get(code, code)} {info}")
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    # the headline: whole steps, no per-kernel events between the launches (those would
    # serialise the dQ kernel behind the dK/dV kernel, which it may otherwise overlap)
    barrier()
    with clk.window():
        ev0.record(stream)
        for _ in range(args.steps):
            step(dv_in, out0)
        ev1.record(stream)
        barrier()
    ms = ev0.elapsed_time(ev1) / args.steps
    ms = max_over_ranks(ms)
    value = world * flops / (ms * 1e-3) / 1e12
    # the per-kernel breakdown (and the roofline's kernel durations): the same steps again,
    # each launch bracketed by the library's own events on the launching stream
    rb.rope_attn_timing_read()
    rb.rope_attn_timing_enable(True)
    barrier()
    with clk.window():
        for _ in range(args.steps):
            step(dv_in, out0)
        barrier()
    rb.rope_attn_timing_enable(False)
    # clocks: the samples taken inside the two timed passes of the same steps
    clk.stop()
    clocks = clk.summary()
    kernels = rb.rope_attn_timing_read()
    launches = sum(c for c, _ in kernels.values())

    # ---------------- end-to-end through host buffers (copies inside the timed region):
    # every step's inputs go host -> device from pinned memory, and every result of the
    # step (O, lse, L, the gradients dQ, dK, dV, and dalpha) comes back device -> host.
    # Steps are pipelined the way a training loop feeds a GPU: step k+1's inputs go up on
    # one copy stream and step k-1's results come down on another while step k computes
    # (both PCIe directions at once), with two device buffer sets; every copy of every
    # timed step lies inside the timed region.
    h2d = sum(host[x].numel() * host[x].element_size() for x in host)
    res_names = ("o", "lse", "L", "dq", "dk", "dv", "dalpha")
    din = [{x: torch.empty_like(dv_in[x]) for x in host} for _ in range(2)]
    dout = [out0, outputs()]
    back = [{x: torch.empty(out0[x].shape, dtype=out0[x].dtype).pin_memory() for x in res_names}
            for _ in range(2)]
    d2h = sum(t.numel() * t.element_size() for t in back[0].values())
    # the same K steps as the headline; the pipeline's fill (the first upload) and drain
    # (the last step's compute and download) fall inside the timed region, once per run
    e2e_steps = max(3, args.steps)
    s_up, s_down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()
    comp_done = [ev(), ev()]   # step on buffer set b finished (its inputs and outputs free)
    up_done = [ev(), ev()]     # inputs of buffer set b on the device
    down_done = [ev(), ev()]   # results of buffer set b back on the host
    started = [False, False]

    def e2e_run(nsteps):
        # the copy streams start no earlier than what the compute stream has reached
        start = ev()
        start.record(stream)
        s_up.wait_event(start)
        s_down.wait_event(start)
        for k in range(nsteps):
            b = k % 2
            with torch.cuda.stream(s_up):
                if started[b]:
                    s_up.wait_event(comp_done[b])
                for x in host:
                    din[b][x].copy_(host[x], non_blocking=True)
                up_done[b].record(s_up)
            stream.wait_event(up_done[b])
            if started[b]:
                stream.wait_event(down_done[b])
            step(din[b], dout[b])
            comp_done[b].record(stream)
            with torch.cuda.stream(s_down):
                s_down.wait_event(comp_done[b])
                for x in res_names:
                    back[b][x].copy_(dout[b][x], non_blocking=True)
                down_done[b].record(s_down)
            started[b] = True
        # the timed region ends when the last results are on the host
        for b in range(2):
            if started[b]:
                stream.wait_event(down_done[b])

    e2e_run(2)
    barrier()
    ev0.record(stream)
    e2e_run(e2e_steps)
    ev1.record(stream)
    barrier()
    e2e_ms = max_over_ranks(ev0.elapsed_time(ev1) / e2e_steps)
    e2e_value = world * flops / (e2e_ms * 1e-3) / 1e12

    if world > 1:
        dist.barrier()
    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return 0

    # ---------------- roofline of the dominant kernel
    peaks, peak_kind = load_peaks()
    f = 0.5 if wl.causal else 1.0
    # algorithmic FLOPs per (batch, head) in units of n^2 d (halved when causal)
    alg = {"fwd_sm100": 4.0, "bwd_dkdv_sm100": 8.0, "bwd_dq_sm100": 2.0}
    per_kernel = {name: {"launches": c, "avg_ms": t / c, "share": t / sum(
        tt for _, tt in kernels.values())} for name, (c, t) in kernels.items()}
    dom = max(kernels, key=lambda k: kernels[k][1])
    dom_avg_s = kernels[dom][1] / kernels[dom][0] * 1e-3
    roof = None
    if dom in alg:
        alg_flops = alg[dom] * wl.B * wl.H * wl.n * wl.n * wl.d * f
        achieved = alg_flops / dom_avg_s / 1e12
        peak = peaks.get("bf16_tflops", FALLBACK["bf16_tflops"])
        roof = {"kernel": dom, "bound": "tensor", "achieved": achieved, "peak": peak,
                "unit": "TFLOP/s", "frac": achieved / peak,
                "peak_source": f"{peak_kind} bf16 burst", "traffic": traffic_for(dom)}
        for name in kernels:
            if name in alg:
                a = alg[name] * wl.B * wl.H * wl.n * wl.n * wl.d * f
                per_kernel[name]["alg_tflops"] = a / (per_kernel[name]["avg_ms"] * 1e-3) / 1e12

    # ---------------- CPU oracle baseline (rank 0, N = 1 only)
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        v, dt, sample, threads = time_oracle(wl)
        cpu = {"value": v, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
               "sample": sample + f" ({dt:.1f} s)"}

    line = {
        "metric": "RoPE-attn fwd+bwd TFLOP/s (bf16, incl. dalpha)",
        "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": config_dict(wl, args.config, world),
        "fwd_tflops_per_gpu": phase_tflops(kernels, FWD_KERNELS, flops_fwd, args.steps),
        "bwd_tflops_per_gpu": phase_tflops(kernels, BWD_KERNELS, flops_bwd, args.steps),
        "pct_of_nominal_bf16_peak": 100 * value / world / NOMINAL_BF16_TFLOPS,
        "pct_of_measured_bf16_peak": 100 * value / world / peaks.get(
            "bf16_tflops", FALLBACK["bf16_tflops"]),
        "roofline": roof,
        "kernels": per_kernel,
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "gpu_launches": launches,
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


# Kernels of each phase (the step's backward takes the table and rotated Q~, K~ from the
# forward, so those run in the forward only).
FWD_KERNELS = {"rope_table": 1.0, "rotate": 1.0, "fwd_sm100": 1.0}
BWD_KERNELS = {"bwd_delta": 1.0, "bwd_dkdv_sm100": 1.0, "bwd_dq_sm100": 1.0,
               "dalpha_final": 1.0}


def phase_tflops(kernels, share, flops, steps):
    ms = sum(w * kernels[k][1] for k, w in share.items() if k in kernels) / steps
    return flops / (ms * 1e-3) / 1e12 if ms > 0 else None


def traffic_for(kernel):
    """DRAM bytes per launch from the committed ncu summary, if the kernel's code (the whole
    file, or the span of it the record names; comments aside) is the one the counters were
    taken on."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f).get(kernel)
    if not rec:
        return None
    src = os.path.join(ROOT, "rope_attention_fwd_b200", "csrc", rec["source"])
    if not os.path.exists(src):
        return None
    text = open(src, encoding="utf-8").read()
    # a record may cover only the kernel's own part of a file that holds several kernels
    if "span_start" in rec:
        if rec["span_start"] not in text:
            return None
        text = text[text.index(rec["span_start"]):]
    if "span_end" in rec:
        if rec["span_end"] not in text:
            return None
        text = text[:text.index(rec["span_end"])]
    sha = hashlib.sha256(code_only(text).encode("utf-8")).hexdigest()
    return rec["bytes_per_launch"] if sha == rec["source_sha256"] else None


def code_only(text):
    """The source without // comments and blank lines: what the counters depend on."""
    import re
    lines = (re.sub(r"//.*$", "", line).rstrip() for line in text.split("\n"))
    return "\n".join(line for line in lines if line)


# ----------------------------------------------------------------- profile mode
def run_profile(args):
    """Whole fwd -> loss -> bwd steps on one problem of any shape, for profilers (ncu wraps
    this): inputs N(0,1) bf16 drawn on the device (the launch sequence matters here, not
    parity), alpha ~ N(0, 0.3^2).  Prints each kernel's average event time over the timed
    steps.  With --d-model > 0 each step also runs the projections around the path
    (q, k, v = x W before; dW and dx after) and prints their times and TFLOP/s."""
    import torch
    from rope_attention_fwd_b200 import binding as rb
    B, H, n, d = args.shape
    g = torch.Generator(device="cuda").manual_seed(0)
    shape = (B, H, n, d)
    q, k, v, e = (torch.randn(shape, device="cuda", generator=g).to(torch.bfloat16)
                  for _ in range(4))
    alpha = 0.3 * torch.randn(d // 2, device="cuda", generator=g)
    ws = rb.workspace(rb.problem(B, H, n, d, torch.bfloat16, args.causal, args.base), "cuda")
    if args.d_model > 0:
        x = torch.randn((B, n, args.d_model), device="cuda", generator=g).to(torch.bfloat16)
        w = [(torch.randn((args.d_model, H * d), device="cuda", generator=g)
              * args.d_model ** -0.5).to(torch.bfloat16) for _ in range(3)]

    def step():
        qq, kk, vv = (q, k, v) if args.d_model <= 0 else rb.rope_attn_proj_fwd(x, *w, H)
        o, lse = rb.rope_attn_fwd(qq, kk, vv, alpha, args.base, args.causal, ws=ws)
        L, dO = rb.rope_attn_loss(o, e, ws=ws)
        grads = rb.rope_attn_bwd_saved(vv, o, lse, dO, alpha, args.base, args.causal, ws)
        if args.d_model > 0:
            rb.rope_attn_proj_bwd(x, *w, *grads[:3])
        return grads

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    rb.rope_attn_timing_read()
    rb.rope_attn_timing_enable(True)
    for _ in range(args.steps):
        step()
    torch.cuda.synchronize()
    rb.rope_attn_timing_enable(False)
    f = 0.5 if args.causal else 1.0
    alg = {"fwd_sm100": 4.0, "bwd_dkdv_sm100": 8.0, "bwd_dq_sm100": 2.0}
    kernels = rb.rope_attn_timing_read()
    prod = 2.0 * B * n * max(args.d_model, 0) * H * d  # FLOPs of one x W product
    for name, (cnt, ms) in kernels.items():
        line = f"{name:16s} {cnt:3d} launches {ms / cnt:8.3f} ms"
        if name in alg:
            tf = alg[name] * B * H * n * n * d * f / (ms / cnt * 1e-3) / 1e12
            line += f"  {tf:7.1f} TFLOP/s algorithmic"
        elif name in ("proj_gemm", "proj_dw_gemm", "proj_dx_gemm"):
            line += f"  {3 * prod / (ms / cnt * 1e-3) / 1e12:7.1f} TFLOP/s"
        print(line)
    if args.d_model > 0:
        parts = {"proj_fwd": ("proj_gemm",),
                 "proj_bwd": ("merge_heads", "proj_dw_gemm", "proj_dx_gemm")}
        for name, nprod in (("proj_fwd", 3), ("proj_bwd", 6)):
            ms = sum(kernels.get(kn, (0, 0.0))[1] for kn in parts[name]) / args.steps
            print(f"{name:16s}   1 launches {ms:8.3f} ms  "
                  f"{nprod * prod / (ms * 1e-3) / 1e12:7.1f} TFLOP/s")
    code, info = rb.rope_attn_device_status(ws)
    if code != 0:
        raise SystemExit(f"device status {rb.STATUS.get(code, code)} {info}")
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", type=int, default=3, choices=[2, 3, 4, 5])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile", action="store_true",
                    help="time the kernels of whole steps on --shape (for profilers); no "
                         "JSON line")
    ap.add_argument("--shape", type=lambda t: tuple(int(x) for x in t.split(",")),
                    default=(2, 16, 8192, 128), help="B,H,n,d of --profile")
    ap.add_argument("--causal", action="store_true", help="causal masking in --profile")
    ap.add_argument("--base", type=float, default=1e4, help="RoPE base in --profile")
    ap.add_argument("--d-model", type=int, default=0,
                    help="--profile: also run the projections with this model width")
    args = ap.parse_args()
    if args.profile:
        return run_profile(args)
    if args.warmup < 3 and args.impl == "ours":
        raise SystemExit("--warmup must be at least 3")
    # the reference arm times a slow CPU program: bound its work per step
    args.steps_ref = max(1, min(args.steps, 3))
    args.warmup_ref = 0
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
