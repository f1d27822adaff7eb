"""Benchmark of the PAB attention stack on B200.

One benchmark step = one whole Pyramid Attention Broadcast sampling run of
the attention stack of a video DiT block over the workload's diffusion steps:
for every step i, spatial attention, temporal attention (layout change of
q, k, v to the temporal view, attention, layout change of the output back)
and cross attention under the PAB schedule (computes on the edge steps and at
the start of every broadcast window, cache hits elsewhere), plus the
attention-difference MSE between each kind's consecutive computed outputs.

Printed (rank 0, one JSON line): dense-equivalent attention TFLOP/s (all
steps' attention flops / run time), executed TFLOP/s, denoising steps/s, the
roofline of the dominant kernel, a CPU baseline (the fp64 oracle on a
bounded sample, on this host's cores) and an end-to-end figure with
host<->device copies inside the timed region.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 480p]
    python bench.py --impl reference ...   # the fp64 oracle arm (CPU)
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402
import torch.distributed as dist  # noqa: E402

import synth  # noqa: E402

METRIC = "attention TFLOP/s & steps/s per DiT attn stack; % of bf16 TC / HBM roofline"
UNIT = "TFLOP/s (dense-equivalent attention)"

# Per-launch DRAM bytes (read + write) measured by ncu for the dominant kernel,
# keyed by (sha256 of the kernel's source, workload); a different source hash
# or a workload without a capture means traffic is null.
MEASURED_TRAFFIC = {
    # flash_tc spatial, one launch of `bench.py --kernel spatial --workload W`
    # (the second of two, as the stack runs it): dram read + write
    ("41c9b98a09ea40c4", "480p"): 176119552 + 38109440,
    ("41c9b98a09ea40c4", "temporal_heavy"): 471980032 + 135882240,
    ("41c9b98a09ea40c4", "720p"): 1603916000 + 512133376,
    # flash_tc sliding tile attention / region-sparse (draft) attention, the
    # second launch of `bench.py --sta` / `bench.py --draft`
    ("41c9b98a09ea40c4", "sta_48x80"): 1719353856 + 545471744,
    ("41c9b98a09ea40c4", "draft_48x80"): 1690944000 + 543200000,
}


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default="480p", choices=("480p", "720p", "temporal_heavy", "tiny", "sta_48x80", "draft_48x80"))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--input-sets", type=int, default=8,
                    help="distinct drifted input sets cycled over the diffusion steps")
    ap.add_argument("--cpu-sample-s", type=float, default=15.0,
                    help="target seconds of oracle work for the CPU baseline sample")
    ap.add_argument("--sta", action="store_true",
                    help="sliding tile attention as the spatial kind (workload sta_48x80 unless "
                         "--workload names another with a spatial window): the kernel against full "
                         "spatial attention, and the PAB stack with each")
    ap.add_argument("--draft", action="store_true",
                    help="draft attention as the spatial kind (workload draft_48x80): pooled sketch and "
                         "selection, region-sparse attention against full spatial attention, and the PAB "
                         "stack with each")
    ap.add_argument("--dsp", action="store_true",
                    help="broadcast sequence parallel: one video's frames sharded over the ranks, two "
                         "all-to-all exchanges per temporal compute (none on broadcast steps); the PAB "
                         "ranges against ranges (1, 1, 1)")
    ap.add_argument("--sweep", action="store_true",
                    help="the 50-step sweep (480p shapes): every range set of the sweep workload timed, "
                         "with the per-step attention difference (MSE) of the all-compute run")
    ap.add_argument("--kernel", choices=("spatial", "temporal", "temporal_sv", "cross", "layout", "mse",
                                         "gemm_qkv", "gemm_mlp_in", "gemm_mlp_out"),
                    help="time one kernel alone on the workload's tensors (one input set, back-to-back "
                         "launches): the single-kernel view used for profiling")
    ap.add_argument("--dit", action="store_true",
                    help="time the synthetic DiT block (projections, norms, MLP around the library's "
                         "attention) with the workload's PAB ranges and with ranges (1, 1, 1)")
    return ap.parse_args(argv)


# ----------------------------------------------------------------- distributed
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def dist_init(world, backend):
    if world > 1 and not dist.is_initialized():
        import datetime
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))


def max_over_ranks(x: float, device) -> float:
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        t = torch.tensor([x], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())
    return x


def barrier(device):
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        if device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ----------------------------------------------------------------- work model
def schedule_counts(w, edge_pct=15):
    """Computes per kind under the PAB schedule (closed form of the plan's rule)."""
    e = -(-edge_pct * w.steps // 100)
    M = max(w.steps - 2 * e, 0)
    return {kind: (w.steps - M) + (-(-M // r)) for kind, r in zip(synth.KINDS, w.ranges)}


def algorithmic_bytes(w):
    v = w.T * w.N * w.C * 2  # one bf16 video tensor
    text = w.text_len * w.C * 2
    return {"spatial": 4 * v, "temporal": 4 * v, "cross": 2 * v + 2 * text,
            "layout": 2 * v, "mse": 2 * v}


def workload_config(w) -> dict:
    """The workload part of the JSON line's config, shared by both arms."""
    return {"workload": w.name, "T": w.T, "H": w.H, "W": w.W, "heads": w.heads, "d": w.d,
            "text_len": w.text_len, "diffusion_steps": w.steps, "ranges": list(w.ranges),
            "step": "one PAB sampling run of the spatial+temporal+cross attention stack"}


def kernel_source_hash(name: str) -> str:
    path = os.path.join(ROOT, "step_reuse_b200", "csrc", name)
    try:
        return hashlib.sha256(open(path, "rb").read()).hexdigest()[:16]
    except OSError:
        return ""


# ----------------------------------------------------------------- peaks
def load_peaks():
    """Roofline denominators: MEASURED_PEAKS.json when present, else the
    pool's earlier measurement (6.65 TB/s copy, 1.59 PFLOP/s bf16 burst)."""
    try:
        peaks = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
        src = "measured"
    except (OSError, ValueError):
        peaks, src = {}, "fallback"
    return {"tc": peaks.get("bf16_tflops", 1590.0), "tc_sustained": peaks.get("bf16_tflops_sustained", 1400.0),
            "hbm": peaks.get("hbm_gbs", 6650.0), "src": src}


def tc_roofline(kernel, achieved, peaks, clk, **extra):
    """Tensor roofline of a kernel timed inside sub-second sampling runs: the
    fraction is taken against the BURST bf16 GEMM peak (the kernels run at or
    near the maximum SM clock there; the sustained figure is a seconds-long
    GEMM loop under the power cap) and the sustained fraction is given beside
    it with the median SM clock of the timed region."""
    d = {"kernel": kernel, "bound": "tensor", "achieved": achieved, "peak": peaks["tc"], "unit": "TFLOP/s",
         "frac": achieved / peaks["tc"], "peak_source": f"{peaks['src']} bf16_tflops (burst)",
         "frac_of_sustained": achieved / peaks["tc_sustained"],
         "sm_mhz_median": (clk or {}).get("sm_mhz")}
    d.update(extra)
    return d


# ----------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled during the timed region."""

    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self._t = None
        self.t_start = self.t_end = None

    def mark_start(self):
        self.t_start = time.time()

    def mark_end(self):
        self.t_end = time.time()

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
            return
        self._t = threading.Thread(target=self._read, daemon=True)
        self._t.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self._t:
            self._t.join(timeout=2)
        sm, mx, reasons = [], None, set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        lo = (self.t_start or 0.0) - 0.05
        hi = (self.t_end or 1e30) + 0.25  # a sample is printed up to one period late
        for ts, ln in self.lines:
            if not (lo <= ts <= hi):
                continue
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------- the stack
class AttentionStack:
    """One PAB sampling run of the three attention kinds through libpab.

    fused=False: temporal attention as the three layouts + temporal-view
    kernel + layout back (every step of the hot path runs);
    fused=True: the temporal kernel reads and writes the spatial view itself
    (pab_plan_set_temporal_view), no layout launches.
    Every compute of a kind after its first is followed by one MSE launch
    against the kind's previous output (the attention-difference diagnostic).
    mse_side (default): those launches run on a side stream once the compute is
    done (an event), where the HBM-bound reduction overlaps the next
    attention kernels; the kind's next compute waits for its MSE (it
    overwrites the slot the MSE reads) and the run ends by joining the side
    stream."""

    def __init__(self, pab, w, device, fused=False, window=(), draft=(), mse_side=True):
        self.pab, self.w, self.dev, self.fused = pab, w, device, fused
        self.side = torch.cuda.Stream(device) if mse_side else None
        self.plan = pab.Plan(w.T, w.H, w.W, w.heads, w.d, w.text_len, w.steps, w.ranges,
                             dtype=torch.bfloat16)
        if fused:
            self.plan.set_temporal_view(True)
        if window:
            self.plan.set_spatial_window(*window)
        if draft:
            self.plan.set_spatial_draft(*draft)
        self.plan.prepare()
        T, N, C = w.T, w.N, w.C
        # temporal-view scratch and the spatial-view copy of the temporal output
        self.tq = torch.empty((N, T, C), dtype=torch.bfloat16, device=device)
        self.tk = torch.empty_like(self.tq)
        self.tv = torch.empty_like(self.tq)
        self.tout = [torch.empty((T, N, C), dtype=torch.bfloat16, device=device) for _ in range(2)]
        self.tslot = 0
        self.mse = torch.zeros((3, w.steps), dtype=torch.float64, device=device)
        self.last_ptr = {}
        self.sched = {k: [self.plan.is_compute(k, i) for i in range(w.steps)] for k in synth.KINDS}
        self.launches_per_run = self._count_launches()

    def _count_launches(self):
        n = 0
        first = {k: True for k in synth.KINDS}
        for i in range(self.w.steps):
            for k in synth.KINDS:
                if self.sched[k][i]:
                    n += 1 if (k != "temporal" or self.fused) else 5  # 3 layouts + attention + layout back
                    if not first[k]:
                        n += 1  # MSE: one launch
                    first[k] = False
        return n

    def run(self, inputs, stream, events=None, only=None):
        """inputs[i][kind] -> dict q,k,v (spatial view for temporal).  With
        `events` (name -> ([starts], [ends])), every launch (of the kernels
        named in `only`, when given) is bracketed by CUDA events on the stream
        it runs on, grouped by kernel.  An event between two launches adds a
        gap of a few microseconds, so runs that set the headline time bracket
        only the dominant kernel."""
        pab, w, plan = self.pab, self.w, self.plan
        plan.reset()
        prev = {}
        T, N, C = w.T, w.N, w.C

        side = self.side
        pending = {}  # kind -> event behind its latest side-stream MSE

        def timed(name, fn, on=stream):
            if events is None or (only is not None and name not in only):
                return fn()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(on)
            r = fn()
            b.record(on)
            events.setdefault(name, ([], []))
            events[name][0].append(a)
            events[name][1].append(b)
            return r

        for i in range(w.steps):
            x = inputs[i % len(inputs)]
            for ki, k in enumerate(synth.KINDS):
                if not self.sched[k][i]:
                    self.last_ptr[k] = plan.attention_ptr(k, i, None, None, None, stream)
                    continue
                if k in pending:  # this compute overwrites what the kind's last MSE reads
                    stream.wait_event(pending.pop(k))
                if k == "temporal" and self.fused:
                    ptr = timed("temporal", lambda: plan.attention_ptr(k, i, x[k]["q"], x[k]["k"], x[k]["v"],
                                                                       stream))
                    self.last_ptr[k] = ptr
                    cur = pab._wrap(ptr, (T, N, C), torch.bfloat16, self.dev)
                elif k == "temporal":
                    for src, dst in ((x[k]["q"], self.tq), (x[k]["k"], self.tk), (x[k]["v"], self.tv)):
                        timed("layout", lambda: pab.layout(src, True, out=dst, stream=stream))
                    ptr = timed("temporal", lambda: plan.attention_ptr(k, i, self.tq, self.tk, self.tv, stream))
                    self.last_ptr[k] = ptr
                    t_out = pab._wrap(ptr, (N, T, C), torch.bfloat16, self.dev)
                    self.tslot ^= 1
                    timed("layout", lambda: pab.layout(t_out, False, out=self.tout[self.tslot], stream=stream))
                    cur = self.tout[self.tslot]
                else:
                    ptr = timed(k, lambda: plan.attention_ptr(k, i, x[k]["q"], x[k]["k"], x[k]["v"], stream))
                    self.last_ptr[k] = ptr
                    shape = (T, N, C) if k == "spatial" else (T * N, C)
                    cur = pab._wrap(ptr, shape, torch.bfloat16, self.dev)
                if k in prev and side is None:
                    timed("mse", lambda: pab.attn_diff_mse_async(cur, prev[k], self.mse[ki, i:i + 1],
                                                                stream=stream))
                elif k in prev:
                    done = torch.cuda.Event()
                    done.record(stream)
                    side.wait_event(done)
                    timed("mse", lambda: pab.attn_diff_mse_async(cur, prev[k], self.mse[ki, i:i + 1],
                                                                stream=side), on=side)
                    pending[k] = torch.cuda.Event()
                    pending[k].record(side)
                prev[k] = cur
        if side is not None:
            stream.wait_stream(side)

    def close(self):
        self.plan.close()


def make_inputs(w, device, n_sets, seed=0):
    """n_sets drifted copies of every kind's q, k, v (temporal inputs in the
    spatial view; the stack changes their layout)."""
    base = synth.initial_inputs(w, device=device, seed=seed)
    tq = {n: base["temporal"][n].reshape(w.N, w.T, w.C).permute(1, 0, 2).contiguous()
          for n in ("q", "k", "v")}
    base["temporal"] = tq
    g = synth.generator(seed + 1, device)
    sets = [base]
    for _ in range(1, n_sets):
        nxt = {k: {n: t.clone() for n, t in v.items()} for k, v in sets[-1].items()}
        synth.drift_(nxt, w.sigma, g)
        sets.append(nxt)
    return sets


def mean_ms(pairs):
    starts, ends = pairs
    if not starts:
        return None
    return sum(s.elapsed_time(e) for s, e in zip(starts, ends)) / len(starts)


# ----------------------------------------------------------------- CPU baseline
def oracle_sample(w, seconds_target=15.0, seed=0):
    """Time the fp64 oracle on a bounded sample of one PAB run: a subset of
    spatial frames, of temporal positions and of cross rows of one computed
    step per kind, scaled to the whole run by unit counts."""
    import numpy as np

    import oracle
    oracle.build()
    rng = np.random.default_rng(seed)
    T, N, C, h, L = w.T, w.N, w.C, w.heads, w.text_len
    flops = w.flops()
    per_unit = {"spatial": flops["spatial"] / T, "temporal": flops["temporal"] / N,
                "cross": flops["cross"] / (T * N)}
    # spend the target time roughly 75/10/15 across the kinds
    rate_guess = 8e9 * max(1, oracle.num_threads()) / 8
    frames = max(1, min(T, int(0.75 * seconds_target * rate_guess / per_unit["spatial"])))
    positions = max(1, min(N, int(0.10 * seconds_target * rate_guess / per_unit["temporal"])))
    rows = max(1, min(T * N, int(0.15 * seconds_target * rate_guess / per_unit["cross"])))

    def bf(shape):
        return torch.randn(shape, generator=torch.Generator().manual_seed(int(rng.integers(1 << 30))))\
            .to(torch.bfloat16).to(torch.float64).numpy()

    t_unit = {}
    q, k, v = bf((frames, N, C)), bf((frames, N, C)), bf((frames, N, C))
    t0 = time.perf_counter()
    oracle.spatial_attention(q, k, v, h)
    t_unit["spatial"] = (time.perf_counter() - t0) / frames
    q, k, v = bf((positions, T, C)), bf((positions, T, C)), bf((positions, T, C))
    t0 = time.perf_counter()
    oracle.temporal_attention(q, k, v, h)
    t_unit["temporal"] = (time.perf_counter() - t0) / positions
    q, kt, vt = bf((rows, C)), bf((L, C)), bf((L, C))
    t0 = time.perf_counter()
    oracle.cross_attention(q, kt, vt, h)
    t_unit["cross"] = (time.perf_counter() - t0) / rows
    units = {"spatial": T, "temporal": N, "cross": T * N}
    counts = schedule_counts(w)
    run_s = sum(counts[k] * units[k] * t_unit[k] for k in synth.KINDS)
    dense = w.steps * sum(flops.values())
    return {
        "value": dense / run_s / 1e12,
        "run_s": run_s,
        "cores": oracle.num_threads(),
        "sample": (f"one computed step per kind on a subset: {frames}/{T} spatial frames, "
                   f"{positions}/{N} temporal positions, {rows}/{T * N} cross rows; "
                   f"run time extrapolated by unit counts over the PAB schedule "
                   f"({counts['spatial']}/{counts['temporal']}/{counts['cross']} computes)"),
    }


# ----------------------------------------------------------------- arms
def run_reference(args):
    world, rank, _ = dist_env()
    if world > 1 and rank != 0:
        return 0
    w = synth.WORKLOADS[args.workload]
    per_step = max(1.0, 60.0 / max(1, args.steps + args.warmup))
    vals = []
    info = None
    for s in range(args.warmup + args.steps):
        info = oracle_sample(w, seconds_target=per_step, seed=s)
        if s >= args.warmup:
            vals.append(info)
    value = statistics.median(v["value"] for v in vals)
    run_s = statistics.median(v["run_s"] for v in vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": run_s * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(w),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": info["cores"], "kind": "oracle",
                         "sample": info["sample"]},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_ours(args):
    world, rank, local = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (no CPU fallback)")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist_init(world, "nccl")
    import step_reuse_b200 as pab

    w = synth.WORKLOADS[args.workload]
    flops = w.flops()
    counts = schedule_counts(w)
    dense_flops = w.steps * sum(flops.values())
    exec_flops = sum(counts[k] * flops[k] for k in synth.KINDS)
    abytes = algorithmic_bytes(w)

    n_sets = max(1, min(w.steps, args.input_sets))
    inputs = make_inputs(w, device, n_sets, seed=rank)
    # the headline stack: temporal attention reads and writes the spatial view
    # (each position's frames gathered with TMA); one MSE launch per compute
    # after a kind's first
    stack = AttentionStack(pab, w, device, fused=True)
    stream = torch.cuda.current_stream(device)

    for _ in range(args.warmup):
        stack.run(inputs, stream)
    torch.cuda.synchronize(device)
    assert pab.device_errors() == 0

    events = {}
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.5)  # let the sampler start before the timed region
    barrier(device)
    torch.cuda.synchronize(device)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    clocks.mark_start()
    t0.record(stream)
    for _ in range(args.steps):
        stack.run(inputs, stream, events, only=("spatial",))
    t1.record(stream)
    torch.cuda.synchronize(device)
    clocks.mark_end()
    barrier(device)
    clk = clocks.stop()
    ms = t0.elapsed_time(t1) / args.steps
    ms = max_over_ranks(ms, device)
    assert pab.device_errors() == 0

    peaks = load_peaks()
    tc_peak, hbm_peak = peaks["tc"], peaks["hbm"]
    # the other kernels' times: a few more runs with every launch bracketed
    # (outside the timed region; the spatial figure is the timed region's)
    bruns = 3
    bevents = {}
    for _ in range(bruns):
        stack.run(inputs, stream, bevents)
    torch.cuda.synchronize(device)
    kms = {name: mean_ms(ev) for name, ev in bevents.items()}
    kms["spatial"] = mean_ms(events["spatial"])
    kernels = {}
    for name in ("spatial", "cross", "temporal", "layout", "mse"):
        t = kms.get(name)
        if not t:
            continue
        fl = flops.get(name, 0.0) if name != "layout" and name != "mse" else 0.0
        by = abytes[name]
        ent = {"ms": t, "launches_per_run": len(bevents[name][0]) // bruns,
               "gbs": by / (t * 1e-3) / 1e9, "frac_hbm": by / (t * 1e-3) / 1e9 / hbm_peak,
               "bytes_per_launch": by}
        if fl:
            ent["tflops"] = fl / (t * 1e-3) / 1e12
            ent["frac_tc"] = ent["tflops"] / tc_peak
        kernels[name] = ent
    sp_ms = kms["spatial"]
    achieved = flops["spatial"] / (sp_ms * 1e-3) / 1e12
    src_hash = kernel_source_hash("flash_tc.cu")
    traffic = MEASURED_TRAFFIC.get((src_hash, args.workload))
    roofline = tc_roofline("spatial flash attention (flash_tc)", achieved, peaks, clk, traffic=traffic,
                           algorithmic_flops_per_launch=flops["spatial"],
                           algorithmic_bytes_per_launch=abytes["spatial"])

    value = world * dense_flops / (ms * 1e-3) / 1e12
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(workload_config(w),
                       l2=f"inputs larger than L2 ({n_sets} drifted input sets of "
                          f"{7 * w.T * w.N * w.C * 2 / 1e6:.0f} MB each, cycled)",
                       parallelism=f"replicas x{world} (one video per GPU)",
                       temporal_view="spatial view: the temporal kernel gathers each position's frames with "
                                     "TMA (the stack with explicit layout launches is reported beside)",
                       mse="attention-difference MSE of every compute after a kind's first, one launch each "
                           "on a side stream (overlapping the next attention kernels)",
                       kernel_times="spatial: CUDA events around its launches in the timed region; the "
                                    "other kernels: three more runs with every launch bracketed; all of them "
                                    "with the side-stream MSE launches overlapping"),
        "denoising_steps_per_s": world * w.steps / (ms * 1e-3),
        "executed_tflops": world * exec_flops / (ms * 1e-3) / 1e12,
        "computes": counts,
        "gpu_launches": stack.launches_per_run * args.steps,
        "roofline": roofline,
        "kernels": kernels,
        "clocks": clk,
    }

    # the same stack with every step computing (ranges 1, 1, 1): the speedup
    # the broadcast buys on this workload
    nstack = AttentionStack(pab, dataclasses.replace(w, ranges=(1, 1, 1)), device, fused=True)
    nstack.run(inputs, stream)
    nsteps = max(3, args.steps // 10)
    barrier(device)
    torch.cuda.synchronize(device)
    n0 = torch.cuda.Event(enable_timing=True)
    n1 = torch.cuda.Event(enable_timing=True)
    n0.record(stream)
    for _ in range(nsteps):
        nstack.run(inputs, stream)
    n1.record(stream)
    torch.cuda.synchronize(device)
    nms = max_over_ranks(n0.elapsed_time(n1) / nsteps, device)
    line["no_broadcast"] = {"ms_per_step": nms, "steps": nsteps,
                            "denoising_steps_per_s": world * w.steps / (nms * 1e-3),
                            "gpu_launches": nstack.launches_per_run * nsteps, "ranges": [1, 1, 1]}
    line["speedup_vs_no_broadcast"] = nms / ms
    nstack.close()

    # the same stack with explicit layout changes around temporal attention
    # (q, k, v to the temporal view, the output back): reported beside the
    # main figure, and the layout kernel's own timing comes from it
    lstack = AttentionStack(pab, w, device, fused=False)
    for _ in range(args.warmup):
        lstack.run(inputs, stream)
    lsteps = max(3, args.steps // 4)
    barrier(device)
    torch.cuda.synchronize(device)
    f0 = torch.cuda.Event(enable_timing=True)
    f1 = torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    for _ in range(lsteps):
        lstack.run(inputs, stream)
    f1.record(stream)
    torch.cuda.synchronize(device)
    lms = max_over_ranks(f0.elapsed_time(f1) / lsteps, device)
    levents = {}
    lstack.run(inputs, stream, levents, only=("layout",))
    torch.cuda.synchronize(device)
    lay = mean_ms(levents["layout"])
    kernels["layout"] = {"ms": lay, "launches_per_run": len(levents["layout"][0]),
                         "gbs": abytes["layout"] / (lay * 1e-3) / 1e9,
                         "frac_hbm": abytes["layout"] / (lay * 1e-3) / 1e9 / hbm_peak}
    line["layout_path"] = {
        "value": world * dense_flops / (lms * 1e-3) / 1e12, "unit": UNIT, "ms_per_step": lms, "steps": lsteps,
        "denoising_steps_per_s": world * w.steps / (lms * 1e-3),
        "gpu_launches": lstack.launches_per_run * lsteps,
        "note": "temporal attention on the temporal view, three layout launches before it and one after"}
    lstack.close()

    if not args.no_e2e:
        line["e2e"] = run_e2e(pab, w, stack, device, stream, args)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb = oracle_sample(w, seconds_target=args.cpu_sample_s)
        line["cpu_baseline"] = {"value": cb["value"], "unit": UNIT, "cores": cb["cores"],
                                "kind": "oracle", "sample": cb["sample"]}
    stack.close()
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist.is_initialized():
        dist.destroy_process_group()
    return 0


def run_e2e(pab, w, stack, device, stream, args):
    """Same metric through the public API with the inputs in pinned HOST
    memory: every computing kind's q, k, v is copied host->device for its
    call (on a copy stream, one step ahead of the compute), and the run's
    result (the last step's three attention outputs and the MSE series) is
    read back to the host, all inside the timed region."""
    host = {}
    for k in synth.KINDS:
        x = stack_inputs_shape(w, k)
        host[k] = {n: torch.randn(shp, dtype=torch.float32).to(torch.bfloat16).pin_memory()
                   for n, shp in x.items()}
    # two device input sets: the copy stream fills the set of step i + 1
    # while step i computes on the other
    dev_in = [{k: {n: torch.empty_like(t, device=device) for n, t in host[k].items()} for k in synth.KINDS}
              for _ in range(2)]
    copy_stream = torch.cuda.Stream(device)
    copied = [torch.cuda.Event(), torch.cuda.Event()]
    outs_host = {k: torch.empty(shp, dtype=torch.bfloat16).pin_memory()
                 for k, shp in (("spatial", (w.T, w.N, w.C)), ("temporal", (w.T, w.N, w.C)),
                                ("cross", (w.T * w.N, w.C)))}
    mse_host = torch.empty((3, w.steps), dtype=torch.float64).pin_memory()
    h2d = sum(stack.sched[k][i] * sum(t.numel() * 2 for t in host[k].values())
              for k in synth.KINDS for i in range(w.steps))
    d2h = sum(t.numel() * 2 for t in outs_host.values()) + mse_host.numel() * 8

    def copy_step(i, after):
        """Host -> device copies of the kinds computing at step i into input
        set i % 2, on the copy stream once `after` (the work enqueued before
        step i - 1 finished using that set) has completed."""
        copy_stream.wait_event(after)
        with torch.cuda.stream(copy_stream):
            for k in synth.KINDS:
                if stack.sched[k][i]:
                    for n in ("q", "k", "v"):
                        dev_in[i % 2][k][n].copy_(host[k][n], non_blocking=True)
        copied[i % 2].record(copy_stream)

    class HostFed:
        """inputs[i]: step i's input set, copied host->device (only the kinds
        computing at step i) while the previous step computed; the copy of
        step i + 1 is issued here too."""

        def __len__(self):
            return w.steps

        def __getitem__(self, i):
            enqueued = torch.cuda.Event()
            enqueued.record(stream)  # every step before i (step i - 1 used set (i + 1) % 2)
            if i == 0:
                copy_step(0, enqueued)
            stream.wait_event(copied[i % 2])
            if i + 1 < w.steps:
                copy_step(i + 1, enqueued)
            return dev_in[i % 2]

    fed = HostFed()

    def one():
        stack.run(fed, stream)
        # results of the run: last step's outputs + the MSE series
        sp = pab._wrap(stack.last_ptr["spatial"], (w.T, w.N, w.C), torch.bfloat16, device)
        cr = pab._wrap(stack.last_ptr["cross"], (w.T * w.N, w.C), torch.bfloat16, device)
        outs_host["spatial"].copy_(sp, non_blocking=True)
        tmp = (pab._wrap(stack.last_ptr["temporal"], (w.T, w.N, w.C), torch.bfloat16, device) if stack.fused
               else stack.tout[stack.tslot])
        outs_host["temporal"].copy_(tmp, non_blocking=True)
        outs_host["cross"].copy_(cr, non_blocking=True)
        mse_host.copy_(stack.mse, non_blocking=True)

    for _ in range(1):
        one()
    torch.cuda.synchronize(device)
    barrier(device)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(args.e2e_steps):
        one()
    b.record(stream)
    torch.cuda.synchronize(device)
    ms = max_over_ranks(a.elapsed_time(b) / args.e2e_steps, device)
    world = dist.get_world_size() if dist.is_initialized() else 1
    dense = w.steps * sum(w.flops().values())
    return {"value": world * dense / (ms * 1e-3) / 1e12, "unit": UNIT, "ms_per_step": ms,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "note": "inputs copied from pinned host memory for every computing kind at every step, on a "
                    "copy stream one step ahead of the compute"}


def stack_inputs_shape(w, kind):
    if kind == "cross":
        return {"q": (w.T * w.N, w.C), "k": (w.text_len, w.C), "v": (w.text_len, w.C)}
    return {"q": (w.T, w.N, w.C), "k": (w.T, w.N, w.C), "v": (w.T, w.N, w.C)}


def dit_flops(w, counts):
    """Algorithmic flops of one sampling run of the DiT block: per computing
    kind 4 C x C projections (cross: q and the output on the video tokens, k and
    v on the text) plus its attention; the MLP (C -> 4C -> C) at every step."""
    R, C, L = w.T * w.N, w.C, w.text_len
    att = w.flops()
    per = {"spatial": 2 * 4 * R * C * C + att["spatial"], "temporal": 2 * 4 * R * C * C + att["temporal"],
           "cross": 2 * 2 * R * C * C + 2 * 2 * L * C * C + att["cross"]}
    mlp = 2 * 2 * R * C * 4 * C
    return sum(counts[k] * per[k] for k in synth.KINDS) + w.steps * mlp


def run_dit(args):
    """The synthetic DiT block over whole sampling runs, PAB ranges against
    ranges (1, 1, 1) (every step computes), device-timed; one JSON line."""
    world, rank, local = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (no CPU fallback)")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist_init(world, "nccl")
    import step_reuse_b200 as pab
    from step_reuse_b200 import dit

    w = synth.WORKLOADS[args.workload]
    xs, text = synth.dit_inputs(w, device=device, seed=rank)
    wts = dit.make_weights(w.C, seed=rank + 1, device=device)
    stream = torch.cuda.current_stream(device)
    res = {}
    runs = max(1, args.steps // 10)
    for label, ranges in (("pab", w.ranges), ("no_broadcast", (1, 1, 1))):
        block = dit.DiTBlock(pab, w.T, w.H, w.W, w.heads, w.d, w.text_len, w.steps, ranges, wts, device)

        def one():
            block.reset()
            for i in range(w.steps):
                block.step(i, xs[i], text, stream)

        for _ in range(args.warmup):
            one()
        torch.cuda.synchronize(device)
        barrier(device)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(runs):
            one()
        b.record(stream)
        torch.cuda.synchronize(device)
        ms = max_over_ranks(a.elapsed_time(b) / runs, device)
        counts = {k: sum(block.plan.is_compute(k, i) for i in range(w.steps)) for k in synth.KINDS}
        tf = dit_flops(w, counts) / (ms * 1e-3) / 1e12
        res[label] = {"ms_per_run": ms, "computes": counts, "tflops": tf,
                      "frac_of_burst_bf16": tf / load_peaks()["tc"]}
        block.close()
    assert pab.device_errors() == 0
    if rank == 0:
        speedup = res["no_broadcast"]["ms_per_run"] / res["pab"]["ms_per_run"]
        line = {
            "metric": "synthetic DiT block: denoising steps/s with PAB broadcast",
            "value": world * w.steps / (res["pab"]["ms_per_run"] * 1e-3), "unit": "steps/s",
            "n_gpus": world, "runs": runs, "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
            "dtype": "bf16", "data": "synthetic (random weights, drifting N(0, 1) residual stream)",
            "config": dict(workload_config(w),
                           step="one sampling run of the DiT block (all diffusion steps)",
                           block="LN -> QKV -> attention -> out-proj per kind, "
                                 "LN -> MLP(4C, tanh GELU); fp32 residual"),
            "speedup_vs_no_broadcast": speedup, "pab": res["pab"], "no_broadcast": res["no_broadcast"],
        }
        print(json.dumps(line), flush=True)
    if dist.is_initialized():
        dist.destroy_process_group()
    return 0


def sta_pairs(w):
    """Query-key pairs per frame of sliding tile attention: every query of
    tile (ty, tx) meets the keys of the window's tiles, clipped at the edge."""
    tile, win_h, win_w = w.spatial_window
    th, tw = w.H // tile, w.W // tile
    rh, rw = (win_h // tile - 1) // 2, (win_w // tile - 1) // 2
    rows = [min(ty + rh + 1, th) - max(ty - rh, 0) for ty in range(th)]
    cols = [min(tx + rw + 1, tw) - max(tx - rw, 0) for tx in range(tw)]
    return (tile * tile) ** 2 * sum(rows) * sum(cols)


def run_sta(args):
    """Sliding tile attention as the spatial kind: the kernel alone against
    full spatial attention on the same tensors, then one PAB sampling run of
    the fused attention stack with each; device-timed; one JSON line."""
    world, rank, local = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (no CPU fallback)")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist_init(world, "nccl")
    import step_reuse_b200 as pab

    name = args.workload if synth.WORKLOADS[args.workload].spatial_window else "sta_48x80"
    w = synth.WORKLOADS[name]
    tile, win_h, win_w = w.spatial_window
    T, N, C = w.T, w.N, w.C
    sta_flops = 4.0 * T * w.heads * w.d * sta_pairs(w)
    full_flops = w.flops()["spatial"]
    n_sets = max(1, min(w.steps, args.input_sets))
    inputs = make_inputs(w, device, n_sets, seed=rank)
    stream = torch.cuda.current_stream(device)
    out = torch.empty((T, N, C), dtype=torch.bfloat16, device=device)
    launches = {
        "sta": lambda x: pab.sta_attention(x["q"], x["k"], x["v"], w.H, w.W, w.heads, tile, win_h, win_w,
                                           out=out, stream=stream),
        "full": lambda x: pab.spatial_attention(x["q"], x["k"], x["v"], w.heads, out=out, stream=stream),
    }
    reps = max(5, args.steps)
    kern = {}
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.5)
    clocks.mark_start()
    for label, fn in launches.items():
        for i in range(args.warmup):
            fn(inputs[i % n_sets]["spatial"])
        torch.cuda.synchronize(device)
        barrier(device)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for i in range(reps):
            fn(inputs[i % n_sets]["spatial"])
        b.record(stream)
        torch.cuda.synchronize(device)
        kern[label] = max_over_ranks(a.elapsed_time(b) / reps, device)
    assert pab.device_errors() == 0
    runs = max(3, args.steps // 10)
    stacks = {}
    for label, window in (("sta", w.spatial_window), ("full", ())):
        st = AttentionStack(pab, w, device, fused=True, window=window)
        for _ in range(args.warmup):
            st.run(inputs, stream)
        torch.cuda.synchronize(device)
        barrier(device)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(runs):
            st.run(inputs, stream)
        b.record(stream)
        torch.cuda.synchronize(device)
        stacks[label] = {"ms_per_run": max_over_ranks(a.elapsed_time(b) / runs, device),
                         "gpu_launches_per_run": st.launches_per_run}
        st.close()
    clocks.mark_end()
    clk = clocks.stop()
    assert pab.device_errors() == 0

    peaks = load_peaks()
    achieved = sta_flops / (kern["sta"] * 1e-3) / 1e12
    if rank == 0:
        line = {
            "metric": "sliding tile attention as the spatial kind: kernel TFLOP/s (window pairs) "
                      "and PAB stack steps/s",
            "value": world * sta_flops / (kern["sta"] * 1e-3) / 1e12, "unit": "TFLOP/s (algorithmic, window)",
            "n_gpus": world, "steps": reps, "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
            "dtype": "bf16", "data": "synthetic",
            "config": dict(workload_config(w), spatial_window={"tile": tile, "win_h": win_h, "win_w": win_w},
                           l2=f"inputs larger than L2 ({n_sets} input sets cycled)"),
            "roofline": tc_roofline("sliding tile attention (flash_tc, window geometry)", achieved, peaks, clk,
                                    traffic=MEASURED_TRAFFIC.get((kernel_source_hash("flash_tc.cu"), name)),
                                    algorithmic_flops_per_launch=sta_flops,
                                    algorithmic_bytes_per_launch=4 * T * N * C * 2),
            "kernel_ms": {"sta": kern["sta"], "full_spatial": kern["full"]},
            "window_share_of_full": sta_flops / full_flops,
            "kernel_speedup_vs_full": kern["full"] / kern["sta"],
            "full_spatial_tflops": full_flops / (kern["full"] * 1e-3) / 1e12,
            "stack": {k: dict(v, denoising_steps_per_s=world * w.steps / (v["ms_per_run"] * 1e-3))
                      for k, v in stacks.items()},
            "stack_speedup_vs_full": stacks["full"]["ms_per_run"] / stacks["sta"]["ms_per_run"],
            # timed launches: the two kernel loops, then `runs` runs of each stack
            "gpu_launches": 2 * reps + runs * sum(v["gpu_launches_per_run"] for v in stacks.values()),
            "clocks": clk,
        }
        print(json.dumps(line), flush=True)
    if dist.is_initialized():
        dist.destroy_process_group()
    return 0


def run_draft(args):
    """Draft attention as the spatial kind: the pooled-sketch selection and
    the region-sparse attention against full spatial attention on the same
    tensors, then one PAB sampling run of the fused stack with each;
    device-timed; one JSON line."""
    world, rank, local = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (no CPU fallback)")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist_init(world, "nccl")
    import step_reuse_b200 as pab

    name = args.workload if synth.WORKLOADS[args.workload].spatial_draft else "draft_48x80"
    w = synth.WORKLOADS[name]
    region, keep = w.spatial_draft
    T, N, C = w.T, w.N, w.C
    R = (w.H // region) * (w.W // region)
    sparse_flops = 4.0 * T * w.heads * w.d * R * keep * (region * region) ** 2
    full_flops = w.flops()["spatial"]
    pool_bytes = 2 * T * N * C * 2 + 2 * T * R * C * 4  # q, k read; the fp32 sketch written
    n_sets = max(1, min(w.steps, args.input_sets))
    inputs = make_inputs(w, device, n_sets, seed=rank)
    stream = torch.cuda.current_stream(device)
    out = torch.empty((T, N, C), dtype=torch.bfloat16, device=device)
    sel = torch.empty((T, w.heads, R, keep), dtype=torch.int32, device=device)
    ws = torch.empty(pab.draft_workspace_bytes(T, w.H, w.W, w.heads, w.d, region), dtype=torch.uint8,
                     device=device)
    launches = {
        "select": lambda x: pab.draft_select(x["q"], x["k"], w.H, w.W, w.heads, keep, region, sel=sel,
                                             workspace=ws, stream=stream),
        "sparse": lambda x: pab.region_sparse_attention(x["q"], x["k"], x["v"], w.H, w.W, w.heads, sel, region,
                                                        out=out, stream=stream),
        "full": lambda x: pab.spatial_attention(x["q"], x["k"], x["v"], w.heads, out=out, stream=stream),
    }
    reps = max(5, args.steps)
    kern = {}
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.5)
    clocks.mark_start()
    for label, fn in launches.items():
        for i in range(args.warmup):
            fn(inputs[i % n_sets]["spatial"])
        torch.cuda.synchronize(device)
        barrier(device)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for i in range(reps):
            fn(inputs[i % n_sets]["spatial"])
        b.record(stream)
        torch.cuda.synchronize(device)
        kern[label] = max_over_ranks(a.elapsed_time(b) / reps, device)
    assert pab.device_errors() == 0
    runs = max(3, args.steps // 10)
    stacks = {}
    for label, draft in (("draft", w.spatial_draft), ("full", ())):
        st = AttentionStack(pab, w, device, fused=True, draft=draft)
        for _ in range(args.warmup):
            st.run(inputs, stream)
        torch.cuda.synchronize(device)
        barrier(device)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(runs):
            st.run(inputs, stream)
        b.record(stream)
        torch.cuda.synchronize(device)
        extra = st.launches_per_run
        if draft:  # each spatial compute is three launches: pool, select, region-sparse attention
            extra += 2 * sum(st.sched["spatial"])
        stacks[label] = {"ms_per_run": max_over_ranks(a.elapsed_time(b) / runs, device),
                         "gpu_launches_per_run": extra}
        st.close()
    clocks.mark_end()
    clk = clocks.stop()
    assert pab.device_errors() == 0

    peaks = load_peaks()
    hbm_peak = peaks["hbm"]
    achieved = sparse_flops / (kern["sparse"] * 1e-3) / 1e12
    total_ms = kern["select"] + kern["sparse"]
    if rank == 0:
        line = {
            "metric": "draft attention as the spatial kind: region-sparse TFLOP/s (kept pairs) and PAB stack "
                      "steps/s",
            "value": world * sparse_flops / (total_ms * 1e-3) / 1e12,
            "unit": "TFLOP/s (algorithmic, kept regions; selection included)",
            "n_gpus": world, "steps": reps, "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
            "dtype": "bf16", "data": "synthetic",
            "config": dict(workload_config(w), spatial_draft={"region": region, "keep": keep, "regions": R},
                           l2=f"inputs larger than L2 ({n_sets} input sets cycled)"),
            "roofline": tc_roofline("region-sparse attention (flash_tc, list geometry)", achieved, peaks, clk,
                                    traffic=MEASURED_TRAFFIC.get((kernel_source_hash("flash_tc.cu"), name)),
                                    algorithmic_flops_per_launch=sparse_flops),
            "select_roofline": {"kernel": "draft pool + select", "bound": "hbm",
                                "achieved": pool_bytes / (kern["select"] * 1e-3) / 1e9, "peak": hbm_peak,
                                "unit": "GB/s", "frac": pool_bytes / (kern["select"] * 1e-3) / 1e9 / hbm_peak,
                                "algorithmic_bytes_per_launch": pool_bytes},
            "kernel_ms": {"select": kern["select"], "sparse": kern["sparse"], "full_spatial": kern["full"]},
            "kept_share_of_full": sparse_flops / full_flops,
            "speedup_vs_full": kern["full"] / total_ms,
            "full_spatial_tflops": full_flops / (kern["full"] * 1e-3) / 1e12,
            "stack": {k: dict(v, denoising_steps_per_s=world * w.steps / (v["ms_per_run"] * 1e-3))
                      for k, v in stacks.items()},
            "stack_speedup_vs_full": stacks["full"]["ms_per_run"] / stacks["draft"]["ms_per_run"],
            # timed launches: pool + select, region-sparse and full loops, then `runs` runs of each stack
            "gpu_launches": 4 * reps + runs * sum(v["gpu_launches_per_run"] for v in stacks.values()),
            "clocks": clk,
        }
        print(json.dumps(line), flush=True)
    if dist.is_initialized():
        dist.destroy_process_group()
    return 0


def run_sweep(args):
    """The sweep workload (480p shapes, 50 steps, inputs drifting 0.2 per
    step on the edge steps and 0.02 in the middle): one sampling run of the
    fused attention stack per range set, device-timed, and the attention
    difference of consecutive steps (MSE) of the all-compute run per kind,
    edges against the middle (the U shape of the PAB report's Fig. 1)."""
    world, rank, local = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (no CPU fallback)")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist_init(world, "nccl")
    import step_reuse_b200 as pab

    w = synth.WORKLOADS["sweep"]
    e = -(-15 * w.steps // 100)
    traj = make_inputs(w, device, 1, seed=rank)  # step 0, then one drift per step
    g = synth.generator(rank + 7, device)
    for i in range(1, w.steps):
        nxt = {k: {n: t.clone() for n, t in v.items()} for k, v in traj[-1].items()}
        synth.drift_(nxt, synth.sigma_at(w, i, e), g)
        traj.append(nxt)
    stream = torch.cuda.current_stream(device)
    runs = max(2, args.steps // 20)
    res, mse = {}, None
    for ranges in w.extra_ranges:
        st = AttentionStack(pab, dataclasses.replace(w, ranges=ranges), device, fused=True)
        for _ in range(max(1, args.warmup)):
            st.run(traj, stream)
        torch.cuda.synchronize(device)
        barrier(device)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(runs):
            st.run(traj, stream)
        b.record(stream)
        torch.cuda.synchronize(device)
        ms = max_over_ranks(a.elapsed_time(b) / runs, device)
        res[str(tuple(ranges))] = {"ms_per_run": ms, "denoising_steps_per_s": world * w.steps / (ms * 1e-3),
                                   "computes": {k: sum(st.sched[k]) for k in synth.KINDS}}
        if tuple(ranges) == (1, 1, 1):
            mse = st.mse.cpu().numpy()
        st.close()
    assert pab.device_errors() == 0
    if rank == 0:
        base = res[str((1, 1, 1))]["ms_per_run"]
        for v in res.values():
            v["speedup_vs_no_broadcast"] = base / v["ms_per_run"]
        u = {}
        for ki, k in enumerate(synth.KINDS):
            edge = [float(mse[ki, i]) for i in list(range(1, e)) + list(range(w.steps - e + 1, w.steps))]
            mid = [float(mse[ki, i]) for i in range(e + 1, w.steps - e)]
            u[k] = {"edge_mean": sum(edge) / len(edge), "middle_mean": sum(mid) / len(mid),
                    "edge_over_middle": (sum(edge) / len(edge)) / (sum(mid) / len(mid))}
        line = {
            "metric": "PAB sweep: denoising steps/s of the attention stack per broadcast range set "
                      "(value: ranges 2/4/6)",
            "value": res[str((2, 4, 6))]["denoising_steps_per_s"],
            "unit": "steps/s", "n_gpus": world, "runs": runs, "higher_is_better": True, "scaling": "weak",
            "dtype": "bf16", "data": "synthetic (drift 0.2 per edge step, 0.02 per middle step)",
            "config": dict(workload_config(w), ranges=[list(r) for r in w.extra_ranges],
                           step="one 50-step sampling run of the fused attention stack"),
            "per_range_set": res, "attention_difference_all_compute": u,
        }
        print(json.dumps(line), flush=True)
    if dist.is_initialized():
        dist.destroy_process_group()
    return 0


def run_dsp(args):
    """One video sharded over the ranks (strong scaling): a sampling run of
    the three attention kinds through DSPStack with the workload's ranges and
    with ranges (1, 1, 1); device-timed, max over ranks; one JSON line with
    the exchanges and bytes each rank sent."""
    world, rank, local = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (no CPU fallback)")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist_init(world, "nccl")
    import step_reuse_b200 as pab
    from step_reuse_b200 import dsp

    w = synth.WORKLOADS[args.workload]
    if w.T % world or w.N % world:
        raise SystemExit(f"{w.name}: T={w.T} and N={w.N} must divide by {world} ranks")
    Tl = w.T // world
    n_sets = max(1, min(w.steps, args.input_sets))
    full = make_inputs(w, device, n_sets, seed=0)  # the same video on every rank; each takes its frames
    fr = slice(rank * Tl, (rank + 1) * Tl)
    inputs = [{k: {n: (x[k][n] if k == "cross" and n != "q" else
                       x[k][n].view(w.T, w.N, w.C)[fr].contiguous() if k != "cross" else
                       x[k][n].view(w.T, w.N, w.C)[fr].reshape(Tl * w.N, w.C).contiguous())
                   for n in ("q", "k", "v")} for k in synth.KINDS} for x in full]
    del full
    stream = torch.cuda.current_stream(device)
    runs = max(2, args.steps // 10)
    res = {}
    for label, ranges in (("pab", w.ranges), ("no_broadcast", (1, 1, 1))):
        st = dsp.DSPStack(pab, w.T, w.H, w.W, w.heads, w.d, w.text_len, w.steps, ranges, device=device)

        def one():
            st.reset()
            for i in range(w.steps):
                x = inputs[i % n_sets]
                for k in synth.KINDS:
                    if st.is_compute(k, i) or k == "temporal":
                        st.attention(k, i, x[k]["q"], x[k]["k"], x[k]["v"], stream)

        for _ in range(args.warmup):
            one()
        torch.cuda.synchronize(device)
        barrier(device)
        ex0, by0 = st.exchanges, st.bytes_sent
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(runs):
            one()
        b.record(stream)
        torch.cuda.synchronize(device)
        ms = max_over_ranks(a.elapsed_time(b) / runs, device)
        res[label] = {"ms_per_run": ms, "denoising_steps_per_s": w.steps / (ms * 1e-3),
                      "exchanges_per_run": (st.exchanges - ex0) // runs,
                      "bytes_sent_per_run_per_rank": (st.bytes_sent - by0) // runs,
                      "temporal_computes": sum(st.is_compute("temporal", i) for i in range(w.steps))}
        st.close()
    assert pab.device_errors() == 0
    if rank == 0:
        ex_p, ex_n = res["pab"]["exchanges_per_run"], res["no_broadcast"]["exchanges_per_run"]
        line = {
            "metric": "broadcast sequence parallel: denoising steps/s of one video over the ranks",
            "value": res["pab"]["denoising_steps_per_s"], "unit": "steps/s", "n_gpus": world, "runs": runs,
            "warmup": args.warmup, "higher_is_better": True, "scaling": "strong", "dtype": "bf16",
            "data": "synthetic",
            "config": dict(workload_config(w), parallelism=f"sequence parallel x{world} (frames; positions "
                                                            f"for temporal attention)"),
            "pab": res["pab"], "no_broadcast": res["no_broadcast"],
            "exchange_reduction": 1.0 - ex_p / ex_n if ex_n else None,
            "speedup_vs_no_broadcast": res["no_broadcast"]["ms_per_run"] / res["pab"]["ms_per_run"],
        }
        print(json.dumps(line), flush=True)
    if dist.is_initialized():
        dist.destroy_process_group()
    return 0


def run_kernel(args):
    """One kernel alone: the workload's tensors for that kernel only (q, k, v
    and the output, or the layout / MSE operands), `warmup` untimed launches,
    then `steps` launches timed with CUDA events; one JSON line with the
    kernel's time and its roofline fraction."""
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (no CPU fallback)")
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    import step_reuse_b200 as pab

    w = synth.WORKLOADS[args.workload]
    T, N, C, L = w.T, w.N, w.C, w.text_len
    g = torch.Generator(device=device).manual_seed(0)
    rnd = lambda *shape: torch.randn(shape, generator=g, device=device).to(torch.bfloat16)
    flops, abytes = w.flops(), algorithmic_bytes(w)
    kind = args.kernel
    if kind == "spatial":
        q, k, v = rnd(T, N, C), rnd(T, N, C), rnd(T, N, C)
        out = torch.empty_like(q)
        fn = lambda: pab.spatial_attention(q, k, v, w.heads, out=out)
    elif kind in ("temporal", "temporal_sv"):
        q, k, v = rnd(T, N, C), rnd(T, N, C), rnd(T, N, C)  # either view holds T*N rows
        out = torch.empty_like(q)
        f = pab.temporal_attention_sv if kind == "temporal_sv" else pab.temporal_attention
        if kind == "temporal":
            q, k, v, out = (t.view(N, T, C) for t in (q, k, v, out))
        fn = lambda: f(q, k, v, w.heads, out=out)
    elif kind == "cross":
        q, kt, vt = rnd(T * N, C), rnd(L, C), rnd(L, C)
        out = torch.empty_like(q)
        fn = lambda: pab.cross_attention(q, kt, vt, w.heads, out=out)
    elif kind == "layout":
        src = rnd(T, N, C)
        dst = torch.empty((N, T, C), dtype=torch.bfloat16, device=device)
        fn = lambda: pab.layout(src, True, out=dst)
    elif kind.startswith("gemm"):
        # the DiT block's projections on this workload's token rows: q | k | v
        # (split into three outputs), the MLP's first GEMM with GELU, its
        # second with the fp32 residual add
        R = T * N
        K, Nn, epi = {"gemm_qkv": (C, 3 * C, pab.GEMM_STORE), "gemm_mlp_in": (C, 4 * C, pab.GEMM_GELU),
                      "gemm_mlp_out": (4 * C, C, pab.GEMM_RESID)}[kind]
        A, B = rnd(R, K), (rnd(K, Nn) * K ** -0.5).to(torch.bfloat16)
        if epi == pab.GEMM_RESID:
            X = torch.zeros((R, Nn), dtype=torch.float32, device=device)
            fn = lambda: pab.block_gemm(A, B, epi, X=X)
            out_bytes = R * Nn * 4 * 2  # fp32 read and written
        elif epi == pab.GEMM_STORE:
            outs = [torch.empty((R, C), dtype=torch.bfloat16, device=device) for _ in range(3)]
            fn = lambda: pab.block_gemm(A, B, epi, outs=outs)
            out_bytes = R * Nn * 2
        else:
            outs = [torch.empty((R, Nn), dtype=torch.bfloat16, device=device)]
            fn = lambda: pab.block_gemm(A, B, epi, outs=outs)
            out_bytes = R * Nn * 2
        flops[kind] = 2.0 * R * K * Nn
        abytes[kind] = R * K * 2 + K * Nn * 2 + out_bytes
    else:
        a, b = rnd(T * N * C), rnd(T * N * C)
        res = torch.zeros(1, dtype=torch.float64, device=device)
        fn = lambda: pab.attn_diff_mse_async(a, b, res)
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize(device)
    clocks = ClockSampler(0)
    clocks.start()
    time.sleep(0.3)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks.mark_start()
    e0.record()
    for _ in range(args.steps):
        fn()
    e1.record()
    torch.cuda.synchronize(device)
    clocks.mark_end()
    clk = clocks.stop()
    assert pab.device_errors() == 0
    ms = e0.elapsed_time(e1) / args.steps
    peaks = load_peaks()
    base = kind.replace("_sv", "")
    by = abytes[base]
    line = {"metric": f"{kind} kernel alone", "workload": w.name, "ms_per_launch": ms, "launches": args.steps,
            "warmup": args.warmup, "gbs": by / (ms * 1e-3) / 1e9, "frac_hbm": by / (ms * 1e-3) / 1e9 / peaks["hbm"],
            "bytes_per_launch": by, "clocks": clk}
    if base in flops:
        tf = flops[base] / (ms * 1e-3) / 1e12
        line.update(tflops=tf, frac_tc=tf / peaks["tc"], flops_per_launch=flops[base])
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    if args.kernel:
        return run_kernel(args)
    if args.sta:
        return run_sta(args)
    if args.draft:
        return run_draft(args)
    if args.dsp:
        return run_dsp(args)
    if args.sweep:
        return run_sweep(args)
    if args.dit:
        return run_dit(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
