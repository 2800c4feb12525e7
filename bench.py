"""Benchmark of the sharded pre-LN transformer layer (forward + backward) on B200.

One step = one pass of the whole hot path over one batch of synthetic input:
tp_layer_fwd followed by tp_layer_bwd of the pre-LN GPT layer
(batch 4 x seq 2048, hidden 4096, 32 heads x 128, ffn 16384, t = 8 shards on
one GPU), the workload the headline metric is quoted on.  Prints ONE JSON
line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--workload NAME]   (any name in synth.WORKLOADS; default the layer)

N > 1 (launched with torch.distributed.run): N data-parallel replicas, one per
GPU, each on its own batch (weak scaling), whose parameter gradients are
all-reduced over NCCL bucket by bucket, each bucket as soon as the backward
has produced it, beside the rest of the backward (--no-dp-allreduce: pure
replicas); the time is the max over ranks.  --dp-allreduce turns the
reduction on at N = 1 too (a one-rank group: it exercises the path).  --impl reference times the fp64 CPU oracle
on the host cores on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from synth import EXTRA_WORKLOADS, WORKLOADS, Workload, make_inputs, to_f64, workload  # noqa: E402

METRIC = "sharded-layer TFLOP/s (bf16 fwd+bwd, 1 B200) and % of dense BF16 peak"
WORKLOAD = "layer_fwdbwd_B4_S2048_D4096_H32_F16384_t8"
NOMINAL_BF16_TFLOPS = 2250.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) per GEMM launch,
# averaged over the 11 GEMM launches of one layer step (dWout and dWqkv share
# one launch), from an ncu capture of the current GEMM kernel (the
# launch-by-launch table is kept with the ncu summaries).  To be re-measured
# whenever the GEMM kernel changes.
GEMM_DRAM_BYTES_PER_LAUNCH = {"layer_fwdbwd_B4_S2048_D4096_H32_F16384_t8": 986.5e6}
PARAMS = ("ln1_g", "ln1_b", "wqkv", "bqkv", "wout", "bout", "ln2_g", "ln2_b", "w1", "b1", "w2", "b2")


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in FALLBACK_PEAKS}, "measured"
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def choose_peak(peaks: dict, clock: dict):
    """The measured bf16 denominator that matches how the timed kernels ran.

    The burst figure (cuBLAS timed alone, clocks free) applies when the median
    SM clock of the timed region stayed within 5 % of its maximum; the
    sustained figure (a seconds-long loop settling under the power cap)
    applies when the clock sagged.  Without a clock record the burst figure
    is used: the larger denominator, the smaller fraction.
    Returns (peak TFLOP/s, name of the figure)."""
    sm, mx = clock.get("sm_mhz"), clock.get("sm_max_mhz")
    if sm and mx and sm < 0.95 * mx:
        return peaks["bf16_tflops_sustained"], "bf16_tflops_sustained"
    return peaks["bf16_tflops"], "bf16_tflops"


def clock_normalised(rate: float, clock: dict):
    """A rate scaled to the maximum SM clock (rate x max MHz / median MHz), or None."""
    sm, mx = clock.get("sm_mhz"), clock.get("sm_max_mhz")
    if not sm or not mx:
        return None
    return rate * mx / sm


def median_step_ms(events) -> float:
    """Median of the per-step durations between consecutive CUDA events."""
    return statistics.median(events[i].elapsed_time(events[i + 1]) for i in range(len(events) - 1))


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(ms: float, device) -> float:
    """The slowest rank's time: every rank returns the same maximum."""
    import torch.distributed as dist
    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size() == 1:
        return ms
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tflops(world: int, flops_per_step_per_rank: float, ms_per_step: float) -> float:
    """Whole-job throughput: all ranks' work over the slowest rank's time."""
    return world * flops_per_step_per_rank / (ms_per_step * 1e-3) / 1e12


# ---------------------------------------------------------------- CPU oracle leg
def oracle_sample(seq: int):
    """A bounded sample of the workload: one sequence of `seq` tokens, full widths."""
    w = workload(WORKLOAD)
    return Workload("sample", "layer_fwdbwd", batch=1, seq=seq, hidden=w.hidden, ffn=w.ffn,
                    heads=w.heads, head_dim=w.head_dim, t=w.t)


def time_oracle(seq: int, reps: int):
    """Times the fp64 oracle's layer forward + backward on the sample; returns (TFLOP/s, s/rep)."""
    from oracle import layer as olayer
    s = oracle_sample(seq)
    inp = make_inputs(s)
    p = {k: to_f64(inp[k]) for k in PARAMS}
    x, dy = to_f64(inp["x"]), to_f64(inp["dy"])
    times = []
    for _ in range(reps):
        t0 = time.perf_counter()
        olayer.layer_fwd(x, p, s.batch, s.heads, s.causal, s.ln_eps)
        olayer.layer_bwd(x, p, dy, s.batch, s.heads, s.causal, s.ln_eps)
        times.append(time.perf_counter() - t0)
    sec = statistics.median(times)
    return s.flops() / sec / 1e12, sec, s


def cores_used():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def base_config(w: Workload, world: int) -> dict:
    """The workload identity both arms report in their JSON line."""
    return {"workload": w.name, "batch": w.batch, "seq": w.seq, "hidden": w.hidden,
            "ffn": w.ffn, "heads": w.heads, "head_dim": w.head_dim, "t": w.t,
            "causal": w.causal, "flop_per_step": w.flops(),
            "parallelism": f"t{w.t} shards on each GPU; {world} independent replica(s)"}


def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return
    seq = 256
    from oracle import layer  # noqa: F401  (import outside the timed region)
    value, sec, s = None, None, None
    for _ in range(args.warmup):
        time_oracle(seq, 1)
    vals = []
    for _ in range(args.steps):
        v, sec, s = time_oracle(seq, 1)
        vals.append(v)
    value = statistics.median(vals)
    sample = (f"one sequence of {seq} tokens of the workload (batch 1, full hidden/ffn/heads), "
              f"fp64 NumPy oracle layer forward+backward, median of {args.steps} steps")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": sec * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": base_config(workload(WORKLOAD), world),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores_used(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        return False

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        try:
            rows = open(self.path).read().strip().splitlines()
        except OSError:
            rows = []
        for row in rows:
            f = [c.strip() for c in row.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for name, val in zip(names, f[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- our arm
class Runner:
    """One step of a workload through the public API, on preallocated buffers."""

    def __init__(self, w: Workload, device, dp: bool = False):
        import tensor_transformer_layer_column_b200 as tl
        from tensor_transformer_layer_column_b200.sublayer import (ShardedAttention, ShardedLayer,
                                                                   ShardedMLP)
        tl.lib()
        self.w = w
        self.host = make_inputs(w, with_dy=w.backward)
        g = {k: v.to(device) for k, v in self.host.items()}
        self.g = g
        dims = tl.Dims.of(w.batch, w.seq, w.hidden, w.ffn, w.heads, w.head_dim, w.t,
                          1 if w.causal else 0, w.ln_eps)
        if w.kind.startswith("layer"):
            self.mod = ShardedLayer(dims, {k: g[k] for k in PARAMS},
                                    placement="post" if "postln" in w.kind else "pre",
                                    recompute="recompute" in w.kind)
            self.acts = self.mod.alloc_acts()
            self.grads = self.mod.alloc_grads()
            self.reducer = None
            if dp:
                from tensor_transformer_layer_column_b200.data_parallel import (
                    GradientAllReduce, sharded_layer_buckets)
                if self.mod.post or self.mod.recompute:
                    raise ValueError("the data-parallel reduction is wired for the pre-LN layer")
                self.buckets, self.grads = sharded_layer_buckets(self.mod, device)
                self.reducer = GradientAllReduce(self.buckets)
                self.ready = self.reducer.events()
        elif w.kind.startswith("attn"):
            self.mod = ShardedAttention(dims, g["wqkv"], g["bqkv"], g["wout"], g["bout"])
        else:
            self.mod = ShardedMLP(dims, g["w1"], g["b1"], g["w2"], g["b2"])
        self.y = torch.empty_like(g["x"])
        self.dx = torch.empty_like(g["x"]) if w.backward else None
        self.fwd_out = None
        self.bwd_out = None

    def step(self, x, dy=None, y=None, dx=None):
        """One step; y and dx name the output buffers (default: the runner's own)."""
        w = self.w
        y = self.y if y is None else y
        dx = self.dx if dx is None else dx
        if w.kind.startswith("layer"):
            self.mod.forward(x, acts=self.acts, y=y)
            if self.reducer is None:
                self.mod.backward(dy, dx=dx, grads=self.grads)
                return
            # Each gradient group's all-reduce waits on its event on a side
            # stream, so it overlaps the rest of the backward; the step ends
            # when the last reduction has landed.
            self.mod.backward(dy, dx=dx, grads=self.grads, ready=self.ready)
            for group in ("mlp", "attn", "ln1"):
                self.reducer.launch(group, self.ready[group])
            self.reducer.finish()
            return
        if self.fwd_out is None:
            self.fwd_out = self.mod.forward(x)
        self.fwd_out["y"] = y
        self.mod.forward(x, out=self.fwd_out)
        if w.backward:
            if self.bwd_out is None:
                self.bwd_out = self.mod.backward(dy)
            self.bwd_out["dx"] = dx
            self.mod.backward(dy, out=self.bwd_out)


def hbm_bytes_per_step(w: Workload) -> dict:
    """Algorithmic DRAM bytes per step of the HBM-bound kernel classes of the
    pre-LN layer (each tensor read or written once; bf16/fp16 activations,
    fp32 statistics).  Empty for other workloads."""
    if w.kind != "layer_fwdbwd":
        return {}
    T, D, F = w.tokens, w.hidden, w.ffn
    BHS = w.batch * w.heads * w.seq
    BHS_pad = w.batch * w.heads * ((w.seq + 127) // 128 * 128)
    return {
        # LN1, LN2: read x, write u (2 bytes each), write mean and rstd
        "ln_fwd": 2 * (4 * T * D + 8 * T),
        # LN2, LN1 backward: read du, the LN input and the residual gradient, write dx
        "ln_bwd": 2 * (8 * T * D + 8 * T),
        # bias gradients db1 and dbqkv: the fp32 column partials that the GeLU'
        # product and the attention backward write (one row per 32 rows), read
        # once, and the bf16 sums written (db2 and dbout come from the LayerNorm
        # backwards)
        "colsum": 4 * (T // 32) * F + 4 * w.batch * ((w.seq + 31) // 32) * 3 * D + 2 * (F + 3 * D),
        # Wqkv to fp16 once per step (the backward reuses the forward's copy)
        "cast": 4 * D * 3 * D,
        # Dv and lse2: read O and dO, read lse, write both padded rows
        "attn_bwd_prep": 4 * T * D + 4 * BHS + 8 * BHS_pad,
    }


def recompute_flops(w: Workload) -> int:
    """FLOPs the recomputing backward adds: the forward without the MLP's
    second product (QKV and output projections, causal core, W1 product)."""
    pairs = w.seq * (w.seq + 1) // 2 if w.causal else w.seq * w.seq
    return (8 * w.tokens * w.hidden * w.hidden + 4 * w.head_dim * w.batch * w.heads * pairs
            + 2 * w.tokens * w.hidden * w.ffn)


def activation_report(w: Workload, mod) -> dict:
    """Activation memory held from forward to backward, and the recomputation cost."""
    rec = bool(getattr(mod, "recompute", False))
    out = {"held_bytes_per_layer": mod.saved_bytes(), "recompute": rec}
    if rec:
        out["recompute_flop_per_step"] = recompute_flops(w)
        out["note"] = ("value counts algorithmic FLOPs only; the recomputed forward's FLOPs "
                       "are extra work inside the timed step")
    return out


def run_ours(args):
    import tensor_transformer_layer_column_b200 as tl
    world, rank, local = dist_env()
    w = workload(args.workload)
    dp = args.dp_allreduce if args.dp_allreduce is not None else world > 1
    dp = dp and w.kind == "layer_fwdbwd"
    if world > 1 or dp:
        import datetime
        import socket
        import torch.distributed as dist
        torch.cuda.set_device(local)
        if world == 1 and "MASTER_PORT" not in os.environ:
            with socket.socket() as sk:
                sk.bind(("127.0.0.1", 0))
                port = sk.getsockname()[1]
            os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK="0",
                              WORLD_SIZE="1")
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    device = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(device)
    run = Runner(w, device, dp=dp)
    g, host_inp = run.g, run.host
    y, dx = run.y, run.dx
    stream = torch.cuda.current_stream(device)
    step = run.step

    for _ in range(args.warmup):
        step(g["x"], g.get("dy"))
    torch.cuda.synchronize(device)
    if tl.check_error() != 0:
        raise RuntimeError("device error word set during warm-up")

    def barrier():
        if world > 1:
            torch.distributed.barrier(device_ids=[device.index])

    # ---- device-resident timed region: K steps, launch trace closed, one
    # event at every step boundary; the step time is the median of the K
    # per-step durations (max over ranks), the total is first to last event.
    bounds = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    # ---- traced region: the same steps again with the launch trace open, for
    # the per-kernel breakdown and the roofline of the dominant kernel class.
    traced_steps = min(args.steps, 20)
    per_step_launches = 64
    trace = tl.LaunchTrace(per_step_launches * traced_steps + 16)
    with ClockSampler(torch.cuda.current_device() if world == 1 else local) as clocks:
        barrier()
        torch.cuda.synchronize(device)
        bounds[0].record(stream)
        for i in range(args.steps):
            step(g["x"], g.get("dy"))
            bounds[i + 1].record(stream)
        torch.cuda.synchronize(device)
        barrier()
        with trace:
            for _ in range(traced_steps):
                step(g["x"], g.get("dy"))
        torch.cuda.synchronize(device)
        barrier()
    ms_total = max_over_ranks(bounds[0].elapsed_time(bounds[-1]), device)
    ms_step = max_over_ranks(median_step_ms(bounds), device)
    clock = clocks.summary()
    records = trace.records()
    launches_per_step = trace.count / traced_steps
    launches = int(round(launches_per_step * args.steps))
    flops_step = w.flops()
    in_bytes = sum(v.numel() * v.element_size() for v in host_inp.values())
    value = job_tflops(world, flops_step, ms_step)

    # ---- end to end through the public API with host buffers
    # Every step uploads its inputs from pinned host memory and downloads its
    # outputs (y, and dx for a backward workload), all inside the timed
    # region.  The copies run on their own streams, double-buffered: step i+1's
    # inputs go up while step i computes, and step i's outputs come down while
    # step i+1 computes, so the two copy engines work beside the kernels.  The
    # first upload and the last download are not overlapped and are counted.
    e2e = None
    if not args.no_e2e:
        hx = host_inp["x"].pin_memory()
        hdy = host_inp["dy"].pin_memory() if w.backward else None
        hy = torch.empty_like(hx).pin_memory()
        hdx = torch.empty_like(hx).pin_memory() if w.backward else None
        xin = [torch.empty_like(g["x"]) for _ in range(2)]
        dyin = [torch.empty_like(g["dy"]) for _ in range(2)] if w.backward else [None, None]
        yout = [torch.empty_like(y) for _ in range(2)]
        dxout = [torch.empty_like(dx) for _ in range(2)] if w.backward else [None, None]
        copy_in = torch.cuda.Stream(device)
        copy_out = torch.cuda.Stream(device)

        def e2e_run(nsteps):
            in_ready = [torch.cuda.Event() for _ in range(2)]
            used = [torch.cuda.Event() for _ in range(2)]       # step done with slot b
            out_done = [torch.cuda.Event() for _ in range(2)]   # slot b's outputs are down
            copy_in.wait_stream(stream)
            copy_out.wait_stream(stream)

            def upload(i):
                b = i % 2
                with torch.cuda.stream(copy_in):
                    if i >= 2:
                        copy_in.wait_event(used[b])
                    xin[b].copy_(hx, non_blocking=True)
                    if w.backward:
                        dyin[b].copy_(hdy, non_blocking=True)
                    in_ready[b].record(copy_in)

            upload(0)
            for i in range(nsteps):
                b = i % 2
                if i + 1 < nsteps:
                    upload(i + 1)
                stream.wait_event(in_ready[b])
                if i >= 2:
                    stream.wait_event(out_done[b])
                step(xin[b], dyin[b], y=yout[b], dx=dxout[b])
                used[b].record(stream)
                with torch.cuda.stream(copy_out):
                    copy_out.wait_event(used[b])
                    hy.copy_(yout[b], non_blocking=True)
                    if w.backward:
                        hdx.copy_(dxout[b], non_blocking=True)
                    out_done[b].record(copy_out)
            stream.wait_event(out_done[(nsteps - 1) % 2])

        e2e_run(args.warmup)
        barrier()
        torch.cuda.synchronize(device)
        s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s2.record(stream)
        e2e_run(args.steps)
        e2.record(stream)
        torch.cuda.synchronize(device)
        barrier()
        e2e_ms = max_over_ranks(s2.elapsed_time(e2), device)
        nb = 2 if w.backward else 1
        e2e = {"value": job_tflops(world, flops_step, e2e_ms / args.steps),
               "unit": "TFLOP/s", "h2d_bytes_per_step": nb * hx.numel() * 2,
               "d2h_bytes_per_step": nb * hy.numel() * 2,
               "copies": "pinned host buffers, own copy streams, double-buffered "
                         "(uploads and downloads overlap neighbouring steps' kernels)"}
    if tl.check_error() != 0:
        raise RuntimeError("device error word set during the timed region")

    # ---- roofline of the dominant kernel class (live CUDA-event durations
    # from the traced region; the denominator follows the sampled clocks)
    peaks, peak_src = load_peaks()
    peak, peak_name = choose_peak(peaks, clock)
    by_kind = {}
    for kind, fl, ms in records:
        d = by_kind.setdefault(kind, [0, 0.0, 0.0])
        d[0] += 1
        d[1] += fl
        d[2] += ms
    dom = max(by_kind, key=lambda k: by_kind[k][2]) if by_kind else None
    roofline = None
    if dom is not None:
        n, fl, ms = by_kind[dom]
        achieved = fl / (ms * 1e-3) / 1e12 if ms > 0 else 0.0
        traffic = GEMM_DRAM_BYTES_PER_LAUNCH.get(w.name) if dom == "gemm" else None
        roofline = {"bound": "tensor", "kernel": f"{dom} (tcgen05)", "achieved": achieved,
                    "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                    "peak_source": f"{peak_src} {peak_name}", "traffic": traffic,
                    "launches": n, "avg_launch_ms": ms / n,
                    "avg_launch_gflop": fl / n / 1e9,
                    "achieved_at_max_clock": clock_normalised(achieved, clock),
                    "frac_of_nominal": achieved / NOMINAL_BF16_TFLOPS,
                    # Against the burst and the sustained figure alike, whichever
                    # the clock record selected for `frac`.
                    "frac_of_burst": achieved / peaks["bf16_tflops"],
                    "frac_of_sustained": achieved / peaks["bf16_tflops_sustained"],
                    "traced_steps": traced_steps}
    hbm = hbm_bytes_per_step(w)
    breakdown = {k: {"launches": v[0], "ms_per_step": v[2] / traced_steps,
                     "share": v[2] / max(1e-9, sum(x[2] for x in by_kind.values())),
                     **({"tflops": v[1] / (v[2] * 1e-3) / 1e12,
                         "frac_of_peak": v[1] / (v[2] * 1e-3) / 1e12 / peak}
                        if v[1] > 0 and v[2] > 0 else {}),
                     **({"algorithmic_bytes_per_step": hbm[k],
                         "gbs": hbm[k] / (v[2] / traced_steps * 1e-3) / 1e9,
                         "frac_of_hbm": hbm[k] / (v[2] / traced_steps * 1e-3) / 1e9 / peaks["hbm_gbs"]}
                        if k in hbm and v[2] > 0 else {})}
                 for k, v in sorted(by_kind.items(), key=lambda kv: -kv[1][2])}

    # ---- CPU oracle baseline (rank 0, N = 1 only), after the GPU timing
    cpu = None
    if world == 1 and not args.no_cpu_baseline and args.workload == WORKLOAD:
        oseq = 1024
        cv, csec, cs = time_oracle(oseq, 2)
        cpu = {"value": cv, "unit": "TFLOP/s", "cores": cores_used(), "kind": "oracle",
               "sample": (f"one sequence of {oseq} tokens of the workload (batch 1, full widths), "
                          f"fp64 NumPy oracle layer forward+backward, median of 2 "
                          f"({csec:.1f} s each)")}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "ms_per_step_mean": ms_total / args.steps,
            "timing": ("median of per-step CUDA-event durations over the timed steps, launch "
                       "trace closed; per-kernel figures from a separate traced pass"),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": {**base_config(w, world),
                       "l2": (f"inputs larger than L2: {in_bytes / 2**20:.0f} MiB of inputs per "
                              "step vs 120 MiB of L2, no flush" if in_bytes > 126e6
                              else "L2 not flushed: inputs smaller than L2")},
            "pct_dense_bf16_peak": 100.0 * value / world / NOMINAL_BF16_TFLOPS,
            "pct_measured_bf16_peak": 100.0 * value / world / peak,
            "peak_source": f"{peak_src} {peak_name}",
            "e2e": e2e,
            "gpu_launches": launches,
            "roofline": roofline,
            "kernels": breakdown,
            "clocks": clock,
            "cpu_baseline": cpu,
        }
        if w.kind.startswith("layer"):
            line["activations"] = activation_report(w, run.mod)
        if dp:
            line["config"]["parallelism"] = (
                f"t{w.t} shards on each GPU; {world} data-parallel replica(s), parameter "
                "gradients all-reduced (NCCL, sum) in 3 buckets, each issued on a side stream "
                "as soon as the backward has produced it")
            line["dp_allreduce"] = {
                "buckets": {g: int(b.numel() * b.element_size())
                            for g, b in run.buckets.flat.items()},
                "bytes_per_step": int(sum(b.numel() * b.element_size()
                                          for b in run.buckets.flat.values()))}
        print(json.dumps(line), flush=True)
    if torch.distributed.is_initialized():
        torch.distributed.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default=WORKLOAD,
                    choices=sorted(WORKLOADS) + sorted(EXTRA_WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true",
                    help="skip the timed CPU oracle sample (for profiler runs)")
    ap.add_argument("--no-e2e", action="store_true",
                    help="skip the host-buffer end-to-end leg (for profiler runs)")
    ap.add_argument("--dp-allreduce", dest="dp_allreduce", action="store_true", default=None,
                    help="all-reduce the layer's parameter gradients over the replicas "
                         "(default with --gpus > 1; at 1 GPU a one-rank group)")
    ap.add_argument("--no-dp-allreduce", dest="dp_allreduce", action="store_false",
                    help="pure replicas: no gradient reduction")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
