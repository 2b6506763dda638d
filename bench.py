"""Benchmark of the sparsely-gated MoE layer forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload zipf] [--impl reference]

One step is one pass of the whole layer (route, permute, expert FFN, combine) over one
batch of synthetic tokens.  The headline workload (default) is the largest single-GPU
one, the skewed dropless top-2 layer (T=65536, d_model=1024, d_ff=4096, E=16, GELU,
bf16, Zipf(1.2) expert load).  The same run also times every other workload (tiny fp32,
Switch top-1, noisy top-4, GShard top-2) with the same step and reports them under
`per_config`.  Under torchrun every rank runs an independent replica on its own GPU (the
layer forward has no exchange step on one device), the step time is the max over ranks,
and the value is the tokens of all ranks per second.

Timing: W untimed warm-up steps; then K steps, each preceded (outside its events) by a
write and read-back of a 256 MB buffer that flushes the 126 MB L2 and by a ~0.2 ms
GPU-side wait, during which the host queues the whole step, so that the step's kernels
run back to back as they do in a CUDA-graph replay (the Python binding's launch latency
is not part of the step); CUDA events on the launching stream bracket each step and each
step call.  The dominant kernel is the
tcgen05 grouped GEMM (two launches per step: up- and down-projection); its roofline uses
the algorithmic bytes/FLOPs of those two launches over the event time of the expert-FFN
call, and its DRAM traffic per launch comes from the committed ncu summary while the
kernel sources match it.  Also reported for the headline workload: the same step
captured into a CUDA graph and replayed (`graph`), and the end-to-end throughput through
MoELayer.forward with every step's inputs copied in from pinned host memory and its
output copied out, consecutive steps pipelined over H2D / compute / D2H streams (`e2e`,
with the serial per-step latency beside it).

The CPU oracle (NumPy fp64) is timed on a fixed sample per workload: each oracle step
routes and dispatches all T tokens (so capacity is the workload's own) and runs the
expert FFN and combine for S fixed tokens (every (T/S)-th); its rate counts those S
tokens.  `cpu_baseline` and `--impl reference` run exactly this step.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import workloads  # noqa: E402

METRIC = "MoE layer fwd tokens/s; expert GEMM TFLOP/s and % of B200 bf16 / HBM roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20
GEMM_SOURCES = ["sparsely_gated_mixture_moe_b200/csrc/grouped_gemm_tc.cu",
                "sparsely_gated_mixture_moe_b200/csrc/common.cuh"]


# ----------------------------------------------------------------------------- helpers

def dist_env():
    """(rank, local_rank, world) from the torchrun environment, or (0, 0, 1)."""
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)),
            int(os.environ.get("WORLD_SIZE", 1)))


def max_over_ranks(x: float, device=None) -> float:
    """Max of a per-rank scalar over the process group (identity without one)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def gemm_source_sha() -> str:
    h = hashlib.sha256()
    for rel in GEMM_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str):
    """DRAM bytes per launch of the grouped GEMM from the committed ncu summary, or None
    when there is none for this workload or the kernel source changed since."""
    p = os.path.join(ROOT, "profiles", "grouped_gemm_traffic.txt")
    if not os.path.exists(p):
        return None
    sha = gemm_source_sha()
    for line in open(p):
        f = dict(kv.split("=", 1) for kv in line.split() if "=" in kv)
        if f.get("workload") == workload and f.get("src_sha") == sha and "bytes_per_launch" in f:
            return float(f["bytes_per_launch"])
    return None


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]
        return False

    def summary(self):
        rows = []
        for l in getattr(self, "lines", []):
            p = [x.strip() for x in l.split(",")]
            if len(p) < 9:
                continue
            try:
                rows.append((float(p[1]), float(p[2]), p[5:9]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, r in rows for i, v in enumerate(r) if v == "Active"})
        top = max(r[0] for r in rows)
        loaded = [r[0] for r in rows if r[0] >= 0.5 * top] or [r[0] for r in rows]
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


# The layer output y is fp32 in every benchmark figure: the workloads' bar (max|err| /
# RMS <= 2e-2 for bf16 layers) leaves no room for a bf16 rounding of y (on the Switch
# workload that rounding alone exceeds it).  --y-bf16 times the bf16-output option of
# the library instead (for callers that round y to bf16 anyway); such a line is labelled
# in its config and is not a figure for these workloads.
Y_BF16 = False


def y_bf16_of(w: workloads.Workload) -> bool:
    """Whether the benchmark runs the layer with a bf16 output y (bf16 layers under
    --y-bf16 only)."""
    return Y_BF16 and w.dtype == "bf16"


def algorithmic(w: workloads.Workload, n_kept: int, counts_kept, fused=False):
    """Algorithmic FLOPs and bytes of each step (kept assignments only, no padding).

    FFN FLOPs 4*N*d*f (two products).  FFN bytes: the weights of the experts that got
    rows, x_perm (dtype) read, y_perm (fp32) written.  Route bytes: x, the gating
    weights, noise, and the chosen indices and gates.  Permute: the chosen experts read,
    slot_pos and perm_src written, counts and offsets, and the kept token rows read from
    x and written to x_perm.  Combine: y_perm rows read, gates and slots, y written (in
    the output type of y_bf16_of).  fused (FFN and combine as one step): the FFN writes
    every row of y and reads each kept row's source index and gate; for k = 2 it also adds
    each kept row into its token's row of y (the up-projection zeroes y); no combine
    bytes."""
    es = 2 if w.dtype == "bf16" else 4
    ys = 2 if y_bf16_of(w) else 4
    T, d, f, E, k = w.T, w.d_model, w.d_ff, w.E, w.k
    active = int(sum(1 for c in counts_kept if c > 0))
    ffn_flops = 4.0 * n_kept * d * f
    ffn_bytes = active * 2.0 * d * f * es + n_kept * d * es + n_kept * d * 4.0
    noisy = w.gating == "noisy_topk"
    route_bytes = T * d * es + E * d * es * (2 if noisy else 1) + (T * E * 4 if noisy else 0) + T * k * 8
    permute_bytes = T * k * 4 * 3 + E * 8.0 + n_kept * d * es * 2
    combine_bytes = n_kept * d * 4.0 + T * k * 8 + T * d * float(ys)
    if fused:
        ffn_bytes = active * 2.0 * d * f * es + n_kept * d * es + T * d * float(ys) + n_kept * 8.0
        ffn_bytes += n_kept * d * 4.0 if k == 2 else T * 4.0
        combine_bytes = 0.0
    return {"ffn_flops": ffn_flops, "ffn_bytes": ffn_bytes, "route_bytes": route_bytes,
            "permute_bytes": permute_bytes, "combine_bytes": combine_bytes}


# ------------------------------------------------------------------------ CPU oracle arm

# Tokens whose expert FFN and combine each oracle step evaluates (every (T/S)-th token);
# routing and dispatch always cover all T tokens.  Sized so that one step takes about one
# to four seconds on a 16-core host.
ORACLE_SAMPLE = {"tiny": 512, "switch": 128, "noisy": 32, "gshard": 32, "zipf": 32,
                 "hierarchical": 32}


def oracle_rows(w):
    S = min(w.T, ORACLE_SAMPLE.get(w.name, 64))
    return [i * w.T // S for i in range(S)]


def oracle_step(w, inp, rows):
    """One oracle step: route and dispatch all T tokens, expert FFN and combine for
    ``rows``.  Returns seconds of wall time."""
    from oracle import moe_oracle as orc
    t0 = time.perf_counter()
    orc.moe_forward_rows(inp, w, rows)
    return time.perf_counter() - t0


def cpu_cores():
    n = len(os.sched_getaffinity(0))
    try:
        from threadpoolctl import threadpool_info
        blas = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:
        blas = n
    return n, blas


def sample_text(w, rows):
    cores, blas = cpu_cores()
    return ("each step: routing and capacity dispatch of all %d tokens, expert FFN and combine "
            "for %d fixed tokens (every %d-th); the rate counts those %d tokens (NumPy fp64; "
            "%d host cores visible, %d BLAS threads)" % (w.T, len(rows), w.T // len(rows),
                                                         len(rows), cores, blas))


def cpu_baseline(w, inp, budget_s=6.0):
    """The oracle as it stands, timed on its fixed sample: one untimed step, then steps
    until about budget_s seconds have been timed (at least two)."""
    rows = oracle_rows(w)
    oracle_step(w, inp, rows)
    times = []
    while len(times) < 2 or sum(times) < budget_s:
        times.append(oracle_step(w, inp, rows))
    _, blas = cpu_cores()
    mean = sum(times) / len(times)
    return {"value": len(rows) / mean, "unit": "tokens/s", "cores": blas, "kind": "oracle",
            "ms_per_step": mean * 1e3, "steps": len(times), "sample": sample_text(w, rows)}


def run_reference(args, w):
    rank, _, world = dist_env()
    if rank != 0:
        return
    inp = workloads.make_inputs(w)
    rows = oracle_rows(w)
    for _ in range(args.warmup):
        oracle_step(w, inp, rows)
    times = [oracle_step(w, inp, rows) for _ in range(args.steps)]
    mean = sum(times) / len(times)
    value = len(rows) / mean
    _, blas = cpu_cores()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": mean * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_json(w),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": blas, "kind": "oracle",
                         "sample": sample_text(w, rows)},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def config_json(w):
    gate = {"noisy_topk": "", "hierarchical": "(%d groups, %d x %d kept)" % (
        w.groups or 0, w.k_primary, w.k // max(w.k_primary, 1))}.get(
        w.gating, "(renorm)" if w.renorm else "(full-softmax gate)")
    c = {"workload": "%s: T=%d d_model=%d d_ff=%d E=%d k=%d gating=%s%s cf=%s act=%s %s%s" % (
        w.name, w.T, w.d_model, w.d_ff, w.E, w.k, w.gating, gate,
        w.capacity_factor, w.act, w.dtype,
        "" if w.zipf_s is None else " zipf_s=%s" % w.zipf_s),
        "T": w.T, "d_model": w.d_model, "d_ff": w.d_ff, "E": w.E, "k": w.k,
        "capacity_factor": w.capacity_factor, "hidden_f16": w.hidden_f16,
        "y": "bf16 (fp32 sums rounded once)" if y_bf16_of(w) else "fp32",
        "l2": "flushed before every timed step (256 MB written, then read back, outside the events)",
        "parallelism": "replicas"}
    return c


# ------------------------------------------------------------------------------ GPU arm

class LayerBench:
    """Device inputs, outputs and workspace of one workload, and its timed step."""

    def __init__(self, moe, w, dev):
        self.moe, self.w, self.dev = moe, w, dev
        self.inp = workloads.make_inputs(w)
        d = {k: v.to(dev) for k, v in self.inp.items()}
        self.cfg = moe.make_config(w.T, w.d_model, w.d_ff, w.E, w.k, gating=w.gating,
                                   renorm=w.renorm, capacity_factor=w.capacity_factor, act=w.act,
                                   dtype=w.dtype, hidden_f16=w.hidden_f16, groups=w.groups,
                                   k_primary=w.k_primary, y_bf16=y_bf16_of(w))
        self.ydt = torch.bfloat16 if y_bf16_of(w) else torch.float32
        self.d = moe.prepare_weights(self.cfg, d)  # fp16 w2 for fp16 hidden (exact re-encoding)
        T, k, E, dm, f = w.T, w.k, w.E, w.d_model, w.d_ff
        self.o = o = dict(
            idx=torch.empty(T, k, dtype=torch.int32, device=dev),
            gate=torch.empty(T, k, dtype=torch.float32, device=dev),
            near=torch.empty(T, dtype=torch.uint8, device=dev),
            counts=torch.empty(E, dtype=torch.int32, device=dev),
            offsets=torch.empty(E + 1, dtype=torch.int32, device=dev),
            perm_src=torch.empty(T * k, dtype=torch.int32, device=dev),
            slot_pos=torch.empty(T * k, dtype=torch.int32, device=dev),
            x_perm=torch.empty(T * k, dm, dtype=w.torch_dtype, device=dev),
            h=torch.empty(T * k, f, dtype=torch.float16 if w.hidden_f16 else w.torch_dtype,
                          device=dev),
            y_perm=torch.empty(T * k, dm, dtype=torch.float32, device=dev),
            y=torch.empty(T, dm, dtype=self.ydt, device=dev))
        self.noisy = w.gating == "noisy_topk"
        o["importance"] = torch.empty(E, dtype=torch.float32, device=dev) if self.noisy else None
        o["load"] = torch.empty(E, dtype=torch.float32, device=dev) if self.noisy and k < E else None
        self.ws = moe.workspace(self.cfg, dev)
        # FFN and combine as one call where moe_forward takes it (top-1)
        self.fused = moe.fused_combine(self.cfg) and self.cfg.k == 1
        self.stream = torch.cuda.current_stream(dev)
        self.launches = 0

    def route(self):
        moe, d, o = self.moe, self.d, self.o
        moe.moe_route(self.cfg, d["x"], d["w_gate"], o["idx"], o["gate"], self.ws,
                      w_noise=d.get("w_noise"), noise=d.get("noise"),
                      logit_bias=d.get("logit_bias"), importance=o["importance"], load=o["load"],
                      near_tie=o["near"])
        return moe.last_launch_count()

    def step(self, evs=None):
        """Route, permute, expert FFN, combine; events (if given) between the calls."""
        moe, d, o, cfg, st = self.moe, self.d, self.o, self.cfg, self.stream
        n = 0
        if evs:
            evs[0].record(st)
        n += self.route()
        if evs:
            evs[1].record(st)
        moe.moe_permute(cfg, o["idx"], d["x"], o["counts"], o["offsets"], o["perm_src"],
                        o["slot_pos"], o["x_perm"], self.ws)
        n += moe.last_launch_count()
        if evs:
            evs[2].record(st)
        if self.fused:
            # top-1: the down-projection writes gate * row straight into y
            moe.moe_expert_ffn_combine(cfg, o["x_perm"], o["offsets"], o["perm_src"],
                                       o["slot_pos"], o["gate"], d["w1"], d["w2"], o["h"], o["y"],
                                       self.ws)
            n += moe.last_launch_count()
            if evs:
                evs[3].record(st)
        else:
            moe.moe_expert_ffn(cfg, o["x_perm"], o["offsets"], d["w1"], d["w2"], o["h"],
                               o["y_perm"], self.ws)
            n += moe.last_launch_count()
            if evs:
                evs[3].record(st)
            moe.moe_combine(cfg, o["y_perm"], o["slot_pos"], o["gate"], o["y"], self.ws)
            n += moe.last_launch_count()
        if evs:
            evs[4].record(st)
        self.launches += n


# GPU clock cycles of the wait queued before each timed step (~0.2 ms): longer than the
# host needs to queue one step's calls
HOST_AHEAD_CYCLES = 400_000


class L2Flusher:
    def __init__(self, dev):
        self.buf = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    def __call__(self, i):
        # write 256 MB (evicts everything), then read it back so the step starts from a cold
        # L2 holding clean lines: the write-back of the flush's own dirty lines is not
        # charged to the first kernel of the step
        self.buf.fill_(float(i))
        self.buf.sum()
        # then keep the GPU busy while the host queues the step, so that no host launch
        # latency falls between the step's kernels
        torch.cuda._sleep(HOST_AHEAD_CYCLES)


def timed_steps(lb, flush, steps, warmup, world, dev, clock_gpu):
    """W warm-up steps, then `steps` timed steps (L2 flushed before each).  Returns the
    per-step phase times [steps, 4] (ms: route, permute, FFN, combine), the clock
    summary, kernels launched in the timed region, and the kept-row counts."""
    import torch.distributed as dist
    moe = lb.moe
    for _ in range(warmup):
        flush(1)
        lb.step()
    torch.cuda.synchronize(dev)
    err = moe.moe_get_error(lb.ws)
    if err:
        raise RuntimeError("%s: device error word %d after warm-up" % (lb.w.name, err))
    offs = lb.o["offsets"].cpu().tolist()
    kept = [offs[e + 1] - offs[e] for e in range(lb.w.E)]
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(steps)]
    lb.launches = 0
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(clock_gpu) as clk:
        for i in range(steps):
            flush(i)
            lb.step(evs[i])
        torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    per = np.array([[evs[i][j].elapsed_time(evs[i][j + 1]) for j in range(4)]
                    for i in range(steps)])
    err = moe.moe_get_error(lb.ws)
    if err:
        raise RuntimeError("%s: device error word %d after the timed steps" % (lb.w.name, err))
    return per, clk.summary(), lb.launches, kept


def summarize(w, per, kept, fused, step_ms_max, world, peaks):
    """Throughput, per-step GB/s with fractions of the HBM peak, and the grouped GEMM's
    roofline against the measured HBM copy and bf16 burst / sustained peaks."""
    n_kept = int(sum(kept))
    alg = algorithmic(w, n_kept, kept, fused)
    ms = per.mean(axis=0)
    ffn_s = ms[2] * 1e-3
    tflops = alg["ffn_flops"] / ffn_s / 1e12
    gbs = alg["ffn_bytes"] / ffn_s / 1e9
    ai = alg["ffn_flops"] / alg["ffn_bytes"]
    ridge = peaks["bf16_tflops_sustained"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    bound = "hbm" if ai < ridge else "tensor"
    hbm = peaks["hbm_gbs"]
    step_gbs = {"route": alg["route_bytes"] / (ms[0] * 1e-3) / 1e9,
                "permute": alg["permute_bytes"] / (ms[1] * 1e-3) / 1e9,
                "combine": None if fused else alg["combine_bytes"] / (ms[3] * 1e-3) / 1e9}
    return {
        "value": w.T * world / (step_ms_max * 1e-3), "unit": "tokens/s",
        "ms_per_step": step_ms_max,
        "steps_ms": {"route": float(ms[0]), "permute": float(ms[1]), "expert_ffn": float(ms[2]),
                     "combine": "fused into expert_ffn" if fused else float(ms[3])},
        "step_gbs": step_gbs,
        "step_hbm_frac": {kk: (None if v is None else v / hbm) for kk, v in step_gbs.items()},
        "expert_gemm": {"tflops": tflops, "frac_of_bf16_burst": tflops / peaks["bf16_tflops"],
                        "frac_of_bf16_sustained": tflops / peaks["bf16_tflops_sustained"],
                        "gbs": gbs, "frac_of_hbm": gbs / hbm, "arith_intensity": ai,
                        "bound": bound,
                        "roofline_frac": gbs / hbm if bound == "hbm"
                        else tflops / peaks["bf16_tflops_sustained"],
                        "compute": "tcgen05 bf16" if w.dtype == "bf16" else "fp32 SIMT FMA"},
        "kept_rows": n_kept,
        "_alg": alg,
    }


def graph_replay(lb, flush, steps, dev, stream):
    """The same step captured once into a CUDA graph and replayed (L2 flushed before each
    replay); returns (mean ms, None) or (inf, reason)."""
    moe = lb.moe
    try:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, capture_error_mode="thread_local"):
            lb.step()
        g_ms = []
        for i in range(steps + 3):
            flush(i)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            graph.replay()
            b.record(stream)
            b.synchronize()
            if i >= 3:
                g_ms.append(a.elapsed_time(b))
        del graph
        if moe.moe_get_error(lb.ws):
            raise RuntimeError("device error word set after the graph replays")
        return float(np.mean(g_ms)), None
    except RuntimeError as ex:
        return float("inf"), str(ex).splitlines()[0][:200]


def end_to_end(lb, flush, steps, world, dev, stream):
    """End to end through the public layer call, host buffers in pinned memory.  Every
    step copies its x (and noise) in from pinned host memory and its y out.  The headline
    figure pipelines consecutive steps the way a caller streaming batches would: H2D on
    one stream, the forward on the compute stream, D2H on a third, two sets of device
    buffers, so that step i's D2H and step i+1's H2D (the two PCIe directions) overlap
    the forwards.  The serial latency of one step (copy in, forward, copy out, nothing
    overlapped) is reported beside it."""
    import torch.distributed as dist
    moe, w, d, inp, noisy = lb.moe, lb.w, lb.d, lb.inp, lb.noisy
    T, dm = w.T, w.d_model
    wl = {kk: v for kk, v in d.items() if kk not in ("x", "noise")}
    layers = [moe.MoELayer(lb.cfg, wl, device=dev) for _ in range(2)]
    x_host = inp["x"].pin_memory()
    noise_host = inp["noise"].pin_memory() if noisy else None
    y_host = [torch.empty(T, dm, dtype=lb.ydt).pin_memory() for _ in range(2)]
    x_dev = [torch.empty_like(d["x"]) for _ in range(2)]
    noise_dev = [torch.empty_like(d["noise"]) if noisy else None for _ in range(2)]
    h2d = x_host.numel() * x_host.element_size() + (noise_host.numel() * 4 if noisy else 0)
    d2h = y_host[0].numel() * y_host[0].element_size()
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_c = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def serial_step():
        x_dev[0].copy_(x_host, non_blocking=True)
        if noisy:
            noise_dev[0].copy_(noise_host, non_blocking=True)
        layers[0].forward(x_dev[0], noise=noise_dev[0])
        y_host[0].copy_(layers[0].y, non_blocking=True)

    def pipelined(n):
        for i in range(n):
            b = i % 2
            if i >= 2:
                s_in.wait_event(ev_c[b])   # the forward of step i-2 has read x_dev[b]
            with torch.cuda.stream(s_in):
                x_dev[b].copy_(x_host, non_blocking=True)
                if noisy:
                    noise_dev[b].copy_(noise_host, non_blocking=True)
                ev_in[b].record(s_in)
            stream.wait_event(ev_in[b])
            if i >= 2:
                stream.wait_event(ev_out[b])  # the D2H of step i-2 has read layers[b].y
            layers[b].forward(x_dev[b], noise=noise_dev[b], stream=stream)
            ev_c[b].record(stream)
            s_out.wait_event(ev_c[b])
            with torch.cuda.stream(s_out):
                y_host[b].copy_(layers[b].y, non_blocking=True)
                ev_out[b].record(s_out)

    for _ in range(3):
        serial_step()
    pipelined(4)
    torch.cuda.synchronize(dev)
    lat_steps = max(3, min(steps, 50))
    lat_ms = []
    for i in range(lat_steps):
        flush(i)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        serial_step()
        b.record(stream)
        b.synchronize()
        lat_ms.append(a.elapsed_time(b))
    lat_mean = max_over_ranks(float(np.mean(lat_ms)), dev)
    if not torch.equal(y_host[0], layers[0].y.cpu()):
        raise RuntimeError("end-to-end output mismatch between host copy and device result")
    e2e_steps = max(4, min(steps, 100))
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    s_in.wait_event(a)
    s_out.wait_event(a)
    pipelined(e2e_steps)
    stream.wait_stream(s_in)
    stream.wait_stream(s_out)
    b.record(stream)
    torch.cuda.synchronize(dev)
    e2e_mean = max_over_ranks(a.elapsed_time(b) / e2e_steps, dev)
    last = (e2e_steps - 1) % 2
    if not torch.equal(y_host[last], layers[last].y.cpu()):
        raise RuntimeError("pipelined end-to-end output mismatch between host copy and device result")
    return {"value": T * world / (e2e_mean * 1e-3), "unit": "tokens/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_mean,
            "serial_latency_ms_per_step": lat_mean,
            "call": "MoELayer.forward (moe_forward); x/noise copied in from pinned host memory and "
                    "y copied out every step; consecutive steps pipelined on three streams "
                    "(H2D / forward / D2H, two buffer sets); no L2 flush between pipelined "
                    "steps (each step's x arrives by H2D)"}


def training_step(lb, flush, steps, world, dev, stream):
    """The training step of the same layer: moe_forward_train, then moe_backward of
    L = sum(dy * y) + 0.01 CV(Importance)^2 (+ 0.01 CV(Load)^2 for noisy gating), timed
    with CUDA events (L2 flushed before each step).  Algorithmic FLOPs: the forward's two
    expert products and the backward's four (dgrad and wgrad of each), 12 N d f."""
    import torch.distributed as dist
    moe, w, d = lb.moe, lb.w, lb.d
    cfg = lb.cfg
    T, k, E, dm, f = w.T, w.k, w.E, w.d_model, w.d_ff
    if moe.lib.moe_train_state_size(__import__("ctypes").byref(cfg)) == 0:
        return {"unavailable": "no backward pass for this configuration"}
    noisy = lb.noisy
    o = {"y": torch.empty(T, dm, dtype=lb.ydt, device=dev),
         "idx": torch.empty(T, k, dtype=torch.int32, device=dev),
         "gate": torch.empty(T, k, device=dev), "counts": torch.empty(E, dtype=torch.int32, device=dev),
         "imp": torch.empty(E, device=dev), "load": torch.empty(E, device=dev) if noisy else None,
         "dx": torch.empty(T, dm, device=dev), "dwg": torch.empty(E, dm, device=dev),
         "dwn": torch.empty(E, dm, device=dev) if noisy else None,
         "dbias": torch.empty(E, device=dev) if "logit_bias" in d else None,
         "dw1": torch.empty(E, f, dm, device=dev), "dw2": torch.empty(E, dm, f, device=dev),
         "dg": torch.empty(T, k, device=dev)}
    g = torch.Generator().manual_seed(77)
    dy = torch.randn(T, dm, generator=g).to(dev)
    state = moe.train_state(cfg, dev)
    ws = moe.backward_workspace(cfg, dev)
    w_load = 0.01 if noisy else 0.0

    def one(evs=None):
        if evs:
            evs[0].record(stream)
        moe.moe_forward_train(cfg, d["x"], d["w_gate"], d["w1"], d["w2"], o["y"], o["idx"], o["gate"],
                              o["counts"], state, ws, w_noise=d.get("w_noise"), noise=d.get("noise"),
                              logit_bias=d.get("logit_bias"), importance=o["imp"], load=o["load"])
        nf = moe.last_launch_count()
        if evs:
            evs[1].record(stream)
        moe.moe_backward(cfg, d["x"], d["w_gate"], d["w1"], d["w2"], o["idx"], o["gate"], state, dy,
                         o["dx"], o["dwg"], o["dw1"], o["dw2"], o["dg"], ws, w_noise=d.get("w_noise"),
                         noise=d.get("noise"), logit_bias=d.get("logit_bias"), importance=o["imp"],
                         load=o["load"], w_importance=0.01, w_load=w_load, dw_noise=o["dwn"],
                         dlogit_bias=o["dbias"])
        if evs:
            evs[2].record(stream)
        return nf + moe.last_launch_count()

    for _ in range(3):
        flush(1)
        one()
    torch.cuda.synchronize(dev)
    if moe.moe_get_error(ws):
        raise RuntimeError("device error word set in the training step")
    n = max(3, min(steps, 20))
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(n)]
    if world > 1:
        dist.barrier()
    launches = 0
    for i in range(n):
        flush(i)
        launches += one(evs[i])
    torch.cuda.synchronize(dev)
    fwd = float(np.mean([e[0].elapsed_time(e[1]) for e in evs]))
    bwd = float(np.mean([e[1].elapsed_time(e[2]) for e in evs]))
    fwd, bwd = max_over_ranks(fwd, dev), max_over_ranks(bwd, dev)
    # kept rows of the training forward: each expert's assignments up to the capacity
    C = moe.moe_capacity(cfg)
    n_kept = sum(min(c, C) if C >= 0 else c for c in o["counts"].cpu().tolist())
    bwd_flops = 8.0 * n_kept * dm * f
    return {"value": T * world / ((fwd + bwd) * 1e-3), "unit": "tokens/s",
            "forward_train_ms": fwd, "backward_ms": bwd, "steps": n,
            "backward_expert_tflops": bwd_flops / (bwd * 1e-3) / 1e12,
            "gpu_launches_per_step": launches / n,
            "loss": "sum(dy*y) + 0.01 CV(Importance)^2" + (" + 0.01 CV(Load)^2" if noisy else ""),
            "note": "backward_expert_tflops counts the four expert products (8 N d f) over the "
                    "whole backward call (router, gate and loss kernels included)"}


def run_gpu(args, w):
    import torch.distributed as dist
    import sparsely_gated_mixture_moe_b200 as moe

    rank, local_rank, world = dist_env()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        dist.init_process_group("nccl", device_id=dev,
                                timeout=__import__("datetime").timedelta(seconds=120))
    clock_gpu = local_rank if "CUDA_VISIBLE_DEVICES" not in os.environ else 0
    peaks, peak_src = load_peaks()
    flush = L2Flusher(dev)
    stream = torch.cuda.current_stream(dev)
    want_cpu = rank == 0 and world == 1 and not args.no_cpu_baseline

    # ---- the headline workload
    lb = LayerBench(moe, w, dev)
    if args.training_only:
        # the training step alone (for profiler captures of the backward pass)
        train = training_step(lb, flush, args.steps, world, dev, stream)
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()
        if rank == 0:
            print(json.dumps({"training_step": train, "config": config_json(w)}), flush=True)
        return
    per, clocks, timed_launches, kept = timed_steps(lb, flush, args.steps, args.warmup, world,
                                                   dev, clock_gpu)
    step_ms_max = max_over_ranks(float(np.mean(per.sum(axis=1))), dev)
    main = summarize(w, per, kept, lb.fused, step_ms_max, world, peaks)
    alg = main.pop("_alg")

    n_graph = max(3, min(args.steps, 200))
    g_local, graph_err = graph_replay(lb, flush, n_graph, dev, stream)
    g_mean = max_over_ranks(g_local, dev)
    if graph_err is not None or not np.isfinite(g_mean):
        graph_info = {"unavailable": graph_err or "capture failed on another rank"}
    else:
        graph_info = {"value": w.T * world / (g_mean * 1e-3), "unit": "tokens/s",
                      "ms_per_step": g_mean, "steps": n_graph,
                      "note": "one step (route, permute, expert FFN, combine) captured once and "
                              "replayed; L2 flushed before each replay"}
    e2e = end_to_end(lb, flush, args.steps, world, dev, stream)
    floor = launch_floor(lb, flush, dev, stream)
    train = training_step(lb, flush, args.steps, world, dev, stream) if not args.no_training else None

    eg = main["expert_gemm"]
    ffn_ms = main["steps_ms"]["expert_ffn"]
    traffic = recorded_traffic(w.name)
    if eg["bound"] == "hbm":
        roof = {"bound": "hbm", "achieved": eg["gbs"], "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": eg["frac_of_hbm"]}
    else:
        roof = {"bound": "tensor", "achieved": eg["tflops"], "peak": peaks["bf16_tflops_sustained"],
                "unit": "TFLOP/s", "frac": eg["frac_of_bf16_sustained"]}
    roof.update({"traffic": traffic,
                 "kernel": "grouped_gemm_tc_kernel (2 launches/step%s)" % (
                     "; the down-projection writes gate * row into y and zeroes dropped "
                     "tokens' rows" if lb.fused else ""),
                 "algorithmic_per_launch": {"flops": alg["ffn_flops"] / 2,
                                            "bytes": alg["ffn_bytes"] / 2},
                 "launch_ms": ffn_ms / 2.0,
                 "peak_source": ("%s (MEASURED_PEAKS.json; %s)" % (
                     peak_src, "bf16 sustained: the kernel runs inside multi-kernel steps"
                     if roof["bound"] == "tensor" else "HBM copy")) if peak_src == "measured"
                 else "fallback"})
    line = {
        "metric": METRIC, "value": main["value"], "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms_max,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
        "data": "synthetic (seeded; random-init weights)", "config": config_json(w),
        "roofline": roof,
    }
    line.update({kk: v for kk, v in main.items() if kk not in ("value", "unit", "ms_per_step")})
    line.update({"e2e": e2e, "graph": graph_info, "gpu_launches": timed_launches, "clocks": clocks,
                 "launch_floor": floor})
    if train is not None:
        line["training_step"] = train
    inp_main = lb.inp
    del lb
    torch.cuda.empty_cache()

    # ---- every other workload: the same timed step, fewer extras
    per_config = {}
    if not args.no_per_config:
        pc_steps = max(3, min(args.steps, 50))
        for name in workloads.ORDER:
            if name == w.name:
                continue
            wk = workloads.WORKLOADS[name]
            lbk = LayerBench(moe, wk, dev)
            perk, clk, nl, keptk = timed_steps(lbk, flush, pc_steps, args.warmup, world, dev,
                                               clock_gpu)
            smax = max_over_ranks(float(np.mean(perk.sum(axis=1))), dev)
            r = summarize(wk, perk, keptk, lbk.fused, smax, world, peaks)
            r.pop("_alg")
            r.update({"steps": pc_steps, "gpu_launches": nl, "clocks": clk,
                      "config": config_json(wk)})
            if want_cpu:
                r["cpu_baseline"] = cpu_baseline(wk, lbk.inp)
            per_config[name] = r
            del lbk
            torch.cuda.empty_cache()
        line["per_config"] = per_config
    if want_cpu:
        line["cpu_baseline"] = cpu_baseline(w, inp_main, budget_s=12.0)
    line["peaks"] = dict(peaks, source=peak_src)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def launch_floor(lb, flush, dev, stream, reps=20):
    """What one launch costs on its own in the step breakdown: event-to-event time of a
    trivial kernel (a one-value fill) with the host ahead of the GPU, and of the router
    alone, against the router's time per launch when 20 run back to back (their launch
    latencies then overlap the previous kernels).  Medians over `reps`, L2 flushed first."""
    small = torch.zeros(1, device=dev)

    def timed(fn, pre=None):
        ts = []
        for i in range(reps + 3):
            flush(i)
            if pre is not None:
                pre()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            b.synchronize()
            if i >= 3:
                ts.append(a.elapsed_time(b) * 1e3)
        return float(np.median(ts))

    trivial = timed(lambda: small.fill_(1.0))
    route = timed(lb.route)

    def twenty():
        for _ in range(20):
            lb.route()

    # a longer GPU-side wait before the first event, so that the host has queued all
    # twenty calls (about 25 us of host time each) before the GPU reaches them
    b2b = timed(twenty, pre=lambda: torch.cuda._sleep(4 * HOST_AHEAD_CYCLES)) / 20.0
    return {"trivial_kernel_us": trivial, "route_us": route, "route_back_to_back_us": b2b,
            "note": "event-to-event times with the host ahead of the GPU; a single launch "
                    "measures at least trivial_kernel_us here, whatever its bytes"}


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="zipf", choices=list(workloads.WORKLOADS))
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="time only the headline workload")
    ap.add_argument("--no-training", action="store_true",
                    help="skip the training-step (forward + backward) figure")
    ap.add_argument("--training-only", action="store_true",
                    help="time only the training step (forward keeping its state, then the "
                         "backward); for profiler captures")
    ap.add_argument("--y-bf16", action="store_true",
                    help="layer output y in bf16 for bf16 layers (outside these workloads' "
                         "error bar; not a benchmark figure)")
    ap.add_argument("--tokens", type=int, default=None,
                    help="run the workload with this many tokens instead of its own T (small "
                         "cases for profiler captures; not a benchmark figure)")
    args = ap.parse_args(argv)
    global Y_BF16
    Y_BF16 = bool(args.y_bf16)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    w = workloads.WORKLOADS[args.workload]
    if args.tokens is not None:
        w = w.scaled(T=args.tokens)
    if args.impl == "reference":
        run_reference(args, w)
    else:
        run_gpu(args, w)


if __name__ == "__main__":
    main()
