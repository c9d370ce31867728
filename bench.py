#!/usr/bin/env python
"""Benchmark of the B200 fused MoE expert layer.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload all|NAME] [--impl ours|reference]

By default every workload is measured in one run: the line's headline
(metric, value, roofline, e2e, cpu_baseline) is the largest, the zipf
training-forward prefill (T=16384, 1.24 TFLOP per step), and a `workloads`
object carries the same figures for each of tiny, decode, dsv3, relu2 and
zipf.  --workload NAME measures one workload only.

A step is one pass of the whole layer over one batch of the workload:
route (top-k gating) -> align (sort/pad by expert) -> gate/up GEMM with the
activation epilogue -> down GEMM with the top-k weights -> scatter-reduce.
Inputs and weights are resident in HBM when the timed region starts.  The K
timed steps run back to back between two CUDA events (one CUDA graph), each
on one of R copies of all inputs, so at least twice the L2 size of other
data is read before a copy is used again; only if that needed more than
MAX_INPUT_COPIES copies (or with --single-copy) is L2 flushed (a write of
twice its size) before every step instead, outside the step's events.  Every kernel of the step is also bracketed by
library-recorded events in a second set of graphs, so the dominant kernel's
duration is measured live over the same number of steps.

Multi-GPU (torchrun, one process per GPU): the layer does not shard, so each
rank runs an independent replica of the workload ("scaling": "weak"); ranks
meet at barriers and the slowest rank's time is reported.

Each workload also carries, measured in the same run: the end-to-end step through
the public API with host buffers (one host-to-device copy of x and logits,
one device-to-host copy of out per step), the dominant kernel's roofline,
the clocks seen, the CPU oracle on a bounded token sample, the router
(moe_router: x . W_g^T and top-k gating, the step before the layer) on its
own with a seeded W_g, and, for the 128-row prefill workloads, the backward
(moe_backward: dx, dW13, dW2 and dL/d topk_weights from a seeded dL/dout)
timed the same way.

--impl reference times the CPU fp64 oracle (test infrastructure) on the host
cores on a bounded sample of the same workload; rank 0 only.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

from grouped_gemm_gating_b200 import workloads as W  # noqa: E402

METRIC = "MoE layer TFLOPS and tokens/s on 1 B200; % of bf16 tensor peak / HBM roofline"

# DRAM bytes (read + write) of one launch of the dominant kernel, from an ncu
# capture of that kernel on that workload (bench.py --workload <w> --steps 3
# --warmup 3 --no-cpu-baseline --single-copy under ncu -k <kernel>).  An
# entry is removed whenever the kernel changes after its capture.
NCU_TRAFFIC = {
    ("decode", "fused_expert"): 201_748_736,
    ("zipf", "gate_up_gemm"): 1_549_468_416,
}
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
CLOCK_QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
               "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
               "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
CLOCK_REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
# input copies for back-to-back timing (the tiny layer needs 159 of its 1.6 MB)
MAX_INPUT_COPIES = 200
# tokens per oracle step for the CPU baseline / reference arm (bounded sample)
CPU_SAMPLE_TOKENS = {"tiny": 32, "decode": 1, "relu2": 2, "dsv3": 8, "zipf": 8}


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="all", choices=["all"] + sorted(W.CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-backward", action="store_true", help="skip the backward leg (block_m = 128 workloads)")
    ap.add_argument("--fp8", action="store_true", help="with --workload NAME: also measure it with fp8 expert weights")
    ap.add_argument("--single-copy", action="store_true",
                    help="one copy of the inputs and an L2 flush before every step (small device footprint, "
                         "e.g. for profiler captures)")
    a = ap.parse_args(argv)
    if a.warmup < 3:
        ap.error("--warmup must be at least 3")
    if a.steps < 1:
        ap.error("--steps must be at least 1")
    return a


def workload_desc(cfg: W.MoEConfig) -> str:
    act = "SwiGLU" if cfg.act == W.ACT_SWIGLU else "relu2"
    s = (f"{cfg.name}: T={cfg.T} d_model={cfg.d} d_ff={cfg.F} E={cfg.E} top_k={cfg.k} {act} "
         f"block_m={cfg.block_m}")
    if cfg.n_group > 1:
        s += f" n_group={cfg.n_group} topk_group={cfg.topk_group}"
    if cfg.n_shared:
        s += f" shared_experts={cfg.n_shared}"
    return s


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def algorithmic(cfg: W.MoEConfig, topk_ids: np.ndarray):
    """FLOPs and bytes of the step and of each GEMM launch (no padding, no re-reads)."""
    S = cfg.T * cfg.k
    U = int(np.unique(topk_ids).size)
    rows = S + cfg.T * cfg.n_shared          # rows through the expert GEMMs
    n_w = U + cfg.n_shared                   # weight matrices read
    n1 = cfg.n1
    g1_flops = 2 * rows * n1 * cfg.d
    g2_flops = 2 * rows * cfg.d * cfg.F
    g1_bytes = n_w * n1 * cfg.d * 2 + cfg.T * cfg.d * 2 + rows * cfg.F * 2
    g2_bytes = n_w * cfg.d * cfg.F * 2 + rows * cfg.F * 2 + rows * cfg.d * 4
    # fused kernel (block_m <= 64): both weight sets of every hit expert, x
    # in, out; h stays in shared memory and the per-slot products are fp32
    # reductions into an L2-resident accumulator, not DRAM traffic
    fused_bytes = n_w * (n1 * cfg.d + cfg.d * cfg.F) * 2 + cfg.T * cfg.d * 2 + cfg.T * cfg.d * 2
    return dict(S=S, U=U, flops_routed=cfg.flops_routed(), flops_total=cfg.flops_total(),
                gate_up_gemm=(g1_flops, g1_bytes), down_gemm=(g2_flops, g2_bytes), fused_bytes=fused_bytes,
                weight_bytes=n_w * (n1 * cfg.d + cfg.d * cfg.F) * 2)


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the GPU works."""

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={CLOCK_QUERY}", "--format=csv,noheader,nounits", "-lms", "20",
                 "-i", str(self.index)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, active = [], [], set()
        for line in out.splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for name, v in zip(CLOCK_REASONS, f[5:9]):
                if v.lower().startswith("active"):
                    active.add(name)
        busy = [s for s in sm if s > 0.5 * max(smax or [1])] or sm
        return {"sm_mhz": statistics.median(busy) if busy else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(active), "samples": len(sm)}


def cpu_info():
    """Host cores and CPU model of the machine the oracle is timed on."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"nproc": os.cpu_count() or 1, "model": model}


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def oracle_step(inp: W.MoEInputs, tokens: np.ndarray):
    """One oracle pass (route, align, forward) over the sampled tokens."""
    import oracle
    c = inp.cfg
    lg = inp.logits[tokens]
    ids, w = oracle.route(lg, c.k, c.n_group, c.topk_group, c.group_score, bool(c.renormalize),
                          c.routed_scaling)
    oracle.align(ids, c.E, c.block_m)
    return oracle.forward(inp.x[tokens], inp.w13, inp.w2, ids, w, c.act, inp.w13_shared, inp.w2_shared)


def time_oracle(inp: W.MoEInputs, steps: int, warmup: int, min_seconds: float = 0.0, max_steps: int = 0,
                threads: int | None = None):
    """Time the oracle on seeded token samples: `warmup` untimed steps, then
    at least `steps` timed steps, and more (up to max_steps, default 10x
    steps) until `min_seconds` of CPU work has been measured.  threads=1
    limits the BLAS pool to one thread."""
    import contextlib
    c = inp.cfg
    n = min(c.T, CPU_SAMPLE_TOKENS.get(c.name, 8))
    rng = np.random.default_rng(c.seed)
    limit = contextlib.nullcontext()
    if threads is not None:
        try:
            from threadpoolctl import threadpool_limits
            limit = threadpool_limits(limits=threads)
        except Exception:
            pass
    cap = max_steps or 10 * steps
    times = []
    with limit:
        cores = blas_threads()
        i = 0
        while True:
            tokens = np.sort(rng.choice(c.T, size=n, replace=False))
            t0 = time.perf_counter()
            oracle_step(inp, tokens)
            if i >= warmup:
                times.append(time.perf_counter() - t0)
            i += 1
            if len(times) >= steps and (sum(times) >= min_seconds or len(times) >= cap):
                break
    sec = float(np.mean(times))
    flops = c.flops_total() * n / c.T
    return {"value": flops / sec / 1e12, "unit": "TFLOPS", "tokens_per_s": n / sec, "cores": cores,
            "kind": "oracle", "steps": len(times), "ms_per_step": sec * 1e3, "tokens": n,
            "sample": f"{n} of {c.T} tokens per step (seeded), {len(times)} steps after {warmup} warm-up "
                      f"({sum(times):.1f} s); route+align+forward in fp64 numpy, {cores} BLAS thread(s)"}


def cpu_baseline(inp: W.MoEInputs, seconds: float):
    """The oracle on the host cores (all BLAS threads) plus a single-thread
    run, each on a bounded token sample of the workload."""
    cb = time_oracle(inp, steps=2, warmup=1, min_seconds=seconds)
    one = time_oracle(inp, steps=1, warmup=0, min_seconds=seconds / 3, threads=1)
    info = cpu_info()
    return {"value": cb["value"], "unit": "TFLOPS", "cores": cb["cores"], "kind": "oracle",
            "sample": cb["sample"], "host_nproc": info["nproc"], "cpu_model": info["model"],
            "single_thread_value": one["value"], "single_thread_sample": one["sample"]}


# --------------------------------------------------------------------------

def dist_setup(gpus: int, backend: str = "nccl"):
    """Rank plumbing for one process per GPU (torchrun env).  "nccl" binds
    the process to its GPU; "gloo" runs the same host logic on the CPU."""
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != gpus:
        raise SystemExit(f"--gpus {gpus} but WORLD_SIZE={world}")
    pg = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        if backend == "nccl":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
        pg = dist
    elif backend == "nccl":
        torch.cuda.set_device(0)
    return world, rank, local, pg


def barrier(pg):
    if pg is not None:
        pg.barrier()


def max_over_ranks(pg, value: float, device: str = "cuda") -> float:
    """The slowest rank's time: every rank runs the same steps, the job
    takes as long as its slowest replica."""
    if pg is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(world: int, flops_per_step: float, ms_total: float, steps: int) -> float:
    """Throughput of all replicas together: world x the per-replica FLOPs of
    a step over the (max-over-ranks) time of one step."""
    return world * flops_per_step / (ms_total / steps / 1e3) / 1e12


# Headline workload when every workload is measured: the largest (1.24
# TFLOP per step), the tensor-bound training-forward prefill.
HEADLINE = "zipf"
# measurement order: the headline first, while the GPU is cool
ORDER = ("zipf", "dsv3", "relu2", "decode", "tiny")
NOMINAL_HBM_GBS = 8000.0


def job_config(cfg: W.MoEConfig, world: int, experts_hit: int) -> dict:
    """The `config` object of a line: the workload only (the same on both arms)."""
    return {"workload": workload_desc(cfg), "global_batch": world * cfg.T,
            "parallelism": f"replicas x{world}", "experts_hit": experts_hit,
            "flops_per_step": cfg.flops_total(), "flops_routed_per_step": cfg.flops_routed()}


def roofline(cfg, alg, stages, total_ms, steps, launches_per_step, rotate, peaks, peak_src):
    """Roofline of the dominant kernel: algorithmic FLOPs (or bytes) of one
    launch over its average launch duration, against the measured peak."""
    dom = max(("gate_up_gemm", "down_gemm", "fused_expert"), key=lambda s: stages[s][0])
    dom_ms, dom_calls = stages[dom]
    per_launch_s = dom_ms / max(dom_calls, 1) / 1e3
    per_launch_src = "CUDA events around the kernel (profiled graphs)"
    if rotate and launches_per_step == 1:
        # the step is this one kernel: its back-to-back step time is its
        # average launch duration, without the events' own launch gap
        per_launch_s = total_ms / steps / 1e3
        per_launch_src = "CUDA events around the back-to-back timed steps (the step is this one kernel)"
    if dom == "fused_expert":   # both GEMMs (and the combine) in one kernel
        fl = alg["gate_up_gemm"][0] + alg["down_gemm"][0]
        by = alg["fused_bytes"]
    else:
        fl, by = alg[dom]
    ridge = peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    src = f"{peak_src} (MEASURED_PEAKS.json)" if peak_src == "measured" else "fallback"
    if fl / by >= ridge:
        achieved = fl / per_launch_s / 1e12
        # the timed region is tens of milliseconds: the burst (not the
        # power-capped sustained) cuBLAS figure is the denominator
        peak = peaks["bf16_tflops"]
        roof = {"bound": "tensor", "unit": "TFLOP/s",
                "frac_of_sustained_peak": round(achieved / peaks["bf16_tflops_sustained"], 4)}
        src += ", burst bf16"
    else:
        achieved = by / per_launch_s / 1e9
        peak = peaks["hbm_gbs"]
        roof = {"bound": "hbm", "unit": "GB/s", "frac_of_nominal_hbm": round(achieved / NOMINAL_HBM_GBS, 4)}
        src += ", HBM copy"
    traffic = NCU_TRAFFIC.get((cfg.name, dom))
    roof.update({"kernel": dom, "achieved": round(achieved, 2), "peak": peak, "peak_source": src,
                 "frac": round(achieved / peak, 4),
                 "traffic": traffic,
                 "traffic_vs_algorithmic": None if traffic is None else round(traffic / by, 3),
                 "per_launch_us": round(per_launch_s * 1e6, 2), "per_launch_source": per_launch_src,
                 "algorithmic_flops": fl, "algorithmic_bytes": by})
    return roof


def measure_workload(name, args, dev, pg, world, rank, cpu_seconds, fp8=False):
    """Every figure of one workload: device-timed steps, per-kernel times,
    roofline, the end-to-end step, the router and the CPU oracle.  With fp8,
    the layer runs on the workload's expert weights quantised to fp8
    (moe_layer_fp8) and only the layer itself is measured."""
    import torch

    from grouped_gemm_gating_b200 import moe as M

    cfg = W.CONFIGS[name]
    inp = W.make_inputs(cfg)
    q8 = W.fp8_weights(inp) if fp8 else None
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size

    def to_dev(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(dev).view(torch.bfloat16)

    # x and logits of a step sit back to back in one device buffer (logits at
    # a 256-byte aligned offset), so the end-to-end step moves them with one
    # host-to-device copy
    x_bytes = cfg.T * cfg.d * 2
    lg_off = -(-x_bytes // 256) * 256
    io_bytes = lg_off + cfg.T * cfg.E * 4

    def io_views(raw):
        return (raw[:x_bytes].view(torch.bfloat16).view(cfg.T, cfg.d),
                raw[lg_off:io_bytes].view(torch.float32).view(cfg.T, cfg.E))

    def input_set():
        io = torch.empty(io_bytes, dtype=torch.uint8, device=dev)
        x_v, lg_v = io_views(io)
        x_v.copy_(to_dev(inp.x))
        lg_v.copy_(torch.from_numpy(inp.logits).to(dev))
        if fp8:
            wq = M.Fp8Experts(*[None if a is None else torch.from_numpy(np.ascontiguousarray(a)).to(dev)
                                for a in q8])
            return dict(io=io, x=x_v, logits=lg_v, wq=wq, w13=None, w2=None, w13s=None, w2s=None)
        return dict(io=io, x=x_v, logits=lg_v,
                    w13=to_dev(inp.w13), w2=to_dev(inp.w2),
                    w13s=to_dev(inp.w13_shared) if cfg.n_shared else None,
                    w2s=to_dev(inp.w2_shared) if cfg.n_shared else None)

    sets = [input_set()]
    buf = M.MoEBuffers(cfg.T, cfg.d, cfg.F, cfg.E, cfg.k, cfg.block_m, cfg.act, cfg.n_shared, dev)
    rk = dict(n_group=cfg.n_group, topk_group=cfg.topk_group, group_score=cfg.group_score,
              renormalize=bool(cfg.renormalize), routed_scaling=cfg.routed_scaling)

    def step(st, xin=None, lgin=None):
        # the whole layer through the public API: route + align + forward
        # (one launch for decode batches)
        if fp8:
            buf.layer_fp8(st["logits"] if lgin is None else lgin, st["x"] if xin is None else xin, st["wq"], **rk)
        else:
            buf.layer(st["logits"] if lgin is None else lgin, st["x"] if xin is None else xin,
                      st["w13"], st["w2"], st["w13s"], st["w2s"], **rk)
        return M.moe_last_launch_count()

    # Cold inputs between steps: the timed steps run back to back, each on one
    # of R copies of all inputs (x, logits, weights), with R chosen so that
    # at least twice the L2 size of other data is read between two uses of a
    # copy.  When that would take more than MAX_INPUT_COPIES copies (or
    # --single-copy is given) L2 is flushed (a write of twice its size) before
    # each step instead, outside the step's events.
    step(sets[0])
    torch.cuda.synchronize(dev)
    topk_ids = buf.topk_ids.cpu().numpy()
    alg = algorithmic(cfg, topk_ids)
    if fp8:
        # the weight stream is one e4m3 byte per weight plus one scale byte
        # per 32 weights
        wb = alg["weight_bytes"] // 2 * 33 // 32
        alg["fused_bytes"] += wb - alg["weight_bytes"]
        alg["weight_bytes"] = wb
    touched = alg["weight_bytes"]
    n_copies = 1 + -(-2 * l2 // touched)
    rotate = n_copies <= MAX_INPUT_COPIES and not args.single_copy
    if not rotate:
        n_copies = 1
    sets += [input_set() for _ in range(n_copies - 1)]
    flush = None if rotate else torch.empty(2 * l2 // 4 + 1024, dtype=torch.float32, device=dev)

    stream = torch.cuda.current_stream(dev)
    launches_per_step = 0
    for i in range(args.warmup):
        launches_per_step = step(sets[i % n_copies])
    torch.cuda.synchronize(dev)
    assert M.moe_read_status(buf.status) == 0, "device status set during warm-up"
    assert np.array_equal(buf.topk_ids.cpu().numpy(), topk_ids)

    def capture(fn):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        return g

    def timed(runs, n, whole=None):
        """Device time of n steps (step i runs runs[i % len(runs)], or one
        call of `whole` runs all n), max over ranks."""
        barrier(pg)
        torch.cuda.synchronize(dev)
        if rotate:
            start = torch.cuda.Event(enable_timing=True)
            end = torch.cuda.Event(enable_timing=True)
            start.record(stream)
            if whole is not None:
                whole()
            else:
                for i in range(n):
                    runs[i % len(runs)]()
            end.record(stream)
            torch.cuda.synchronize(dev)
            ms = start.elapsed_time(end)
        else:
            starts = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
            ends = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
            for i in range(n):
                flush.zero_()
                starts[i].record(stream)
                runs[i % len(runs)]()
                ends[i].record(stream)
            torch.cuda.synchronize(dev)
            ms = sum(s_.elapsed_time(e_) for s_, e_ in zip(starts, ends))
        barrier(pg)
        return max_over_ranks(pg, ms)

    # The step's launches are replayed from CUDA graphs (kernels chained by
    # programmatic dependent launch), one graph per input copy; back to back,
    # the K timed steps are one graph (as in a captured model forward).
    g_main = [capture(lambda st=st: step(st)) for st in sets]
    g_steps = None
    if rotate:
        g_steps = capture(lambda: [step(sets[i % n_copies]) for i in range(args.steps)])
    for g in g_main:
        g.replay()
    if g_steps is not None:
        g_steps.replay()
    torch.cuda.synchronize(dev)

    # ---- device-timed region: inputs resident in HBM ----
    clocks = ClockSampler(dev.index if dev.index is not None else 0)
    clocks.start()
    time.sleep(0.1)  # the sampler is running before the timed region starts
    total_ms = timed([g.replay for g in g_main], args.steps, g_steps.replay if g_steps is not None else None)
    clk = clocks.stop()
    launches = launches_per_step * args.steps
    assert M.moe_read_status(buf.status) == 0, "device status set during the timed region"

    # ---- per-kernel durations: a second set of graphs carries
    # library-recorded events around every kernel, replayed over the same
    # number of steps ----
    M.moe_profile_enable(True)
    g_prof = [capture(lambda st=st: step(st)) for st in sets]
    M.moe_profile_enable(False)
    for g in g_prof:
        g.replay()
    torch.cuda.synchronize(dev)
    stages = {k_: [0.0, 0] for k_ in M.STAGES}
    for _ in range(-(-args.steps // n_copies)):
        # every graph is replayed once per round: each graph's events hold
        # its latest replay
        for g in g_prof:
            if not rotate:
                flush.zero_()
            g.replay()
        torch.cuda.synchronize(dev)
        for k_, (ms, c) in M.moe_profile_collect(release=False).items():
            stages[k_][0] += ms
            stages[k_][1] += c
    M.moe_profile_collect(release=True)

    # ---- the same steps enqueued eagerly from Python (no graph), for context ----
    eager_ms = timed([lambda st=st: step(st) for st in sets], args.steps)

    # ---- end to end through the public API with pinned host buffers ----
    io_h = torch.empty(io_bytes, dtype=torch.uint8).pin_memory()
    x_h, lg_h = io_views(io_h)
    x_h.copy_(torch.from_numpy(np.ascontiguousarray(inp.x).view(np.int16)).view(torch.bfloat16))
    lg_h.copy_(torch.from_numpy(inp.logits))
    out_h = torch.empty((cfg.T, cfg.d), dtype=torch.bfloat16).pin_memory()

    def e2e_step(st):
        st["io"].copy_(io_h, non_blocking=True)  # x and logits, one copy
        step(st)
        out_h.copy_(buf.out, non_blocking=True)

    e2e_step(sets[0])
    torch.cuda.synchronize(dev)
    g_e2e = [capture(lambda st=st: e2e_step(st)) for st in sets]
    g_e2e_steps = None
    if rotate:
        g_e2e_steps = capture(lambda: [e2e_step(sets[i % n_copies]) for i in range(args.steps)])
        g_e2e_steps.replay()
        torch.cuda.synchronize(dev)
    e2e_ms = timed([g.replay for g in g_e2e], args.steps, g_e2e_steps.replay if g_e2e_steps is not None else None)
    assert torch.equal(out_h.view(torch.int16), buf.out.cpu().view(torch.int16))
    del g_main, g_prof, g_e2e, g_steps, g_e2e_steps

    if fp8:
        sec_per_step = total_ms / args.steps / 1e3
        peaks, peak_src = load_peaks()
        res = {
            "value": round(whole_job_tflops(world, alg["flops_total"], total_ms, args.steps), 4), "unit": "TFLOPS",
            "ms_per_step": round(total_ms / args.steps, 5), "tokens_per_s": round(world * cfg.T / sec_per_step, 1),
            "config": dict(job_config(cfg, world, alg["U"]), weights="fp8 e4m3, power-of-two scale per 32 K values"),
            "stages_us": {k: round(v[0] / max(v[1], 1) * 1e3, 2) for k, v in stages.items() if v[1]},
            "roofline": roofline(cfg, alg, stages, total_ms, args.steps, launches_per_step, rotate, peaks, peak_src),
            "e2e": {"value": round(whole_job_tflops(world, alg["flops_total"], e2e_ms, args.steps), 4),
                    "unit": "TFLOPS", "ms_per_step": round(e2e_ms / args.steps, 5),
                    "h2d_bytes_per_step": int(io_bytes), "d2h_bytes_per_step": int(cfg.T * cfg.d * 2)},
            "gpu_launches": int(launches), "launches_per_step": int(launches_per_step),
            "clocks": {k: clk[k] for k in ("sm_mhz", "sm_max_mhz", "reasons")},
        }
        res["roofline"]["traffic"] = None
        res["roofline"]["traffic_vs_algorithmic"] = None
        del sets, buf, flush
        torch.cuda.synchronize(dev)
        torch.cuda.empty_cache()
        return res

    # ---- the gate before the layer (moe_router: x . W_g^T + top-k), on its
    # own: same x copies, a seeded W_g ~ N(0, 0.02), the same timing rule ----
    wg = to_dev(W.router_inputs(1, cfg.d, cfg.E, seed=cfg.seed + 7)[1])
    r_logits = torch.empty((cfg.T, cfg.E), dtype=torch.float32, device=dev)
    r_ids = torch.empty((cfg.T, cfg.k), dtype=torch.int32, device=dev)
    r_w = torch.empty((cfg.T, cfg.k), dtype=torch.float32, device=dev)

    def router_call(st):
        M.moe_router(st["x"], wg, cfg.k, r_logits, r_ids, r_w, **rk)
        return M.moe_last_launch_count()

    r_launches = router_call(sets[0])
    torch.cuda.synchronize(dev)
    g_router = [capture(lambda st=st: router_call(st)) for st in sets]
    g_router_steps = None
    if rotate:
        g_router_steps = capture(lambda: [router_call(sets[i % n_copies]) for i in range(args.steps)])
        g_router_steps.replay()
        torch.cuda.synchronize(dev)
    router_ms = timed([g.replay for g in g_router], args.steps,
                      g_router_steps.replay if g_router_steps is not None else None)
    del g_router, g_router_steps

    # ---- the backward (moe_backward: dx, dW13, dW2, dL/dw) on the 128-row
    # layout, with a seeded dL/dout per input copy; same timing rule ----
    backward = None
    if cfg.block_m == 128 and not args.no_backward:
        grads = M.MoEGradBuffers(cfg.T, cfg.d, cfg.F, cfg.E, cfg.k, cfg.act, cfg.n_shared, dev)
        for i, st in enumerate(sets):
            st["dout"] = to_dev(W.grad_output(cfg.T, cfg.d, seed=cfg.seed + 50 + i))

        def bwd_call(st):
            grads.backward(buf, st["x"], st["w13"], st["w2"], st["dout"], st["w13s"], st["w2s"])
            return M.moe_last_launch_count()

        b_launches = 0
        for i in range(args.warmup):
            b_launches = bwd_call(sets[i % n_copies])
        torch.cuda.synchronize(dev)
        g_bwd = [capture(lambda st=st: bwd_call(st)) for st in sets]
        g_bwd_steps = None
        if rotate:
            g_bwd_steps = capture(lambda: [bwd_call(sets[i % n_copies]) for i in range(args.steps)])
            g_bwd_steps.replay()
            torch.cuda.synchronize(dev)
        bwd_ms = timed([g.replay for g in g_bwd], args.steps, g_bwd_steps.replay if g_bwd_steps is not None else None)
        assert M.moe_read_status(buf.status) == 0, "device status set during the backward"
        M.moe_profile_enable(True)
        g_bprof = [capture(lambda st=st: bwd_call(st)) for st in sets]
        M.moe_profile_enable(False)
        b_stages = {k_: [0.0, 0] for k_ in M.STAGES}
        for _ in range(-(-args.steps // n_copies)):
            for g in g_bprof:
                if not rotate:
                    flush.zero_()
                g.replay()
            torch.cuda.synchronize(dev)
            for k_, (ms, c) in M.moe_profile_collect(release=False).items():
                b_stages[k_][0] += ms
                b_stages[k_][1] += c
        M.moe_profile_collect(release=True)
        del g_bwd, g_bwd_steps, g_bprof
        rows = cfg.T * cfg.k + cfg.T * cfg.n_shared
        # algorithmic: dh (2 rows d F), dx (2 rows n1 d), dW13 (2 rows n1 d),
        # dW2 (2 rows d F) = twice the forward; the recomputed gate/up
        # pre-activations (2 rows n1 d) are reported on top
        b_flops = 2 * cfg.flops_total()
        recompute = 2 * rows * cfg.n1 * cfg.d
        b_s = bwd_ms / args.steps / 1e3
        bst = {k: round(v[0] / max(v[1], 1) * 1e3, 2) for k, v in b_stages.items() if v[1]}
        dom = max(("bwd_recompute", "bwd_dh_gemm", "bwd_dx_gemm", "bwd_dw13_gemm", "bwd_dw2_gemm"),
                  key=lambda k_: b_stages[k_][0])
        dom_flops = {"bwd_recompute": recompute, "bwd_dh_gemm": 2 * rows * cfg.d * cfg.F,
                     "bwd_dx_gemm": 2 * rows * cfg.n1 * cfg.d, "bwd_dw13_gemm": 2 * rows * cfg.n1 * cfg.d,
                     "bwd_dw2_gemm": 2 * rows * cfg.d * cfg.F}[dom]
        dom_s = b_stages[dom][0] / max(b_stages[dom][1], 1) / 1e3
        peaks_b, _ = load_peaks()
        backward = {"ms_per_step": round(bwd_ms / args.steps, 5),
                    "value": round(world * b_flops / b_s / 1e12, 4), "unit": "TFLOPS",
                    "algorithmic_flops": int(b_flops), "recompute_flops": int(recompute),
                    "tflops_incl_recompute": round(world * (b_flops + recompute) / b_s / 1e12, 4),
                    "launches_per_step": int(b_launches), "gpu_launches": int(b_launches * args.steps),
                    "stages_us": bst,
                    "roofline": {"bound": "tensor", "kernel": dom, "unit": "TFLOP/s",
                                 "achieved": round(dom_flops / dom_s / 1e12, 2), "peak": peaks_b["bf16_tflops"],
                                 "frac": round(dom_flops / dom_s / 1e12 / peaks_b["bf16_tflops"], 4),
                                 "per_launch_us": round(dom_s * 1e6, 2), "algorithmic_flops": int(dom_flops)}}
        del grads
        for st in sets:
            st.pop("dout", None)

    sec_per_step = total_ms / args.steps / 1e3
    value = whole_job_tflops(world, alg["flops_total"], total_ms, args.steps)
    e2e_value = whole_job_tflops(world, alg["flops_total"], e2e_ms, args.steps)
    peaks, peak_src = load_peaks()
    roof = roofline(cfg, alg, stages, total_ms, args.steps, launches_per_step, rotate, peaks, peak_src)

    r_s = router_ms / args.steps / 1e3
    r_flops = 2.0 * cfg.T * cfg.E * cfg.d
    r_bytes = cfg.T * cfg.d * 2 + cfg.E * cfg.d * 2 + cfg.T * cfg.E * 4 + cfg.T * cfg.k * 8
    r_t_min = max(r_flops / (peaks["bf16_tflops"] * 1e12), r_bytes / (peaks["hbm_gbs"] * 1e9))
    router = {"us_per_call": round(r_s * 1e6, 2), "launches": int(r_launches),
              "tflops": round(r_flops / r_s / 1e12, 3), "gbs": round(r_bytes / r_s / 1e9, 1),
              "algorithmic_flops": int(r_flops), "algorithmic_bytes": int(r_bytes),
              "roofline_frac": round(r_t_min / r_s, 4),
              "roofline_note": "time at the slower of FLOPs / burst bf16 peak and bytes / HBM copy bandwidth, "
                               "over the measured time"}

    res = {
        "value": round(value, 4), "unit": "TFLOPS", "ms_per_step": round(total_ms / args.steps, 5),
        "tokens_per_s": round(world * cfg.T / sec_per_step, 1),
        "config": job_config(cfg, world, alg["U"]),
        "timing": {"l2": (f"inputs larger than L2: steps run back to back, each on one of {n_copies} copies of "
                          f"x, logits and the expert weights ({touched / 1e6:.1f} MB of weights read per step; "
                          f"a copy is reused after >= 2x L2 of other data)") if rotate else
                         "flushed before every timed step (write of 2x L2), outside the step's events",
                   "launch": ("one CUDA graph of the K timed steps, kernels chained by programmatic dependent "
                              "launch") if rotate else
                             "CUDA graph of the step, kernels chained by programmatic dependent launch"},
        "ms_per_step_eager": round(eager_ms / args.steps, 5),
        "stages_us": {k: round(v[0] / max(v[1], 1) * 1e3, 2) for k, v in stages.items() if v[1]},
        "stages_source": "CUDA events around each kernel in replayed graphs of the step",
        "roofline": roof,
        "router": router,
        "e2e": {"value": round(e2e_value, 4), "unit": "TFLOPS", "ms_per_step": round(e2e_ms / args.steps, 5),
                "h2d_bytes_per_step": int(io_bytes),
                "d2h_bytes_per_step": int(cfg.T * cfg.d * 2)},
        "gpu_launches": int(launches),
        "launches_per_step": int(launches_per_step),
        "clocks": {k: clk[k] for k in ("sm_mhz", "sm_max_mhz", "reasons")},
    }
    if backward is not None:
        res["backward"] = backward
    # free this workload's device memory before the next one
    del sets, buf, wg, r_logits, r_ids, r_w, flush
    torch.cuda.synchronize(dev)
    torch.cuda.empty_cache()
    if rank == 0 and world == 1 and cpu_seconds > 0:
        res["cpu_baseline"] = cpu_baseline(inp, cpu_seconds)
    return res


def run_ours(args):
    import torch

    from grouped_gemm_gating_b200 import moe as M

    world, rank, local, pg = dist_setup(args.gpus)
    dev = torch.device("cuda", local if world > 1 else 0)
    M.load_library()
    names = ORDER if args.workload == "all" else (args.workload,)
    head = HEADLINE if args.workload == "all" else args.workload
    results = {}
    for name in names:
        cpu_s = 0.0 if args.no_cpu_baseline else (10.0 if name == head else 3.0)
        results[name] = measure_workload(name, args, dev, pg, world, rank, cpu_s)
    if args.workload == "all" or args.fp8:
        # the bandwidth-bound shapes again with fp8 expert weights
        for name in [n for n in names if W.CONFIGS[n].block_m <= 64 and n != "tiny"]:
            results[name + "_fp8"] = measure_workload(name, args, dev, pg, world, rank, 0.0, fp8=True)
    h = results[head]
    line = {
        "metric": METRIC, "value": h["value"], "unit": "TFLOPS", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": h["ms_per_step"],
        "tokens_per_s": h["tokens_per_s"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded; random-init expert weights ~N(0,0.02))",
        "config": h["config"],
        "timing": h["timing"],
        "ms_per_step_eager": h["ms_per_step_eager"],
        "stages_us": h["stages_us"],
        "stages_source": h["stages_source"],
        "roofline": h["roofline"],
        "router": h["router"],
        "backward": h.get("backward"),
        "e2e": h["e2e"],
        "gpu_launches": h["gpu_launches"],
        "clocks": h["clocks"],
    }
    if "cpu_baseline" in h:
        line["cpu_baseline"] = h["cpu_baseline"]
    if len(results) > 1:
        line["workloads"] = dict(results)
    if pg is not None:
        pg.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_reference(args):
    """The CPU oracle, as it stands, on the host cores: the headline
    workload's config, metric and unit, the same K steps after the same W
    warm-up steps, each step a bounded token sample of the workload."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    name = HEADLINE if args.workload == "all" else args.workload
    cfg = W.CONFIGS[name]
    inp = W.make_inputs(cfg)
    import oracle
    ids, _ = oracle.route(inp.logits, cfg.k, cfg.n_group, cfg.topk_group, cfg.group_score,
                          bool(cfg.renormalize), cfg.routed_scaling)
    experts_hit = int(np.unique(ids).size)
    cb = time_oracle(inp, steps=args.steps, warmup=args.warmup, max_steps=args.steps)
    info = cpu_info()
    line = {
        "impl": "reference", "metric": METRIC, "value": round(cb["value"], 6), "unit": "TFLOPS",
        "n_gpus": world, "steps": cb["steps"], "warmup": args.warmup,
        "ms_per_step": round(cb["ms_per_step"], 3), "tokens_per_s": round(cb["tokens_per_s"], 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded)",
        "config": job_config(cfg, world, experts_hit),
        "cpu_baseline": {"value": round(cb["value"], 6), "unit": "TFLOPS", "cores": cb["cores"],
                         "kind": "oracle", "sample": cb["sample"], "host_nproc": info["nproc"],
                         "cpu_model": info["model"]},
        "e2e": {"value": round(cb["value"], 6), "unit": "TFLOPS", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
