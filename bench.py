"""Benchmark of the hot path: metadata prepare + KV append + sparse attention.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--only]

A step is one pass of the whole path (metadata prepare, KV append,
attention) over one batch of a workload.  The headline workload is the
GPT-OSS-like paged decode (B=32, S_q=1, H_q=64, H_kv=8, D=64, block 16,
lengths U[512, 8192], causal window 128, learned sinks, fp16); unless
--only is given, every other named workload (tiny fp32 decode,
selected-token bf16 decode, local-plus-selected INT8 decode, ragged prefill,
windowed chunked prefill, the QKV-prologue decode) is measured the same way
and listed under "workloads" in the same JSON line.  Inputs are resident in
HBM when the timed region starts; each step reads a different one of enough
independent device instances that the attended bytes of one cycle exceed
twice the L2, so every step reads its keys from HBM.  The K timed steps
are captured as one CUDA graph (one per 1000 steps) and timed with CUDA
events on the launching stream.

Under torchrun (N > 1) every rank runs its own batch (weak scaling, no data
collective); the time is the maximum over ranks.

Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "decode attended-KV GB/s and tokens/s per B200, % of HBM roofline"
DEFAULT_WORKLOAD = "gptoss_paged_decode_f16"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


# ---------------------------------------------------------------------------
# bookkeeping shared by both arms
# ---------------------------------------------------------------------------

def _token_set(wl, tokens):
    return set(range(wl.T)) if tokens is None else {int(t) for t in tokens}


def attended_kv_bytes(wl, tokens=None) -> int:
    """Algorithmic attended K+V bytes of one step: for every (request, kv
    head), the union over the request's query tokens (those in ``tokens``
    when given) of the attended keys, times D times the cache element size,
    for K and V."""
    elt = {"f32": 4, "f16": 2, "bf16": 2, "i8": 1}[wl.cache]
    keep = _token_set(wl, tokens)
    total = 0
    a = wl.arrays
    cu = [int(x) for x in a["cu_seqlens_q"]]
    for b in range(wl.B):
        q, p0 = wl.q_lens[b], wl.past[b]
        toks = [t for t in range(cu[b], cu[b + 1]) if t in keep]
        if q == 0 or not toks:
            continue
        L = p0 + q
        for h in range(wl.H_kv):
            n = 0
            if wl.sel_mode == "main":
                rows = [b] if wl.sel_per_request else toks
                s = set()
                for r in rows:
                    s |= {int(i) for i in a["selected_idx"][r, h] if 0 <= i < L}
                n = len(s)
            else:
                ps = [p0 + t - cu[b] for t in toks]
                lo = max(0, min(ps) - wl.window + 1) if wl.window > 0 else 0
                n = max(ps) + 1 - lo
                if wl.sel_mode == "aux":
                    rows = [b] if wl.sel_per_request else toks
                    s = set()
                    for r in rows:
                        s |= {int(i) for i in a["selected_idx"][r, h] if 0 <= i < int(a["aux_seqlens"][b])}
                    n += len(s)
            total += n * wl.D * elt * 2
    return total


def attention_flops(wl, tokens=None) -> int:
    """Algorithmic FLOPs of QK^T and PV over the attended (causal) pairs of
    the query tokens (those in ``tokens`` when given)."""
    keep = _token_set(wl, tokens)
    pairs = 0
    t = 0
    for b in range(wl.B):
        q, p0 = wl.q_lens[b], wl.past[b]
        for i in range(q):
            if t in keep:
                p = p0 + i
                lo = max(0, p - wl.window + 1) if wl.window > 0 else 0
                pairs += p - lo + 1
            t += 1
    return 4 * wl.D * wl.H_q * pairs


def is_prefill(wl) -> bool:
    return wl.max_seqlen_q > 16 and wl.sel_mode is None


def work_of(wl, tokens=None):
    """(amount, unit scale, unit) of the metric for a step over ``tokens``:
    attended K+V bytes in GB/s for decode, attention FLOPs in TFLOP/s for
    prefill."""
    if is_prefill(wl):
        return attention_flops(wl, tokens), 1e12, "TFLOP/s"
    return attended_kv_bytes(wl, tokens), 1e9, "GB/s"


L2_NOTE = ("inputs larger than L2: each step reads a different one of several independent device "
           "copies of the workload, whose attended bytes per cycle exceed twice the L2")


def workload_config(wl, world: int) -> dict:
    """The `config` object of a JSON line: the workload, identical in both arms."""
    return {"workload": wl.name, "B": wl.B, "S_q": wl.max_seqlen_q, "T": wl.T, "H_q": wl.H_q,
            "H_kv": wl.H_kv, "D": wl.D, "block_size": wl.block_size, "window": wl.window,
            "max_seqlen_k": wl.max_seqlen_k, "selection": wl.sel_mode, "sel_width": wl.sel_width,
            "sinks": wl.has_sinks, "act": wl.act, "cache": wl.cache,
            "prologue": bool(getattr(wl, "prologue", None)),
            "parallelism": f"dp{world}" if world > 1 else "single", "l2": L2_NOTE}


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return (float(pk["hbm_gbs"]), float(pk["bf16_tflops"]),
                float(pk.get("bf16_tflops_sustained", pk["bf16_tflops"])), "measured")
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "selected_token_sparse_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel sources; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    e = rec.get(f"{kernel}|{workload}")
    if not e or e.get("source_hash") != kernel_source_hash():
        return None
    return e.get("dram_bytes_per_launch")


# ---------------------------------------------------------------------------
# distributed helpers (gloo-testable)
# ---------------------------------------------------------------------------

def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def reduce_max(x: float, device=None) -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ---------------------------------------------------------------------------
# clocks
# ---------------------------------------------------------------------------

_REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
            0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
            0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
            0x100: "display_clock_setting"}


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""

    def __init__(self, index: int, period_s: float = 0.005):
        self.index, self.period = index, period_s
        self.samples, self.reasons = [], 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _reasons(self):
        fn = getattr(self.nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            getattr(self.nv, "nvmlDeviceGetCurrentClocksThrottleReasons")
        return int(fn(self.h))

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.reasons |= self._reasons()
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nv is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._t is not None:
            self._t.join()
        if self.nv is not None:   # one sample after the region as well
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.reasons |= self._reasons()
            except Exception:
                pass

    def summary(self):
        if self.nv is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "samples": len(self.samples),
                "reasons": [n for bit, n in _REASONS.items() if self.reasons & bit and bit != 0x1]}


# ---------------------------------------------------------------------------
# the CPU baseline (fp64 oracle)
# ---------------------------------------------------------------------------

def oracle_sample(wl, budget_s: float):
    """Token sample of one oracle step that takes about budget_s / 3 on this
    host: every token when a whole step fits, else evenly spaced tokens (the
    metadata and the append always run in full).  The step's fixed cost and
    its cost per token are estimated from steps over one and over four
    tokens.  Returns the token list, or None for whole steps."""
    from oracle import spa_oracle as O

    def spaced(n):
        return [int(x) for x in np.linspace(0, wl.T - 1, n).round().astype(int)]

    def seconds(tokens):
        t0 = time.perf_counter()
        O.run_step(wl, tokens=tokens)
        return time.perf_counter() - t0

    if wl.T <= 4:
        return None
    seconds(spaced(1))                       # first touch of the arrays
    t1 = seconds(spaced(1))
    t4 = seconds(spaced(4))
    per_tok = max((t4 - t1) / 3.0, 1e-6)
    fixed = max(t1 - per_tok, 0.0)
    n = int((budget_s / 3.0 - fixed) / per_tok)
    if n >= wl.T:
        return None
    return spaced(max(1, n))


def cpu_baseline(wl, budget_s: float = 10.0, max_steps: int = 1000):
    """Time the oracle as it stands on the host: steps of the workload (each
    over a bounded token sample) until the budget is spent.  Returns the
    cpu_baseline object."""
    from oracle import spa_oracle as O
    tokens = oracle_sample(wl, budget_s)
    n = 0
    t0, c0 = time.perf_counter(), time.process_time()
    while n < 1 or (time.perf_counter() - t0 < budget_s and n < max_steps):
        O.run_step(wl, tokens=tokens)
        n += 1
    wall = time.perf_counter() - t0
    cores = max(1, int(round((time.process_time() - c0) / wall)))
    amount, scale, unit = work_of(wl, tokens)
    sample = (f"{n} whole step(s)" if tokens is None else
              f"{n} step(s) over {len(tokens)} of {wl.T} query tokens (metadata and append in full)")
    return {"value": amount / (wall / n) / scale, "unit": unit, "cores": cores,
            "host_cores": host_cores(), "kind": "oracle",
            "sample": sample + " of the same workload, fp64 numpy oracle, single-threaded"}


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

GRAPH_CHUNK = 1000   # steps per captured graph; K steps replay ceil(K / chunk) graphs


class Graphs:
    """K consecutive steps captured as few CUDA graphs as possible (one when
    K <= GRAPH_CHUNK), each step on the next device instance in turn."""

    def __init__(self, stream, step_fns, k: int, start: int = 0):
        import torch
        self.graphs = []
        R = len(step_fns)
        i = start
        left = k
        while left > 0:
            n = min(left, GRAPH_CHUNK)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for j in range(n):
                    step_fns[(i + j) % R]()
            self.graphs.append(g)
            i += n
            left -= n

    def replay(self):
        for g in self.graphs:
            g.replay()

    def upload(self, stream) -> bool:
        """Upload the instantiated graphs to the device ahead of their first
        replay, so that the timed replay does not pay for it."""
        try:
            from cuda.bindings import driver as cu
            for g in self.graphs:
                err, = cu.cuGraphUpload(cu.CUgraphExec(int(g.raw_cuda_graph_exec())),
                                        cu.CUstream(int(stream.cuda_stream)))
                if err != cu.CUresult.CUDA_SUCCESS:
                    return False
            return True
        except Exception:
            return False


# Cycles the GPU spins (torch.cuda._sleep) ahead of the first timing event,
# so that the host has submitted the graphs before the event is recorded:
# the events then bracket device execution only (about 100 us at 1.9 GHz).
LEAD_CYCLES = 200_000


def timed(dev, stream, graphs: Graphs, sampler=None):
    """Device time (ms) of one replay of `graphs`, bracketed by a barrier and a
    synchronize on both sides; the maximum over ranks."""
    import torch
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(dev)
    torch.cuda.synchronize(dev)
    if sampler is not None:
        sampler.__enter__()
    with torch.cuda.stream(stream):
        torch.cuda._sleep(LEAD_CYCLES)
        ev0.record(stream)
        graphs.replay()
        ev1.record(stream)
    torch.cuda.synchronize(dev)
    if sampler is not None:
        sampler.__exit__(None, None, None)
    barrier(dev)
    return reduce_max(ev0.elapsed_time(ev1), dev)


def measure(name, args, dev, rank, world, headline: bool):
    """Time K steps of one workload (and its dominant kernel); returns the
    per-workload result object."""
    import torch

    from selected_token_sparse_b200 import pipeline, spa, workloads as W

    # rank 0 draws the named workload's own seed; other ranks draw other batches
    wl = W.by_name(name) if rank == 0 else W.by_name(name, seed=1000 * rank + len(name))
    amount, scale, unit = work_of(wl)
    prefill = is_prefill(wl)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    K = args.steps if headline else min(args.steps, GRAPH_CHUNK)
    Wm = args.warmup if headline else min(args.warmup, 50)

    # independent device instances so that a cycle's attended bytes exceed 2x L2
    base = pipeline.to_device(wl, dev)
    per_inst = (attended_kv_bytes(wl) if not prefill else 0) + sum(
        base[k].numel() * base[k].element_size() for k in ("q", "k_new", "v_new") if k in base)
    R = args.instances or max(2, min(64, math.ceil(2 * l2 / max(per_inst, 1))))
    insts = []
    for i in range(R):
        d = {k: (v.clone() if k in ("k_cache", "v_cache", "q", "k_new", "v_new", "qkv", "block_table",
                                   "cu_seqlens_q", "past_seqlens", "selected_idx") else v)
             for k, v in base.items()}
        insts.append(pipeline.Step(wl, d, num_splits=args.splits, mode=args.mode))
    del base
    step0 = insts[0]
    plan = spa.attention_plan(step0.args)
    launches_per_step = step0.launches()
    single = launches_per_step == 1
    kind_name = {0: "decode_scalar", 1: "decode_mma", 2: "prefill_tcgen05", 3: "decode_tc"}[plan["kind"]]
    if single:
        kind_name += "_step"

    stream = torch.cuda.Stream(dev)
    torch.cuda.synchronize(dev)
    with torch.cuda.stream(stream):
        for st in insts:      # load modules, set attributes outside capture
            st()
    torch.cuda.synchronize(dev)

    g_warm = Graphs(stream, insts, Wm)
    g_steps = Graphs(stream, insts, K, start=Wm)
    with torch.cuda.stream(stream):
        g_warm.replay()
    uploaded = g_steps.upload(stream)
    torch.cuda.synchronize(dev)
    clk = ClockSampler(dev.index)
    ms = timed(dev, stream, g_steps, clk)
    ms_per_step = ms / K
    del g_steps

    # the dominant kernel: a one-launch step is that kernel; otherwise the
    # step's attention launch alone, over the same rotation
    if single:
        attn_ms = ms_per_step
    else:
        attn = [lambda st=st: spa.run_attention(st.args, st.workspace) for st in insts]
        ka = max(K, R)
        ga_warm = Graphs(stream, attn, Wm)
        ga = Graphs(stream, attn, ka, start=Wm)
        with torch.cuda.stream(stream):
            ga_warm.replay()
        ga.upload(stream)
        torch.cuda.synchronize(dev)
        attn_ms = timed(dev, stream, ga) / ka
        del ga, ga_warm
    del g_warm

    e2e = None
    if headline and not args.no_e2e:
        e2e = measure_e2e(wl, args, dev, stream, insts, amount, scale, unit, world)

    status = int(insts[0].status.item())
    hbm, bf16, bf16_sus, peak_src = load_peaks()
    achieved = amount / (attn_ms * 1e-3) / scale
    if prefill:
        roof = {"bound": "tensor", "achieved": achieved, "peak": bf16, "unit": unit,
                "frac": achieved / bf16, "peak_source": f"{peak_src} bf16 dense burst (fp16 same rate)"}
    else:
        roof = {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": unit,
                "frac": achieved / hbm, "peak_source": f"{peak_src} HBM copy"}
    entry = "spa_prepare_append_attention" if single else "spa_attention"
    roof.update({"kernel": f"{entry} ({kind_name}, 1 launch, {plan['num_splits']} split(s))",
                 "us_per_launch": attn_ms * 1e3, "algorithmic_per_launch": amount,
                 "traffic": recorded_traffic(kind_name, name)})
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl, budget_s=10.0 if headline else 3.0)
    res = {"workload": name, "dtype": wl.act, "value": world * amount / (ms_per_step * 1e-3) / scale, "unit": unit,
           "ms_per_step": ms_per_step, "steps": K, "warmup": Wm,
           "tokens_per_s": world * wl.T / (ms_per_step * 1e-3),
           "algorithmic_per_step": amount, "roofline": roof, "cpu_baseline": cpu, "e2e": e2e,
           "gpu_launches": K * launches_per_step, "launches_per_step": launches_per_step,
           "num_splits": plan["num_splits"], "clocks": clk.summary(), "status": status,
           "config": workload_config(wl, world),
           "run": {"instances": R,
                   "l2": f"rotating {R} device instances, attended+q/k/v bytes per cycle "
                         f"{R * per_inst / 1e6:.0f} MB vs L2 {l2 / 1e6:.0f} MB",
                   "timing": f"{K} steps captured in {math.ceil(K / GRAPH_CHUNK)} CUDA graph(s)"
                             f"{' uploaded before the timed replay' if uploaded else ''}; CUDA events on the "
                             "launching stream, recorded after a GPU-side lead so that they bracket device "
                             "execution",
                   "step_entry": ("spa_prepare_qkv_append + spa_attention" if getattr(wl, "prologue", None) else
                                  {"step": "spa_prepare_append_attention",
                                   "prepare_append": "spa_prepare_append_kv + spa_attention",
                                   "staged": "spa_prepare_metadata + spa_append_kv + spa_attention"}[args.mode])}}
    del insts
    torch.cuda.empty_cache()
    return res


def select_bytes(sw) -> int:
    """Algorithmic bytes of one selection-producer launch: every candidate
    score read once (keys 0..bound of each row) and every output slot written."""
    cand = sum(min(int(b), sw.n_keys - 1) + 1 for b in sw.bound if b >= 0)
    return 4 * sw.H * cand + 4 * sw.R * sw.H * sw.sel_width


def measure_select(name, args, dev, rank, world):
    """Time K launches of the selection producer (spa_select_topk) over
    rotating device copies of its scores."""
    import torch

    from selected_token_sparse_b200 import spa, workloads as W
    sw = getattr(W, name)() if rank == 0 else getattr(W, name)(seed=1000 * rank + 7)
    amount = select_bytes(sw)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    R = args.instances or max(2, min(64, math.ceil(2 * l2 / amount)))
    K = min(args.steps, GRAPH_CHUNK)
    Wm = min(args.warmup, 50)
    sc0 = torch.from_numpy(sw.scores).to(dev)
    bound = torch.from_numpy(sw.bound).to(dev)
    scores = [sc0.clone() for _ in range(R)]
    del sc0
    outs = [torch.empty(sw.R, sw.H, sw.sel_width, dtype=torch.int32, device=dev) for _ in range(R)]
    fns = [lambda i=i: spa.select_topk(scores[i], bound, sw.top_k, sw.sel_width, out=outs[i]) for i in range(R)]
    stream = torch.cuda.Stream(dev)
    torch.cuda.synchronize(dev)
    with torch.cuda.stream(stream):
        for f in fns:
            f()
    torch.cuda.synchronize(dev)
    g_warm = Graphs(stream, fns, Wm)
    g = Graphs(stream, fns, K, start=Wm)
    with torch.cuda.stream(stream):
        g_warm.replay()
    g.upload(stream)
    torch.cuda.synchronize(dev)
    clk = ClockSampler(dev.index)
    ms = timed(dev, stream, g, clk) / K
    hbm, _, _, peak_src = load_peaks()
    achieved = amount / (ms * 1e-3) / 1e9
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        from oracle import spa_oracle as O
        n, t0, c0 = 0, time.perf_counter(), time.process_time()
        while n < 1 or time.perf_counter() - t0 < 3.0:
            O.select_topk(sw.scores, sw.bound, sw.top_k, sw.sel_width)
            n += 1
        wall = time.perf_counter() - t0
        cpu = {"value": amount / (wall / n) / 1e9, "unit": "GB/s",
               "cores": max(1, int(round((time.process_time() - c0) / wall))), "host_cores": host_cores(),
               "kind": "oracle", "sample": f"{n} whole call(s) of the same workload, numpy/Python oracle"}
    res = {"workload": name, "dtype": "f32", "value": world * amount / (ms * 1e-3) / 1e9, "unit": "GB/s",
           "ms_per_step": ms, "steps": K, "warmup": Wm, "algorithmic_per_step": amount,
           "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                        "peak_source": f"{peak_src} HBM copy", "kernel": "spa_select_topk (select_topk_kernel, 1 launch)",
                        "us_per_launch": ms * 1e3, "algorithmic_per_launch": amount,
                        "traffic": recorded_traffic("select_topk", name)},
           "cpu_baseline": cpu, "gpu_launches": K, "launches_per_step": 1, "num_splits": 1,
           "clocks": clk.summary(), "status": 0,
           "config": {"workload": name, "R": sw.R, "H_kv": sw.H, "n_keys": sw.n_keys, "top_k": sw.top_k,
                      "sel_width": sw.sel_width, "scores": "f32 N(0,1)",
                      "parallelism": f"dp{world}" if world > 1 else "single", "l2": L2_NOTE},
           "run": {"instances": R, "timing": f"{K} launches captured in one CUDA graph; CUDA events"}}
    del g, g_warm, scores, outs
    torch.cuda.empty_cache()
    return res


def measure_e2e(wl, args, dev, stream, insts, amount, scale, unit, world):
    """The metric end to end through the Python API: every step copies its
    inputs from pinned host memory to the device and reads the output back."""
    import torch

    from selected_token_sparse_b200 import pipeline
    R = len(insts)
    host = pipeline.to_device(wl, pin=True)
    packed = bool(getattr(wl, "prologue", None) and wl.prologue.get("packed"))
    inputs = (("qkv",) if packed else ("q", "k_new", "v_new")) + (
        "cu_seqlens_q", "past_seqlens", "block_table", "selected_idx", "position_ids")
    names = [n for n in inputs if n in host]
    # a step's inputs travel as ONE host->device copy: they sit in one pinned
    # host buffer and, on the device, in one buffer whose 256-byte-aligned
    # slices are the tensors the step reads (the caches stay per instance)
    offs, total = {}, 0
    for n in names:
        offs[n] = total
        total += (host[n].numel() * host[n].element_size() + 255) // 256 * 256
    hbuf = torch.empty(total, dtype=torch.uint8, pin_memory=True)
    for n in names:
        nb = host[n].numel() * host[n].element_size()
        hbuf[offs[n]:offs[n] + nb].copy_(host[n].contiguous().view(-1).view(torch.uint8))
    e2e_insts = []
    for st in insts:
        dbuf = torch.empty(total, dtype=torch.uint8, device=dev)
        d2 = dict(st.d)
        for n in names:
            nb = host[n].numel() * host[n].element_size()
            d2[n] = dbuf[offs[n]:offs[n] + nb].view(host[n].dtype).view(host[n].shape)
            d2[n].copy_(st.d[n])
        e2e_insts.append((dbuf, pipeline.Step(wl, d2, num_splits=args.splits, want_lse=False,
                                              mode=args.mode)))
    out_host = torch.empty(insts[0].out.shape, dtype=insts[0].out.dtype, pin_memory=True)
    d2h = out_host.numel() * out_host.element_size()
    ke = min(args.steps, 2000)

    def e2e_step(i):
        dbuf, st = e2e_insts[i % R]
        dbuf.copy_(hbuf, non_blocking=True)
        st()
        out_host.copy_(st.out, non_blocking=True)

    with torch.cuda.stream(stream):
        for i in range(min(args.warmup, 50)):
            e2e_step(i)
    torch.cuda.synchronize(dev)
    barrier(dev)
    x0, x1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        x0.record(stream)
        for i in range(ke):
            e2e_step(i)
        x1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = reduce_max(x0.elapsed_time(x1), dev) / ke
    return {"value": world * amount / (e2e_ms * 1e-3) / scale, "unit": unit,
            "h2d_bytes_per_step": int(total), "d2h_bytes_per_step": int(d2h),
            "ms_per_step": e2e_ms, "steps": ke}


def measure_seq_shard(args, dev, rank, world):
    """One batch's keys split across the ranks by position (sequence-sharded
    split-KV): every rank attends its kv_range (partial state, no sink), the
    states are all-gathered over NCCL and merged with the sink.  Strong
    scaling: the total work is the same batch at every N."""
    import torch

    from selected_token_sparse_b200 import pipeline, shard, spa, workloads as W
    wl = W.by_name(args.workload)        # the same requests on every rank
    amount, scale, unit = work_of(wl)
    a = wl.arrays
    lengths = [p + q for p, q in zip(wl.past, wl.q_lens)]
    rng = shard.sequence_ranges(lengths, world, rank, wl.block_size)
    d = pipeline.to_device(wl, dev)
    st = pipeline.Step(wl, d, want_lse=True)
    st()                                 # metadata and append (every rank; the new rows land in its cache)
    torch.cuda.synchronize(dev)
    bt = torch.from_numpy(shard.shard_block_table(a["block_table"], rng, wl.block_size)).to(dev)
    meta = dict(st.meta, cu_seqlens_q=d["cu_seqlens_q"])
    po = torch.empty(wl.T, wl.H_q, wl.D, dtype=torch.float32, device=dev)
    pl = torch.empty(wl.T, wl.H_q, dtype=torch.float32, device=dev)
    kw = dict(st.kw)
    if wl.sel_mode == "aux" and rank != 0:
        kw.update(selected_idx=None, sel_target=0, aux_k=None, aux_v=None, aux_seqlens=None)
    rng_d = torch.from_numpy(rng).to(dev)    # the arguments hold its address for every step
    args_p = spa.attention_args(d["q"], d["k_cache"], d["v_cache"], bt, meta, max_seqlen_q=wl.max_seqlen_q,
                                max_seqlen_k=wl.max_seqlen_k, out=po, lse=pl, num_splits=args.splits,
                                status=st.status, kv_range=rng_d, partial=True, **kw)
    ws = spa.new_workspace(spa.workspace_size(args_p), dev)
    out = torch.empty_like(st.out)
    lse = torch.empty(wl.T, wl.H_q, dtype=torch.float32, device=dev)
    gpo = torch.empty(world, *po.shape, dtype=po.dtype, device=dev)
    gpl = torch.empty(world, *pl.shape, dtype=pl.dtype, device=dev)

    def step():
        spa.run_attention(args_p, ws)
        if world > 1:
            import torch.distributed as dist
            dist.all_gather_into_tensor(gpo, po)
            dist.all_gather_into_tensor(gpl, pl)
            spa.merge_partials(gpo, gpl, d.get("sinks"), out, lse)
        else:
            spa.merge_partials(po.unsqueeze(0), pl.unsqueeze(0), d.get("sinks"), out, lse)

    stream = torch.cuda.current_stream(dev)
    K, Wm = args.steps, args.warmup
    for _ in range(Wm):
        step()
    torch.cuda.synchronize(dev)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(dev)
    torch.cuda.synchronize(dev)
    clk = ClockSampler(dev.index)
    with clk:
        ev0.record(stream)
        for _ in range(K):
            step()
        ev1.record(stream)
        torch.cuda.synchronize(dev)
    barrier(dev)
    ms = reduce_max(ev0.elapsed_time(ev1), dev) / K
    status = int(st.status.item())
    hbm, _, _, peak_src = load_peaks()
    return {"workload": wl.name, "dtype": wl.act, "value": amount / (ms * 1e-3) / scale, "unit": unit,
            "ms_per_step": ms, "steps": K, "warmup": Wm, "tokens_per_s": wl.T / (ms * 1e-3),
            "algorithmic_per_step": amount, "status": status, "clocks": clk.summary(),
            "scaling": "strong", "gpu_launches": K * 2,
            "config": dict(workload_config(wl, world), parallelism=f"sequence-sharded split-KV over {world} rank(s)"),
            "run": {"timing": "eager launches (partial attention, NCCL all-gather of the partial states, merge); "
                              "CUDA events on the current stream, maximum over ranks",
                    "roofline_per_rank_bytes": amount / world, "hbm_peak": hbm, "peak_source": peak_src}}


def run_ours(args):
    import torch
    import torch.distributed as dist

    from selected_token_sparse_b200 import workloads as W

    rank, world, local = dist_env()
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", device_id=torch.device("cuda", local),
                                timeout=__import__("datetime").timedelta(seconds=120))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    if args.seq_shard:
        r = measure_seq_shard(args, dev, rank, world)
        line = {"metric": METRIC, "value": r["value"], "unit": r["unit"], "n_gpus": world, "steps": r["steps"],
                "warmup": r["warmup"], "ms_per_step": r["ms_per_step"], "higher_is_better": True,
                "scaling": "strong", "vs_baseline": None, "dtype": r["dtype"], "data": "synthetic",
                "config": r["config"], "tokens_per_s": r["tokens_per_s"], "gpu_launches": r["gpu_launches"],
                "clocks": r["clocks"], "status": r["status"], "run": r["run"], "roofline": None,
                "cpu_baseline": None, "e2e": None}
        if world > 1:
            dist.barrier(device_ids=[dev.index])
            dist.destroy_process_group()
        if rank == 0:
            print(json.dumps(line), flush=True)
        return
    if args.workload in W.SELECTION_WORKLOADS:   # the selection producer as the headline
        results = [measure_select(args.workload, args, dev, rank, world)]
        results[0]["e2e"] = None
    else:
        names = [args.workload]
        if not args.only:
            names += [n for n in W.WORKLOADS + W.PROLOGUE_WORKLOADS if n != args.workload]
        results = [measure(n, args, dev, rank, world, headline=(i == 0)) for i, n in enumerate(names)]
        if not args.only:
            results += [measure_select(n, args, dev, rank, world) for n in W.SELECTION_WORKLOADS]
    h = results[0]
    line = {
        "metric": METRIC, "value": h["value"], "unit": h["unit"], "n_gpus": world, "steps": h["steps"],
        "warmup": h["warmup"], "ms_per_step": h["ms_per_step"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": h["dtype"], "data": "synthetic",
        "config": h["config"], "tokens_per_s": h.get("tokens_per_s"),
        "algorithmic_per_step": h["algorithmic_per_step"],
        "roofline": h["roofline"], "cpu_baseline": h["cpu_baseline"], "e2e": h["e2e"],
        "gpu_launches": h["gpu_launches"], "clocks": h["clocks"], "status": h["status"],
        "run": h["run"],
        "workloads": [{k: v for k, v in r.items() if k != "e2e"} for r in results],
    }
    if world > 1:
        dist.barrier(device_ids=[dev.index])
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# reference arm: the oracle on the host cores
# ---------------------------------------------------------------------------

def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    from oracle import spa_oracle as O
    from selected_token_sparse_b200 import workloads as W
    wl = W.by_name(args.workload)
    budget = 120.0 / max(1, args.steps + args.warmup)     # seconds per step
    tokens = oracle_sample(wl, 3.0 * budget)
    for _ in range(args.warmup):
        O.run_step(wl, tokens=tokens)
    c0 = time.process_time()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        O.run_step(wl, tokens=tokens)
    wall = time.perf_counter() - t0
    cores = max(1, int(round((time.process_time() - c0) / wall)))
    amount, scale, unit = work_of(wl, tokens)
    sec = wall / args.steps
    value = amount / sec / scale
    sample = ("whole steps" if tokens is None else
              f"{len(tokens)} of {wl.T} query tokens per step (metadata and append in full)")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": unit, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(wl, world),
            "cpu_baseline": {"value": value, "unit": unit, "cores": cores, "host_cores": host_cores(),
                             "kind": "oracle", "sample": sample + ", fp64 numpy oracle, single-threaded"},
            "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=100)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, help="the headline workload")
    ap.add_argument("--only", action="store_true", help="measure the headline workload only")
    ap.add_argument("--instances", type=int, default=0)
    ap.add_argument("--splits", type=int, default=0, help="key splits per unit (0 = automatic)")
    ap.add_argument("--mode", choices=["step", "prepare_append", "staged"], default="step",
                    help="entry points of one step: the fused step call, prepare+append then attention, "
                         "or the three staged calls")
    ap.add_argument("--seq-shard", action="store_true",
                    help="split one batch's keys across the ranks (partial states, all-gather, merge)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.steps < 1:
        args.steps = 1
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
