"""Benchmark of the hot path: metadata prepare + KV append + sparse attention.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME]

A step is one pass of the whole path (spa_prepare_metadata, spa_append_kv,
spa_attention) over one batch of the GPT-OSS-like paged decode workload
(B=32, S_q=1, H_q=64, H_kv=8, D=64, block 16, lengths U[512, 8192], causal
window 128, learned sinks, fp16).  Inputs are resident in HBM when the timed
region starts; the step cycles through enough independent cache instances
that the attended bytes of one cycle exceed twice the L2, so every step
reads its keys from HBM.  Steps are replayed from CUDA graphs and timed with
CUDA events on the launching stream.

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

def attended_kv_bytes(wl) -> int:
    """Algorithmic attended K+V bytes of one step: for every (request, kv
    head), the union over the request's query tokens of the attended keys,
    times D times the cache element size, for K and V."""
    elt = {"f32": 4, "f16": 2, "bf16": 2, "i8": 1}[wl.cache]
    total = 0
    a = wl.arrays
    for b in range(wl.B):
        q, p0 = wl.q_lens[b], wl.past[b]
        if q == 0:
            continue
        L = p0 + q
        for h in range(wl.H_kv):
            n = 0
            if wl.sel_mode == "main":
                rows = [b] if wl.sel_per_request else list(range(int(a["cu_seqlens_q"][b]),
                                                                 int(a["cu_seqlens_q"][b + 1])))
                s = set()
                for r in rows:
                    s |= {int(i) for i in a["selected_idx"][r, h] if 0 <= i < L}
                n = len(s)
            else:
                lo = max(0, p0 - wl.window + 1) if wl.window > 0 else 0
                n = L - lo
                if wl.sel_mode == "aux":
                    rows = [b] if wl.sel_per_request else list(range(int(a["cu_seqlens_q"][b]),
                                                                     int(a["cu_seqlens_q"][b + 1])))
                    s = set()
                    for r in rows:
                        s |= {int(i) for i in a["selected_idx"][r, h] if 0 <= i < int(a["aux_seqlens"][b])}
                    n += len(s)
            total += n * wl.D * elt * 2
    return total


def attention_flops(wl) -> int:
    """Algorithmic FLOPs of QK^T and PV over the attended (causal) pairs."""
    pairs = 0
    for b in range(wl.B):
        q, p0 = wl.q_lens[b], wl.past[b]
        for i in range(q):
            p = p0 + i
            lo = max(0, p - wl.window + 1) if wl.window > 0 else 0
            pairs += p - lo + 1
    return 4 * wl.D * wl.H_q * pairs


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

def cpu_baseline(wl, budget_s: float = 12.0, max_steps: int = 1000, min_steps: int = 1):
    """Time the oracle as it stands on the host: whole steps of the workload
    until the budget is spent.  Returns (seconds per step, steps, cores)."""
    from oracle import spa_oracle as O
    n = 0
    t0, c0 = time.perf_counter(), time.process_time()
    while n < min_steps or (time.perf_counter() - t0 < budget_s and n < max_steps):
        O.run_step(wl)
        n += 1
    wall = time.perf_counter() - t0
    cpu = time.process_time() - c0
    cores = max(1, int(round(cpu / wall)))
    return wall / n, n, cores


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def run_ours(args):
    import torch
    import torch.distributed as dist

    from selected_token_sparse_b200 import pipeline, spa, workloads as W

    rank, world, local = dist_env()
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", device_id=torch.device("cuda", local),
                                timeout=__import__("datetime").timedelta(seconds=120))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    seed_off = 100 * rank
    wl = W.by_name(args.workload, seed=None if rank == 0 else 1 + seed_off)
    alg_bytes = attended_kv_bytes(wl)
    flops = attention_flops(wl)
    is_prefill = wl.max_seqlen_q > 16 and wl.sel_mode is None
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size

    # independent device instances so that a cycle's attended bytes exceed 2x L2
    base = pipeline.to_device(wl, dev)
    per_inst = alg_bytes + sum(base[k].numel() * base[k].element_size()
                               for k in ("q", "k_new", "v_new"))
    R = args.instances or max(2, min(64, math.ceil(2 * l2 / max(per_inst, 1))))
    if is_prefill:
        R = args.instances or 2
    insts = []
    for i in range(R):
        d = {k: (v.clone() if k in ("k_cache", "v_cache", "q", "k_new", "v_new", "block_table",
                                   "cu_seqlens_q", "past_seqlens", "selected_idx") else v)
             for k, v in base.items()}
        insts.append(pipeline.Step(wl, d, num_splits=args.splits, mode=args.mode))
    del base
    step0 = insts[0]
    plan = spa.attention_plan(step0.args)
    launches_per_step = step0.launches()
    # one launch per step: the fused step kernel is the whole step
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

    # CUDA graphs: one per instance, plus one chaining all instances
    def capture(fn):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            fn()
        return g

    g_one = [capture(st) for st in insts]
    g_all = capture(lambda: [st() for st in insts])

    def attn_only(st):
        def f():
            spa.run_attention(st.args, st.workspace)   # the step's own attention call
        return f

    ga_one = [capture(attn_only(st)) for st in insts]
    ga_all = capture(lambda: [attn_only(st)() for st in insts])

    def replay(graph_all, graph_one, k):
        q, r = divmod(k, R)
        for _ in range(q):
            graph_all.replay()
        for i in range(r):
            graph_one[i].replay()

    K, Wm = args.steps, args.warmup
    with torch.cuda.stream(stream):
        replay(g_all, g_one, Wm)
    torch.cuda.synchronize(dev)

    # ---- timed region: exactly K steps
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(dev)
    torch.cuda.synchronize(dev)
    with ClockSampler(dev.index) as clk:
        with torch.cuda.stream(stream):
            ev0.record(stream)
            replay(g_all, g_one, K)
            ev1.record(stream)
        torch.cuda.synchronize(dev)
    barrier(dev)
    ms = ev0.elapsed_time(ev1)
    ms = reduce_max(ms, dev)
    ms_per_step = ms / K

    # ---- dominant kernel alone (same rotation), for the roofline; a fused
    # step is one launch, so the timed steps above time that kernel
    if single:
        attn_ms = ms_per_step
    else:
        with torch.cuda.stream(stream):
            replay(ga_all, ga_one, Wm)
        torch.cuda.synchronize(dev)
        ka = max(K, R)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            replay(ga_all, ga_one, ka)
            e1.record(stream)
        torch.cuda.synchronize(dev)
        attn_ms = e0.elapsed_time(e1) / ka

    # ---- end to end through the Python API with host buffers
    e2e = None
    if not args.no_e2e:
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
        h2d = total
        out_host = torch.empty(step0.out.shape, dtype=step0.out.dtype, pin_memory=True)
        d2h = out_host.numel() * out_host.element_size()
        ke = min(K, 2000)

        def e2e_step(i):
            dbuf, st = e2e_insts[i % R]
            dbuf.copy_(hbuf, non_blocking=True)
            st()
            out_host.copy_(st.out, non_blocking=True)

        with torch.cuda.stream(stream):
            for i in range(min(Wm, 50)):
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
        if is_prefill:
            e2e = {"value": world * flops / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s"}
        else:
            e2e = {"value": world * alg_bytes / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s"}
        e2e.update({"h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                    "ms_per_step": e2e_ms, "steps": ke})

    status = int(insts[0].status.item())
    hbm, bf16, bf16_sus, peak_src = load_peaks()
    if is_prefill:
        achieved = flops / (attn_ms * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": bf16, "unit": "TFLOP/s",
                "frac": achieved / bf16, "peak_source": f"{peak_src} bf16 dense (fp16 same rate)"}
        value = world * flops / (ms_per_step * 1e-3) / 1e12
        unit = "TFLOP/s"
    else:
        achieved = alg_bytes / (attn_ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                "frac": achieved / hbm, "peak_source": f"{peak_src} HBM copy"}
        value = world * alg_bytes / (ms_per_step * 1e-3) / 1e9
        unit = "GB/s"
    entry = "spa_prepare_append_attention" if single else "spa_attention"
    roof.update({"kernel": f"{entry} ({kind_name}, 1 launch, {plan['num_splits']} split(s))",
                 "us_per_launch": attn_ms * 1e3,
                 "algorithmic_per_launch": flops if is_prefill else alg_bytes,
                 "traffic": recorded_traffic(kind_name, args.workload)})

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        sec, n, cores = cpu_baseline(wl)
        cv = (flops / sec / 1e12) if is_prefill else (alg_bytes / sec / 1e9)
        cpu = {"value": cv, "unit": unit, "cores": cores, "kind": "oracle",
               "sample": f"{n} whole step(s) of the same workload (metadata, append, attention "
                         f"for all {wl.T} tokens), fp64 numpy oracle"}

    line = {
        "metric": METRIC, "value": value, "unit": unit, "n_gpus": world, "steps": K,
        "warmup": Wm, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": wl.act, "data": "synthetic",
        "config": {"workload": args.workload, "B": wl.B, "S_q": wl.max_seqlen_q, "H_q": wl.H_q,
                   "H_kv": wl.H_kv, "D": wl.D, "block_size": wl.block_size, "window": wl.window,
                   "max_seqlen_k": wl.max_seqlen_k, "sinks": wl.has_sinks, "cache": wl.cache,
                   "parallelism": f"dp{world}" if world > 1 else "single",
                   "l2": f"rotating {R} device instances, attended+q/k/v bytes per cycle "
                         f"{R * per_inst / 1e6:.0f} MB vs L2 {l2 / 1e6:.0f} MB",
                   "timing": "CUDA graphs of whole steps, CUDA events on the launching stream",
                   "step_entry": {"step": "spa_prepare_append_attention",
                                  "prepare_append": "spa_prepare_append_kv + spa_attention",
                                  "staged": "spa_prepare_metadata + spa_append_kv + spa_attention"}[args.mode],
                   "launches_per_step": launches_per_step,
                   "num_splits": plan["num_splits"]},
        "tokens_per_s": world * wl.T / (ms_per_step * 1e-3),
        "attended_kv_bytes_per_step": alg_bytes,
        "roofline": roof, "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": K * launches_per_step,
        "clocks": clk.summary(), "status": status,
    }
    if world > 1:
        del g_one, g_all, ga_one, ga_all
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
    alg_bytes = attended_kv_bytes(wl)
    flops = attention_flops(wl)
    is_prefill = wl.max_seqlen_q > 16 and wl.sel_mode is None
    budget = 120.0 / max(1, args.steps + args.warmup)     # seconds per step
    # whole steps when they fit the per-step budget, otherwise a token sample
    t0 = time.perf_counter()
    O.run_step(wl)
    full = time.perf_counter() - t0
    frac = 1.0 if full <= budget else max(budget / full, 1.0 / wl.T)
    ntok = max(1, int(round(frac * wl.T)))
    tokens = None if ntok >= wl.T else list(np.linspace(0, wl.T - 1, ntok).astype(int))
    for _ in range(args.warmup):
        O.run_step(wl, tokens=tokens)
    c0 = time.process_time()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        O.run_step(wl, tokens=tokens)
    wall = time.perf_counter() - t0
    cores = max(1, int(round((time.process_time() - c0) / wall)))
    share = 1.0 if tokens is None else len(tokens) / wl.T
    sec = wall / args.steps
    if is_prefill:
        value, unit = share * flops / sec / 1e12, "TFLOP/s"
    else:
        value, unit = share * alg_bytes / sec / 1e9, "GB/s"
    sample = ("whole steps" if tokens is None else
              f"{len(tokens)} of {wl.T} tokens per step (metadata and append in full)")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": unit, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": args.workload},
            "cpu_baseline": {"value": value, "unit": unit, "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=100)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--instances", type=int, default=0)
    ap.add_argument("--splits", type=int, default=0, help="key splits per unit (0 = automatic)")
    ap.add_argument("--mode", choices=["step", "prepare_append", "staged"], default="step",
                    help="entry points of one step: the fused step call, prepare+append then attention, "
                         "or the three staged calls")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
