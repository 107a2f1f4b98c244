"""Warm, in-graph phase breakdown of the decode kernels (warp-MMA and tcgen05)
and of the tcgen05 prefill.

    python -m selected_token_sparse_b200.phase_probe [--workload NAME] [--lib PATH]

Builds (or loads) the probe variant of libspa (build.py --probe: the same
sources compiled with -DSPA_PHASE_PROBE, where thread 0 of every CTA stamps
%globaltimer at the kernel's phase boundaries), captures K steps of the
workload over rotating device instances in one CUDA graph, replays it twice
(warm), clears the stamps, replays it once more and reads back the stamps of
the graph's last step -- a step that ran right after another one, as in the
benchmark.  Prints the median / p90 duration of each phase over the CTAs.

Phase stamps of decode_mma_kernel (those of decode_tc_kernel are listed in
TC_PHASES below):
  0 entry (before griddepcontrol.wait)   1 predecessor complete (wait released)
  2 unit decoded (metadata, fused scan)  3 Q staged, before the candidates
  4 first candidate chunk resolved       5 first K/V stages issued
  6 key loop done (all copies landed)    7 output / partial state written
  8 fused metadata + append tail done    9 split merge done (CTA end)
  10 cluster barrier passed               11 merged rows written (cluster merge)
"""
from __future__ import annotations

import argparse
import ctypes
import math
import os

import numpy as np
import torch

from . import build, pipeline, spa, workloads as W

TC_PHASES = [(0, 1, "wait for the predecessor (PDL)"), (1, 2, "unit metadata (cumulative-length scan)"),
             (2, 3, "producers: to their first candidates"), (3, 4, "producers: candidates of chunk 0"),
             (4, 5, "producers: INT8 staging, tile 0 copied, converted, published"),
             (4, 13, "producers: this step's rows quantised (INT8) and appended"),
             (13, 14, "producers: copies of tiles 0-1 issued"), (14, 15, "producers: tile 0 landed"),
             (15, 5, "producers: tile 0 converted and published"),
             (2, 6, "softmax warps: Q (x key scale, hi / lo) into tensor memory"),
             (6, 7, "softmax warps: wait for S(0)"), (7, 8, "key loop (S, softmax, PV per tile)"),
             (8, 9, "epilogue: normalise, write output / partial"), (9, 10, "split merge"),
             (9, 11, "merge: cluster barrier"), (11, 12, "merge: rows from the workspace"),
             (1, 10, "CTA after the wait"), (0, 10, "CTA incl. the wait")]
PHASES = [(0, 1, "wait for the predecessor (PDL)"), (1, 2, "unit metadata (cumulative-length scan)"),
          (2, 3, "Q rows to shared memory"), (3, 4, "candidates: block ids, row offsets"),
          (4, 5, "issue the first K/V stages; first token's append"), (5, 6, "key loop (copies, QK, softmax, PV)"),
          (6, 7, "epilogue: normalise, write output"), (7, 8, "fused metadata / append tail"),
          (8, 9, "split merge"), (8, 10, "merge: cluster barrier"),
          (10, 11, "merge: rows from the workspace"),
          (1, 9, "CTA after the wait"), (0, 9, "CTA incl. the wait")]


# Stamps of prefill_tcgen05_kernel (slot: point).  Softmax thread 0 of group
# A (q tile A) uses slots 1-9 for its first item and 11-19 for its second,
# thread 0 of group B slots 21-29 / 31-39: +0 geometry known, +1 S(0) ready,
# +2 P(0) handed over, +3 / +4 the same for key step 1, +5 / +6 step 2,
# +7 last PV complete, +8 epilogue stored.  40-43: the producer issued K/V
# tiles 0-3 of the CTA's stream; 44: first Q issued; 45 / 46: the first
# item's first K tile / Q landed (MMA thread), 47 / 48 the second item's;
# 0 / 50: CTA start / end (thread 0); 51-53: inside group A's softmax of its
# first item's key step 1 (row max known, rescale done, P stores issued).
PF_PHASES = [(0, 1, "A item 0: geometry (metadata loads)"), (44, 46, "item 0: Q copy"),
             (40, 45, "item 0: first K tile copy (from issue)"),
             (1, 2, "A item 0: wait for S(0)"), (2, 3, "A item 0: softmax of key step 0"),
             (3, 4, "A item 0: P(0) -> S(1) (PV + S on the tensor core)"), (4, 5, "A item 0: softmax of step 1"),
             (4, 51, "A step 1: max pass (4 TMEM loads)"), (51, 52, "A step 1: rescale check"),
             (52, 53, "A step 1: exp pass, P stores issued"), (53, 5, "A step 1: P stores complete, arrive"),
             (5, 6, "A item 0: P(1) -> S(2)"), (6, 7, "A item 0: softmax of step 2"),
             (8, 9, "A item 0: epilogue (O out of TMEM, stores)"), (9, 11, "A: next item's geometry"),
             (11, 12, "A item 1: wait for S(0)"), (12, 13, "A item 1: softmax of step 0"),
             (13, 14, "A item 1: P(0) -> S(1)"), (22, 23, "B item 0: softmax of step 0"),
             (23, 24, "B item 0: P(0) -> S(1)"), (29, 31, "B: next item's geometry"),
             (31, 32, "B item 1: wait for S(0)"), (0, 50, "CTA")]


def run_pf(lib, insts, steps, R, raw=None):
    clear, read = lib.spa_probe_clear_pf, lib.spa_probe_read_pf
    stream = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(steps):
            insts[i % R]()
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    assert clear() == 0
    torch.cuda.synchronize()
    g.replay()
    torch.cuda.synchronize()
    nct, slots = 2048, 64
    buf = np.zeros(nct * slots, dtype=np.uint64)
    assert read(buf.ctypes.data, buf.nbytes) == 0
    P = buf.reshape(nct, slots).astype(np.int64)
    if raw:
        np.save(raw, P)
    P = P[P[:, 0] > 0]
    lines = [f"prefill kernel: {len(P)} CTAs of the graph's last step ({steps} steps, {R} instances); "
             f"span {(P[:, 50].max() - P[:, 0].min()) / 1e3:.2f} us", "",
             "| interval | CTAs | median us | p90 us | max us |", "|---|---|---|---|---|"]
    for a, b, name in PF_PHASES:
        ok = (P[:, a] > 0) & (P[:, b] > 0)
        if ok.any():
            x = (P[ok, b] - P[ok, a]) / 1e3
            lines.append(f"| {a}->{b} {name} | {int(ok.sum())} | {np.median(x):.2f} | {np.percentile(x, 90):.2f} | "
                         f"{x.max():.2f} |")
    return "\n".join(lines)


def run(workload: str, lib_path: str, steps: int = 64, raw: str = None):
    lib = spa.load_library(lib_path)
    for k in ("mma", "tc", "pf"):
        getattr(lib, f"spa_probe_read_{k}").restype = ctypes.c_int
        getattr(lib, f"spa_probe_read_{k}").argtypes = [ctypes.c_void_p, ctypes.c_size_t]
        getattr(lib, f"spa_probe_clear_{k}").restype = ctypes.c_int
    spa._LIB = lib
    wl = W.by_name(workload)
    base = pipeline.to_device(wl)
    l2 = torch.cuda.get_device_properties(0).L2_cache_size
    per = sum(base[k].numel() * base[k].element_size() for k in ("k_cache", "v_cache"))
    R = max(2, min(16, math.ceil(2 * l2 / per) + 1))
    insts = []
    for _ in range(R):
        d = {k: (v.clone() if k in ("k_cache", "v_cache", "q", "k_new", "v_new", "block_table", "cu_seqlens_q",
                                   "past_seqlens", "selected_idx") else v) for k, v in base.items()}
        insts.append(pipeline.Step(wl, d))
    kind = spa.attention_plan(insts[0].args)["kind"]
    if kind == 2:
        with torch.cuda.stream(torch.cuda.Stream()):
            for st in insts:
                st()
        torch.cuda.synchronize()
        return run_pf(lib, insts, steps, R, raw)
    assert kind in (1, 3), "the workload runs neither the warp-MMA nor the tcgen05 decode kernel"
    tag, phases, last, nct = ("mma", PHASES, 9, 8192) if kind == 1 else ("tc", TC_PHASES, 10, 4096)
    clear = getattr(lib, f"spa_probe_clear_{tag}")
    read = getattr(lib, f"spa_probe_read_{tag}")
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        for st in insts:
            st()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(steps):
            insts[i % R]()
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    assert clear() == 0
    torch.cuda.synchronize()
    g.replay()
    torch.cuda.synchronize()
    buf = np.zeros(nct * 16, dtype=np.uint64)
    assert read(buf.ctypes.data, buf.nbytes) == 0
    P = buf.reshape(nct, 16).astype(np.int64)
    if raw:   # every CTA's stamps, indexed blockIdx.y * gridDim.x + blockIdx.x (0: not stamped)
        np.save(raw, P)
    P = P[P[:, 0] > 0]
    lines = [f"workload {workload} ({tag} kernel): {len(P)} CTAs of the graph's last step ({steps} steps, "
             f"{R} instances)",
             f"CTA span (first entry to last end): {(P[:, last].max() - P[:, 0].min()) / 1e3:.2f} us; "
             f"from the first wait release: {(P[:, last].max() - P[:, 1].min()) / 1e3:.2f} us",
             "", "| phase | median us | p90 us | max us |", "|---|---|---|---|"]
    for a, b, name in phases:
        ok = (P[:, a] > 0) & (P[:, b] > 0)
        if ok.any():
            x = (P[ok, b] - P[ok, a]) / 1e3
            lines.append(f"| {a}->{b} {name} | {np.median(x):.2f} | {np.percentile(x, 90):.2f} | {x.max():.2f} |")
    t0 = P[:, 1].min()
    lines += ["", "stamp offsets from the first wait release (us), percentiles 0 / 50 / 100:"]
    for k in range(last + 1):
        ok = P[:, k] > 0
        if ok.any():
            q = np.percentile((P[ok, k] - t0) / 1e3, [0, 50, 100])
            lines.append(f"  stamp {k}: {q[0]:.2f} / {q[1]:.2f} / {q[2]:.2f}")
    return "\n".join(lines)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="gptoss_paged_decode_f16")
    ap.add_argument("--lib", default=None, help="probe library (default: build it with build.py --probe)")
    ap.add_argument("--steps", type=int, default=64)
    ap.add_argument("--raw", default=None, help="also save the raw stamps (.npy)")
    a = ap.parse_args()
    lib = a.lib or (build.PROBE_LIB if os.path.exists(build.PROBE_LIB) else build.build_probe())
    print(run(a.workload, lib, a.steps, a.raw))


if __name__ == "__main__":
    main()
