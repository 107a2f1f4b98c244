"""Seeded synthetic inputs for paged / selected-token sparse attention.

This module only draws random inputs and lays them out; it holds none of the
attention method's arithmetic (no metadata derivation, no KV append, no index
gathering, no softmax).  Both the fp64 CPU oracle (through the tests and the
bench's CPU baseline) and the CUDA path consume the same arrays.

Shapes follow the operator inputs described on the pages:
  q           [T, H_q, D]            activation dtype
  k_new/v_new [T, H_kv, D]           activation dtype (tokens appended this step)
  k_cache     [NB, block_size, H_kv, D] cache dtype (activation dtype or int8)
  block_table [B, MB] int32          physical block id per logical block, -1 unused
  cu_seqlens_q [B+1], past_seqlens [B] int32
  selected_idx [B or T, H_kv, K_sel] int32, -1 padded
  aux_k/aux_v [B, aux_cap, H_kv, D]  cache dtype; aux_seqlens [B] int32
  sinks [H_q] fp32; k_scale/v_scale [H_kv, D] fp32

bf16 arrays are carried as uint16 bit patterns (numpy has no bfloat16); the
``dtypes`` map of a workload names the logical dtype of every array.

The five named workloads are the ones the headline measurements are quoted on
(tiny fp32 decode, GPT-OSS-like paged decode, selected-token decode,
local-plus-selected INT8 decode, ragged causal prefill); ``small=True`` gives a
reduced copy with the same structure for fast parity tests.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional

import numpy as np


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round finite float32 values to bfloat16 (round-to-nearest-even); return the bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).reshape(-1).view(np.uint32)
    out = np.empty(u.shape, dtype=np.uint16)
    step = 1 << 24
    for i in range(0, u.size, step):
        c = u[i:i + step]
        # finite values stay below 2**32 after adding the bias
        out[i:i + step] = ((c + (np.uint32(0x7FFF) + ((c >> np.uint32(16)) & np.uint32(1))))
                           >> np.uint32(16)).astype(np.uint16)
    return out.reshape(np.shape(x))


_NORMAL_TABLE = {}


def _normal_table(act: str) -> np.ndarray:
    """N(0, 1) quantiles at the midpoints of 65536 equal-probability cells,
    encoded in the activation dtype."""
    if act not in _NORMAL_TABLE:
        from scipy.special import ndtri
        z = ndtri((np.arange(65536, dtype=np.float64) + 0.5) / 65536.0).astype(np.float32)
        if act == "f32":
            tab = z
        elif act == "f16":
            tab = z.astype(np.float16)
        else:
            tab = f32_to_bf16_bits(z)
        _NORMAL_TABLE[act] = tab
    return _NORMAL_TABLE[act]


def _act_array(rng: np.random.Generator, shape, act: str) -> np.ndarray:
    """Seeded N(0, 1) draws in the activation dtype: 16 uniform random bits per
    element select one of 65536 equal-probability normal quantiles."""
    if act not in ("f32", "f16", "bf16"):
        raise ValueError(act)
    n = int(np.prod(shape))
    bits = rng.integers(0, 65536, size=n, dtype=np.uint16)
    return _normal_table(act)[bits].reshape(shape)


@dataclasses.dataclass
class Workload:
    name: str
    act: str                      # 'f32' | 'f16' | 'bf16'
    cache: str                    # 'f32' | 'f16' | 'bf16' | 'i8'
    B: int
    H_q: int
    H_kv: int
    D: int
    block_size: int
    q_lens: List[int]
    past: List[int]
    window: int
    sel_mode: Optional[str]       # None | 'main' | 'aux'
    sel_per_request: int
    sel_width: int
    aux_cap: int
    has_sinks: bool
    scale: float
    seed: int
    arrays: Dict[str, np.ndarray] = dataclasses.field(default_factory=dict)
    dtypes: Dict[str, str] = dataclasses.field(default_factory=dict)
    # optional QKV prologue ahead of the append: packed (bool), qk_norm (bool),
    # eps, rotary_dim, interleaved (bool), max_pos, pos_ids (bool), rotary_offset
    prologue: Optional[Dict] = None

    @property
    def T(self) -> int:
        return int(sum(self.q_lens))

    @property
    def G(self) -> int:
        return self.H_q // self.H_kv

    @property
    def NB(self) -> int:
        return int(self.arrays["k_cache"].shape[0])

    @property
    def MB(self) -> int:
        return int(self.arrays["block_table"].shape[1])

    @property
    def max_seqlen_q(self) -> int:
        return int(max(self.q_lens)) if self.q_lens else 0

    @property
    def max_seqlen_k(self) -> int:
        return int(max(p + q for p, q in zip(self.past, self.q_lens))) if self.q_lens else 0

    def __getitem__(self, k):
        return self.arrays[k]


def make_workload(*, name="custom", act="f16", cache=None, B=2, H_q=8, H_kv=2, D=64,
                  block_size=16, q_lens=None, past=None, window=0, sel_mode=None,
                  sel_per_request=1, sel_width=0, sel_valid=None, sel_sorted=False,
                  sel_tail_pad=0, aux_cap=0, aux_lens=None, has_sinks=True, scale=0.0,
                  int8_history=False, kv_scale_range=(0.01, 0.05), spare_blocks=0,
                  prologue: Optional[Dict] = None, seed=0) -> Workload:
    """Draw one seeded workload.

    Lengths: request b has ``past[b]`` resident tokens and ``q_lens[b]`` new
    tokens.  Each request owns ceil((past+q)/block_size) physical blocks taken
    in order from a random permutation of all blocks (``spare_blocks`` extra
    unowned blocks are added so that unmapped cache rows exist).

    Selection: ``sel_width`` slots per row.  ``sel_valid`` (int or per-row
    callable) entries are unique draws from the addressable range (positions
    of the request for 'main', [0, aux_len) for 'aux'); the remaining slots are
    -1.  With ``sel_tail_pad`` the padding sits at the tail of a sorted list;
    otherwise the list keeps draw order with the padding at the tail too.
    """
    cache = cache or act
    q_lens = list(q_lens if q_lens is not None else [1] * B)
    past = list(past if past is not None else [0] * B)
    assert len(q_lens) == B and len(past) == B
    rng = np.random.default_rng(seed)
    T = int(sum(q_lens))
    totals = [p + q for p, q in zip(past, q_lens)]
    nblk = [(t + block_size - 1) // block_size for t in totals]
    MB = max(max(nblk) if nblk else 1, 1)
    NB = int(sum(nblk)) + spare_blocks
    NB = max(NB, 1)
    perm = rng.permutation(NB).astype(np.int32)
    block_table = np.full((B, MB), -1, dtype=np.int32)
    off = 0
    for b in range(B):
        block_table[b, :nblk[b]] = perm[off:off + nblk[b]]
        off += nblk[b]
    cu = np.zeros(B + 1, dtype=np.int32)
    cu[1:] = np.cumsum(q_lens)
    arrays: Dict[str, np.ndarray] = {}
    dtypes: Dict[str, str] = {}
    arrays["q"] = _act_array(rng, (T, H_q, D), act); dtypes["q"] = act
    arrays["k_new"] = _act_array(rng, (T, H_kv, D), act); dtypes["k_new"] = act
    arrays["v_new"] = _act_array(rng, (T, H_kv, D), act); dtypes["v_new"] = act
    cache_shape = (NB, block_size, H_kv, D)
    if cache == "i8":
        for nm in ("k_cache", "v_cache"):
            arrays[nm] = rng.integers(-127, 128, size=cache_shape, dtype=np.int16).astype(np.int8)
            dtypes[nm] = "i8"
        lo, hi = kv_scale_range
        arrays["k_scale"] = rng.uniform(lo, hi, size=(H_kv, D)).astype(np.float32)
        arrays["v_scale"] = rng.uniform(lo, hi, size=(H_kv, D)).astype(np.float32)
        dtypes["k_scale"] = dtypes["v_scale"] = "f32"
    else:
        for nm in ("k_cache", "v_cache"):
            arrays[nm] = _act_array(rng, cache_shape, cache)
            dtypes[nm] = cache
    arrays["block_table"] = block_table
    arrays["cu_seqlens_q"] = cu
    arrays["past_seqlens"] = np.asarray(past, dtype=np.int32)
    for nm in ("block_table", "cu_seqlens_q", "past_seqlens"):
        dtypes[nm] = "i32"
    if has_sinks:
        arrays["sinks"] = rng.standard_normal(H_q).astype(np.float32)
        dtypes["sinks"] = "f32"
    if sel_mode == "aux":
        aux_lens = list(aux_lens if aux_lens is not None else [aux_cap] * B)
        shape = (B, aux_cap, H_kv, D)
        if cache == "i8":
            arrays["aux_k"] = rng.integers(-127, 128, size=shape, dtype=np.int16).astype(np.int8)
            arrays["aux_v"] = rng.integers(-127, 128, size=shape, dtype=np.int16).astype(np.int8)
        else:
            arrays["aux_k"] = _act_array(rng, shape, cache)
            arrays["aux_v"] = _act_array(rng, shape, cache)
        dtypes["aux_k"] = dtypes["aux_v"] = cache
        arrays["aux_seqlens"] = np.asarray(aux_lens, dtype=np.int32)
        dtypes["aux_seqlens"] = "i32"
    if sel_mode is not None:
        rows = B if sel_per_request else T
        sel = np.full((rows, H_kv, sel_width), -1, dtype=np.int32)
        tok_req = np.repeat(np.arange(B), q_lens) if T else np.zeros(0, dtype=np.int64)
        for r in range(rows):
            b = r if sel_per_request else int(tok_req[r])
            if sel_mode == "main":
                rng_hi = totals[b]
            else:
                rng_hi = aux_lens[b]
            for h in range(H_kv):
                if callable(sel_valid):
                    nv = int(sel_valid(r, h))
                elif sel_valid is None:
                    nv = sel_width - sel_tail_pad
                else:
                    nv = int(sel_valid)
                nv = max(0, min(nv, sel_width, rng_hi))
                idx = rng.permutation(rng_hi)[:nv].astype(np.int32)
                if sel_sorted:
                    idx = np.sort(idx)
                sel[r, h, :nv] = idx
        arrays["selected_idx"] = sel
        dtypes["selected_idx"] = "i32"
    pro = None
    if prologue:
        # drawn from a stream of its own, so the arrays above do not change
        pro = dict(prologue)
        prng = np.random.default_rng(seed + 7919)
        if pro.get("packed"):
            arrays["qkv"] = np.concatenate([arrays["q"], arrays["k_new"], arrays["v_new"]], axis=1)
            dtypes["qkv"] = act
        if pro.get("qk_norm"):
            arrays["q_norm_weight"] = prng.uniform(0.5, 1.5, size=D).astype(np.float32)
            arrays["k_norm_weight"] = prng.uniform(0.5, 1.5, size=D).astype(np.float32)
            dtypes["q_norm_weight"] = dtypes["k_norm_weight"] = "f32"
        rd = int(pro.get("rotary_dim", 0))
        if rd:
            max_pos = int(pro.get("max_pos", (max(totals) if totals else 0) + 64))
            pro["max_pos"] = max_pos
            inv_freq = float(pro.get("base", 10000.0)) ** (-np.arange(0, rd, 2, dtype=np.float64) / rd)
            angle = np.arange(max_pos, dtype=np.float64)[:, None] * inv_freq[None, :]
            arrays["cos_cache"] = np.cos(angle).astype(np.float32)
            arrays["sin_cache"] = np.sin(angle).astype(np.float32)
            dtypes["cos_cache"] = dtypes["sin_cache"] = "f32"
        if pro.get("pos_ids"):
            shift = int(pro.get("pos_shift", 3))
            pos = [past[b] + i + shift for b in range(B) for i in range(q_lens[b])]
            arrays["position_ids"] = np.asarray(pos, dtype=np.int32).reshape(T)
            dtypes["position_ids"] = "i32"
    wl = Workload(name=name, act=act, cache=cache, B=B, H_q=H_q, H_kv=H_kv, D=D,
                  block_size=block_size, q_lens=q_lens, past=past, window=window,
                  sel_mode=sel_mode, sel_per_request=sel_per_request, sel_width=sel_width,
                  aux_cap=aux_cap, has_sinks=has_sinks, scale=scale, seed=seed,
                  arrays=arrays, dtypes=dtypes, prologue=pro)
    return wl


# ---------------------------------------------------------------------------
# The five named workloads.
# ---------------------------------------------------------------------------

WORKLOADS = ("tiny_decode_f32", "gptoss_paged_decode_f16", "selected_decode_bf16",
             "local_plus_selected_int8", "ragged_prefill_f16", "windowed_chunked_prefill_f16")


def tiny_decode_f32(seed: int = 0, small: bool = False) -> Workload:
    """B=2 decode, H_q=4, H_kv=2, D=64, block 16, lengths {37, 100}, 16 selected
    indices per (request, kv head) of which the last 3 are -1, sinks on, fp32."""
    totals = [37, 100]
    return make_workload(name="tiny_decode_f32", act="f32", B=2, H_q=4, H_kv=2, D=64,
                         block_size=16, q_lens=[1, 1], past=[t - 1 for t in totals],
                         sel_mode="main", sel_per_request=1, sel_width=16, sel_valid=13,
                         has_sinks=True, seed=seed)


def gptoss_paged_decode_f16(seed: int = 1, small: bool = False) -> Workload:
    """B=32 decode, H_q=64, H_kv=8, D=64, block 16, lengths U[512, 8192],
    causal local window 128, learned sink per q head, fp16."""
    rng = np.random.default_rng(seed + 1000)
    B = 4 if small else 32
    hi = 700 if small else 8192
    totals = [int(x) for x in rng.integers(512 if not small else 100, hi + 1, size=B)]
    if small:
        totals[0] = 3           # shorter than the window
        totals[1] = 128         # exactly the window
    return make_workload(name="gptoss_paged_decode_f16", act="f16", B=B, H_q=64, H_kv=8,
                         D=64, block_size=16, q_lens=[1] * B, past=[t - 1 for t in totals],
                         window=128, has_sinks=True, seed=seed)


def selected_decode_bf16(seed: int = 2, small: bool = False) -> Workload:
    """B=16 decode, H_q=32, H_kv=4, D=128, cache length 32768 paged in blocks of 64,
    2048 sorted unique selected indices per (request, kv head) with 5% -1 padding
    at the tail, sinks on, bf16."""
    B = 2 if small else 16
    L = 1000 if small else 32768
    W = 200 if small else 2048
    pad = int(0.05 * W)
    return make_workload(name="selected_decode_bf16", act="bf16", B=B, H_q=32, H_kv=4, D=128,
                         block_size=64, q_lens=[1] * B, past=[L - 1] * B, sel_mode="main",
                         sel_per_request=1, sel_width=W, sel_tail_pad=pad, sel_sorted=True,
                         has_sinks=True, seed=seed)


def local_plus_selected_int8(seed: int = 3, small: bool = False) -> Workload:
    """S_q=8 multi-query decode, B=8, H_q=48, H_kv=4 (12 q heads per kv head),
    D=128, window 128 on the main cache plus 512 selected indices into an
    auxiliary store of 4096 tokens, INT8 per-channel K/V with scales U[0.01, 0.05]."""
    B = 2 if small else 8
    past = 300 if small else 4088
    aux = 600 if small else 4096
    W_sel = 100 if small else 512
    return make_workload(name="local_plus_selected_int8", act="f16", cache="i8", B=B, H_q=48,
                         H_kv=4, D=128, block_size=64, q_lens=[8] * B, past=[past] * B,
                         window=128, sel_mode="aux", sel_per_request=1, sel_width=W_sel,
                         sel_sorted=True, aux_cap=aux, has_sinks=True, seed=seed)


def ragged_prefill_f16(seed: int = 4, small: bool = False) -> Workload:
    """Ragged causal prefill, B=4, lengths {512, 1024, 2048, 3072}, H_q=32, H_kv=8,
    D=128, paged block 64, no selection, no window, sinks on, fp16."""
    lens = [70, 130, 257, 300] if small else [512, 1024, 2048, 3072]
    return make_workload(name="ragged_prefill_f16", act="f16", B=4, H_q=32, H_kv=8, D=128,
                         block_size=64, q_lens=lens, past=[0] * 4, has_sinks=True, seed=seed)


def windowed_chunked_prefill_f16(seed: int = 5, small: bool = False) -> Workload:
    """Chunked prefill of GPT-OSS-like local (sliding-window) layers: B=4 chunks
    of {2048, 1024, 512, 1536} tokens after {0, 1024, 3000, 512} resident
    tokens, H_q=64, H_kv=8, D=64, paged block 16, window 128, sinks on, fp16."""
    if small:
        q_lens, past = [150, 64, 40, 97], [0, 70, 300, 33]
    else:
        q_lens, past = [2048, 1024, 512, 1536], [0, 1024, 3000, 512]
    return make_workload(name="windowed_chunked_prefill_f16", act="f16", B=4, H_q=64, H_kv=8, D=64,
                         block_size=16, q_lens=q_lens, past=past, window=128, has_sinks=True, seed=seed)


# Workloads that run the QKV prologue ahead of the append.
PROLOGUE_WORKLOADS = ("qkv_prologue_selected_decode_bf16",)


def qkv_prologue_selected_decode_bf16(seed: int = 6, small: bool = False) -> Workload:
    """Selected-token decode fed by the QKV prologue: packed QKV, QK RMSNorm and
    rotary embedding over all D channels (half-split pairs) ahead of the append;
    B=16, H_q=32, H_kv=4, D=128, cache length 8192 paged in blocks of 64, 1024
    sorted selected indices per (request, kv head) with 5% -1 padding, sinks, bf16."""
    B = 3 if small else 16
    L = 700 if small else 8192
    W_sel = 100 if small else 1024
    return make_workload(name="qkv_prologue_selected_decode_bf16", act="bf16", B=B, H_q=32, H_kv=4,
                         D=128, block_size=64, q_lens=[1] * B, past=[L - 1] * B, sel_mode="main",
                         sel_per_request=1, sel_width=W_sel, sel_sorted=True,
                         sel_tail_pad=W_sel // 20, has_sinks=True,
                         prologue=dict(packed=True, qk_norm=True, rotary_dim=128), seed=seed)


# Inputs of the selection producer (TopK over per-key scores).
@dataclasses.dataclass
class SelectionWorkload:
    name: str
    R: int
    H: int
    n_keys: int
    top_k: int
    sel_width: int
    scores: np.ndarray            # [R, H, n_keys] fp32
    bound: np.ndarray             # [R] int32: last eligible key of each row


SELECTION_WORKLOADS = ("topk_selection_f32",)


def topk_selection_f32(seed: int = 7, small: bool = False) -> SelectionWorkload:
    """Scores for the selected-token decode shape: 16 requests x 4 kv heads x
    32768 keys, N(0, 1) fp32, every key of a request eligible (bound = 32767);
    1946 kept in rows of capacity 2048 (the decode workload's 5% padding)."""
    R, H, N, W = (2, 4, 1000, 200) if small else (16, 4, 32768, 2048)
    rng = np.random.default_rng(seed)
    scores = rng.standard_normal((R, H, N)).astype(np.float32)
    return SelectionWorkload(name="topk_selection_f32", R=R, H=H, n_keys=N, top_k=W - W // 20, sel_width=W,
                             scores=scores, bound=np.full(R, N - 1, dtype=np.int32))


def by_name(name: str, small: bool = False, seed: Optional[int] = None) -> Workload:
    fn = {n: globals()[n] for n in WORKLOADS + PROLOGUE_WORKLOADS}[name]
    if seed is None:
        return fn(small=small)
    return fn(seed=seed, small=small)
