"""fp64 CPU oracle for paged / selected-token sparse attention.

TEST INFRASTRUCTURE.  Only the tests, the smoke check and the bench's CPU
baseline leg may import this module.  The product path (the CUDA library and
its Python binding) never calls it and shares no code with it.

It is a plain, slow restatement of what the pages define, written in the order
the pages describe the pipeline:

  0. selection producer -- onnxruntime PR #33472, Key Changes
     (PackedSparseAttentionIndexer: QSA TopK selection) and experiments note
     (compact TopK keeps stable keys, causal tails, capacity padding and
     overflow handling): the top_k keys of per-key scores, as selected
     indices for step 3.
  1. metadata prepare  -- "[WebGPU] Add PagedAttention metadata and GPT-OSS
     support" (onnxruntime PR #32277), Description and Changes (exact
     per-request seqlen_k / seqlens_q derived on device), review item T1
     (worked cases new_seqlens=[1, 2] and [2, 0], seqlen_k = -1 sentinel);
     "[WebGPU] Add SparsePagedAttention" (PR #32533), File summaries
     (token_meta: sanitised per-token metadata) and review note on malformed
     cumulative_sequence_length.
  2. KV append scatter -- "[WebGPU] Add SparsePagedAttention", File summaries
     (scatter current K/V into the cache using slot_mapping); INT8 per-channel
     cache from onnxruntime PR #33472, Key Changes (key_scale / value_scale).
  3. attended-key gather -- PR #32277 review item Q3 (window start
     max(0, causal_end - local_window_size), causal_end = past + q_idx + 1);
     "[WebGPU] Add DynamicSparseAttention" (PR #32529), Description/Attention
     (selected main-cache and local-plus-auxiliary modes, guarded indices,
     padding) and QKV and cache (GQA head mapping); "ai.onnx.LinearAttention"
     Description (H_q a positive multiple of H_kv).
  4. scaled QK + joint FP32 softmax with a learned per-head sink --
     PR #32529 Description/Attention ("joint FP32 stable softmax with optional
     sink"); PR #32277 Description (learned head-sink term); scale = 0 selects
     1/sqrt(D) as in "ai.onnx.LinearAttention", Attributes.
  5. split-KV partial + log-sum-exp combine -- PR #32533 follow-up Description
     (FP32 partial softmax state merged in a finalize stage).  The combine is
     exact in real arithmetic, so the oracle computes the single-pass
     definition: softmax over the whole attended set plus the sink.
  5b. sequence-sharded split-KV -- the same finalize merge over shards of a
     sequence split across devices: attention() over one shard's key range
     (kv_range) without the sink, then merge_partials() with the sink once.

Readings where the pages are silent (all listed in the design notes):
  * KV cache layout [num_blocks, block_size, H_kv, D]; slot = block*bs + offset.
  * malformed cu_seqlens are clamped to a non-decreasing sequence in [0, T]
    and flagged; negative past lengths are clamped to 0 and flagged.
  * seqlen_k = past + q_len - 1 (total - 1); a request with no tokens at all
    gives -1.
  * INT8 quantise: q8 = clamp(rint(float32(x) / float32(scale)), -128, 127),
    IEEE fp32 division, round-half-even; dequantise q8 * scale.
  * the sink is a logit (not multiplied by the softmax scale) that adds
    exp(sink - m) to the denominator and nothing to the numerator.
  * window W > 0 keeps keys j with max(0, p - W + 1) <= j <= p; W <= 0 is off.
  * selected main-cache indices i are attended iff 0 <= i <= p; -1 is
    padding; i < -1 or i >= L_b sets BAD_IDX (skipped).  Auxiliary indices
    are attended iff 0 <= i < aux_len[b]; others (except -1) set BAD_IDX.
  * all auxiliary entries are visible to every query token of the request.
  * a selected entry repeated in a list counts once per occurrence.
  * an empty attended set with no sink gives output 0 and lse = -inf.
  * keys whose logical block is unmapped (CAPACITY / BAD_BLOCK) are skipped.

Every floating-point step runs in float64; inputs are decoded exactly from
their fp32 / fp16 / bf16 / int8 encodings.
"""
from __future__ import annotations

import math
from typing import Dict, Iterable, Optional, Sequence, Tuple

import numpy as np

# status bits (device status word of the library; same numbering here)
ST_BAD_CU = 0x1
ST_CAPACITY = 0x2
ST_BAD_BLOCK = 0x4
ST_BOUNDS = 0x8
ST_BAD_IDX = 0x10


def decode(x: np.ndarray, dtype: str) -> np.ndarray:
    """Exact float64 value of an encoded array ('f32','f16','bf16' bits,'i8')."""
    if dtype in ("f32", "f16", "i8", "f64"):
        return np.asarray(x).astype(np.float64)
    if dtype == "bf16":
        bits = np.asarray(x, dtype=np.uint16).astype(np.uint32) << 16
        return bits.view(np.float32).astype(np.float64)
    raise ValueError(dtype)


# ---------------------------------------------------------------------------
# 0. selection producer (TopK over per-key scores)
# ---------------------------------------------------------------------------
#
# onnxruntime PR #33472, Key Changes (PackedSparseAttentionIndexer: QSA block
# scoring and hierarchical / compact TopK selection feeding the selected
# indices of DynamicSparseAttention) and the experiments note on compact TopK
# (it keeps stable keys, causal tails, capacity stride / padding and overflow
# handling).  The pages never define the score itself, so the scores are an
# input here.  Readings:
#   * a row's eligible keys are j <= bound (the causal tail: a request's
#     last position, seqlen_k = total - 1, or a token's own position) with a
#     score that is neither NaN nor -inf (-inf masks a key);
#   * the top_k eligible keys by score are kept; equal scores keep the lower
#     key index first (stable);
#   * the kept indices are written in increasing order at the start of the
#     row, and the rest of the row (its capacity, sel_width) is -1;
#   * fewer eligible keys than top_k: all of them are kept (no overflow).

def select_topk(scores: np.ndarray, bound: np.ndarray, top_k: int, sel_width: int) -> np.ndarray:
    """selected_idx [R, H, sel_width] of fp32 scores [R, H, N] with per-row bounds [R]."""
    scores = np.asarray(scores, dtype=np.float32)
    R, H, N = scores.shape
    out = np.full((R, H, sel_width), -1, dtype=np.int32)
    for r in range(R):
        last = min(int(bound[r]), N - 1)
        for h in range(H):
            row = [float(v) for v in scores[r, h]]
            eligible = [j for j in range(last + 1) if not math.isnan(row[j]) and row[j] != -math.inf]
            ranked = sorted(eligible, key=lambda j: (-row[j], j))
            kept = sorted(ranked[:top_k])
            out[r, h, :len(kept)] = kept
    return out


# ---------------------------------------------------------------------------
# 1. metadata prepare
# ---------------------------------------------------------------------------

def prepare_metadata(cu_seqlens_q: np.ndarray, past_seqlens: np.ndarray,
                     block_table: np.ndarray, T: int, max_seqlen_q: int,
                     max_seqlen_k: int, block_size: int, num_blocks: int) -> Dict[str, np.ndarray]:
    """Per-request lengths and per-token (request, position, slot).

    Returns seqlens_q[B], seqlen_k[B] (total-1, -1 for a request with no
    tokens), token_batch[T], token_pos[T], slot_mapping[T] (-1 where the
    token has no valid slot) and the status word.
    """
    cu = [int(v) for v in cu_seqlens_q]
    B = len(cu) - 1
    MB = block_table.shape[1] if block_table.ndim == 2 else 0
    status = 0
    # sanitised cumulative lengths: non-decreasing, starting at 0, within [0, T]
    cs = [0] * (B + 1)
    for b in range(1, B + 1):
        cs[b] = min(max(cu[b], cs[b - 1]), T)
    if any(cu[b] != cs[b] for b in range(B + 1)) or cs[B] != T:
        status |= ST_BAD_CU
    past = []
    for b in range(B):
        p = int(past_seqlens[b])
        if p < 0:
            status |= ST_BAD_CU
            p = 0
        past.append(p)
    seqlens_q = np.zeros(B, dtype=np.int32)
    seqlen_k = np.zeros(B, dtype=np.int32)
    for b in range(B):
        q_len = cs[b + 1] - cs[b]
        total = past[b] + q_len
        seqlens_q[b] = q_len
        seqlen_k[b] = total - 1
        if q_len > max_seqlen_q or total > max_seqlen_k:
            status |= ST_BOUNDS
    token_batch = np.full(T, -1, dtype=np.int32)
    token_pos = np.full(T, -1, dtype=np.int32)
    slot = np.full(T, -1, dtype=np.int32)
    for t in range(T):
        owner = -1
        for b in range(B):
            if cs[b] <= t < cs[b + 1]:
                owner = b
                break
        if owner < 0:
            continue
        p = past[owner] + (t - cs[owner])
        token_batch[t] = owner
        token_pos[t] = p
        lb = p // block_size
        if lb >= MB:
            status |= ST_CAPACITY
            continue
        blk = int(block_table[owner, lb])
        if blk < 0 or blk >= num_blocks:
            status |= ST_BAD_BLOCK
            continue
        slot[t] = blk * block_size + p % block_size
    return {"seqlens_q": seqlens_q, "seqlen_k": seqlen_k, "token_batch": token_batch,
            "token_pos": token_pos, "slot_mapping": slot, "status": status}


# ---------------------------------------------------------------------------
# 1b. QKV prologue (optional, between metadata and append)
# ---------------------------------------------------------------------------
#
# "[WebGPU] Add DynamicSparseAttention", Description: QKV and cache (packed
# and unpacked QKV), Position processing (QK RMSNorm; partial and interleaved
# RoPE; rotary offsets and explicit position IDs); "[WebGPU] Add
# SparsePagedAttention", Description (the prologue -- packed-QKV split, RoPE
# -- ahead of the block-table scatter).  Readings where the pages are silent:
#   * packed QKV is [T, H_q + 2*H_kv, D]: q heads, then k heads, then v heads;
#   * RMSNorm over each head's D channels, y = x / sqrt(mean(x^2) + eps) * w,
#     one fp32 weight vector [D] for q and one for k; applied before RoPE;
#   * RoPE rotates the first rotary_dim channels by the angle whose cos / sin
#     are the caches' row `position` (fp32 [max_pos, rotary_dim / 2]); pairs
#     are (i, i + rotary_dim/2) ("half-split") or (2i, 2i+1) ("interleaved"):
#       (a, b) -> (a cos - b sin, b cos + a sin);
#   * position = position_ids[t] when given, else token_pos[t] + offset; a
#     position outside [0, max_pos) is left unrotated and sets BOUNDS;
#   * q, k and v leave the prologue rounded to the activation dtype (round to
#     nearest even), then k and v go through the append unchanged.

def encode(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round float64 values to `dtype`'s encoding (nearest even); bf16 as uint16 bits."""
    x = np.asarray(x, dtype=np.float64)
    if dtype == "f32":
        return x.astype(np.float32)
    if dtype == "f16":
        return x.astype(np.float16)
    if dtype == "bf16":
        # the two bf16 neighbours of x, and the nearer one (ties to the even code)
        lo = (np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64) >> 16) << 16
        cand = [lo - (1 << 16), lo, lo + (1 << 16)]
        vals = [c.astype(np.uint32).view(np.float32).astype(np.float64) for c in cand]
        best = cand[1].copy()
        bestd = np.abs(vals[1] - x)
        for c, v in ((cand[0], vals[0]), (cand[2], vals[2])):
            d = np.abs(v - x)
            better = (d < bestd) | ((d == bestd) & (((c >> 16) & 1) == 0) & (((best >> 16) & 1) == 1))
            best = np.where(better, c, best)
            bestd = np.where(better, d, bestd)
        return (best >> 16).astype(np.uint16)
    raise ValueError(dtype)


def split_packed(qkv: np.ndarray, H_q: int, H_kv: int) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """q [T, H_q, D], k and v [T, H_kv, D] of a packed [T, H_q + 2 H_kv, D] array."""
    return qkv[:, :H_q], qkv[:, H_q:H_q + H_kv], qkv[:, H_q + H_kv:]


def rms_norm(x: np.ndarray, weight: np.ndarray, eps: float) -> np.ndarray:
    """x / sqrt(mean(x^2) + eps) * weight over the last axis (float64)."""
    x = np.asarray(x, dtype=np.float64)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + float(eps)) * np.asarray(weight, dtype=np.float64)


def rotate(x: np.ndarray, cos: np.ndarray, sin: np.ndarray, rotary_dim: int,
           interleaved: bool) -> np.ndarray:
    """Rotary embedding of the first rotary_dim channels of x [D]; cos / sin [rotary_dim / 2]."""
    y = np.array(x, dtype=np.float64)
    half = rotary_dim // 2
    c = np.asarray(cos, dtype=np.float64)[:half]
    s = np.asarray(sin, dtype=np.float64)[:half]
    if interleaved:
        a, b = y[0:rotary_dim:2].copy(), y[1:rotary_dim:2].copy()
        y[0:rotary_dim:2] = a * c - b * s
        y[1:rotary_dim:2] = b * c + a * s
    else:
        a, b = y[:half].copy(), y[half:rotary_dim].copy()
        y[:half] = a * c - b * s
        y[half:rotary_dim] = b * c + a * s
    return y


def qkv_prologue(q: np.ndarray, k: np.ndarray, v: np.ndarray, act: str, token_pos: np.ndarray,
                 q_norm_weight: Optional[np.ndarray] = None,
                 k_norm_weight: Optional[np.ndarray] = None, eps: float = 1e-6,
                 cos_cache: Optional[np.ndarray] = None, sin_cache: Optional[np.ndarray] = None,
                 rotary_dim: int = 0, interleaved: bool = False,
                 position_ids: Optional[np.ndarray] = None, rotary_offset: int = 0):
    """Per token and head: RMSNorm (if its weight is given), then RoPE (if the
    caches are given) of q and k; v passes through.  Inputs and outputs are
    encoded in `act`.  Returns (q_out, k_out, v_out, status)."""
    T = q.shape[0]
    status = 0
    qo = decode(q, act).copy()
    ko = decode(k, act).copy()
    rope = cos_cache is not None and rotary_dim > 0
    max_pos = cos_cache.shape[0] if rope else 0
    for t in range(T):
        pos = int(position_ids[t]) if position_ids is not None else int(token_pos[t]) + int(rotary_offset)
        rot_ok = rope and 0 <= pos < max_pos
        if rope and not rot_ok:
            status |= ST_BOUNDS
        for x, w in ((qo, q_norm_weight), (ko, k_norm_weight)):
            for h in range(x.shape[1]):
                r = x[t, h]
                if w is not None:
                    r = rms_norm(r, w, eps)
                if rot_ok:
                    r = rotate(r, cos_cache[pos], sin_cache[pos], rotary_dim, interleaved)
                x[t, h] = r
    return encode(qo, act), encode(ko, act), np.array(v, copy=True), status


# ---------------------------------------------------------------------------
# 2. KV append scatter
# ---------------------------------------------------------------------------

def quantize_int8(x_f32: np.ndarray, scale_f32: np.ndarray) -> np.ndarray:
    """q8 = clamp(rint(x / scale), -128, 127), division and rounding in fp32."""
    r = np.rint(np.asarray(x_f32, dtype=np.float32) / np.asarray(scale_f32, dtype=np.float32))
    return np.clip(r, -128, 127).astype(np.int8)


def append_kv(k_new: np.ndarray, v_new: np.ndarray, act: str, k_cache: np.ndarray,
              v_cache: np.ndarray, cache: str, slot_mapping: np.ndarray,
              k_scale: Optional[np.ndarray] = None,
              v_scale: Optional[np.ndarray] = None) -> Tuple[np.ndarray, np.ndarray]:
    """Write token t's K/V rows to cache slot slot_mapping[t]; returns new caches.

    Float caches receive an exact copy of the encoded values.  An int8 cache
    receives the per-channel quantised values.  Slots equal to -1 are skipped.
    """
    kc = k_cache.copy()
    vc = v_cache.copy()
    bs = kc.shape[1]
    for t, s in enumerate(np.asarray(slot_mapping)):
        s = int(s)
        if s < 0:
            continue
        blk, off = divmod(s, bs)
        if cache == "i8":
            kc[blk, off] = quantize_int8(decode(k_new[t], act).astype(np.float32), k_scale)
            vc[blk, off] = quantize_int8(decode(v_new[t], act).astype(np.float32), v_scale)
        else:
            kc[blk, off] = k_new[t]
            vc[blk, off] = v_new[t]
    return kc, vc


# ---------------------------------------------------------------------------
# 3.-5. attention
# ---------------------------------------------------------------------------

def attended_keys(t: int, h_kv: int, meta: Dict[str, np.ndarray], block_table: np.ndarray,
                  block_size: int, num_blocks: int, window: int,
                  selected_idx: Optional[np.ndarray], sel_per_request: int, sel_target: int,
                  aux_seqlens: Optional[np.ndarray], kv_range: Optional[np.ndarray] = None):
    """The attended set of token t under kv head h_kv.

    With ``kv_range`` ([B, 2]) only the main-cache positions lo <= j < hi of
    the token's request are kept (one shard of a sequence split across
    devices); they are dropped before any block-table lookup.

    Returns (blocks, offsets, aux_pos, status): the physical main-cache rows
    (block id, row within block) and the auxiliary positions of request b,
    each as an int64 array in attended order.
    """
    status = 0
    empty = np.zeros(0, dtype=np.int64)
    b = int(meta["token_batch"][t])
    if b < 0:
        return empty, empty, empty, status
    p = int(meta["token_pos"][t])
    L = int(meta["seqlen_k"][b]) + 1
    MB = block_table.shape[1]
    sel = None
    if selected_idx is not None:
        sel = np.asarray(selected_idx[b if sel_per_request else t, h_kv], dtype=np.int64)
        bad = (sel < -1) | ((sel >= 0) & (sel >= (L if sel_target == 0 else int(aux_seqlens[b]))))
        if bad.any():
            status |= ST_BAD_IDX
    if sel is not None and sel_target == 0:
        # selected main-cache entries: valid, and causal for this token
        main_pos = sel[(sel >= 0) & (sel < L) & (sel <= p)]
    else:
        # causal local window (or dense causal when the window is off)
        lo = max(0, p - window + 1) if window > 0 else 0
        main_pos = np.arange(lo, p + 1, dtype=np.int64)
    if kv_range is not None:
        main_pos = main_pos[(main_pos >= int(kv_range[b][0])) & (main_pos < int(kv_range[b][1]))]
    if sel is not None and sel_target == 1:
        aux_pos = sel[(sel >= 0) & (sel < int(aux_seqlens[b]))]
    else:
        aux_pos = empty
    lb = main_pos // block_size
    in_table = lb < MB
    if not in_table.all():
        status |= ST_CAPACITY
    main_pos, lb = main_pos[in_table], lb[in_table]
    blk = block_table[b, lb].astype(np.int64)
    ok = (blk >= 0) & (blk < num_blocks)
    if not ok.all():
        status |= ST_BAD_BLOCK
    return blk[ok], (main_pos % block_size)[ok], aux_pos, status


def attention(q: np.ndarray, act: str, k_cache: np.ndarray, v_cache: np.ndarray, cache: str,
              block_table: np.ndarray, meta: Dict[str, np.ndarray], *, H_kv: int,
              window: int = 0, selected_idx: Optional[np.ndarray] = None,
              sel_per_request: int = 1, sel_target: int = 0,
              aux_k: Optional[np.ndarray] = None, aux_v: Optional[np.ndarray] = None,
              aux_seqlens: Optional[np.ndarray] = None, sinks: Optional[np.ndarray] = None,
              scale: float = 0.0, k_scale: Optional[np.ndarray] = None,
              v_scale: Optional[np.ndarray] = None,
              tokens: Optional[Iterable[int]] = None,
              kv_range: Optional[np.ndarray] = None) -> Dict[str, np.ndarray]:
    """Output o[T, H_q, D] (float64) and lse[T, H_q] of the attention step.

    For token t at position p in request b and q head h (kv head h // G):
      s_j = scale * <q[t, h], k_j>                    over the attended set
      m   = max(max_j s_j, sink_h)
      l   = sum_j exp(s_j - m) + exp(sink_h - m)
      o   = sum_j exp(s_j - m) v_j / l,  lse = m + log(l)
    With ``tokens`` only those rows are computed (others stay NaN).
    """
    T, H_q, D = q.shape
    G = H_q // H_kv
    NB, bs = k_cache.shape[0], k_cache.shape[1]
    sc = 1.0 / math.sqrt(D) if scale == 0.0 else float(np.float32(scale))
    out = np.full((T, H_q, D), np.nan)
    lse = np.full((T, H_q), np.nan)
    status = 0
    toks = range(T) if tokens is None else tokens
    for t in toks:
        qt = decode(q[t], act)                        # [H_q, D]
        b = int(meta["token_batch"][t])
        for h_kv in range(H_kv):
            blk, off, aux_pos, st = attended_keys(
                t, h_kv, meta, block_table, bs, NB, window, selected_idx,
                sel_per_request, sel_target, aux_seqlens, kv_range)
            status |= st
            K = decode(k_cache[blk, off, h_kv], cache)           # [n_main, D]
            V = decode(v_cache[blk, off, h_kv], cache)
            if aux_pos.size:
                K = np.concatenate([K, decode(aux_k[b, aux_pos, h_kv], cache)])
                V = np.concatenate([V, decode(aux_v[b, aux_pos, h_kv], cache)])
            if cache == "i8":                                    # per-channel dequantise
                K = K * k_scale[h_kv].astype(np.float64)
                V = V * v_scale[h_kv].astype(np.float64)
            for g in range(G):
                h = h_kv * G + g
                sink = -math.inf if sinks is None else float(sinks[h])
                s = sc * (K @ qt[h])                   # [n]
                m = max(float(s.max()) if s.size else -math.inf, sink)
                if m == -math.inf:
                    out[t, h] = 0.0
                    lse[t, h] = -math.inf
                    continue
                e = np.exp(s - m)
                l = float(e.sum()) + math.exp(sink - m)
                out[t, h] = (e @ V) / l
                lse[t, h] = m + math.log(l)
    return {"out": out, "lse": lse, "status": status}


# ---------------------------------------------------------------------------
# 5b. sequence-sharded split-KV: merge of per-shard partial states
# ---------------------------------------------------------------------------
#
# "[WebGPU] Add SparsePagedAttention", File summaries: the main and the
# auxiliary pass each leave a partial FP32 softmax state, and a finalize stage
# merges them and applies the sink.  A sequence split across devices is the
# same merge over shards: shard r attends only its key range (attention()
# with kv_range and no sink) and leaves o_r (normalised over its keys, 0 when
# it has none) and lse_r = m_r + log(l_r) (-inf when it has none).  Then
#   M   = max(sink, max_r lse_r)
#   L   = exp(sink - M) + sum_r exp(lse_r - M)
#   out = sum_r exp(lse_r - M) o_r / L,   lse = M + log(L)
# (out = 0 and lse = -inf when M = -inf): the sink is counted once.

def merge_partials(outs: np.ndarray, lses: np.ndarray, sinks: Optional[np.ndarray]):
    """Merge R shards' partial states outs [R, T, H_q, D], lses [R, T, H_q]
    with the per-head sinks [H_q] (or none).  Returns (out, lse) in float64."""
    outs = np.asarray(outs, dtype=np.float64)
    lses = np.asarray(lses, dtype=np.float64)
    R, T, H_q, D = outs.shape
    out = np.zeros((T, H_q, D))
    lse = np.full((T, H_q), -math.inf)
    for t in range(T):
        for h in range(H_q):
            sink = -math.inf if sinks is None else float(sinks[h])
            M = max([sink] + [float(lses[r, t, h]) for r in range(R)])
            if M == -math.inf:
                continue
            w = [math.exp(float(lses[r, t, h]) - M) for r in range(R)]
            L = math.exp(sink - M) + sum(w)
            out[t, h] = sum(w[r] * outs[r, t, h] for r in range(R)) / L
            lse[t, h] = M + math.log(L)
    return out, lse


# ---------------------------------------------------------------------------
# the whole step
# ---------------------------------------------------------------------------

def run_step(wl, tokens: Optional[Sequence[int]] = None) -> Dict[str, np.ndarray]:
    """Metadata prepare, KV append, attention over one synthetic workload.

    ``wl`` is a workload object exposing the named arrays and parameters.
    """
    a = wl.arrays
    meta = prepare_metadata(a["cu_seqlens_q"], a["past_seqlens"], a["block_table"], wl.T,
                            wl.max_seqlen_q, wl.max_seqlen_k, wl.block_size, wl.NB)
    q, k_new, v_new = a["q"], a["k_new"], a["v_new"]
    pro = getattr(wl, "prologue", None)
    if pro:
        if pro.get("packed"):
            q, k_new, v_new = split_packed(a["qkv"], wl.H_q, wl.H_kv)
        q, k_new, v_new, st = qkv_prologue(
            q, k_new, v_new, wl.act, meta["token_pos"], a.get("q_norm_weight"),
            a.get("k_norm_weight"), pro.get("eps", 1e-6), a.get("cos_cache"), a.get("sin_cache"),
            pro.get("rotary_dim", 0), pro.get("interleaved", False), a.get("position_ids"),
            pro.get("rotary_offset", 0))
        meta = dict(meta, status=meta["status"] | st)
    kc, vc = append_kv(k_new, v_new, wl.act, a["k_cache"], a["v_cache"], wl.cache,
                       meta["slot_mapping"], a.get("k_scale"), a.get("v_scale"))
    sel = a.get("selected_idx")
    res = attention(q, wl.act, kc, vc, wl.cache, a["block_table"], meta, H_kv=wl.H_kv,
                    window=wl.window, selected_idx=sel, sel_per_request=wl.sel_per_request,
                    sel_target=1 if wl.sel_mode == "aux" else 0, aux_k=a.get("aux_k"),
                    aux_v=a.get("aux_v"), aux_seqlens=a.get("aux_seqlens"),
                    sinks=a.get("sinks"), scale=wl.scale, k_scale=a.get("k_scale"),
                    v_scale=a.get("v_scale"), tokens=tokens)
    res["meta"] = meta
    res["k_cache"] = kc
    res["v_cache"] = vc
    if pro:
        res["q_out"] = q
    res["status"] = res["status"] | meta["status"]
    return res
