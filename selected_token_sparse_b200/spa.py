"""Thin Python binding of libspa (ctypes).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels.  Tensors must be CUDA tensors; outputs are allocated with torch on
the input's device (the library itself never allocates).  Work is enqueued on
torch's current stream.  If libspa.so is missing the import fails loudly --
there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libspa.so")

SPA_F32, SPA_F16, SPA_BF16, SPA_I8 = 0, 1, 2, 3
SPA_OK, SPA_ERR_INVALID_ARG, SPA_ERR_UNSUPPORTED, SPA_ERR_WORKSPACE, SPA_ERR_CUDA = 0, -1, -2, -3, -4
ST_BAD_CU, ST_CAPACITY, ST_BAD_BLOCK, ST_BOUNDS, ST_BAD_IDX = 0x1, 0x2, 0x4, 0x8, 0x10

EXPORTED = ("spa_prepare_metadata", "spa_append_kv", "spa_prepare_append_kv", "spa_prepare_qkv_append",
            "spa_attention", "spa_attention_workspace_size", "spa_attention_plan",
            "spa_prepare_append_attention", "spa_prepare_append_attention_launches",
            "spa_attention_noalloc", "spa_select_topk", "spa_merge_partials", "spa_error_string")

_DT = {torch.float32: SPA_F32, torch.float16: SPA_F16, torch.bfloat16: SPA_BF16, torch.int8: SPA_I8}

_vp = ctypes.c_void_p
_i32 = ctypes.c_int32


class AttentionArgs(ctypes.Structure):
    """Mirror of spa_attention_args_t (include/spa.h)."""
    _fields_ = [
        ("struct_size", ctypes.c_size_t),
        ("q", _vp), ("out", _vp), ("act", _i32),
        ("T", _i32), ("B", _i32), ("H_q", _i32), ("H_kv", _i32), ("D", _i32),
        ("k_cache", _vp), ("v_cache", _vp), ("cache", _i32),
        ("k_scale", _vp), ("v_scale", _vp),
        ("block_table", _vp),
        ("MB", _i32), ("block_size", _i32), ("num_blocks", _i32),
        ("cu_seqlens_q", _vp), ("seqlens_q", _vp), ("seqlen_k", _vp),
        ("token_batch", _vp), ("token_pos", _vp),
        ("max_seqlen_q", _i32), ("max_seqlen_k", _i32),
        ("is_causal", _i32), ("window", _i32),
        ("selected_idx", _vp), ("sel_width", _i32), ("sel_per_request", _i32), ("sel_target", _i32),
        ("aux_k", _vp), ("aux_v", _vp), ("aux_cap", _i32), ("aux_seqlens", _vp),
        ("sinks", _vp), ("scale", ctypes.c_float), ("lse", _vp),
        ("num_splits", _i32), ("status", _vp),
        ("kv_range", _vp), ("partial", _i32), ("test_expire_wait", _i32),
    ]


class QkvArgs(ctypes.Structure):
    """Mirror of spa_qkv_args_t (include/spa.h)."""
    _fields_ = [
        ("struct_size", ctypes.c_size_t),
        ("cu_seqlens_q", _vp), ("past_seqlens", _vp), ("block_table", _vp),
        ("B", _i32), ("T", _i32), ("max_seqlen_q", _i32), ("max_seqlen_k", _i32), ("MB", _i32),
        ("block_size", _i32), ("num_blocks", _i32),
        ("seqlens_q", _vp), ("seqlen_k", _vp), ("token_batch", _vp), ("token_pos", _vp),
        ("slot_mapping", _vp),
        ("act", _i32), ("H_q", _i32), ("H_kv", _i32), ("D", _i32),
        ("qkv", _vp), ("q", _vp), ("k", _vp), ("v", _vp),
        ("q_norm_weight", _vp), ("k_norm_weight", _vp), ("norm_eps", ctypes.c_float),
        ("cos_cache", _vp), ("sin_cache", _vp),
        ("max_pos", _i32), ("rotary_dim", _i32), ("rotary_interleaved", _i32),
        ("position_ids", _vp), ("rotary_offset", _i32),
        ("q_out", _vp), ("k_cache", _vp), ("v_cache", _vp), ("cache", _i32),
        ("k_scale", _vp), ("v_scale", _vp), ("status", _vp),
    ]


class SpaError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {error_string(code)} (code {code})")
        self.code = code


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise RuntimeError(f"libspa.so not found at {path}; build it with "
                           "`python -m selected_token_sparse_b200.build`")
    lib = ctypes.CDLL(path)
    lib.spa_prepare_metadata.restype = ctypes.c_int
    lib.spa_prepare_metadata.argtypes = [_vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _i32,
                                         _vp, _vp, _vp, _vp, _vp, _vp, _vp]
    lib.spa_append_kv.restype = ctypes.c_int
    lib.spa_append_kv.argtypes = [_vp, _vp, _i32, _vp, _vp, _i32, _vp, _vp, _vp, _i32, _i32, _i32,
                                  _i32, _i32, _vp, _vp]
    lib.spa_prepare_append_kv.restype = ctypes.c_int
    lib.spa_prepare_append_kv.argtypes = [_vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _i32,
                                          _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _vp, _vp, _i32,
                                          _vp, _vp, _i32, _i32, _vp, _vp]
    lib.spa_attention_workspace_size.restype = ctypes.c_size_t
    lib.spa_attention_workspace_size.argtypes = [ctypes.POINTER(AttentionArgs)]
    lib.spa_attention.restype = ctypes.c_int
    lib.spa_attention.argtypes = [ctypes.POINTER(AttentionArgs), _vp, ctypes.c_size_t, _vp]
    lib.spa_attention_plan.restype = ctypes.c_int
    lib.spa_attention_plan.argtypes = [ctypes.POINTER(AttentionArgs), _vp, _vp, _vp]
    lib.spa_prepare_append_attention.restype = ctypes.c_int
    lib.spa_prepare_append_attention.argtypes = [ctypes.POINTER(AttentionArgs), _vp, _vp, _vp, _vp, _vp,
                                                 ctypes.c_size_t, _vp]
    lib.spa_prepare_append_attention_launches.restype = ctypes.c_int
    lib.spa_prepare_append_attention_launches.argtypes = [ctypes.POINTER(AttentionArgs)]
    lib.spa_prepare_qkv_append.restype = ctypes.c_int
    lib.spa_prepare_qkv_append.argtypes = [ctypes.POINTER(QkvArgs), _vp]
    lib.spa_merge_partials.restype = ctypes.c_int
    lib.spa_merge_partials.argtypes = [_vp, _vp, _i32, _i32, _i32, _i32, _vp, _i32, _vp, _vp, _vp]
    lib.spa_select_topk.restype = ctypes.c_int
    lib.spa_select_topk.argtypes = [_vp, _i32, _i32, _i32, _vp, _i32, _i32, _vp, _vp]
    lib.spa_error_string.restype = ctypes.c_char_p
    lib.spa_error_string.argtypes = [ctypes.c_int]
    return lib


_LIB: Optional[ctypes.CDLL] = None


def lib() -> ctypes.CDLL:
    global _LIB
    if _LIB is None:
        _LIB = load_library()
    return _LIB


def error_string(code: int) -> str:
    return lib().spa_error_string(code).decode()


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libspa takes CUDA tensors")
    if not t.is_contiguous():
        raise ValueError("libspa takes contiguous tensors")
    return t.data_ptr()


def _stream(device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _check(code: int, what: str):
    if code != SPA_OK:
        raise SpaError(code, what)


def new_status(device) -> torch.Tensor:
    return torch.zeros(1, dtype=torch.int32, device=device)


def prepare_metadata(cu_seqlens_q: torch.Tensor, past_seqlens: torch.Tensor,
                     block_table: torch.Tensor, T: int, max_seqlen_q: int, max_seqlen_k: int,
                     block_size: int, num_blocks: int, status: Optional[torch.Tensor] = None,
                     out: Optional[Dict[str, torch.Tensor]] = None) -> Dict[str, torch.Tensor]:
    """Step 1: per-request seqlens_q / seqlen_k and per-token batch / pos / slot."""
    dev = cu_seqlens_q.device
    B = cu_seqlens_q.numel() - 1
    MB = block_table.shape[1] if block_table.dim() == 2 else 0
    if out is None:
        i32 = dict(dtype=torch.int32, device=dev)
        out = {"seqlens_q": torch.empty(B, **i32), "seqlen_k": torch.empty(B, **i32),
               "token_batch": torch.empty(T, **i32), "token_pos": torch.empty(T, **i32),
               "slot_mapping": torch.empty(T, **i32)}
    if status is None:
        status = new_status(dev)
    out["status"] = status
    rc = lib().spa_prepare_metadata(
        _ptr(cu_seqlens_q), _ptr(past_seqlens), _ptr(block_table), B, T, max_seqlen_q,
        max_seqlen_k, MB, block_size, num_blocks, _ptr(out["seqlens_q"]), _ptr(out["seqlen_k"]),
        _ptr(out["token_batch"]), _ptr(out["token_pos"]), _ptr(out["slot_mapping"]),
        _ptr(status), _stream(dev))
    _check(rc, "spa_prepare_metadata")
    out["cu_seqlens_q"] = cu_seqlens_q
    return out


def append_kv(k_new: torch.Tensor, v_new: torch.Tensor, k_cache: torch.Tensor,
              v_cache: torch.Tensor, slot_mapping: torch.Tensor,
              k_scale: Optional[torch.Tensor] = None, v_scale: Optional[torch.Tensor] = None,
              status: Optional[torch.Tensor] = None) -> None:
    """Step 2: scatter k_new/v_new [T, H_kv, D] into the paged cache [NB, bs, H_kv, D]."""
    T, H_kv, D = k_new.shape
    NB, bs = k_cache.shape[0], k_cache.shape[1]
    if status is None:
        status = new_status(k_new.device)
    rc = lib().spa_append_kv(_ptr(k_new), _ptr(v_new), _DT[k_new.dtype], _ptr(k_cache),
                             _ptr(v_cache), _DT[k_cache.dtype], _ptr(k_scale), _ptr(v_scale),
                             _ptr(slot_mapping), T, H_kv, D, bs, NB, _ptr(status),
                             _stream(k_new.device))
    _check(rc, "spa_append_kv")


def prepare_append_kv(cu_seqlens_q: torch.Tensor, past_seqlens: torch.Tensor,
                      block_table: torch.Tensor, T: int, max_seqlen_q: int, max_seqlen_k: int,
                      k_new: torch.Tensor, v_new: torch.Tensor, k_cache: torch.Tensor,
                      v_cache: torch.Tensor, k_scale: Optional[torch.Tensor] = None,
                      v_scale: Optional[torch.Tensor] = None, status: Optional[torch.Tensor] = None,
                      out: Optional[Dict[str, torch.Tensor]] = None) -> Dict[str, torch.Tensor]:
    """Steps 1 + 2 in one launch (same results as prepare_metadata then append_kv)."""
    dev = cu_seqlens_q.device
    B = cu_seqlens_q.numel() - 1
    MB = block_table.shape[1] if block_table.dim() == 2 else 0
    NB, bs, H_kv, D = k_cache.shape
    if out is None:
        i32 = dict(dtype=torch.int32, device=dev)
        out = {"seqlens_q": torch.empty(B, **i32), "seqlen_k": torch.empty(B, **i32),
               "token_batch": torch.empty(T, **i32), "token_pos": torch.empty(T, **i32),
               "slot_mapping": torch.empty(T, **i32)}
    if status is None:
        status = new_status(dev)
    out["status"] = status
    rc = lib().spa_prepare_append_kv(
        _ptr(cu_seqlens_q), _ptr(past_seqlens), _ptr(block_table), B, T, max_seqlen_q,
        max_seqlen_k, MB, bs, NB, _ptr(out["seqlens_q"]), _ptr(out["seqlen_k"]),
        _ptr(out["token_batch"]), _ptr(out["token_pos"]), _ptr(out["slot_mapping"]),
        _ptr(k_new), _ptr(v_new), _DT[k_new.dtype], _ptr(k_cache), _ptr(v_cache),
        _DT[k_cache.dtype], _ptr(k_scale), _ptr(v_scale), H_kv, D, _ptr(status), _stream(dev))
    _check(rc, "spa_prepare_append_kv")
    out["cu_seqlens_q"] = cu_seqlens_q
    return out


def qkv_args(cu_seqlens_q: torch.Tensor, past_seqlens: torch.Tensor, block_table: torch.Tensor, T: int,
             max_seqlen_q: int, max_seqlen_k: int, meta: Dict[str, torch.Tensor], *, H_q: int,
             q_out: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
             qkv: Optional[torch.Tensor] = None, q: Optional[torch.Tensor] = None,
             k: Optional[torch.Tensor] = None, v: Optional[torch.Tensor] = None,
             q_norm_weight: Optional[torch.Tensor] = None, k_norm_weight: Optional[torch.Tensor] = None,
             norm_eps: float = 1e-6, cos_cache: Optional[torch.Tensor] = None,
             sin_cache: Optional[torch.Tensor] = None, rotary_dim: int = 0, rotary_interleaved: bool = False,
             position_ids: Optional[torch.Tensor] = None, rotary_offset: int = 0,
             k_scale: Optional[torch.Tensor] = None, v_scale: Optional[torch.Tensor] = None,
             status: Optional[torch.Tensor] = None) -> QkvArgs:
    """Arguments of spa_prepare_qkv_append (steps 1, prologue, 2); `meta` holds the
    five metadata output arrays."""
    NB, bs, H_kv, D = k_cache.shape
    a = QkvArgs()
    a.struct_size = ctypes.sizeof(QkvArgs)
    a.cu_seqlens_q, a.past_seqlens, a.block_table = _ptr(cu_seqlens_q), _ptr(past_seqlens), _ptr(block_table)
    a.B, a.T = cu_seqlens_q.numel() - 1, T
    a.max_seqlen_q, a.max_seqlen_k = max_seqlen_q, max_seqlen_k
    a.MB = block_table.shape[1] if block_table.dim() == 2 else 0
    a.block_size, a.num_blocks = bs, NB
    a.seqlens_q, a.seqlen_k = _ptr(meta["seqlens_q"]), _ptr(meta["seqlen_k"])
    a.token_batch, a.token_pos, a.slot_mapping = (_ptr(meta["token_batch"]), _ptr(meta["token_pos"]),
                                                  _ptr(meta["slot_mapping"]))
    a.act = _DT[q_out.dtype]
    a.H_q, a.H_kv, a.D = H_q, H_kv, D
    a.qkv, a.q, a.k, a.v = _ptr(qkv), _ptr(q), _ptr(k), _ptr(v)
    a.q_norm_weight, a.k_norm_weight, a.norm_eps = _ptr(q_norm_weight), _ptr(k_norm_weight), float(norm_eps)
    a.cos_cache, a.sin_cache = _ptr(cos_cache), _ptr(sin_cache)
    a.max_pos = cos_cache.shape[0] if cos_cache is not None else 0
    a.rotary_dim = rotary_dim if cos_cache is not None else 0
    a.rotary_interleaved = 1 if rotary_interleaved else 0
    a.position_ids, a.rotary_offset = _ptr(position_ids), rotary_offset
    a.q_out, a.k_cache, a.v_cache, a.cache = _ptr(q_out), _ptr(k_cache), _ptr(v_cache), _DT[k_cache.dtype]
    a.k_scale, a.v_scale = _ptr(k_scale), _ptr(v_scale)
    a.status = _ptr(status)
    return a


def run_prepare_qkv_append(args: QkvArgs, device) -> None:
    """Enqueue spa_prepare_qkv_append for prepared arguments on the current stream."""
    _check(lib().spa_prepare_qkv_append(ctypes.byref(args), _stream(device)), "spa_prepare_qkv_append")


def attention_args(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                   block_table: torch.Tensor, meta: Dict[str, torch.Tensor], *,
                   max_seqlen_q: int, max_seqlen_k: int, out: torch.Tensor,
                   lse: Optional[torch.Tensor] = None, window: int = 0,
                   selected_idx: Optional[torch.Tensor] = None, sel_per_request: int = 1,
                   sel_target: int = 0, aux_k: Optional[torch.Tensor] = None,
                   aux_v: Optional[torch.Tensor] = None, aux_seqlens: Optional[torch.Tensor] = None,
                   sinks: Optional[torch.Tensor] = None, scale: float = 0.0,
                   k_scale: Optional[torch.Tensor] = None, v_scale: Optional[torch.Tensor] = None,
                   num_splits: int = 0, status: Optional[torch.Tensor] = None,
                   is_causal: int = 1, kv_range: Optional[torch.Tensor] = None,
                   partial: bool = False) -> AttentionArgs:
    """Argument struct of spa_attention.  It holds raw device addresses: every
    tensor passed here must stay alive for as long as the struct is used."""
    T, H_q, D = q.shape
    a = AttentionArgs()
    a.struct_size = ctypes.sizeof(AttentionArgs)
    a.q, a.out, a.act = _ptr(q), _ptr(out), _DT[q.dtype]
    a.T, a.B, a.H_q, a.H_kv, a.D = T, meta["seqlens_q"].numel(), H_q, k_cache.shape[2], D
    a.k_cache, a.v_cache, a.cache = _ptr(k_cache), _ptr(v_cache), _DT[k_cache.dtype]
    a.k_scale, a.v_scale = _ptr(k_scale), _ptr(v_scale)
    a.block_table = _ptr(block_table)
    a.MB, a.block_size, a.num_blocks = block_table.shape[1], k_cache.shape[1], k_cache.shape[0]
    a.cu_seqlens_q = _ptr(meta["cu_seqlens_q"])
    a.seqlens_q, a.seqlen_k = _ptr(meta["seqlens_q"]), _ptr(meta["seqlen_k"])
    a.token_batch, a.token_pos = _ptr(meta["token_batch"]), _ptr(meta["token_pos"])
    a.max_seqlen_q, a.max_seqlen_k = max_seqlen_q, max_seqlen_k
    a.is_causal, a.window = is_causal, window
    a.selected_idx = _ptr(selected_idx)
    a.sel_width = selected_idx.shape[-1] if selected_idx is not None else 0
    a.sel_per_request, a.sel_target = sel_per_request, sel_target
    a.aux_k, a.aux_v = _ptr(aux_k), _ptr(aux_v)
    a.aux_cap = aux_k.shape[1] if aux_k is not None else 0
    a.aux_seqlens = _ptr(aux_seqlens)
    a.sinks, a.scale, a.lse = _ptr(sinks), float(scale), _ptr(lse)
    a.num_splits = num_splits
    a.status = _ptr(status if status is not None else meta.get("status"))
    a.kv_range = _ptr(kv_range)
    a.partial = 1 if partial else 0
    return a


def new_workspace(nbytes: int, device) -> torch.Tensor:
    """A zero-filled workspace (its tickets and work counter must start at zero)."""
    return torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def workspace_size(args: AttentionArgs) -> int:
    return int(lib().spa_attention_workspace_size(ctypes.byref(args)))


def attention_plan(args: AttentionArgs) -> Dict[str, int]:
    """What spa_attention would launch: splits, launches, kernel kind."""
    ns, nl, kk = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
    rc = lib().spa_attention_plan(ctypes.byref(args), ctypes.addressof(ns), ctypes.addressof(nl),
                                  ctypes.addressof(kk))
    _check(rc, "spa_attention_plan")
    return {"num_splits": ns.value, "launches": nl.value, "kind": kk.value}


def run_attention(args: AttentionArgs, workspace: Optional[torch.Tensor]) -> None:
    """Enqueue spa_attention for prepared arguments on the current stream."""
    need = workspace_size(args)
    if need and (workspace is None or workspace.numel() < need):
        raise SpaError(SPA_ERR_WORKSPACE, "spa_attention")
    ws = _ptr(workspace) if need else None
    dev = workspace.device if workspace is not None else torch.device("cuda")
    rc = lib().spa_attention(ctypes.byref(args), ws, need, _stream(dev))
    _check(rc, "spa_attention")


def run_prepare_append_attention(args: AttentionArgs, past_seqlens: torch.Tensor, k_new: torch.Tensor,
                                 v_new: torch.Tensor, slot_mapping: torch.Tensor,
                                 workspace: Optional[torch.Tensor]) -> None:
    """Enqueue steps 1-5 (spa_prepare_append_attention) for prepared arguments on the
    current stream; the metadata arrays `args` points at are written."""
    need = workspace_size(args)
    if need and (workspace is None or workspace.numel() < need):
        raise SpaError(SPA_ERR_WORKSPACE, "spa_prepare_append_attention")
    rc = lib().spa_prepare_append_attention(ctypes.byref(args), _ptr(past_seqlens), _ptr(k_new),
                                            _ptr(v_new), _ptr(slot_mapping), _ptr(workspace) if need else None,
                                            need, _stream(k_new.device))
    _check(rc, "spa_prepare_append_attention")


class BoundStep:
    """spa_prepare_append_attention with every argument marshalled once: each
    call passes the prepared pointers and the current stream, nothing else.
    The tensors the arguments point at must stay alive and in place."""

    def __init__(self, args: AttentionArgs, past_seqlens: torch.Tensor, k_new: torch.Tensor,
                 v_new: torch.Tensor, slot_mapping: torch.Tensor, workspace: Optional[torch.Tensor]):
        need = workspace_size(args)
        if need and (workspace is None or workspace.numel() < need):
            raise SpaError(SPA_ERR_WORKSPACE, "spa_prepare_append_attention")
        self._fn = lib().spa_prepare_append_attention
        self._args = ctypes.byref(args)
        self._ptrs = (_ptr(past_seqlens), _ptr(k_new), _ptr(v_new), _ptr(slot_mapping),
                      _ptr(workspace) if need else None, need)
        self._dev = k_new.device
        self._keep = (args, past_seqlens, k_new, v_new, slot_mapping, workspace)

    def __call__(self) -> None:
        rc = self._fn(self._args, *self._ptrs, torch.cuda.current_stream(self._dev).cuda_stream)
        if rc != SPA_OK:
            raise SpaError(rc, "spa_prepare_append_attention")


def prepare_append_attention_launches(args: AttentionArgs) -> int:
    """Kernel launches spa_prepare_append_attention makes for these arguments (1 or 2)."""
    rc = int(lib().spa_prepare_append_attention_launches(ctypes.byref(args)))
    if rc < 0:
        _check(rc, "spa_prepare_append_attention_launches")
    return rc


def attention(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
              block_table: torch.Tensor, meta: Dict[str, torch.Tensor], *, max_seqlen_q: int,
              max_seqlen_k: int, out: Optional[torch.Tensor] = None, want_lse: bool = False,
              workspace: Optional[torch.Tensor] = None, **kw):
    """Steps 3-5: sparse / paged attention; returns (out, lse or None)."""
    if out is None:
        out = torch.empty_like(q)
    lse = torch.empty(q.shape[0], q.shape[1], dtype=torch.float32, device=q.device) if want_lse else None
    a = attention_args(q, k_cache, v_cache, block_table, meta, max_seqlen_q=max_seqlen_q,
                       max_seqlen_k=max_seqlen_k, out=out, lse=lse, **kw)
    need = workspace_size(a)
    if need and (workspace is None or workspace.numel() < need):
        workspace = new_workspace(need, q.device)
    rc = lib().spa_attention(ctypes.byref(a), _ptr(workspace) if need else None, need,
                             _stream(q.device))
    _check(rc, "spa_attention")
    return out, lse


def select_topk(scores: torch.Tensor, bound: torch.Tensor, top_k: int, sel_width: int,
                out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Selection producer: the top_k keys of fp32 scores [R, H, n_keys] per row,
    keys 0..bound[r] eligible; returns selected_idx [R, H, sel_width] (increasing,
    -1 padded), the layout spa_attention's selected mode reads."""
    R, H, N = scores.shape
    if scores.dtype != torch.float32 or bound.dtype != torch.int32:
        raise ValueError("select_topk takes fp32 scores and int32 bounds")
    if out is None:
        out = torch.empty(R, H, sel_width, dtype=torch.int32, device=scores.device)
    rc = lib().spa_select_topk(_ptr(scores), R, H, N, _ptr(bound), int(top_k), int(sel_width), _ptr(out),
                               _stream(scores.device))
    _check(rc, "spa_select_topk")
    return out


def merge_partials(part_out: torch.Tensor, part_lse: torch.Tensor, sinks: Optional[torch.Tensor],
                   out: torch.Tensor, lse: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Merge R shards' partial states part_out [R, T, H_q, D] fp32 and
    part_lse [R, T, H_q] (spa_attention with partial=1 over each shard's
    kv_range) into out [T, H_q, D] (its own dtype), the sink counted once."""
    R, T, H_q, D = part_out.shape
    rc = lib().spa_merge_partials(_ptr(part_out), _ptr(part_lse), R, T, H_q, D, _ptr(sinks), _DT[out.dtype],
                                  _ptr(out), _ptr(lse), _stream(out.device))
    _check(rc, "spa_merge_partials")
    return out
