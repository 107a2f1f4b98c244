"""One pass of the hot path through the C ABI: metadata prepare, KV append,
attention.  Used by the tests, the bench and the smoke check; contains no
arithmetic of the method (that all runs in libspa's kernels).
"""
from __future__ import annotations

from typing import Dict, Optional

import numpy as np
import torch

from . import spa

_TORCH = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16, "i8": torch.int8,
          "i32": torch.int32}


def tensor_of(arr: np.ndarray, dtype: str) -> torch.Tensor:
    """Host tensor for a workload array (bf16 arrays are carried as uint16 bits)."""
    t = torch.from_numpy(np.ascontiguousarray(arr))
    if dtype == "bf16":
        return t.view(torch.int16).view(torch.bfloat16)
    return t.to(_TORCH[dtype]) if t.dtype != _TORCH[dtype] else t


def to_device(wl, device="cuda", pin: bool = False) -> Dict[str, torch.Tensor]:
    out = {}
    for k, arr in wl.arrays.items():
        t = tensor_of(arr, wl.dtypes[k])
        out[k] = t.pin_memory() if pin else t.to(device)
    return out


def attention_kwargs(wl, d: Dict[str, torch.Tensor]) -> dict:
    return dict(window=wl.window, selected_idx=d.get("selected_idx"),
                sel_per_request=wl.sel_per_request, sel_target=1 if wl.sel_mode == "aux" else 0,
                aux_k=d.get("aux_k"), aux_v=d.get("aux_v"), aux_seqlens=d.get("aux_seqlens"),
                sinks=d.get("sinks"), scale=wl.scale, k_scale=d.get("k_scale"),
                v_scale=d.get("v_scale"))


MODES = ("step", "prepare_append", "staged")


class Step:
    """Pre-allocated buffers for repeated steps of one workload on one device.

    mode "step": spa_prepare_append_attention (one launch where the path
    allows it); "prepare_append": spa_prepare_append_kv then spa_attention;
    "staged": spa_prepare_metadata, spa_append_kv, spa_attention.  A workload
    with a QKV prologue runs spa_prepare_qkv_append (metadata, prologue,
    append) and then spa_attention on the prologue's q, whatever the mode.
    """

    def __init__(self, wl, d: Dict[str, torch.Tensor], num_splits: int = 0,
                 want_lse: bool = False, mode: str = "step"):
        if mode not in MODES:
            raise ValueError(f"mode must be one of {MODES}")
        self.wl, self.d, self.mode = wl, d, mode
        dev = d["q"].device
        i32 = dict(dtype=torch.int32, device=dev)
        B, T = wl.B, wl.T
        self.meta = {"seqlens_q": torch.empty(B, **i32), "seqlen_k": torch.empty(B, **i32),
                     "token_batch": torch.empty(T, **i32), "token_pos": torch.empty(T, **i32),
                     "slot_mapping": torch.empty(T, **i32)}
        self.status = torch.zeros(1, **i32)
        self.out = torch.empty_like(d["q"])
        self.lse = torch.empty(T, wl.H_q, dtype=torch.float32, device=dev) if want_lse else None
        self.num_splits = num_splits
        self.kw = attention_kwargs(wl, d)
        meta = dict(self.meta, cu_seqlens_q=d["cu_seqlens_q"], status=self.status)
        self.pro = getattr(wl, "prologue", None)
        q_att = d["q"]
        if self.pro:
            self.q_pro = torch.empty_like(d["q"])
            q_att = self.q_pro
            packed = bool(self.pro.get("packed"))
            self.qargs = spa.qkv_args(
                d["cu_seqlens_q"], d["past_seqlens"], d["block_table"], T, wl.max_seqlen_q,
                wl.max_seqlen_k, self.meta, H_q=wl.H_q, q_out=self.q_pro, k_cache=d["k_cache"],
                v_cache=d["v_cache"], qkv=d["qkv"] if packed else None,
                q=None if packed else d["q"], k=None if packed else d["k_new"],
                v=None if packed else d["v_new"], q_norm_weight=d.get("q_norm_weight"),
                k_norm_weight=d.get("k_norm_weight"), norm_eps=self.pro.get("eps", 1e-6),
                cos_cache=d.get("cos_cache"), sin_cache=d.get("sin_cache"),
                rotary_dim=self.pro.get("rotary_dim", 0),
                rotary_interleaved=self.pro.get("interleaved", False),
                position_ids=d.get("position_ids"), rotary_offset=self.pro.get("rotary_offset", 0),
                k_scale=d.get("k_scale"), v_scale=d.get("v_scale"), status=self.status)
        self.args = spa.attention_args(q_att, d["k_cache"], d["v_cache"], d["block_table"], meta,
                                       max_seqlen_q=wl.max_seqlen_q, max_seqlen_k=wl.max_seqlen_k,
                                       out=self.out, lse=self.lse, num_splits=num_splits,
                                       status=self.status, **self.kw)
        self.workspace = spa.new_workspace(spa.workspace_size(self.args), dev)
        self._bound = None
        if mode == "step" and not self.pro:
            self._bound = spa.BoundStep(self.args, d["past_seqlens"], d["k_new"], d["v_new"],
                                        self.meta["slot_mapping"], self.workspace)

    def launches(self) -> int:
        """Kernel launches one call makes."""
        if self.pro:
            return 1 + spa.attention_plan(self.args)["launches"]
        if self.mode == "step":
            return spa.prepare_append_attention_launches(self.args)
        return (1 if self.mode == "prepare_append" else 2) + spa.attention_plan(self.args)["launches"]

    def __call__(self):
        wl, d = self.wl, self.d
        if self.pro:
            spa.run_prepare_qkv_append(self.qargs, d["q"].device)
            spa.run_attention(self.args, self.workspace)
            return self.out
        if self.mode == "step":
            self._bound()   # spa_prepare_append_attention, arguments marshalled once
            return self.out
        if self.mode == "prepare_append":
            spa.prepare_append_kv(d["cu_seqlens_q"], d["past_seqlens"], d["block_table"],
                                  wl.T, wl.max_seqlen_q, wl.max_seqlen_k, d["k_new"],
                                  d["v_new"], d["k_cache"], d["v_cache"],
                                  k_scale=d.get("k_scale"), v_scale=d.get("v_scale"),
                                  status=self.status, out=self.meta)
        else:
            spa.prepare_metadata(d["cu_seqlens_q"], d["past_seqlens"], d["block_table"],
                                 wl.T, wl.max_seqlen_q, wl.max_seqlen_k, wl.block_size,
                                 wl.NB, status=self.status, out=self.meta)
            spa.append_kv(d["k_new"], d["v_new"], d["k_cache"], d["v_cache"],
                          self.meta["slot_mapping"], k_scale=d.get("k_scale"),
                          v_scale=d.get("v_scale"), status=self.status)
        spa.run_attention(self.args, self.workspace)
        return self.out


def run_step(wl, device="cuda", num_splits: int = 0, want_lse: bool = True, mode: str = "step"):
    """Run one step on fresh device copies; returns host numpy results."""
    d = to_device(wl, device)
    st = Step(wl, d, num_splits=num_splits, want_lse=want_lse, mode=mode)
    st()
    torch.cuda.synchronize(device)
    res = {k: v.cpu().numpy() for k, v in st.meta.items()}
    res["status"] = int(st.status.item())
    res["out"] = st.out.float().cpu().numpy().astype(np.float64)
    if st.lse is not None:
        res["lse"] = st.lse.cpu().numpy().astype(np.float64)
    res["k_cache"] = d["k_cache"].cpu()
    res["v_cache"] = d["v_cache"].cpu()
    if st.pro:
        res["q_out"] = st.q_pro.cpu()
    return res
