"""The host-side planner needs no GPU.

spa_attention_plan and spa_prepare_append_attention_launches decide, from
shapes alone, which kernel runs, into how many splits the keys go and how many
launches a call makes.  The pointers below are placeholders: the planner only
checks them for presence and 16-byte alignment and never dereferences them.
"""
import ctypes

import pytest

from selected_token_sparse_b200 import spa
from selected_token_sparse_b200 import workloads as W

CODE = {"f32": spa.SPA_F32, "f16": spa.SPA_F16, "bf16": spa.SPA_BF16, "i8": spa.SPA_I8}
SCALAR, MMA, PREFILL, TC = 0, 1, 2, 3


def args_for(wl, num_splits=0):
    a = spa.AttentionArgs()
    a.struct_size = ctypes.sizeof(spa.AttentionArgs)
    addrs = iter(range(1, 1000))

    def ptr():
        return next(addrs) << 20

    arr = wl.arrays
    a.q, a.out, a.act = ptr(), ptr(), CODE[wl.act]
    a.T, a.B, a.H_q, a.H_kv, a.D = wl.T, wl.B, wl.H_q, wl.H_kv, wl.D
    a.k_cache, a.v_cache, a.cache = ptr(), ptr(), CODE[wl.cache]
    if wl.cache == "i8":
        a.k_scale, a.v_scale = ptr(), ptr()
    a.block_table, a.MB, a.block_size, a.num_blocks = ptr(), wl.MB, wl.block_size, wl.NB
    a.cu_seqlens_q, a.seqlens_q, a.seqlen_k = ptr(), ptr(), ptr()
    a.token_batch, a.token_pos = ptr(), ptr()
    a.max_seqlen_q, a.max_seqlen_k = wl.max_seqlen_q, wl.max_seqlen_k
    a.is_causal, a.window = 1, wl.window
    if "selected_idx" in arr:
        a.selected_idx, a.sel_width = ptr(), arr["selected_idx"].shape[-1]
    a.sel_per_request, a.sel_target = wl.sel_per_request, 1 if wl.sel_mode == "aux" else 0
    if "aux_k" in arr:
        a.aux_k, a.aux_v, a.aux_seqlens, a.aux_cap = ptr(), ptr(), ptr(), arr["aux_k"].shape[1]
    if "sinks" in arr:
        a.sinks = ptr()
    a.scale, a.num_splits, a.status = wl.scale, num_splits, ptr()
    return a


# (workload, kernel, launches of the one-call step at full size)
CASES = [
    ("tiny_decode_f32", SCALAR, 2),           # fp32 activations: CUDA cores, staged
    ("gptoss_paged_decode_f16", MMA, 1),      # warp-MMA kernel, fused one-launch step
    ("selected_decode_bf16", MMA, 1),
    ("local_plus_selected_int8", TC, 1),      # 96-row units: tcgen05 kernel, fused one-launch step
]


@pytest.mark.parametrize("name", ["ragged_prefill_f16", "windowed_chunked_prefill_f16"])
def test_plan_of_prefill(name):
    # the tcgen05 prefill needs the driver's tensor-map encoder; without a
    # driver (this host) the planner falls back to the warp-MMA kernel
    a = args_for(W.by_name(name, small=False))
    kind = spa.attention_plan(a)["kind"]
    assert kind in (PREFILL, MMA)
    # the prefill kernel has no fused step; the warp-MMA fallback has one
    assert spa.prepare_append_attention_launches(a) == (2 if kind == PREFILL else 1)


@pytest.mark.parametrize("name,kind,step_launches", CASES)
def test_plan_of_each_workload(name, kind, step_launches):
    wl = W.by_name(name, small=False)
    a = args_for(wl)
    plan = spa.attention_plan(a)
    assert plan["kind"] == kind
    assert plan["launches"] == 1
    assert plan["num_splits"] >= 1
    assert spa.prepare_append_attention_launches(a) == step_launches


def test_automatic_splits_fill_one_wave():
    # selected decode: 64 units; two CTAs per SM on 148 SMs leave room for 4 splits
    plan = spa.attention_plan(args_for(W.by_name("selected_decode_bf16")))
    assert plan["num_splits"] == 4
    # INT8 multi-token decode on tcgen05 (one CTA per SM): 32 units x 4 splits <= 148
    plan = spa.attention_plan(args_for(W.by_name("local_plus_selected_int8")))
    assert plan["num_splits"] == 4
    # GPT-OSS decode already fills the GPU with 256 units: no split
    plan = spa.attention_plan(args_for(W.by_name("gptoss_paged_decode_f16")))
    assert plan["num_splits"] == 1


def test_requested_splits_are_kept():
    a = args_for(W.by_name("selected_decode_bf16"), num_splits=3)
    assert spa.attention_plan(a)["num_splits"] == 3


def test_misaligned_pointer_is_rejected():
    a = args_for(W.by_name("gptoss_paged_decode_f16"))
    a.k_cache = a.k_cache + 8
    with pytest.raises(spa.SpaError):
        spa.attention_plan(a)
