"""spa_attention_noalloc: the attention entry point for callers that cannot
allocate device memory (inside a CUDA graph capture, under a host runtime that
owns every allocation, ...).  It must give the results of spa_attention with a
caller workspace, call after call, from the library's own static scratch.

This file is collected last on purpose, so that a run stopping at its first
failure has run every other test before it.
"""
import ctypes

import numpy as np
import pytest
import torch

from selected_token_sparse_b200 import pipeline, spa, workloads as W
from tests.gpu_util import LSE_TOL, TOL, oracle_step, rounding_incurred

SCRATCH_LIMIT = 8 << 20
SPA_ERR_SCRATCH_LIMIT = -5


def _entry(lib):
    fn = lib.spa_attention_noalloc
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.POINTER(spa.AttentionArgs), ctypes.c_void_p]
    return fn


# Every split plan's partial states travel through the scratch array: up to 8
# splits on the tensor-core kernels (one cluster per unit, merged after a
# cluster barrier), more than 8 there (the last CTA of a unit merges, with
# tickets), and the CUDA-core kernel (tickets); the windowed prefill's
# persistent schedule keeps its work counter there.  The sequence mixes
# workloads so that a call finds the previous call's partials (of another
# shape) in the array -- the prefill's counter words among them.
CASES = [("gptoss_paged_decode_f16", 16), ("tiny_decode_f32", 3), ("local_plus_selected_int8", 12),
         ("windowed_chunked_prefill_f16", 1), ("selected_decode_bf16", 4), ("selected_decode_bf16", 32),
         ("local_plus_selected_int8", 3), ("windowed_chunked_prefill_f16", 1), ("tiny_decode_f32", 5),
         ("gptoss_paged_decode_f16", 2), ("gptoss_paged_decode_f16", 16)]


def _prepare(name, splits):
    wl = W.by_name(name, small=True)
    d = pipeline.to_device(wl)
    st = pipeline.Step(wl, d, num_splits=splits, want_lse=True)
    assert spa.attention_plan(st.args)["num_splits"] == splits
    st()                                    # metadata, append, spa_attention with a workspace
    torch.cuda.synchronize()
    out = torch.empty_like(st.out)
    lse = torch.empty_like(st.lse)
    meta = dict(st.meta, cu_seqlens_q=d["cu_seqlens_q"])
    args = spa.attention_args(d["q"], d["k_cache"], d["v_cache"], d["block_table"], meta,
                              max_seqlen_q=wl.max_seqlen_q, max_seqlen_k=wl.max_seqlen_k,
                              out=out, lse=lse, num_splits=splits, status=st.status, **st.kw)
    need = spa.workspace_size(args)
    assert 0 < need <= SCRATCH_LIMIT        # partials or counters go through the scratch, and they fit
    return wl, st, args, out, lse


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_and_oracle():
    fn = _entry(spa.lib())
    stream = torch.cuda.current_stream().cuda_stream
    prepared = [_prepare(name, splits) for name, splits in CASES]
    for (name, splits), (wl, st, args, out, lse) in zip(CASES, prepared):
        ref = oracle_step(wl)
        ref_out, ref_lse = ref["out"], ref["lse"]
        for _ in range(2):                  # two calls in a row share the static scratch
            out.fill_(float("nan"))
            lse.fill_(float("nan"))
            rc = fn(ctypes.byref(args), stream)
            assert rc == 0, spa.error_string(rc)
            torch.cuda.synchronize()
            # the same kernels and plan as spa_attention with a workspace: identical bits
            assert torch.equal(out.view(torch.int16) if out.element_size() == 2 else out.view(torch.int32),
                               st.out.view(torch.int16) if out.element_size() == 2 else st.out.view(torch.int32)), name
            got = out.float().cpu().numpy().astype(np.float64)
            assert np.isfinite(got).all()
            err = np.abs(got - ref_out)
            assert (err <= TOL[wl.act] + rounding_incurred(ref_out, wl.act)).all(), (name, splits, err.max())
            assert err.max() <= TOL[wl.act], (name, splits, err.max())
            gl = lse.cpu().numpy().astype(np.float64)
            both_inf = np.isneginf(gl) & np.isneginf(ref_lse)
            assert np.abs(np.where(both_inf, 0.0, gl - ref_lse)).max() <= LSE_TOL, name
        assert int(st.status.item()) == 0


def test_noalloc_rejects_calls_beyond_the_scratch_limit():
    """Host-side check only: nothing is enqueued, so no GPU is needed."""
    lib = spa.load_library()
    fn = _entry(lib)
    a = spa.AttentionArgs()
    a.struct_size = ctypes.sizeof(spa.AttentionArgs)
    fake = 1 << 20                          # never dereferenced: the call is rejected first
    a.q = a.out = a.k_cache = a.v_cache = fake
    a.block_table = a.cu_seqlens_q = a.seqlens_q = a.seqlen_k = a.token_batch = a.token_pos = fake
    a.act = a.cache = spa.SPA_F16
    a.T, a.B, a.H_q, a.H_kv, a.D = 64, 64, 128, 8, 128
    a.MB, a.block_size, a.num_blocks = 64, 64, 4096
    a.max_seqlen_q, a.max_seqlen_k = 1, 4096
    a.is_causal = 1
    a.num_splits = 16                       # 16 x 64 x 128 x 128 x 4 bytes of partials = 64 MiB
    assert lib.spa_attention_workspace_size(ctypes.byref(a)) > SCRATCH_LIMIT
    assert fn(ctypes.byref(a), None) == SPA_ERR_SCRATCH_LIMIT
    assert b"scratch" in lib.spa_error_string(SPA_ERR_SCRATCH_LIMIT)
