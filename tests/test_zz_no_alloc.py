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
from tests.gpu_util import LSE_TOL, TOL, half_ulp

SCRATCH_LIMIT = 8 << 20
SPA_ERR_SCRATCH_LIMIT = -5


def _entry(lib):
    fn = lib.spa_attention_noalloc
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.POINTER(spa.AttentionArgs), ctypes.c_void_p]
    return fn


@pytest.mark.gpu
@pytest.mark.parametrize("name,splits", [("selected_decode_bf16", 0), ("local_plus_selected_int8", 3),
                                         ("gptoss_paged_decode_f16", 4)])
def test_noalloc_matches_workspace_entry_point(name, splits):
    wl = W.by_name(name, small=True)
    d = pipeline.to_device(wl)
    st = pipeline.Step(wl, d, num_splits=splits, want_lse=True)
    st()                                    # metadata, append, spa_attention with a workspace
    torch.cuda.synchronize()
    ref_out = st.out.float().cpu().numpy().astype(np.float64)
    ref_lse = st.lse.cpu().numpy().astype(np.float64)

    out = torch.empty_like(st.out)
    lse = torch.empty_like(st.lse)
    meta = dict(st.meta, cu_seqlens_q=d["cu_seqlens_q"])
    args = spa.attention_args(d["q"], d["k_cache"], d["v_cache"], d["block_table"], meta,
                              max_seqlen_q=wl.max_seqlen_q, max_seqlen_k=wl.max_seqlen_k,
                              out=out, lse=lse, num_splits=splits, status=st.status, **st.kw)
    need = spa.workspace_size(args)
    assert 0 < need <= SCRATCH_LIMIT       # the call really uses scratch, and it fits
    fn = _entry(spa.lib())
    stream = torch.cuda.current_stream().cuda_stream
    for _ in range(2):                      # two calls in a row share the static scratch
        out.fill_(float("nan"))
        lse.fill_(float("nan"))
        rc = fn(ctypes.byref(args), stream)
        assert rc == 0, spa.error_string(rc)
        torch.cuda.synchronize()
        got = out.float().cpu().numpy().astype(np.float64)
        assert np.isfinite(got).all()
        bound = TOL[wl.act] + half_ulp(ref_out, wl.act)
        assert (np.abs(got - ref_out) <= bound).all()
        gl = lse.cpu().numpy().astype(np.float64)
        assert np.allclose(gl, ref_lse, atol=LSE_TOL, rtol=0)
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
    a.num_splits = 8                        # 8 x 64 x 128 x 128 x 4 bytes of partials = 32 MiB
    assert lib.spa_attention_workspace_size(ctypes.byref(a)) > SCRATCH_LIMIT
    assert fn(ctypes.byref(a), None) == SPA_ERR_SCRATCH_LIMIT
    assert b"scratch" in lib.spa_error_string(SPA_ERR_SCRATCH_LIMIT)
