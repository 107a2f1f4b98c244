"""Failure detection of the bounded on-chip waits, made to fire without a GPU
fault: the test hook test_expire_wait makes the tcgen05 prefill kernel drop
one barrier arrival per CTA (on a barrier that guards no copy and no MMA) and
poll for it only briefly.  The launch must return, the status word must carry
SPA_ST_TIMEOUT, and the next normal call on the same stream must be correct,
so the context stays usable."""
import numpy as np
import pytest
import torch

from selected_token_sparse_b200 import pipeline, spa, workloads as W
from tests.gpu_util import compare, oracle_step

pytestmark = pytest.mark.gpu

SPA_ST_TIMEOUT = 0x20


def _result(wl, st, d):
    got = {k: v.cpu().numpy() for k, v in st.meta.items()}
    got.update(status=int(st.status.item()), out=st.out.float().cpu().numpy().astype(np.float64),
               lse=st.lse.cpu().numpy().astype(np.float64), k_cache=d["k_cache"].cpu(), v_cache=d["v_cache"].cpu())
    return got


def _counter_words(st):
    """The persistent schedule's work counter and ticket (zero between calls)."""
    if spa.workspace_size(st.args) == 0:
        return [0, 0]
    return st.workspace[:8].view(torch.int32).tolist()


# one CTA per item (causal) and the persistent schedule with its work counter (window)
@pytest.mark.parametrize("name", ["ragged_prefill_f16", "windowed_chunked_prefill_f16"])
def test_expired_wait_sets_timeout_and_the_next_call_is_correct(name):
    wl = W.by_name(name, small=True)
    d = pipeline.to_device(wl)
    st = pipeline.Step(wl, d, want_lse=True)
    assert spa.attention_plan(st.args)["kind"] == 2          # the tcgen05 prefill kernel
    if name.startswith("windowed"):
        assert spa.workspace_size(st.args) > 0              # the counter lives in the workspace
    ref = oracle_step(wl)
    st()                                                     # metadata, append, attention
    torch.cuda.synchronize()
    compare(wl, _result(wl, st, d), ref, strict=True)
    assert _counter_words(st) == [0, 0]

    # the same attention call with the hook: a wait expires in every CTA
    st.status.zero_()
    st.args.test_expire_wait = 1
    spa.run_attention(st.args, st.workspace)                 # returns: nothing hangs
    torch.cuda.synchronize()
    assert int(st.status.item()) & SPA_ST_TIMEOUT
    assert _counter_words(st) == [0, 0]                      # put back although the CTAs gave up

    # the context is intact: the next normal calls on the stream are correct
    st.args.test_expire_wait = 0
    for _ in range(2):
        st.status.zero_()
        st.out.fill_(float("nan"))
        spa.run_attention(st.args, st.workspace)
        torch.cuda.synchronize()
        compare(wl, _result(wl, st, d), ref, strict=True)
        assert _counter_words(st) == [0, 0]
