"""Sequence-sharded split-KV on one GPU: R shards of each request's keys are
attended one after another (spa_attention with partial = 1 over each shard's
kv_range, with a block table that maps only that shard's blocks), then
spa_merge_partials combines them.  Each partial state matches the oracle's
attention over the shard without the sink, no status bit is set by the other
shards' unmapped blocks, and the merged output matches the oracle's unsharded
attention.  (Shards on several GPUs exchange the same states with one
all-gather; that plumbing is tested on CPU in tests/test_shard_dist.py.)"""
import numpy as np
import pytest
import torch

from oracle import spa_oracle as O
from selected_token_sparse_b200 import pipeline, shard, spa, workloads as W
from tests.gpu_util import LSE_TOL, TOL, rounding_incurred

pytestmark = pytest.mark.gpu


def _lse_err(a, b):
    both = np.isneginf(a) & np.isneginf(b)
    return float(np.abs(np.where(both, 0.0, a - b)).max()) if a.size else 0.0


def run_sharded(wl, R, num_splits=0):
    d = pipeline.to_device(wl)
    st = pipeline.Step(wl, d, want_lse=True)      # metadata + append (and the unsharded call)
    st()
    torch.cuda.synchronize()
    a = wl.arrays
    meta_h = O.prepare_metadata(a["cu_seqlens_q"], a["past_seqlens"], a["block_table"], wl.T, wl.max_seqlen_q,
                                wl.max_seqlen_k, wl.block_size, wl.NB)
    kc, vc = O.append_kv(a["k_new"], a["v_new"], wl.act, a["k_cache"], a["v_cache"], wl.cache,
                         meta_h["slot_mapping"], a.get("k_scale"), a.get("v_scale"))
    lengths = [p + q for p, q in zip(wl.past, wl.q_lens)]
    meta = dict(st.meta, cu_seqlens_q=d["cu_seqlens_q"])
    outs, lses = [], []
    for r in range(R):
        rng = shard.sequence_ranges(lengths, R, r, wl.block_size)
        bt = torch.from_numpy(shard.shard_block_table(a["block_table"], rng, wl.block_size)).cuda()
        kw = dict(st.kw)
        aux_here = wl.sel_mode == "aux" and r == 0      # the auxiliary entries belong to one shard
        if wl.sel_mode == "aux" and not aux_here:
            kw.update(selected_idx=None, sel_target=0, aux_k=None, aux_v=None, aux_seqlens=None)
        po = torch.full((wl.T, wl.H_q, wl.D), float("nan"), dtype=torch.float32, device="cuda")
        pl = torch.full((wl.T, wl.H_q), float("nan"), dtype=torch.float32, device="cuda")
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        rng_d = torch.from_numpy(rng).cuda()          # the arguments hold its address: keep it alive
        args = spa.attention_args(d["q"], d["k_cache"], d["v_cache"], bt, meta, max_seqlen_q=wl.max_seqlen_q,
                                  max_seqlen_k=wl.max_seqlen_k, out=po, lse=pl, num_splits=num_splits,
                                  status=status, kv_range=rng_d, partial=True, **kw)
        ws = spa.new_workspace(spa.workspace_size(args), "cuda")
        spa.run_attention(args, ws)
        torch.cuda.synchronize()
        assert int(status.item()) == 0, hex(int(status.item()))
        ref = O.attention(a["q"], wl.act, kc, vc, wl.cache, a["block_table"], meta_h, H_kv=wl.H_kv,
                          window=wl.window, selected_idx=a.get("selected_idx") if (wl.sel_mode == "main" or aux_here)
                          else None, sel_per_request=wl.sel_per_request, sel_target=1 if aux_here else 0,
                          aux_k=a.get("aux_k"), aux_v=a.get("aux_v"), aux_seqlens=a.get("aux_seqlens"),
                          sinks=None, scale=wl.scale, k_scale=a.get("k_scale"), v_scale=a.get("v_scale"),
                          kv_range=rng)
        g = po.cpu().numpy().astype(np.float64)
        assert np.isfinite(g).all()
        assert np.abs(g - ref["out"]).max() <= TOL[wl.act], (r, np.abs(g - ref["out"]).max())
        assert _lse_err(pl.cpu().numpy().astype(np.float64), ref["lse"]) <= LSE_TOL
        outs.append(po)
        lses.append(pl)
    out = torch.empty_like(st.out)
    lse = torch.empty(wl.T, wl.H_q, dtype=torch.float32, device="cuda")
    spa.merge_partials(torch.stack(outs), torch.stack(lses), d.get("sinks"), out, lse)
    torch.cuda.synchronize()
    return out.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("name,R,splits", [
    ("gptoss_paged_decode_f16", 2, 0), ("gptoss_paged_decode_f16", 3, 16),
    ("selected_decode_bf16", 4, 0), ("selected_decode_bf16", 3, 3),
    ("local_plus_selected_int8", 2, 0), ("local_plus_selected_int8", 3, 12),
    ("tiny_decode_f32", 2, 0), ("ragged_prefill_f16", 3, 0), ("windowed_chunked_prefill_f16", 2, 0),
    ("windowed_chunked_prefill_f16", 3, 0), ("windowed_chunked_prefill_f16", 4, 0)])
def test_sharded_partials_merge_to_the_oracle(name, R, splits):
    wl = W.by_name(name, small=True)
    out, lse = run_sharded(wl, R, splits)
    ref = O.run_step(wl)
    err = np.abs(out - ref["out"])
    assert (err <= TOL[wl.act] + rounding_incurred(ref["out"], wl.act)).all(), err.max()
    assert err.max() <= TOL[wl.act], err.max()
    assert _lse_err(lse, ref["lse"]) <= LSE_TOL


def test_sharded_selected_decode_full_size():
    """The selected-token decode at full size (32768 keys per request) over 4 shards."""
    wl = W.by_name("selected_decode_bf16")
    out, lse = run_sharded(wl, 4)
    ref = O.run_step(wl)
    assert np.abs(out - ref["out"]).max() <= TOL[wl.act]
    assert _lse_err(lse, ref["lse"]) <= LSE_TOL


def test_merge_of_empty_shards_and_one_shard():
    """All shards empty: 0 and -inf without a sink, 0 and the sink with one;
    a single shard without a sink is returned unchanged (to fp32 rounding)."""
    T, H, D = 3, 4, 64
    po = torch.zeros(2, T, H, D, device="cuda")
    pl = torch.full((2, T, H), float("-inf"), device="cuda")
    out = torch.empty(T, H, D, dtype=torch.float32, device="cuda")
    lse = torch.empty(T, H, device="cuda")
    spa.merge_partials(po, pl, None, out, lse)
    assert (out == 0).all() and torch.isneginf(lse).all()
    sinks = torch.tensor([0.5, -1.0, 2.0, 0.0], device="cuda")
    spa.merge_partials(po, pl, sinks, out, lse)
    assert (out == 0).all()
    assert torch.allclose(lse, sinks.expand(T, H), atol=1e-6)
    x = torch.randn(1, T, H, D, device="cuda")
    l = torch.randn(1, T, H, device="cuda")
    spa.merge_partials(x, l, None, out, lse)
    assert torch.allclose(out, x[0], atol=1e-6, rtol=1e-6)
    assert torch.allclose(lse, l[0], atol=1e-5)
