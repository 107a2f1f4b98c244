"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the
same seeded inputs.  Metadata, slots, cache contents, index handling and
status bits are compared bit for bit; outputs within max-abs 1e-5 (fp32) or
3e-3 (fp16 / bf16; INT8 caches are compared with the oracle run on the
dequantised values)."""
import numpy as np
import pytest
import torch

from selected_token_sparse_b200 import pipeline, workloads as W
from tests.gpu_util import compare, oracle_step

pytestmark = pytest.mark.gpu


def run(wl, **kw):  # noqa: D103
    return pipeline.run_step(wl, **kw)


@pytest.mark.parametrize("name", W.WORKLOADS)
def test_workload_small(name):
    wl = W.by_name(name, small=True)
    compare(wl, run(wl), oracle_step(wl), strict=True)


@pytest.mark.parametrize("name", W.WORKLOADS)
def test_workload_full_size(name):
    """The workloads at full size; prefill outputs are sampled rows: each
    request's first and last two rows, six random rows, and one random row of
    every 128-row q tile (every head of a sampled row is compared, so every
    prefill work item is checked)."""
    wl = W.by_name(name, small=False)
    tokens = None
    if name in ("ragged_prefill_f16", "windowed_chunked_prefill_f16"):
        rng = np.random.default_rng(0)
        cu = wl["cu_seqlens_q"]
        picks = set()
        for b in range(wl.B):
            picks |= {int(cu[b]), int(cu[b]) + 1, int(cu[b + 1]) - 1, int(cu[b + 1]) - 2}
            picks |= set(int(x) for x in rng.integers(cu[b], cu[b + 1], size=6))
            for q0 in range(int(cu[b]), int(cu[b + 1]), 128):
                picks.add(int(rng.integers(q0, min(q0 + 128, int(cu[b + 1])))))
        tokens = sorted(picks)
    got = run(wl)
    ref = oracle_step(wl, tokens=tokens)
    compare(wl, got, ref, tokens=tokens, strict=True)


@pytest.mark.parametrize("name", ["tiny_decode_f32", "gptoss_paged_decode_f16",
                                  "selected_decode_bf16", "local_plus_selected_int8"])
@pytest.mark.parametrize("splits", [1, 2, 3, 7, 32])
def test_forced_splits(name, splits):
    wl = W.by_name(name, small=True)
    compare(wl, run(wl, num_splits=splits), oracle_step(wl))


@pytest.mark.parametrize("name", W.WORKLOADS)
def test_deterministic(name):
    wl = W.by_name(name, small=True)
    a, b = run(wl), run(wl)
    assert np.array_equal(a["out"], b["out"])
    assert np.array_equal(a["lse"], b["lse"], equal_nan=True)


# ---------------------------------------------------------------------------
# edge cases
# ---------------------------------------------------------------------------

EDGE = {
    "empty_requests_decode": dict(act="f16", B=4, H_q=8, H_kv=2, D=64, block_size=16,
                                  q_lens=[1, 0, 1, 0], past=[40, 17, 0, 0], window=16),
    "no_tokens": dict(act="f16", B=2, H_q=4, H_kv=2, D=64, block_size=16, q_lens=[0, 0],
                      past=[5, 0]),
    "window_larger_than_history": dict(act="bf16", B=3, H_q=8, H_kv=1, D=128, block_size=64,
                                       q_lens=[1, 1, 1], past=[3, 64, 200], window=1000),
    "window_one": dict(act="f16", B=2, H_q=4, H_kv=4, D=64, block_size=16, q_lens=[1, 1],
                       past=[10, 0], window=1),
    "no_sink_mha": dict(act="f32", B=2, H_q=2, H_kv=2, D=64, block_size=16, q_lens=[1, 1],
                        past=[30, 5], window=8, has_sinks=False),
    "gqa16": dict(act="bf16", B=2, H_q=32, H_kv=2, D=64, block_size=16, q_lens=[1, 1],
                  past=[100, 33], window=64),
    "all_padding_selection": dict(act="f16", B=2, H_q=4, H_kv=2, D=64, block_size=16,
                                  q_lens=[1, 1], past=[20, 9], sel_mode="main", sel_width=8,
                                  sel_valid=0),
    "all_padding_selection_no_sink": dict(act="f16", B=2, H_q=4, H_kv=2, D=64, block_size=16,
                                          q_lens=[1, 1], past=[20, 9], sel_mode="main",
                                          sel_width=8, sel_valid=0, has_sinks=False),
    "per_token_selection_multi_query": dict(act="bf16", B=2, H_q=8, H_kv=2, D=128, block_size=64,
                                            q_lens=[4, 3], past=[150, 70], sel_mode="main",
                                            sel_per_request=0, sel_width=40, sel_valid=33),
    "per_request_selection_multi_query": dict(act="f16", B=2, H_q=8, H_kv=2, D=64, block_size=16,
                                              q_lens=[5, 2], past=[60, 7], sel_mode="main",
                                              sel_per_request=1, sel_width=30, sel_valid=25),
    "aux_short_lengths": dict(act="f16", cache="i8", B=3, H_q=12, H_kv=2, D=128, block_size=64,
                              q_lens=[2, 1, 3], past=[100, 5, 64], window=32, sel_mode="aux",
                              sel_width=20, aux_cap=50, aux_lens=[50, 10, 0]),
    "aux_without_window": dict(act="bf16", B=2, H_q=4, H_kv=2, D=64, block_size=16, q_lens=[1, 2],
                               past=[20, 30], window=0, sel_mode="aux", sel_width=12, aux_cap=30),
    "int8_bf16_act": dict(act="bf16", cache="i8", B=2, H_q=8, H_kv=2, D=128, block_size=64,
                          q_lens=[1, 1], past=[300, 77], window=128),
    "int8_f32_act": dict(act="f32", cache="i8", B=2, H_q=4, H_kv=2, D=64, block_size=16,
                         q_lens=[1, 1], past=[50, 7], window=20),
    "explicit_scale": dict(act="f16", B=2, H_q=4, H_kv=2, D=128, block_size=16, q_lens=[1, 1],
                           past=[50, 7], window=20, scale=0.3),
    "chunked_prefill_dense": dict(act="f16", B=3, H_q=8, H_kv=2, D=64, block_size=16,
                                  q_lens=[7, 1, 12], past=[20, 3, 0]),
    "chunked_prefill_window": dict(act="bf16", B=2, H_q=4, H_kv=1, D=128, block_size=64,
                                   q_lens=[40, 9], past=[100, 0], window=24),
    "long_prefill_per_token_fallback": dict(act="f32", B=2, H_q=4, H_kv=2, D=64, block_size=16,
                                            q_lens=[70, 33], past=[0, 5]),
    # units of more than 32 rows (G x S_q) take the tcgen05 decode kernel
    "tc_bf16_window_64_rows": dict(act="bf16", B=3, H_q=32, H_kv=2, D=128, block_size=64,
                                   q_lens=[4, 2, 3], past=[200, 30, 0], window=100),
    "tc_int8_d64_aux_40_rows": dict(act="f16", cache="i8", B=2, H_q=20, H_kv=2, D=64, block_size=16,
                                    q_lens=[4, 4], past=[130, 70], window=40, sel_mode="aux",
                                    sel_width=50, aux_cap=90, aux_lens=[90, 33]),
    "tc_sel_main_48_rows": dict(act="f16", B=2, H_q=16, H_kv=2, D=128, block_size=64, q_lens=[6, 5],
                                past=[400, 250], sel_mode="main", sel_per_request=1, sel_width=300,
                                sel_valid=280),
    "tc_empty_selection": dict(act="bf16", cache="i8", B=2, H_q=48, H_kv=4, D=128, block_size=64,
                               q_lens=[8, 3], past=[60, 10], sel_mode="main", sel_per_request=1,
                               sel_width=16, sel_valid=0),
    # tcgen05 prefill work items: an odd group size pairs consecutive q tiles
    # of one head (the last pair of a request may hold one tile), an even one
    # pairs two heads; more items than SMs make the persistent (windowed)
    # schedule claim further items and reuse its Q buffers and K/V stages
    "prefill_tile_pairs_window_claimed": dict(act="f16", B=4, H_q=15, H_kv=5, D=64, block_size=16,
                                              q_lens=[600, 260, 100, 513], past=[50, 0, 900, 7],
                                              window=64),
    "prefill_tile_pairs_causal_d128": dict(act="f16", B=2, H_q=3, H_kv=1, D=128, block_size=64,
                                           q_lens=[300, 140], past=[0, 20]),
    "prefill_head_pairs_window_d128_claimed": dict(act="bf16", B=2, H_q=32, H_kv=8, D=128, block_size=64,
                                                   q_lens=[700, 500], past=[30, 0], window=200),
}


@pytest.mark.parametrize("case", sorted(EDGE))
def test_edge_case(case):
    wl = W.make_workload(name=case, seed=11, **EDGE[case])
    compare(wl, run(wl), oracle_step(wl))


def test_bad_selected_indices_flagged_and_skipped():
    wl = W.make_workload(act="f16", B=2, H_q=4, H_kv=2, D=64, block_size=16, q_lens=[1, 1],
                         past=[30, 12], sel_mode="main", sel_width=10, sel_valid=7, seed=5)
    sel = wl.arrays["selected_idx"]
    sel[0, 0, 7] = 31 + 5        # beyond the request's length
    sel[1, 1, 8] = -9            # below the padding value
    ref = oracle_step(wl)
    assert ref["status"] == 0x10
    compare(wl, run(wl), ref)


def test_bad_aux_indices_flagged_and_skipped():
    wl = W.make_workload(act="f16", cache="i8", B=2, H_q=8, H_kv=2, D=128, block_size=64,
                         q_lens=[2, 1], past=[70, 3], window=16, sel_mode="aux", sel_width=12,
                         aux_cap=40, aux_lens=[40, 9], seed=6)
    sel = wl.arrays["selected_idx"]
    sel[1, 0, 11] = 20           # within capacity, beyond request 1's aux length
    sel[0, 1, 10] = 40           # beyond capacity
    ref = oracle_step(wl)
    assert ref["status"] == 0x10
    compare(wl, run(wl), ref)


@pytest.mark.parametrize("which", ["decreasing_cu", "short_cu", "bad_block", "capacity",
                                   "negative_past"])
def test_malformed_metadata_status(which):
    """Malformed inputs: status bits and metadata match the oracle, caches stay
    bit-exact (no write outside a valid slot); outputs are unspecified."""
    wl = W.make_workload(act="f16", B=3, H_q=4, H_kv=2, D=64, block_size=16, q_lens=[2, 1, 3],
                         past=[20, 5, 40], window=8, spare_blocks=2, seed=9)
    a = wl.arrays
    if which == "decreasing_cu":
        a["cu_seqlens_q"][2] = 1
    elif which == "short_cu":
        a["cu_seqlens_q"][3] = 4
    elif which == "bad_block":
        a["block_table"][2, 2] = wl.NB + 3
        a["block_table"][0, 0] = -1
    elif which == "capacity":
        a["past_seqlens"][0] = wl.MB * wl.block_size - 1
    elif which == "negative_past":
        a["past_seqlens"][1] = -4
    ref = oracle_step(wl)
    assert ref["status"] != 0
    got = run(wl)
    compare(wl, got, ref, check_out=False)


def test_status_accumulates_and_is_not_cleared():
    wl = W.make_workload(act="f16", B=1, H_q=4, H_kv=2, D=64, block_size=16, q_lens=[1],
                         past=[5], sel_mode="main", sel_width=4, sel_valid=2, seed=3)
    wl.arrays["selected_idx"][0, 0, 3] = 100
    d = pipeline.to_device(wl)
    st = pipeline.Step(wl, d)
    st.status.fill_(0x40)
    st()
    torch.cuda.synchronize()
    assert int(st.status.item()) == 0x50


# ---------------------------------------------------------------------------
# fused prepare + append against the staged entry points; workspace reuse
# ---------------------------------------------------------------------------

def _all_equal(a, b):
    for k in ("seqlens_q", "seqlen_k", "token_batch", "token_pos", "slot_mapping"):
        assert np.array_equal(a[k], b[k]), k
    assert a["status"] == b["status"]
    for k in ("k_cache", "v_cache"):
        assert torch.equal(a[k].view(torch.uint8) if a[k].element_size() == 1 else
                           a[k].view(torch.int16) if a[k].element_size() == 2 else
                           a[k].view(torch.int32),
                           b[k].view(torch.uint8) if b[k].element_size() == 1 else
                           b[k].view(torch.int16) if b[k].element_size() == 2 else
                           b[k].view(torch.int32)), k


@pytest.mark.parametrize("name", W.WORKLOADS)
@pytest.mark.parametrize("mode", ["step", "prepare_append"])
def test_fused_entry_points_match_staged(name, mode):
    """spa_prepare_append_attention and spa_prepare_append_kv + spa_attention give
    the staged sequence's metadata, caches, status, out and lse bit for bit."""
    wl = W.by_name(name, small=True)
    a = run(wl, mode=mode)
    b = run(wl, mode="staged")
    _all_equal(a, b)
    assert np.array_equal(a["out"], b["out"])
    assert np.array_equal(a["lse"], b["lse"], equal_nan=True)


@pytest.mark.parametrize("which", ["decreasing_cu", "bad_block", "capacity"])
def test_fused_prepare_append_malformed(which):
    wl = W.make_workload(act="f16", cache="i8", B=3, H_q=8, H_kv=2, D=64, block_size=16,
                         q_lens=[2, 1, 3], past=[20, 5, 40], window=8, spare_blocks=2, seed=19)
    a_ = wl.arrays
    if which == "decreasing_cu":
        a_["cu_seqlens_q"][2] = 1
    elif which == "bad_block":
        a_["block_table"][2, 2] = wl.NB + 3
    else:
        a_["past_seqlens"][0] = wl.MB * wl.block_size - 1
    _all_equal(run(wl, mode="prepare_append"), run(wl, mode="staged"))


def _step_launches(wl, **kw):
    d = pipeline.to_device(wl)
    return pipeline.Step(wl, d, **kw).launches()


# One-launch step (warp-MMA decode on a 16-bit cache): metadata from the raw
# cumulative lengths in every CTA, this step's own rows read from k_new / v_new.
STEP_CASES = {
    # GQA decode, one token per request (per-token units)
    "decode_f16": dict(act="f16", B=4, H_q=16, H_kv=2, D=64, block_size=16, q_lens=[1, 1, 1, 1],
                       past=[0, 15, 40, 200], window=32),
    # several tokens per request, grouped by request: new rows of earlier tokens
    # of the same request are read from k_new
    "multi_token_grouped_bf16": dict(act="bf16", B=3, H_q=8, H_kv=2, D=128, block_size=16,
                                     q_lens=[3, 1, 4], past=[5, 0, 30]),
    # several tokens per request with per-token selections: per-token units
    # reading other units' new rows from k_new
    "multi_token_per_token_sel": dict(act="f16", B=2, H_q=8, H_kv=2, D=64, block_size=16,
                                      q_lens=[3, 2], past=[10, 4], sel_mode="main", sel_per_request=0,
                                      sel_width=12, sel_valid=10),
    # malformed: decreasing cumulative lengths, a bad block id, a position past the table
    "malformed_cu": dict(act="f16", B=3, H_q=8, H_kv=2, D=64, block_size=16, q_lens=[2, 1, 3],
                         past=[20, 5, 40], window=8, spare_blocks=2),
    "empty_request": dict(act="f16", B=3, H_q=8, H_kv=2, D=64, block_size=16, q_lens=[1, 0, 1],
                          past=[7, 3, 0]),
    # multi-token units of 36-96 rows run on the tcgen05 kernel: INT8 rows of
    # this step's tokens are quantised from k_new by the reader
    "tc_int8_window_aux": dict(act="f16", cache="i8", B=3, H_q=48, H_kv=4, D=128, block_size=16,
                               q_lens=[8, 3, 5], past=[70, 6, 200], window=32, sel_mode="aux",
                               sel_width=40, sel_valid=33, aux_cap=90, aux_lens=[90, 40, 60]),
    "tc_int8_dense_d64": dict(act="bf16", cache="i8", B=2, H_q=32, H_kv=2, D=64, block_size=16,
                              q_lens=[4, 6], past=[33, 120]),
    "tc_bf16_window": dict(act="bf16", B=3, H_q=48, H_kv=4, D=128, block_size=16, q_lens=[8, 0, 4],
                           past=[100, 9, 3], window=64),
    "tc_int8_malformed_cu": dict(act="f16", cache="i8", B=3, H_q=48, H_kv=4, D=128, block_size=16,
                                 q_lens=[4, 3, 6], past=[20, 5, 40], window=8, spare_blocks=2),
    # more new tokens than the staging area holds: quantised where a tile needs them
    "tc_int8_many_new_tokens": dict(act="f16", cache="i8", B=2, H_q=2, H_kv=2, D=128, block_size=16,
                                    q_lens=[80, 70], past=[30, 0]),
    # 64 q heads per kv head: one token per unit (per-token units on tcgen05)
    "tc_int8_per_token_units": dict(act="bf16", cache="i8", B=2, H_q=64, H_kv=1, D=64, block_size=16,
                                    q_lens=[3, 2], past=[40, 9], window=16),
}


@pytest.mark.parametrize("case", list(STEP_CASES))
@pytest.mark.parametrize("splits", [0, 1, 3])
def test_step_matches_staged(case, splits):
    wl = W.make_workload(seed=31, has_sinks=True, **STEP_CASES[case])
    if case in ("malformed_cu", "tc_int8_malformed_cu"):
        wl.arrays["cu_seqlens_q"][2] = 1
        wl.arrays["block_table"][2, 2] = wl.NB + 3
        wl.arrays["past_seqlens"][0] = wl.MB * wl.block_size - 1
    assert _step_launches(wl, num_splits=splits) == 1
    a = run(wl, mode="step", num_splits=splits)
    b = run(wl, mode="staged", num_splits=splits)
    _all_equal(a, b)
    rows = slice(None)
    if "malformed" in case:
        # only the rows some unit writes: a token of a request, within the
        # first max_seqlen_q tokens of it (the bounds status flags the rest)
        tb = a["token_batch"]
        starts = np.concatenate([[0], np.cumsum(a["seqlens_q"])])
        rows = [t for t in range(wl.T) if tb[t] >= 0 and t - starts[tb[t]] < wl.max_seqlen_q]
    assert np.array_equal(a["out"][rows], b["out"][rows])
    assert np.array_equal(a["lse"][rows], b["lse"][rows], equal_nan=True)
    if "malformed" not in case:
        compare(wl, a, oracle_step(wl))


def test_step_launch_counts():
    assert _step_launches(W.by_name("gptoss_paged_decode_f16", small=True)) == 1
    assert _step_launches(W.by_name("selected_decode_bf16", small=True)) == 1
    assert _step_launches(W.by_name("tiny_decode_f32", small=True)) == 2        # fp32: scalar kernel
    assert _step_launches(W.by_name("local_plus_selected_int8", small=True)) == 1   # fused tcgen05 step
    assert _step_launches(W.by_name("ragged_prefill_f16", small=True)) == 2


@pytest.mark.parametrize("name", ["selected_decode_bf16", "local_plus_selected_int8"])
def test_workspace_reuse_across_calls(name):
    """Split tickets are left at zero, so the same workspace serves call after call."""
    wl = W.by_name(name, small=True)
    d = pipeline.to_device(wl)
    st = pipeline.Step(wl, d, num_splits=3, want_lse=True)
    outs = []
    for _ in range(3):
        st()
        torch.cuda.synchronize()
        outs.append(st.out.clone())
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[1], outs[2])
    ref = oracle_step(wl)
    got = {k: v.cpu().numpy() for k, v in st.meta.items()}
    got.update(status=int(st.status.item()), out=outs[-1].float().cpu().numpy().astype(np.float64),
               k_cache=d["k_cache"].cpu(), v_cache=d["v_cache"].cpu())
    compare(wl, got, ref)
