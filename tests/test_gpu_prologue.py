"""GPU parity of the QKV prologue (spa_prepare_qkv_append) against the fp64
oracle: metadata, status and v rows bit for bit; the processed q and k rows
within two units in the last place of the activation dtype (the kernel
computes the norm and the rotation in fp32, the oracle in fp64); INT8 k codes
within one step where the two sides' values straddle a rounding boundary
(rare); the attention output within the dtype's tolerance plus rounding."""
import numpy as np
import pytest
import torch

from oracle import spa_oracle as O
from selected_token_sparse_b200 import pipeline, workloads as W
from tests.gpu_util import compare, oracle_step

pytestmark = pytest.mark.gpu

MANT = {"f16": 10, "bf16": 7, "f32": 23}


def _values(x, dtype):
    """float64 values of an encoded host array (torch or numpy)."""
    if isinstance(x, torch.Tensor):
        x = x.float().numpy() if x.dtype != torch.int8 else x.numpy()
        return np.asarray(x, dtype=np.float64)
    return O.decode(x, dtype)


def _within_ulps(got, ref, dtype, n=2):
    """|got - ref| <= n ulp(ref) + ulp(max |ref| of the head's row): a rotation
    output is a difference of products, so its rounding error scales with the
    row's magnitude, not with the (possibly cancelled) value."""
    ref = np.asarray(ref, dtype=np.float64)
    got = np.asarray(got, dtype=np.float64).reshape(ref.shape)
    e = np.floor(np.log2(np.maximum(np.abs(ref), 2.0 ** -14)))
    ulp = 2.0 ** (e - MANT[dtype])
    rowmax = np.max(np.abs(ref), axis=-1, keepdims=True)
    bound = n * ulp + rowmax * 2.0 ** -MANT[dtype] + 1e-30
    bad = np.abs(got - ref) > bound
    assert not bad.any(), f"{int(bad.sum())} values beyond the bound; worst {float(np.abs(got - ref).max())}"


CASES = {
    "f16_unpacked_norm_rope": dict(act="f16", B=3, H_q=8, H_kv=2, D=64, block_size=16, q_lens=[1, 3, 2],
                                   past=[10, 40, 0], window=32,
                                   prologue=dict(qk_norm=True, rotary_dim=64)),
    "bf16_packed_interleaved_partial_posids": dict(
        act="bf16", B=2, H_q=8, H_kv=4, D=128, block_size=64, q_lens=[2, 5], past=[100, 7],
        prologue=dict(packed=True, qk_norm=True, rotary_dim=32, interleaved=True, pos_ids=True)),
    "int8_cache_norm_rope_offset": dict(act="f16", cache="i8", B=2, H_q=12, H_kv=4, D=128, block_size=64,
                                        q_lens=[4, 3], past=[70, 200], window=64,
                                        prologue=dict(packed=True, qk_norm=True, rotary_dim=128,
                                                      rotary_offset=5)),
    "f32_rope_only": dict(act="f32", B=2, H_q=4, H_kv=2, D=64, block_size=16, q_lens=[1, 1], past=[33, 5],
                          prologue=dict(rotary_dim=48, interleaved=True)),
    "positions_out_of_range": dict(act="f16", B=2, H_q=4, H_kv=2, D=64, block_size=16, q_lens=[2, 1],
                                   past=[5, 9], prologue=dict(qk_norm=True, rotary_dim=64, pos_ids=True,
                                                              pos_shift=10 ** 6)),
    "decode_packed_gqa": dict(act="bf16", B=6, H_q=32, H_kv=4, D=128, block_size=16, q_lens=[1] * 6,
                              past=[0, 3, 17, 64, 100, 250], window=128,
                              prologue=dict(packed=True, qk_norm=True, rotary_dim=128)),
}


@pytest.mark.parametrize("case", list(CASES))
def test_prologue_matches_oracle(case):
    wl = W.make_workload(seed=41, has_sinks=True, **CASES[case])
    got = pipeline.run_step(wl)
    ref = oracle_step(wl)
    # metadata and status bit for bit; the caches and q within rounding
    compare(wl, got, ref, check_out=False, check_cache=False)
    _within_ulps(_values(got["q_out"], wl.act), _values(ref["q_out"], wl.act), wl.act)
    slots = ref["meta"]["slot_mapping"]
    bs = wl.block_size
    for name in ("k_cache", "v_cache"):
        g, r = got[name], ref[name]
        for s in slots:
            if s < 0:
                continue
            gb, rb = g[s // bs, s % bs], r[s // bs, s % bs]
            if wl.cache == "i8":
                d = np.abs(gb.numpy().astype(np.int32) - rb.astype(np.int32))
                assert d.max() <= (1 if name == "k_cache" else 0), name
            elif name == "v_cache":
                assert torch.equal(gb.view(torch.int16) if gb.element_size() == 2 else gb,
                                   torch.from_numpy(np.asarray(rb)).view(torch.int16)
                                   if gb.element_size() == 2 else torch.from_numpy(np.asarray(rb)))
            else:
                _within_ulps(_values(gb, wl.cache), _values(rb, wl.cache), wl.cache)
    if wl.cache == "i8":
        # codes off by one are rounding-boundary cases: rare
        kd = np.abs(got["k_cache"].numpy().astype(np.int32) - ref["k_cache"].astype(np.int32))
        assert (kd > 0).mean() < 0.01
    # untouched cache rows bit for bit
    mask = np.ones(got["k_cache"].shape[:2], dtype=bool)
    for s in slots:
        if s >= 0:
            mask[s // bs, s % bs] = False
    for name in ("k_cache", "v_cache"):
        g = got[name][torch.from_numpy(mask)]
        r = np.asarray(ref[name])[mask]
        gv = g.view(torch.int16).numpy() if g.element_size() == 2 else g.numpy()
        rv = r.view(np.int16) if r.dtype in (np.float16, np.uint16) else r
        assert np.array_equal(np.asarray(gv).reshape(-1).view(np.uint8), np.asarray(rv).reshape(-1).view(np.uint8))
    # attention on the processed q: within the dtype tolerance (+ rounding)
    compare(wl, got, ref, check_cache=False)


def test_prologue_identity_is_bit_exact():
    """Without norm and rotation the prologue is the packed split plus the append."""
    wl = W.make_workload(act="f16", B=2, H_q=8, H_kv=2, D=64, block_size=16, q_lens=[3, 2], past=[9, 30],
                         window=16, prologue=dict(packed=True), seed=43)
    got = pipeline.run_step(wl)
    ref = oracle_step(wl)
    compare(wl, got, ref)
    assert np.array_equal(got["q_out"].view(torch.int16).numpy(), wl["q"].view(np.int16))


@pytest.mark.parametrize("small", [True, False])
def test_named_prologue_workload(small):
    wl = W.by_name("qkv_prologue_selected_decode_bf16", small=small)
    got = pipeline.run_step(wl)
    ref = oracle_step(wl)
    compare(wl, got, ref, check_out=False, check_cache=False)
    _within_ulps(_values(got["q_out"], wl.act), _values(ref["q_out"], wl.act), wl.act)
    compare(wl, got, ref, check_cache=False, strict=True)
