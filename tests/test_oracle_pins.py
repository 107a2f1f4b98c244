"""Pins for the fp64 oracle: it is checked against things other than itself.

* values the pages print or fix for worked examples (tests/golden/*.json),
* PyTorch's scaled_dot_product_attention (float64, CPU) as an independent
  library formulation of causal / windowed / selected attention, with the
  learned sink expressed as an extra zero-valued key whose logit is the sink,
* closed forms (constant V, single key, q = 0, window of one key, empty set),
* brute-force enumeration for the metadata, and invariants the method fixes
  (paged == contiguous, selection order, select-all == dense causal).

The test builds every expected value itself from logical (unpaged) K/V
sequences; only the oracle reads the paged cache.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import spa_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------------------
# helpers: a logical workload, laid out in a paged cache by the test itself
# ---------------------------------------------------------------------------

class Logical:
    """Per-request logical K/V sequences and their paged placement."""

    def __init__(self, q_lens, past, H_q, H_kv, D, bs, seed, spare=3, identity=False,
                 cache="f16"):
        rng = np.random.default_rng(seed)
        self.B = len(q_lens)
        self.q_lens, self.past = list(q_lens), list(past)
        self.H_q, self.H_kv, self.D, self.bs = H_q, H_kv, D, bs
        self.T = sum(q_lens)
        self.L = [p + q for p, q in zip(past, q_lens)]
        # logical sequences, exactly representable in fp16
        self.K = [rng.standard_normal((L, H_kv, D)).astype(np.float16) for L in self.L]
        self.V = [rng.standard_normal((L, H_kv, D)).astype(np.float16) for L in self.L]
        self.Q = rng.standard_normal((self.T, H_q, D)).astype(np.float16)
        nblk = [(L + bs - 1) // bs for L in self.L]
        MB = max(max(nblk), 1)
        NB = sum(nblk) + spare
        order = np.arange(NB) if identity else rng.permutation(NB)
        self.block_table = np.full((self.B, MB), -1, dtype=np.int32)
        o = 0
        for b in range(self.B):
            self.block_table[b, :nblk[b]] = order[o:o + nblk[b]]
            o += nblk[b]
        # garbage everywhere, then the history rows placed by hand
        self.k_cache = rng.standard_normal((NB, bs, H_kv, D)).astype(np.float16)
        self.v_cache = rng.standard_normal((NB, bs, H_kv, D)).astype(np.float16)
        for b in range(self.B):
            for j in range(self.past[b]):
                blk = self.block_table[b, j // bs]
                self.k_cache[blk, j % bs] = self.K[b][j]
                self.v_cache[blk, j % bs] = self.V[b][j]
        self.cu = np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int32)
        self.k_new = np.concatenate([self.K[b][self.past[b]:] for b in range(self.B)])
        self.v_new = np.concatenate([self.V[b][self.past[b]:] for b in range(self.B)])
        self.NB = NB

    def run(self, **kw):
        meta = O.prepare_metadata(self.cu, np.asarray(self.past, np.int32), self.block_table,
                                  self.T, max(self.q_lens), max(self.L), self.bs, self.NB)
        kc, vc = O.append_kv(self.k_new, self.v_new, "f16", self.k_cache, self.v_cache, "f16",
                             meta["slot_mapping"])
        return O.attention(self.Q, "f16", kc, vc, "f16", self.block_table, meta,
                           H_kv=self.H_kv, **kw)

    def sdpa(self, b, mask, sinks=None, extra_k=None, extra_v=None):
        """torch SDPA (float64) for request b with a boolean mask [H_q|1, q, L]."""
        G = self.H_q // self.H_kv
        t0 = int(self.cu[b])
        q = torch.from_numpy(self.Q[t0:t0 + self.q_lens[b]].astype(np.float64)).permute(1, 0, 2)
        k = torch.from_numpy(self.K[b].astype(np.float64)).permute(1, 0, 2)
        v = torch.from_numpy(self.V[b].astype(np.float64)).permute(1, 0, 2)
        if extra_k is not None:
            k = torch.cat([k, extra_k], dim=1)
            v = torch.cat([v, extra_v], dim=1)
        k = k.repeat_interleave(G, dim=0)
        v = v.repeat_interleave(G, dim=0)
        mask = torch.as_tensor(mask).expand(self.H_q, -1, -1)
        add = torch.where(mask, 0.0, -math.inf).to(torch.float64)
        if sinks is not None:
            # sink == one more key with q.k = 0 and value 0, logit biased to sink_h
            k = torch.cat([k, torch.zeros(self.H_q, 1, self.D, dtype=torch.float64)], dim=1)
            v = torch.cat([v, torch.zeros(self.H_q, 1, self.D, dtype=torch.float64)], dim=1)
            sk = torch.from_numpy(np.asarray(sinks, np.float64)).view(self.H_q, 1, 1)
            add = torch.cat([add, sk.expand(-1, add.shape[1], 1)], dim=2)
        o = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=add)
        return o.permute(1, 0, 2).numpy()

    def causal_mask(self, b):
        return torch.ones(self.q_lens[b], self.L[b], dtype=torch.bool).tril(diagonal=self.past[b])


# ---------------------------------------------------------------------------
# metadata
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("name", ["metadata_ragged_1_2.json", "metadata_empty_2_0.json",
                                  "metadata_uniform_decode.json"])
def test_metadata_golden(name):
    g = load(name)
    B = len(g["cu_seqlens_q"]) - 1
    bs = 16
    MB = 8
    bt = np.arange(B * MB, dtype=np.int32).reshape(B, MB)
    m = O.prepare_metadata(np.array(g["cu_seqlens_q"], np.int32), np.array(g["past_seqlens"], np.int32),
                           bt, g["T"], g["max_seqlen_q"], g["max_seqlen_k"], bs, B * MB)
    e = g["expect"]
    for k in ("seqlens_q", "seqlen_k", "token_batch", "token_pos"):
        assert m[k].tolist() == e[k], k
    assert m["status"] == e["status"]
    if "attended_positions" in e:
        for t, exp in enumerate(e["attended_positions"]):
            blk, off, aux, st = O.attended_keys(t, 0, m, bt, bs, B * MB, 0, None, 1, 0, None)
            b = m["token_batch"][t]
            pos = [int(list(bt[b]).index(x)) * bs + int(o) for x, o in zip(blk, off)]
            assert pos == exp
    if "over_bound_past_seqlens" in g:
        m2 = O.prepare_metadata(np.array(g["cu_seqlens_q"], np.int32),
                                np.array(g["over_bound_past_seqlens"], np.int32), bt, g["T"],
                                g["max_seqlen_q"], g["max_seqlen_k"], bs, B * MB)
        assert m2["status"] == g["over_bound_status"]


def test_window_golden():
    g = load("window_start_q3.json")
    for c in g["cases"]:
        B, bs = 1, 4
        L = c["past"] + c["q_len"]
        MB = (L + bs - 1) // bs
        bt = np.arange(MB, dtype=np.int32)[None]
        m = O.prepare_metadata(np.array([0, c["q_len"]], np.int32), np.array([c["past"]], np.int32),
                               bt, c["q_len"], c["q_len"], L, bs, MB)
        for t in range(c["q_len"]):
            blk, off, _, _ = O.attended_keys(t, 0, m, bt, bs, MB, c["window"], None, 1, 0, None)
            assert (blk * bs + off).tolist() == c["visible"][t]


def test_metadata_bruteforce():
    rng = np.random.default_rng(7)
    for trial in range(40):
        B = int(rng.integers(1, 6))
        q_lens = [int(x) for x in rng.integers(0, 5, size=B)]
        past = [int(x) for x in rng.integers(0, 40, size=B)]
        bs = int(rng.choice([1, 2, 4, 16]))
        T = sum(q_lens)
        MB = max((p + q + bs - 1) // bs for p, q in zip(past, q_lens)) + 1
        NB = B * MB
        bt = rng.permutation(NB).astype(np.int32).reshape(B, MB)
        cu = np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int32)
        m = O.prepare_metadata(cu, np.array(past, np.int32), bt, T, max(q_lens),
                               max(p + q for p, q in zip(past, q_lens)), bs, NB)
        # forward enumeration: request by request, token by token
        tb, tp, sl = [], [], []
        for b in range(B):
            for i in range(q_lens[b]):
                pos = past[b] + i
                tb.append(b)
                tp.append(pos)
                sl.append(int(bt[b, pos // bs]) * bs + pos % bs)
        assert m["token_batch"].tolist() == tb
        assert m["token_pos"].tolist() == tp
        assert m["slot_mapping"].tolist() == sl
        assert m["seqlens_q"].tolist() == q_lens
        assert m["seqlen_k"].tolist() == [p + q - 1 for p, q in zip(past, q_lens)]
        assert m["status"] == 0


def test_metadata_malformed_status():
    bt = np.array([[0, 1], [2, 3]], np.int32)
    base = dict(block_table=bt, T=4, max_seqlen_q=4, max_seqlen_k=8, block_size=4, num_blocks=4)
    ok = O.prepare_metadata(np.array([0, 2, 4], np.int32), np.array([0, 0], np.int32), **base)
    assert ok["status"] == 0
    # decreasing cumulative lengths: clamped, flagged
    m = O.prepare_metadata(np.array([0, 3, 2], np.int32), np.array([0, 0], np.int32), **base)
    assert m["status"] & O.ST_BAD_CU
    assert m["seqlens_q"].tolist() == [3, 0]
    assert m["token_batch"].tolist() == [0, 0, 0, -1]
    # last entry short of T: trailing token has no owner
    m = O.prepare_metadata(np.array([0, 1, 3], np.int32), np.array([0, 0], np.int32), **base)
    assert m["status"] & O.ST_BAD_CU and m["token_batch"][3] == -1 and m["slot_mapping"][3] == -1
    # negative past
    m = O.prepare_metadata(np.array([0, 2, 4], np.int32), np.array([-5, 0], np.int32), **base)
    assert m["status"] & O.ST_BAD_CU and m["token_pos"].tolist() == [0, 1, 0, 1]
    # position beyond the table
    m = O.prepare_metadata(np.array([0, 2, 4], np.int32), np.array([7, 0], np.int32), **base)
    assert m["status"] == O.ST_CAPACITY | O.ST_BOUNDS
    assert m["slot_mapping"].tolist() == [1 * 4 + 3, -1, 8, 9]
    # invalid block id
    bt2 = np.array([[0, -1], [2, 9]], np.int32)
    m = O.prepare_metadata(np.array([0, 2, 4], np.int32), np.array([3, 3], np.int32), bt2, 4, 4, 8, 4, 4)
    assert m["status"] == O.ST_BAD_BLOCK
    assert m["slot_mapping"].tolist() == [3, -1, 11, -1]


# ---------------------------------------------------------------------------
# append
# ---------------------------------------------------------------------------

def test_append_readback_and_untouched():
    lw = Logical([3, 1, 5], [10, 0, 20], H_q=4, H_kv=2, D=8, bs=4, seed=1)
    meta = O.prepare_metadata(lw.cu, np.asarray(lw.past, np.int32), lw.block_table, lw.T,
                              5, max(lw.L), lw.bs, lw.NB)
    kc, vc = O.append_kv(lw.k_new, lw.v_new, "f16", lw.k_cache, lw.v_cache, "f16", meta["slot_mapping"])
    touched = np.zeros(lw.k_cache.shape[:2], bool)
    for b in range(lw.B):
        for j in range(lw.L[b]):
            blk = lw.block_table[b, j // lw.bs]
            assert np.array_equal(kc[blk, j % lw.bs].view(np.uint16), lw.K[b][j].view(np.uint16))
            assert np.array_equal(vc[blk, j % lw.bs].view(np.uint16), lw.V[b][j].view(np.uint16))
            if j >= lw.past[b]:
                touched[blk, j % lw.bs] = True
    assert np.array_equal(kc[~touched].view(np.uint16), lw.k_cache[~touched].view(np.uint16))


def test_int8_quantize_reading():
    s = np.float32(1.0)
    x = np.array([2.5, 3.5, -2.5, -3.5, 0.5, 1.5, 300.0, -300.0, 127.4, -128.6, 126.5],
                 dtype=np.float32)
    q = O.quantize_int8(x, np.full_like(x, s))
    assert q.tolist() == [2, 4, -2, -4, 0, 2, 127, -128, 127, -128, 126]
    rng = np.random.default_rng(3)
    xs = rng.standard_normal(10000).astype(np.float32)
    sc = rng.uniform(0.01, 0.05, 10000).astype(np.float32)
    q = O.quantize_int8(xs, sc).astype(np.float64)
    r = xs.astype(np.float64) / sc.astype(np.float64)
    inr = (r > -128.5) & (r < 127.5)
    assert np.all(np.abs(q[inr] - r[inr]) <= 0.5 + 1e-6)
    assert np.all(q[r >= 127.5] == 127) and np.all(q[r <= -128.5] == -128)


# ---------------------------------------------------------------------------
# attention against the library formulation
# ---------------------------------------------------------------------------

def _cmp(lw, res, b, ref, tol=1e-10):
    t0 = int(lw.cu[b])
    got = res["out"][t0:t0 + lw.q_lens[b]]
    np.testing.assert_allclose(got, ref, atol=tol, rtol=0)


@pytest.mark.parametrize("G", [1, 4])
def test_dense_causal_vs_sdpa(G):
    lw = Logical([5, 1, 9], [0, 12, 7], H_q=2 * G, H_kv=2, D=16, bs=4, seed=10 + G)
    res = lw.run()
    for b in range(lw.B):
        _cmp(lw, res, b, lw.sdpa(b, lw.causal_mask(b)))


def test_sink_vs_sdpa_extra_key():
    lw = Logical([4, 1], [3, 20], H_q=6, H_kv=3, D=8, bs=4, seed=21)
    sinks = np.random.default_rng(0).standard_normal(6).astype(np.float32) * 2
    res = lw.run(sinks=sinks)
    for b in range(lw.B):
        _cmp(lw, res, b, lw.sdpa(b, lw.causal_mask(b), sinks=sinks))


@pytest.mark.parametrize("W", [1, 3, 8, 1000])
def test_window_vs_sdpa_band(W):
    lw = Logical([6, 1, 3], [0, 30, 9], H_q=4, H_kv=2, D=8, bs=4, seed=30 + W)
    sinks = np.linspace(-1, 1, 4).astype(np.float32)
    res = lw.run(window=W, sinks=sinks)
    for b in range(lw.B):
        band = lw.causal_mask(b) & torch.ones(lw.q_lens[b], lw.L[b], dtype=torch.bool).triu(
            diagonal=lw.past[b] - W + 1)
        _cmp(lw, res, b, lw.sdpa(b, band, sinks=sinks))


def test_selected_main_vs_sdpa_per_head():
    lw = Logical([1, 1, 3], [40, 17, 25], H_q=6, H_kv=3, D=8, bs=4, seed=41)
    rng = np.random.default_rng(5)
    K = 7
    sel = np.full((lw.B, lw.H_kv, K), -1, np.int32)
    for b in range(lw.B):
        for h in range(lw.H_kv):
            n = int(rng.integers(0, K + 1))
            sel[b, h, :n] = rng.permutation(lw.L[b])[:n]
    sinks = rng.standard_normal(6).astype(np.float32)
    res = lw.run(selected_idx=sel, sel_per_request=1, sel_target=0, sinks=sinks)
    G = lw.H_q // lw.H_kv
    for b in range(lw.B):
        mask = torch.zeros(lw.H_q, lw.q_lens[b], lw.L[b], dtype=torch.bool)
        for h in range(lw.H_q):
            idx = [int(i) for i in sel[b, h // G] if i >= 0]
            mask[h][:, idx] = True
        mask &= lw.causal_mask(b)
        _cmp(lw, res, b, lw.sdpa(b, mask, sinks=sinks))


def test_aux_vs_sdpa():
    lw = Logical([2, 1], [9, 30], H_q=4, H_kv=2, D=8, bs=4, seed=51)
    rng = np.random.default_rng(8)
    cap, W, K = 12, 5, 6
    aux_k = rng.standard_normal((lw.B, cap, lw.H_kv, lw.D)).astype(np.float16)
    aux_v = rng.standard_normal((lw.B, cap, lw.H_kv, lw.D)).astype(np.float16)
    aux_len = np.array([12, 7], np.int32)
    sel = np.full((lw.B, lw.H_kv, K), -1, np.int32)
    for b in range(lw.B):
        for h in range(lw.H_kv):
            n = int(rng.integers(1, K + 1))
            sel[b, h, :n] = rng.permutation(int(aux_len[b]))[:n]
    sel[1, 0, -1] = 9            # inside the store's capacity but beyond request 1's aux length
    sinks = rng.standard_normal(4).astype(np.float32)
    res = lw.run(window=W, selected_idx=sel, sel_per_request=1, sel_target=1, aux_k=aux_k,
                 aux_v=aux_v, aux_seqlens=aux_len, sinks=sinks)
    assert res["status"] == O.ST_BAD_IDX
    G = lw.H_q // lw.H_kv
    for b in range(lw.B):
        ek = torch.from_numpy(aux_k[b].astype(np.float64)).permute(1, 0, 2)   # [H_kv, cap, D]
        ev = torch.from_numpy(aux_v[b].astype(np.float64)).permute(1, 0, 2)
        band = lw.causal_mask(b) & torch.ones(lw.q_lens[b], lw.L[b], dtype=torch.bool).triu(
            diagonal=lw.past[b] - W + 1)
        mask = torch.zeros(lw.H_q, lw.q_lens[b], lw.L[b] + cap, dtype=torch.bool)
        mask[:, :, :lw.L[b]] = band
        for h in range(lw.H_q):
            idx = [lw.L[b] + int(i) for i in sel[b, h // G] if 0 <= i < aux_len[b]]
            mask[h][:, idx] = True
        _cmp(lw, res, b, lw.sdpa(b, mask, sinks=sinks, extra_k=ek, extra_v=ev))


def test_int8_attention_vs_dequantized_sdpa():
    rng = np.random.default_rng(61)
    B, H_q, H_kv, D, bs, past = 2, 4, 2, 8, 4, [10, 6]
    L = [p + 1 for p in past]
    NB = sum((x + bs - 1) // bs for x in L)
    bt = np.full((B, 3), -1, np.int32)
    perm = rng.permutation(NB)
    o = 0
    for b in range(B):
        n = (L[b] + bs - 1) // bs
        bt[b, :n] = perm[o:o + n]
        o += n
    kc = rng.integers(-127, 128, (NB, bs, H_kv, D)).astype(np.int8)
    vc = rng.integers(-127, 128, (NB, bs, H_kv, D)).astype(np.int8)
    ks = rng.uniform(0.01, 0.05, (H_kv, D)).astype(np.float32)
    vs = rng.uniform(0.01, 0.05, (H_kv, D)).astype(np.float32)
    q = rng.standard_normal((B, H_q, D)).astype(np.float16)
    kn = rng.standard_normal((B, H_kv, D)).astype(np.float16)
    vn = rng.standard_normal((B, H_kv, D)).astype(np.float16)
    cu = np.arange(B + 1, dtype=np.int32)
    meta = O.prepare_metadata(cu, np.array(past, np.int32), bt, B, 1, max(L), bs, NB)
    kc2, vc2 = O.append_kv(kn, vn, "f16", kc, vc, "i8", meta["slot_mapping"], ks, vs)
    res = O.attention(q, "f16", kc2, vc2, "i8", bt, meta, H_kv=H_kv, k_scale=ks, v_scale=vs)
    for b in range(B):
        rows = [(bt[b, j // bs], j % bs) for j in range(L[b])]
        Kd = np.stack([kc2[r] for r in rows]).astype(np.float64) * ks.astype(np.float64)
        Vd = np.stack([vc2[r] for r in rows]).astype(np.float64) * vs.astype(np.float64)
        # new token went through the quantiser
        np.testing.assert_array_equal(kc2[rows[-1]], O.quantize_int8(kn[b].astype(np.float32), ks))
        qq = torch.from_numpy(q[b].astype(np.float64))[:, None]
        kk = torch.from_numpy(Kd).permute(1, 0, 2).repeat_interleave(2, 0)
        vv = torch.from_numpy(Vd).permute(1, 0, 2).repeat_interleave(2, 0)
        ref = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv)[:, 0].numpy()
        np.testing.assert_allclose(res["out"][b], ref, atol=1e-12, rtol=0)


def test_lse_vs_logsumexp():
    lw = Logical([3], [5], H_q=2, H_kv=1, D=8, bs=4, seed=71)
    sinks = np.array([0.3, -2.0], np.float32)
    res = lw.run(sinks=sinks)
    q = torch.from_numpy(lw.Q.astype(np.float64))
    k = torch.from_numpy(lw.K[0].astype(np.float64))[:, 0]
    for i in range(3):
        p = 5 + i
        for h in range(2):
            s = (k[:p + 1] @ q[i, h]) / math.sqrt(8)
            ref = torch.logsumexp(torch.cat([s, torch.tensor([float(sinks[h])], dtype=torch.float64)]), 0)
            assert abs(res["lse"][i, h] - float(ref)) < 1e-12


def test_default_scale_matches_library_default():
    lw = Logical([1], [9], H_q=2, H_kv=2, D=16, bs=4, seed=72)
    a = lw.run(scale=0.0)["out"]
    b = lw.run(scale=0.5)["out"]
    ref = lw.sdpa(0, lw.causal_mask(0))          # library default 1/sqrt(D)
    np.testing.assert_allclose(a[0], ref[0], atol=1e-12)
    assert np.abs(a - b).max() > 1e-6


# ---------------------------------------------------------------------------
# closed forms
# ---------------------------------------------------------------------------

def _single(q, Ks, Vs, sink=None, **kw):
    """One request, one kv head, logical keys Ks [L, D]; returns out [H_q, D]."""
    L, D = Ks.shape
    H_q = q.shape[0]
    bs = 4
    nb = (L + bs - 1) // bs
    bt = np.arange(nb, dtype=np.int32)[None, ::-1].copy()        # reversed placement
    kc = np.zeros((nb, bs, 1, D), np.float64)
    vc = np.zeros((nb, bs, 1, D), np.float64)
    for j in range(L):
        kc[bt[0, j // bs], j % bs, 0] = Ks[j]
        vc[bt[0, j // bs], j % bs, 0] = Vs[j]
    meta = O.prepare_metadata(np.array([0, 1], np.int32), np.array([L - 1], np.int32), bt, 1, 1,
                              L, bs, nb)
    sinks = None if sink is None else np.full(H_q, sink, np.float32)
    r = O.attention(q[None].astype(np.float64), "f64", kc, vc, "f64", bt, meta, H_kv=1,
                    sinks=sinks, **kw)
    return r["out"][0], r["lse"][0]


def test_closed_form_constant_v():
    rng = np.random.default_rng(80)
    L, D = 11, 8
    v = rng.standard_normal(D)
    Vs = np.tile(v, (L, 1))
    Ks = rng.standard_normal((L, D))
    q = rng.standard_normal((3, D))
    out, _ = _single(q, Ks, Vs)
    np.testing.assert_allclose(out, np.tile(v, (3, 1)), atol=1e-13)
    # q = 0: all logits are 0, so the weights are uniform; the sink takes e^sink
    out, lse = _single(np.zeros((2, D)), Ks, Vs, sink=0.7)
    np.testing.assert_allclose(out, np.tile(L * v / (L + math.exp(0.7)), (2, 1)), atol=1e-13)
    np.testing.assert_allclose(lse, np.log(L + math.exp(0.7)), atol=1e-13)


def test_closed_form_single_key_and_window_one():
    rng = np.random.default_rng(81)
    D = 8
    Ks = rng.standard_normal((1, D))
    Vs = rng.standard_normal((1, D))
    q = rng.standard_normal((2, D))
    out, _ = _single(q, Ks, Vs)
    np.testing.assert_array_equal(out, np.tile(Vs[0], (2, 1)))
    # window of one key with a sink: v_p * e^{s_p} / (e^{s_p} + e^{sink})
    L = 9
    Ks = rng.standard_normal((L, D))
    Vs = rng.standard_normal((L, D))
    out, _ = _single(q, Ks, Vs, sink=-0.4, window=1)
    s = (q @ Ks[-1]) / math.sqrt(D)
    w = np.exp(s) / (np.exp(s) + math.exp(-0.4))
    np.testing.assert_allclose(out, w[:, None] * Vs[-1][None], atol=1e-13)


def test_closed_form_empty_selection():
    rng = np.random.default_rng(82)
    L, D = 6, 8
    Ks, Vs = rng.standard_normal((L, D)), rng.standard_normal((L, D))
    q = rng.standard_normal((2, D))
    sel = np.full((1, 1, 4), -1, np.int32)
    out, lse = _single(q, Ks, Vs, selected_idx=sel, sel_per_request=1, sel_target=0)
    assert np.all(out == 0) and np.all(np.isneginf(lse))
    out, lse = _single(q, Ks, Vs, sink=1.5, selected_idx=sel, sel_per_request=1, sel_target=0)
    assert np.all(out == 0)
    np.testing.assert_allclose(lse, 1.5)


# ---------------------------------------------------------------------------
# invariants
# ---------------------------------------------------------------------------

def test_select_all_equals_dense_and_order_invariance():
    lw = Logical([1, 1], [23, 50], H_q=4, H_kv=2, D=8, bs=4, seed=90)
    sinks = np.array([0.1, -0.3, 2.0, -1.0], np.float32)
    dense = lw.run(sinks=sinks)["out"]
    Kw = 64
    rng = np.random.default_rng(1)
    sel = np.full((2, 2, Kw), -1, np.int32)
    for b in range(2):
        for h in range(2):
            sel[b, h, :lw.L[b]] = rng.permutation(lw.L[b])
    a = lw.run(sinks=sinks, selected_idx=sel, sel_per_request=1, sel_target=0)["out"]
    np.testing.assert_allclose(a, dense, atol=1e-13)
    sel2 = sel[:, :, ::-1].copy()
    c = lw.run(sinks=sinks, selected_idx=sel2, sel_per_request=1, sel_target=0)["out"]
    np.testing.assert_allclose(c, dense, atol=1e-13)


def test_paged_equals_contiguous():
    a = Logical([3, 1], [13, 6], H_q=4, H_kv=2, D=8, bs=4, seed=91, identity=False)
    b = Logical([3, 1], [13, 6], H_q=4, H_kv=2, D=8, bs=4, seed=91, identity=True)
    for lw in (a, b):
        lw.Q = a.Q
    np.testing.assert_array_equal(a.run(window=5)["out"], b.run(window=5)["out"])


def test_bad_index_flag_and_skip():
    lw = Logical([1], [9], H_q=2, H_kv=1, D=8, bs=4, seed=92)
    sel = np.array([[[3, -1, 10, -7, 5]]], np.int32)      # 10 >= L, -7 < -1
    r = lw.run(selected_idx=sel, sel_per_request=1, sel_target=0)
    assert r["status"] == O.ST_BAD_IDX
    ok = lw.run(selected_idx=np.array([[[3, 5]]], np.int32), sel_per_request=1, sel_target=0)
    np.testing.assert_array_equal(r["out"], ok["out"])


# ---------------------------------------------------------------------------
# QKV prologue: RMSNorm, rotary embedding, rounding to the activation dtype
# ---------------------------------------------------------------------------

def test_rms_norm_worked_example():
    # [3, 4]: mean square 12.5, so [3, 4] / sqrt(12.5) scaled by [1, 2]
    got = O.rms_norm(np.array([3.0, 4.0]), np.array([1.0, 2.0]), 0.0)
    r = math.sqrt(12.5)
    np.testing.assert_allclose(got, [3.0 / r, 8.0 / r], rtol=0, atol=1e-15)


def test_rms_norm_matches_torch_and_eps():
    rng = np.random.default_rng(11)
    x = rng.standard_normal((5, 64))
    w = rng.uniform(0.5, 1.5, 64)
    for eps in (0.0, 1e-6, 0.5):
        ref = torch.nn.functional.rms_norm(torch.from_numpy(x), (64,), torch.from_numpy(w), eps)
        np.testing.assert_allclose(O.rms_norm(x, w, eps), ref.numpy(), rtol=1e-13, atol=1e-14)
    # scale invariance without eps
    np.testing.assert_allclose(O.rms_norm(7.5 * x, w, 0.0), O.rms_norm(x, w, 0.0), rtol=1e-13)


def test_rotate_quarter_turn():
    x = np.array([1.0, 2.0, 3.0, 4.0, 5.0])
    c, s = np.zeros(2), np.ones(2)
    # half-split pairs (0, 2), (1, 3): (a, b) -> (-b, a); channel 4 is past rotary_dim
    np.testing.assert_array_equal(O.rotate(x, c, s, 4, False), [-3.0, -4.0, 1.0, 2.0, 5.0])
    # interleaved pairs (0, 1), (2, 3)
    np.testing.assert_array_equal(O.rotate(x, c, s, 4, True), [-2.0, 1.0, -4.0, 3.0, 5.0])


def test_rotate_zero_angle_and_partial_tail():
    rng = np.random.default_rng(12)
    x = rng.standard_normal(64)
    np.testing.assert_array_equal(O.rotate(x, np.ones(16), np.zeros(16), 32, True), x)
    y = O.rotate(x, *np.split(rng.standard_normal(32), 2), 32, False)
    np.testing.assert_array_equal(y[32:], x[32:])


def _theta(pos, rd, base=10000.0):
    inv = base ** (-np.arange(0, rd, 2) / rd)
    return np.cos(pos * inv), np.sin(pos * inv)


@pytest.mark.parametrize("interleaved", [False, True])
def test_rotate_as_complex_multiplication(interleaved):
    """Each channel pair (a, b) is the complex number a + ib times exp(i theta)."""
    rng = np.random.default_rng(13)
    rd, x = 48, rng.standard_normal(64)
    c, s = _theta(37, rd)
    if interleaved:
        a, b = x[0:rd:2], x[1:rd:2]
    else:
        a, b = x[:rd // 2], x[rd // 2:rd]
    z = (a + 1j * b) * np.exp(1j * np.arctan2(s, c))
    y = O.rotate(x, c, s, rd, interleaved)
    ya, yb = (y[0:rd:2], y[1:rd:2]) if interleaved else (y[:rd // 2], y[rd // 2:rd])
    np.testing.assert_allclose(ya, z.real, atol=1e-13)
    np.testing.assert_allclose(yb, z.imag, atol=1e-13)


def test_rope_relative_position_and_norm():
    rng = np.random.default_rng(14)
    rd = 64
    q, k = rng.standard_normal(64), rng.standard_normal(64)
    dots = []
    for p in (5, 40, 300):
        qr = O.rotate(q, *_theta(p + 9, rd), rd, False)
        kr = O.rotate(k, *_theta(p, rd), rd, False)
        np.testing.assert_allclose(np.linalg.norm(qr), np.linalg.norm(q), rtol=1e-13)
        dots.append(float(qr @ kr))
    np.testing.assert_allclose(dots, dots[0], rtol=1e-11)


def test_interleaved_is_half_split_of_permuted_channels():
    rng = np.random.default_rng(15)
    rd, x = 32, rng.standard_normal(64)
    c, s = _theta(21, rd)
    perm = np.concatenate([np.arange(0, rd, 2), np.arange(1, rd, 2), np.arange(rd, 64)])
    # interleaved on x == half-split on x[perm], read back through the permutation
    got = O.rotate(x, c, s, rd, True)
    via = np.empty(64)
    via[perm] = O.rotate(x[perm], c, s, rd, False)
    np.testing.assert_allclose(got, via, atol=1e-14)


def test_encode_rounds_to_nearest_even():
    # bf16 spacing at 1 is 2^-7: 1 + 2^-8 is a tie (to 1.0, the even code);
    # 1 + 2^-8 + 2^-9 rounds up; -2.5e-3 and pi round to their bf16 neighbours
    x = np.array([1.0, 1.0 + 2.0 ** -8, 1.0 + 2.0 ** -8 + 2.0 ** -9, 1.0 + 3 * 2.0 ** -8])
    np.testing.assert_array_equal(O.encode(x, "bf16"), [0x3F80, 0x3F80, 0x3F81, 0x3F82])
    h = O.encode(np.array([1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11]), "f16")
    np.testing.assert_array_equal(h.view(np.uint16), [0x3C00, 0x3C02])


def test_bf16_decode_bit_patterns():
    """bf16 codes read by hand from the format (1 sign, 8 exponent, 7 fraction
    bits, bias 127): the value is the code placed in the upper half of a
    binary32 word."""
    codes = np.array([0x3F80, 0xC040, 0x0001, 0x4049, 0x3F81, 0x7F7F, 0x8000, 0x0080, 0x7F80, 0xFF80],
                     dtype=np.uint16)
    want = [1.0, -3.0, 2.0 ** -133, 3.140625, 1.0 + 2.0 ** -7, (2.0 - 2.0 ** -7) * 2.0 ** 127, -0.0,
            2.0 ** -126, math.inf, -math.inf]
    got = O.decode(codes, "bf16")
    assert got.dtype == np.float64
    np.testing.assert_array_equal(got, want)
    assert math.copysign(1.0, got[6]) == -1.0


def test_bf16_decode_encode_round_trip():
    """Every non-NaN bf16 code decodes to a value that encodes back to itself."""
    codes = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    exp = (codes.astype(np.uint32) >> 7) & 0xFF
    frac = codes.astype(np.uint32) & 0x7F
    keep = ~((exp == 0xFF) & (frac != 0))
    codes = codes[keep]
    np.testing.assert_array_equal(O.encode(O.decode(codes, "bf16"), "bf16"), codes)


def _prologue_wl(**pro):
    from selected_token_sparse_b200 import workloads as W
    return W.make_workload(act="f16", B=2, H_q=4, H_kv=2, D=64, block_size=16, q_lens=[3, 2],
                           past=[7, 20], window=16, prologue=pro, seed=21)


def test_prologue_without_norm_or_rope_is_identity():
    wl = _prologue_wl(packed=True)
    q, k, v = O.split_packed(wl["qkv"], wl.H_q, wl.H_kv)
    meta = O.prepare_metadata(wl["cu_seqlens_q"], wl["past_seqlens"], wl["block_table"], wl.T,
                              wl.max_seqlen_q, wl.max_seqlen_k, wl.block_size, wl.NB)
    qo, ko, vo, st = O.qkv_prologue(q, k, v, "f16", meta["token_pos"])
    assert st == 0
    for a, b in ((qo, wl["q"]), (ko, wl["k_new"]), (vo, wl["v_new"])):
        np.testing.assert_array_equal(a.view(np.uint16), b.view(np.uint16))


def test_prologue_position_ids_equal_offset():
    """Explicit positions p + 3 give what the metadata positions with offset 3 give."""
    a = O.run_step(_prologue_wl(qk_norm=True, rotary_dim=32, interleaved=True, pos_ids=True,
                                pos_shift=3))
    b = O.run_step(_prologue_wl(qk_norm=True, rotary_dim=32, interleaved=True, rotary_offset=3))
    np.testing.assert_array_equal(a["q_out"].view(np.uint16), b["q_out"].view(np.uint16))
    np.testing.assert_allclose(a["out"], b["out"], rtol=0, atol=0)


def test_prologue_rotation_uses_the_token_position():
    """q_out of a token equals RMSNorm then rotation at past + index, rounded."""
    wl = _prologue_wl(qk_norm=True, rotary_dim=64, interleaved=False)
    r = O.run_step(wl)
    t, h = 4, 1                        # request 1, second token: position 20 + 1
    x = O.decode(wl["q"][t, h], "f16")
    y = O.rotate(O.rms_norm(x, wl["q_norm_weight"], 1e-6), wl["cos_cache"][21], wl["sin_cache"][21],
                 64, False)
    np.testing.assert_array_equal(r["q_out"][t, h], y.astype(np.float16))


def test_prologue_out_of_range_position_flags_bounds():
    wl = _prologue_wl(rotary_dim=32, pos_ids=True, pos_shift=10 ** 6)
    r = O.run_step(wl)
    assert r["status"] & O.ST_BOUNDS
    np.testing.assert_array_equal(r["q_out"].view(np.uint16), wl["q"].view(np.uint16))


# ---------------------------------------------------------------------------
# selection producer (TopK over per-key scores)
# ---------------------------------------------------------------------------

def test_topk_worked_examples():
    g = load("topk_worked.json")
    for c in g["cases"]:
        got = O.select_topk(np.array(c["scores"], dtype=np.float32), np.array(c["bound"]), c["top_k"],
                            c["sel_width"])
        np.testing.assert_array_equal(got, np.array(c["expected"]), err_msg=c["name"])


def _topk_by_dominance(row, last, k):
    """The unique set S of min(k, E) eligible keys such that every kept key
    beats every eligible key left out (higher score, or an equal score and a
    lower index), found by enumerating all subsets of a tiny row."""
    import itertools
    elig = [j for j in range(min(last, len(row) - 1) + 1) if not math.isnan(row[j]) and row[j] != -math.inf]
    n = min(k, len(elig))
    found = []
    for S in itertools.combinations(elig, n):
        rest = [j for j in elig if j not in S]
        if all(row[i] > row[j] or (row[i] == row[j] and i < j) for i in S for j in rest):
            found.append(list(S))
    assert len(found) == 1
    return found[0]


def test_topk_brute_force_dominance():
    rng = np.random.default_rng(7)
    for trial in range(300):
        n = int(rng.integers(1, 9))
        # few distinct values, so that ties are common; some masked keys
        row = rng.integers(-2, 3, size=n).astype(np.float32)
        row[rng.random(n) < 0.15] = -np.inf
        row[rng.random(n) < 0.1] = np.nan
        last = int(rng.integers(-1, n + 2))
        k = int(rng.integers(1, n + 2))
        W = k + int(rng.integers(0, 3))
        got = O.select_topk(row.reshape(1, 1, n), np.array([last]), k, W)[0, 0]
        want = _topk_by_dominance([float(v) for v in row], last, k)
        np.testing.assert_array_equal(got[:len(want)], want)
        assert (got[len(want):] == -1).all()


def test_topk_matches_stable_lexsort():
    """numpy's lexsort (score descending, then index) gives the same kept set
    on a larger row; the kept indices come out increasing."""
    rng = np.random.default_rng(8)
    R, H, N = 3, 2, 500
    scores = np.round(rng.standard_normal((R, H, N)), 1).astype(np.float32)   # many ties
    bound = np.array([499, 250, 37])
    got = O.select_topk(scores, bound, 60, 64)
    for r in range(R):
        for h in range(H):
            idx = np.arange(bound[r] + 1)
            order = np.lexsort((idx, -scores[r, h, :bound[r] + 1].astype(np.float64)))
            want = np.sort(order[:60])
            np.testing.assert_array_equal(got[r, h, :len(want)], want)
            assert (got[r, h, len(want):] == -1).all()
            assert (np.diff(got[r, h, :len(want)]) > 0).all()


# ---------------------------------------------------------------------------
# sequence-sharded split-KV: shard partials and their merge
# ---------------------------------------------------------------------------

def _ranges(lw, cuts):
    """kv_range [B, 2] of shard `cuts` = (lo, hi) for every request."""
    return np.array([[lo, hi] for lo, hi in cuts], dtype=np.int64)


def test_shard_partial_vs_sdpa_without_sink():
    """A shard's partial is plain softmax attention over the keys of its range
    (no sink): SDPA with the causal mask restricted to the range."""
    lw = Logical([3, 1], [40, 70], H_q=4, H_kv=2, D=64, bs=16, seed=31)
    rng = [(10, 30), (45, 71)]
    r = lw.run(window=0, kv_range=_ranges(lw, rng))
    for b in range(lw.B):
        lo, hi = rng[b]
        cols = torch.arange(lw.L[b])
        mask = lw.causal_mask(b) & ((cols >= lo) & (cols < hi))[None, :]
        want = lw.sdpa(b, mask)
        t0 = int(lw.cu[b])
        np.testing.assert_allclose(r["out"][t0:t0 + lw.q_lens[b]], want, atol=1e-12)


def test_merged_shards_equal_unsharded_sdpa_with_sink():
    """Partials over a partition of the keys (one shard empty for some rows),
    merged with the sink once, equal SDPA over all keys with the sink as an
    extra key."""
    lw = Logical([2, 1, 3], [50, 9, 100], H_q=6, H_kv=3, D=64, bs=16, seed=32)
    sinks = np.random.default_rng(5).standard_normal(6)
    cuts = [[(0, 20), (0, 4), (0, 0)], [(20, 45), (4, 10), (0, 60)], [(45, 1000), (10, 1000), (60, 1000)]]
    parts = [lw.run(window=0, kv_range=_ranges(lw, c)) for c in cuts]
    out, lse = O.merge_partials(np.stack([p["out"] for p in parts]), np.stack([p["lse"] for p in parts]), sinks)
    for b in range(lw.B):
        want = lw.sdpa(b, lw.causal_mask(b), sinks=sinks)
        t0 = int(lw.cu[b])
        np.testing.assert_allclose(out[t0:t0 + lw.q_lens[b]], want, atol=1e-12)
    whole = lw.run(window=0, sinks=sinks)
    np.testing.assert_allclose(lse, whole["lse"], atol=1e-12)


def test_merge_closed_forms():
    """One shard and no sink: the merge returns the shard's state.  All shards
    empty: 0 and -inf.  A sink alone over one shard rescales by l / (l + e^sink)."""
    rng = np.random.default_rng(6)
    o = rng.standard_normal((1, 2, 3, 8))
    l = rng.standard_normal((1, 2, 3))
    out, lse = O.merge_partials(o, l, None)
    np.testing.assert_allclose(out, o[0], atol=1e-15)
    np.testing.assert_allclose(lse, l[0], atol=1e-15)
    out, lse = O.merge_partials(np.zeros((2, 1, 1, 4)), np.full((2, 1, 1), -np.inf), None)
    assert (out == 0).all() and np.isneginf(lse).all()
    # every shard empty but a finite sink: the denominator is the sink alone
    out, lse = O.merge_partials(np.zeros((2, 1, 1, 4)), np.full((2, 1, 1), -np.inf), np.array([0.3]))
    assert (out == 0).all()
    np.testing.assert_allclose(lse, [[0.3]], atol=1e-15)
    sink = np.array([0.7, -1.0, 2.0])
    out, lse = O.merge_partials(o, l, sink)
    f = np.exp(l[0]) / (np.exp(l[0]) + np.exp(sink)[None, :])
    np.testing.assert_allclose(out, o[0] * f[..., None], atol=1e-12)
    np.testing.assert_allclose(lse, np.log(np.exp(l[0]) + np.exp(sink)[None, :]), atol=1e-12)
