"""Sequence-sharded split-KV, host side, on CPU: the shard ranges, the
shard's block table, and the gather of partial states over a world-size-2
gloo group.  Each rank computes its shard's partial state with the oracle
(there is no GPU here); the gathered states merged by the oracle's merge equal
the oracle's unsharded attention.  The CUDA partial and merge kernels are
compared with the oracle in tests/test_gpu_shard.py."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import spa_oracle as O
from selected_token_sparse_b200 import shard, workloads as W


def test_sequence_ranges_partition_block_aligned():
    lengths = [1, 16, 17, 100, 1000, 0]
    for world in (1, 2, 3, 4, 7):
        parts = [shard.sequence_ranges(lengths, world, r, 16) for r in range(world)]
        for b, L in enumerate(lengths):
            cover = []
            for r in range(world):
                lo, hi = parts[r][b]
                assert 0 <= lo <= hi <= L
                assert lo % 16 == 0
                cover.extend(range(lo, hi))
            assert cover == list(range(L))          # contiguous, disjoint, complete


def test_shard_block_table_maps_only_its_range():
    bt = np.arange(24, dtype=np.int32).reshape(2, 12)
    rng = np.array([[16, 40], [0, 0]], dtype=np.int32)
    got = shard.shard_block_table(bt, rng, 16)
    np.testing.assert_array_equal(got[0], [-1, 1, 2, -1, -1, -1, -1, -1, -1, -1, -1, -1])
    assert (got[1] == -1).all()


def _wl():
    return W.make_workload(act="f16", B=3, H_q=8, H_kv=2, D=64, block_size=16, q_lens=[1, 2, 1],
                           past=[90, 40, 7], window=0, has_sinks=True, seed=41)


def _oracle_partial(wl, kv_range):
    a = wl.arrays
    meta = O.prepare_metadata(a["cu_seqlens_q"], a["past_seqlens"], a["block_table"], wl.T,
                              wl.max_seqlen_q, wl.max_seqlen_k, wl.block_size, wl.NB)
    kc, vc = O.append_kv(a["k_new"], a["v_new"], wl.act, a["k_cache"], a["v_cache"], wl.cache,
                         meta["slot_mapping"])
    return O.attention(a["q"], wl.act, kc, vc, wl.cache, a["block_table"], meta, H_kv=wl.H_kv,
                       kv_range=kv_range, sinks=None)


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        wl = _wl()
        lengths = [p + n for p, n in zip(wl.past, wl.q_lens)]
        rng = shard.sequence_ranges(lengths, world, rank, wl.block_size)
        part = _oracle_partial(wl, rng)
        po, pl = shard.all_gather_partials(torch.from_numpy(part["out"]), torch.from_numpy(part["lse"]))
        q.put((rank, po.numpy(), pl.numpy()))
    finally:
        dist.destroy_process_group()


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def test_two_gloo_ranks_merge_to_the_unsharded_attention():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted([q.get(timeout=300) for _ in procs], key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    wl = _wl()
    full = O.run_step(wl)
    for rank, po, pl in res:
        assert po.shape[0] == 2
        out, lse = O.merge_partials(po, pl, wl.arrays["sinks"])
        np.testing.assert_allclose(out, full["out"], atol=1e-12)
        np.testing.assert_allclose(lse, full["lse"], atol=1e-12)
    # both ranks gathered the same states; each shard holds keys of some
    # request, and the one-block request is empty on rank 0 (lse -inf)
    np.testing.assert_array_equal(res[0][1], res[1][1])
    pl = res[0][2]
    assert np.isfinite(pl[0]).any() and np.isfinite(pl[1]).all()
    assert np.isneginf(pl[0, 3]).all()
