"""The bench's multi-rank bookkeeping on CPU with gloo, world size 2: the
timed duration is the maximum over ranks, and the barrier is taken by every
rank.  Also checks the algorithmic byte / FLOP accounting on small cases."""
import os
import socket

import numpy as np
import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from selected_token_sparse_b200 import workloads as W


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = 1.5 + 2.0 * rank
        got = bench.reduce_max(mine)
        bench.barrier()
        q.put((rank, got, bench.dist_env()))
    finally:
        dist.destroy_process_group()


def test_reduce_max_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, env in res:
        assert got == 3.5
        assert env == (rank, 2, rank)


def test_reduce_max_single_process_is_identity():
    assert bench.reduce_max(4.25) == 4.25


def test_attended_bytes_window_and_selection():
    wl = W.make_workload(act="f16", B=2, H_q=4, H_kv=2, D=64, block_size=16, q_lens=[1, 1],
                         past=[10, 300], window=128, seed=0)
    # request 0 attends all 11 keys, request 1 its 128-key window; K and V, 2 bytes
    assert bench.attended_kv_bytes(wl) == (11 + 128) * 2 * 64 * 2 * 2
    wl = W.make_workload(act="bf16", B=1, H_q=2, H_kv=1, D=128, block_size=64, q_lens=[1],
                         past=[99], sel_mode="main", sel_width=10, sel_valid=7, seed=1)
    assert bench.attended_kv_bytes(wl) == 7 * 128 * 2 * 2


def test_attention_flops_causal():
    wl = W.make_workload(act="f16", B=2, H_q=2, H_kv=1, D=8, block_size=16, q_lens=[3, 2],
                         past=[0, 4], seed=0)
    pairs = (1 + 2 + 3) + (5 + 6)
    assert bench.attention_flops(wl) == 4 * 8 * 2 * pairs


def test_attended_bytes_of_a_token_subset():
    # two requests of 3 tokens each, window 4: request 0 tokens at 10, 11, 12
    wl = W.make_workload(act="f16", B=2, H_q=2, H_kv=1, D=64, block_size=16, q_lens=[3, 3],
                         past=[10, 2], window=4, seed=0)
    row = 64 * 2 * 2
    # all tokens: request 0 keys 7..12 (6), request 1 keys 0..4 (5)
    assert bench.attended_kv_bytes(wl) == (6 + 5) * row
    # token 1 alone (position 11): keys 8..11
    assert bench.attended_kv_bytes(wl, tokens=[1]) == 4 * row
    # token 3 (request 1, position 2): keys 0..2
    assert bench.attended_kv_bytes(wl, tokens=[1, 3]) == (4 + 3) * row
    assert bench.attention_flops(wl, tokens=[0]) == 4 * 64 * 2 * 4


def test_reference_arm_prints_our_config(capsys):
    """The reference arm (the oracle on the host) reports the same config object
    as our arm would for the same workload."""
    import json
    import sys
    argv = sys.argv
    sys.argv = ["bench.py", "--impl", "reference", "--workload", "tiny_decode_f32", "--steps", "1",
                "--warmup", "3"]
    try:
        bench.main()
    finally:
        sys.argv = argv
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert line["config"] == bench.workload_config(W.by_name("tiny_decode_f32"), 1)
    assert line["cpu_baseline"]["host_cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0


def test_select_bytes():
    sw = W.topk_selection_f32(small=True)
    sw.bound[:] = [9, -1]
    # row 0: keys 0..9 of H heads read; every output slot written
    assert bench.select_bytes(sw) == 4 * sw.H * 10 + 4 * sw.R * sw.H * sw.sel_width
