"""GPU parity of the selection producer (spa_select_topk) against the oracle's
select_topk, bit for bit: the kept indices, their order and the -1 padding.
Then the producer's rows feed spa_attention's selected mode, and the output
matches the oracle's attention over the oracle's own selection."""
import numpy as np
import pytest
import torch

from oracle import spa_oracle as O
from selected_token_sparse_b200 import pipeline, spa, workloads as W
from tests.gpu_util import compare, oracle_step

pytestmark = pytest.mark.gpu


def _scores(rng, R, H, N, ties=False, special=False):
    s = rng.standard_normal((R, H, N)).astype(np.float32)
    if ties:
        s = np.round(s, 1).astype(np.float32)      # many equal scores
    if special:
        m = rng.random((R, H, N))
        s[m < 0.03] = -np.inf
        s[(m >= 0.03) & (m < 0.05)] = np.nan
        s[(m >= 0.05) & (m < 0.06)] = np.inf
        s[(m >= 0.06) & (m < 0.08)] = -0.0
        s[(m >= 0.08) & (m < 0.10)] = 0.0
    return s


def _run(scores, bound, top_k, width):
    got = spa.select_topk(torch.from_numpy(scores).cuda(), torch.from_numpy(bound.astype(np.int32)).cuda(),
                          top_k, width)
    torch.cuda.synchronize()
    return got.cpu().numpy()


CASES = {
    # the selected-token decode shape: 16 requests x 4 kv heads x 32768 keys,
    # 1946 kept in rows of 2048 (the workload's 5% padding)
    "selected_decode_shape": dict(R=16, H=4, N=32768, top_k=1946, width=2048, bounds="full"),
    "ties_ragged_bounds": dict(R=5, H=3, N=3001, top_k=700, width=777, bounds="ragged", ties=True),
    "specials": dict(R=4, H=2, N=2000, top_k=300, width=300, bounds="ragged", special=True, ties=True),
    "fewer_eligible_than_k": dict(R=3, H=2, N=500, top_k=400, width=512, bounds="short"),
    "top_k_zero": dict(R=2, H=2, N=100, top_k=0, width=8, bounds="full"),
    "one_key": dict(R=2, H=1, N=1, top_k=1, width=4, bounds="full"),
    # beyond the shared-memory staging capacity: the passes re-read global memory
    "long_rows_global_path": dict(R=2, H=2, N=70001, top_k=4096, width=4100, bounds="ragged", ties=True),
    "all_ties": dict(R=2, H=2, N=5000, top_k=1234, width=1300, bounds="full", const=True),
}


@pytest.mark.parametrize("case", list(CASES))
def test_select_topk_matches_oracle(case):
    c = dict(CASES[case])
    rng = np.random.default_rng(hash(case) % (2 ** 32))
    R, H, N = c["R"], c["H"], c["N"]
    s = _scores(rng, R, H, N, ties=c.get("ties", False), special=c.get("special", False))
    if c.get("const"):
        s[:] = 0.5
    if c["bounds"] == "full":
        bound = np.full(R, N - 1)
    elif c["bounds"] == "short":
        bound = rng.integers(-1, 300, size=R)
    else:
        bound = rng.integers(0, N + 50, size=R)
        bound[0] = -1 if R > 2 else bound[0]
        bound[-1] = N - 1
    got = _run(s, bound, c["top_k"], c["width"])
    want = O.select_topk(s, bound, c["top_k"], c["width"])
    np.testing.assert_array_equal(got, want)


def test_select_topk_twice_same_buffer():
    """A second call into the same output rows gives the same bits (nothing is
    left over from the first call)."""
    rng = np.random.default_rng(3)
    s = _scores(rng, 3, 2, 1500, ties=True)
    bound = np.array([1499, 700, 20])
    sc, bd = torch.from_numpy(s).cuda(), torch.from_numpy(bound.astype(np.int32)).cuda()
    out = torch.full((3, 2, 600), 12345, dtype=torch.int32, device="cuda")
    spa.select_topk(sc, bd, 512, 600, out=out)
    first = out.clone()
    spa.select_topk(sc, bd, 512, 600, out=out)
    torch.cuda.synchronize()
    assert torch.equal(first, out)
    np.testing.assert_array_equal(out.cpu().numpy(), O.select_topk(s, bound, 512, 600))


@pytest.mark.parametrize("small", [True, False])
def test_producer_feeds_attention(small):
    """Scores -> spa_select_topk -> the selected-token decode step; the output
    and the metadata match the oracle run on the oracle's selection."""
    wl = W.by_name("selected_decode_bf16", small=small)
    rng = np.random.default_rng(17)
    N = wl.max_seqlen_k
    scores = rng.standard_normal((wl.B, wl.H_kv, N)).astype(np.float32)
    top_k = wl.sel_width - wl.sel_width // 20
    bound = np.array([p + q - 1 for p, q in zip(wl.past, wl.q_lens)], dtype=np.int32)   # seqlen_k
    sel = O.select_topk(scores, bound, top_k, wl.sel_width)
    wl.arrays["selected_idx"] = sel          # the oracle's selection
    d = pipeline.to_device(wl)
    # the device rows come from the producer, written over the uploaded ones
    d["selected_idx"].fill_(7)
    spa.select_topk(torch.from_numpy(scores).cuda(), torch.from_numpy(bound).cuda(), top_k, wl.sel_width,
                    out=d["selected_idx"])
    st = pipeline.Step(wl, d, want_lse=True)
    st()
    torch.cuda.synchronize()
    np.testing.assert_array_equal(d["selected_idx"].cpu().numpy(), sel)
    got = {k: v.cpu().numpy() for k, v in st.meta.items()}
    got.update(status=int(st.status.item()), out=st.out.float().cpu().numpy().astype(np.float64),
               lse=st.lse.cpu().numpy().astype(np.float64), k_cache=d["k_cache"].cpu(),
               v_cache=d["v_cache"].cpu())
    compare(wl, got, oracle_step(wl), strict=True)
