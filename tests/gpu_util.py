"""Helpers for the GPU parity tests: run a workload through the C ABI and
through the oracle, and compare the two."""
import numpy as np

from oracle import spa_oracle as O

TOL = {"f32": 1e-5, "f16": 3e-3, "bf16": 3e-3}
LSE_TOL = 2e-4


def rounding_incurred(ref, act):
    """|round_act(ref) - ref|: the rounding error the reference value itself
    incurs when it is written in the activation dtype (nearest even).  A
    kernel writes its output in that dtype, so this part of the difference is
    not the kernel's."""
    ref = np.asarray(ref, dtype=np.float64)
    if act == "f32":
        return np.abs(ref.astype(np.float32).astype(np.float64) - ref)
    return np.abs(O.decode(O.encode(ref, act), act) - ref)


def oracle_step(wl, tokens=None):
    return O.run_step(wl, tokens=tokens)


def _bits(x):
    x = np.asarray(x)
    if x.dtype == np.float16:
        return x.view(np.uint16)
    if x.dtype == np.float32:
        return x.view(np.uint32)
    return x


def compare(wl, got, ref, tokens=None, check_out=True, check_cache=True, strict=False):
    """Bit-exact metadata / status / cache; output within the dtype's tolerance.

    Every output element must lie within TOL plus the rounding the reference
    value incurs in the output format, |round_act(ref) - ref| (for bf16 that
    reaches 3e-3 only at |ref| >= 0.77).  With ``strict`` the plain max-abs
    TOL must hold as well (the named workloads)."""
    for k in ("seqlens_q", "seqlen_k", "token_batch", "token_pos", "slot_mapping"):
        np.testing.assert_array_equal(got[k], ref["meta"][k], err_msg=k)
    assert got["status"] == ref["status"], (hex(got["status"]), hex(ref["status"]))
    if check_cache:
        for k in ("k_cache", "v_cache"):
            g = got[k]
            if g.dtype.is_floating_point and g.element_size() == 2:
                g = g.view(__import__("torch").int16)
            g = g.numpy()
            r = np.asarray(ref[k])
            if r.dtype == np.float16:
                r = r.view(np.int16)
            elif r.dtype == np.uint16:
                r = r.view(np.int16)
            assert np.array_equal(g.reshape(-1).view(np.uint8), r.reshape(-1).view(np.uint8)), k
    if not check_out:
        return None
    rows = np.arange(wl.T) if tokens is None else np.asarray(tokens)
    go, ro = got["out"][rows], ref["out"][rows]
    assert np.isfinite(go).all()
    diff = np.abs(go - ro)
    err = float(diff.max()) if go.size else 0.0
    bound = TOL[wl.act] + rounding_incurred(ro, wl.act)
    worst = float((diff - bound).max()) if go.size else -1.0
    assert worst <= 0, f"max-abs error {err}; exceeds tolerance + rounding floor by {worst}"
    if strict:
        assert err <= TOL[wl.act], f"max-abs error {err} > {TOL[wl.act]}"
    if "lse" in got:
        gl, rl = got["lse"][rows], ref["lse"][rows]
        both_inf = np.isneginf(gl) & np.isneginf(rl)
        lerr = float(np.abs(np.where(both_inf, 0.0, gl - rl)).max()) if gl.size else 0.0
        assert lerr <= LSE_TOL, f"lse error {lerr}"
    return err
