"""The oracle's pins are discriminating: a plausible mistake planted in a copy
of the oracle (on the CPU) makes at least one pin fail.

Each mutation rewrites one expression of the oracle's source text, loads the
result as a separate module and runs the pin tests against it.
"""
import importlib.util
import inspect
import types

import pytest

from oracle import spa_oracle
import tests.test_oracle_pins as pins

MUTATIONS = [
    # (description, original text, planted mistake)
    ("window off by one", "max(0, p - window + 1)", "max(0, p - window)"),
    ("window not clamped at zero", "max(0, p - window + 1) if window > 0 else 0",
     "(p - window + 1) if window > 0 else 0"),
    ("sink dropped from the denominator", "float(e.sum()) + math.exp(sink - m)", "float(e.sum())"),
    ("sink multiplied by the scale", "sink = -math.inf if sinks is None else float(sinks[h])",
     "sink = -math.inf if sinks is None else float(sinks[h]) * sc"),
    ("sink ignored in the max", "m = max(float(s.max()) if s.size else -math.inf, sink)",
     "m = float(s.max()) if s.size else -math.inf"),
    ("GQA head mapping interleaved", "h = h_kv * G + g", "h = g * H_kv + h_kv"),
    ("scale not applied", "s = sc * (K @ qt[h])", "s = (K @ qt[h])"),
    ("seqlen_k not total-1", "seqlen_k[b] = total - 1", "seqlen_k[b] = total"),
    ("per-token position ignores past", "p = past[owner] + (t - cs[owner])", "p = t - cs[owner]"),
    ("slot offset uses the position", "slot[t] = blk * block_size + p % block_size",
     "slot[t] = blk * block_size + (t % block_size)"),
    ("causal check dropped for selections",
     "main_pos = sel[(sel >= 0) & (sel < L) & (sel <= p)]", "main_pos = sel[(sel >= 0) & (sel < L)]"),
    ("value scale used for keys", "K = K * k_scale[h_kv].astype(np.float64)",
     "K = K * v_scale[h_kv].astype(np.float64)"),
    ("int8 rounding truncates", "r = np.rint(", "r = np.trunc("),
    ("aux length bound ignored", "aux_pos = sel[(sel >= 0) & (sel < int(aux_seqlens[b]))]",
     "aux_pos = sel[(sel >= 0)]"),
    ("lse without the max", "lse[t, h] = m + math.log(l)", "lse[t, h] = math.log(l)"),
    ("rotation sign flipped", "y[:half] = a * c - b * s", "y[:half] = a * c + b * s"),
    ("interleaved pair order swapped", "a, b = y[0:rotary_dim:2].copy(), y[1:rotary_dim:2].copy()",
     "b, a = y[0:rotary_dim:2].copy(), y[1:rotary_dim:2].copy()"),
    ("RMS over the sum, not the mean", "ms = np.mean(x * x, axis=-1, keepdims=True)",
     "ms = np.sum(x * x, axis=-1, keepdims=True)"),
    ("RMSNorm eps dropped", "np.sqrt(ms + float(eps))", "np.sqrt(ms)"),
    ("rotary offset ignored", "int(token_pos[t]) + int(rotary_offset)", "int(token_pos[t])"),
    ("bf16 decode without the shift", "bits = np.asarray(x, dtype=np.uint16).astype(np.uint32) << 16",
     "bits = np.asarray(x, dtype=np.uint16).astype(np.uint32)"),
    ("bf16 decode shifted by 15", "bits = np.asarray(x, dtype=np.uint16).astype(np.uint32) << 16",
     "bits = np.asarray(x, dtype=np.uint16).astype(np.uint32) << 15"),
    ("bf16 bits read as float16", "return bits.view(np.float32).astype(np.float64)",
     "return np.asarray(x, dtype=np.uint16).view(np.float16).astype(np.float64)"),
    ("topk ties keep the higher index", "key=lambda j: (-row[j], j)", "key=lambda j: (-row[j], -j)"),
    ("topk bound exclusive", "for j in range(last + 1) if not", "for j in range(last) if not"),
    ("topk -inf eligible", "not math.isnan(row[j]) and row[j] != -math.inf]", "not math.isnan(row[j])]"),
    ("topk kept in rank order", "kept = sorted(ranked[:top_k])", "kept = ranked[:top_k]"),
    ("topk padded with zeros", "out = np.full((R, H, sel_width), -1, dtype=np.int32)",
     "out = np.full((R, H, sel_width), 0, dtype=np.int32)"),
    ("topk smallest scores", "ranked = sorted(eligible, key=lambda j: (-row[j], j))",
     "ranked = sorted(eligible, key=lambda j: (row[j], j))"),
    ("shard range inclusive of hi", "(main_pos < int(kv_range[b][1]))]", "(main_pos <= int(kv_range[b][1]))]"),
    ("merge drops the sink", "L = math.exp(sink - M) + sum(w)", "L = sum(w)"),
    ("merge counts the sink per shard", "L = math.exp(sink - M) + sum(w)", "L = R * math.exp(sink - M) + sum(w)"),
    ("merge lse without log L", "lse[t, h] = M + math.log(L)", "lse[t, h] = M"),
    ("merge ignores the sink in the max", "M = max([sink] + [float(lses[r, t, h]) for r in range(R)])",
     "M = max([float(lses[r, t, h]) for r in range(R)])"),
    ("bf16 ties away from even", "(((c >> 16) & 1) == 0) & (((best >> 16) & 1) == 1)",
     "(((c >> 16) & 1) == 1) & (((best >> 16) & 1) == 0)"),
]


def _mutant(orig, new):
    src = inspect.getsource(spa_oracle)
    assert src.count(orig) >= 1, orig
    mod = types.ModuleType("spa_oracle_mutant")
    exec(compile(src.replace(orig, new), "spa_oracle_mutant", "exec"), mod.__dict__)
    return mod


def _pin_cases():
    cases = []
    for name, fn in inspect.getmembers(pins, inspect.isfunction):
        if not name.startswith("test_"):
            continue
        marks = getattr(fn, "pytestmark", [])
        params = [m for m in marks if m.name == "parametrize"]
        if params:
            argname, values = params[0].args
            for v in values:
                cases.append((fn, {argname: v}))
        else:
            cases.append((fn, {}))
    return cases


@pytest.mark.parametrize("desc,orig,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_mistake_is_caught(desc, orig, new, monkeypatch):
    mod = _mutant(orig, new)
    monkeypatch.setattr(pins, "O", mod)
    failed = []
    for fn, kw in _pin_cases():
        try:
            fn(**kw)
        except Exception:
            failed.append(fn.__name__)
    assert failed, f"no pin caught the planted mistake: {desc}"
