"""Plant plausible mistakes in a copy of the oracle and check the pins catch each.

The copy is built from the oracle's source text with one edit applied and run
on the CPU; the real oracle is never modified.
"""
import inspect
import types

import pytest

from oracle import misa_oracle
import tests.test_oracle_dosa as dosa_pins
import tests.test_oracle_pins as pins

MUTATIONS = {
    "score_without_relu": ("I += w[j] * np.maximum(A[r], 0.0)", "I += w[j] * A[r]"),
    "router_signed_w": ("return np.abs(w64) * A.sum(axis=1)", "return w64 * A.sum(axis=1)"),
    "router_without_relu": ("A = np.maximum(head_token_scores(q, pooled, range(q.shape[0]), counter), 0.0)",
                            "A = head_token_scores(q, pooled, range(q.shape[0]), counter)"),
    "pool_divides_by_B": ("out[m] = blk.sum(axis=0) / blk.shape[0]", "out[m] = blk.sum(axis=0) / B"),
    "pool_full_block_tail": ("blk = K[m * B:min((m + 1) * B, L)]", "blk = K[m * B:(m + 1) * B]"),
    "topk_ties_to_high_index": ("order = np.lexsort((idx, -I))", "order = np.lexsort((-idx, -I))"),
    "toph_ties_to_high_index": ("order = np.lexsort((np.arange(r.shape[0]), -r))",
                                "order = np.lexsort((-np.arange(r.shape[0]), -r))"),
    "prefix_excludes_query": ("I = index_scores(q, w, K[:L_i], heads, counter)",
                              "I = index_scores(q, w, K[:L_i - 1], heads, counter)"),
    "e4m3_wrong_bias": ("* 2.0 ** (e - 7)", "* 2.0 ** (e - 8)"),
    "fp8_scale_dropped": ("return decode_e4m3(keys) * np.asarray(scale, dtype=np.float64)[:, None]",
                          "return decode_e4m3(keys)"),
    "rerank_ties_by_position": ("topk=top_k(I, k, index=c))", "topk=top_k(I, k))"),
    "weights_not_per_head": ("I += w[j] * np.maximum", "I += w[0] * np.maximum"),
    "dense_misses_a_head": ("I = index_scores(q, w, K[:L_i], range(q.shape[0]), counter)",
                            "I = index_scores(q, w, K[:L_i], range(q.shape[0] - 1), counter)"),
}

# the certified pruning of the dense indexer, against its own pins
DOSA_MUTATIONS = {
    "dosa_residual_sign": ("U += w[j] * max(a + qn[j] * rho, 0.0)", "U += w[j] * max(a - qn[j] * rho, 0.0)"),
    "dosa_negative_heads_upper": ("U += w[j] * max(a - qn[j] * rho, 0.0)",
                                  "U += w[j] * max(a + qn[j] * rho, 0.0)"),
    "dosa_negative_heads_dropped": ("U += w[j] * max(a - qn[j] * rho, 0.0)", "U += 0.0"),
    "dosa_prunes_at_equality": ("pruned = U < tau", "pruned = U <= tau"),
    "dosa_threshold_from_top_seed": ("[::-1][k - 1])", "[::-1][0])"),
    "dosa_radius_from_first_token": ("rho = float(np.sqrt(np.sum((Kb - c) ** 2, axis=1)).max())",
                                     "rho = float(np.sqrt(np.sum((Kb[0] - c) ** 2)))"),
}

PIN_TESTS = [(n, f) for n, f in inspect.getmembers(pins, inspect.isfunction) if n.startswith("test_")]
DOSA_PIN_TESTS = [(n, f) for n, f in inspect.getmembers(dosa_pins, inspect.isfunction)
                  if n.startswith("test_") and n != "test_certificate_on_the_workloads"]


def _mutant(src_from, src_to):
    src = inspect.getsource(misa_oracle)
    assert src.count(src_from) >= 1, src_from
    mod = types.ModuleType("misa_oracle_mutant")
    exec(compile(src.replace(src_from, src_to), "misa_oracle_mutant", "exec"), mod.__dict__)
    return mod


def _params(fn):
    marks = getattr(fn, "pytestmark", [])
    for m in marks:
        if m.name == "parametrize":
            names = [s.strip() for s in m.args[0].split(",")]
            for vals in m.args[1]:
                vals = vals if isinstance(vals, tuple) else (vals,)
                yield dict(zip(names, vals))
            return
    yield {}


def _caught(tests):
    caught = []
    for tname, fn in tests:
        for kw in _params(fn):
            try:
                fn(**kw)
            except Exception:
                caught.append(tname)
                break
        if caught:
            break
    return caught


@pytest.mark.parametrize("name", sorted(DOSA_MUTATIONS))
def test_dosa_pins_catch_mutation(name, monkeypatch):
    monkeypatch.setattr(dosa_pins, "O", _mutant(*DOSA_MUTATIONS[name]))
    assert _caught(DOSA_PIN_TESTS), f"no pin caught mutation {name}"


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_mutation(name, monkeypatch):
    monkeypatch.setattr(pins, "O", _mutant(*MUTATIONS[name]))
    caught = []
    for tname, fn in PIN_TESTS:
        for kw in _params(fn):
            try:
                fn(**kw)
            except Exception:
                caught.append(tname)
                break
        if caught:
            break
    assert caught, f"no pin caught mutation {name}"
