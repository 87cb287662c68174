"""GPU parity at the five workloads' full sizes.

Every workload runs whole on the GPU (all queries, full L); the oracle then
recomputes queries one by one: every query of the decode workloads, and 32
queries spread evenly over each prefill chunk (so over its query groups of
the tensor-core path) plus every needle's target query.  The MISA-dagger
decode runs as the captured decode step (append + route + routed top-k' +
re-rank in one call), the launch configuration the throughput measurement
replays.

Checks per sampled query (tolerances as in the smaller parity tests):
router scores within tolerance and head set equal up to boundary ties; the
routed per-token scores, computed with the GPU's head set, within tolerance
over the whole prefix; the routed top-k (k' for MISA-dagger) equal up to
boundary ties; dense DSA scores and top-k the same way; for MISA-dagger the
step's final top-k equal to the oracle's re-rank of the GPU's candidates up
to boundary ties; the routed and dense top-k of the call without scores_out
(scores in the workspace) equal to those with it on every query.
The boundary-tie counts are printed per workload.
"""
import numpy as np
import pytest
import torch

from long_context_misa_b200 import inputs as G
from long_context_misa_b200 import misa as M
from oracle import misa_oracle as O
from tests.parity import assert_close, compare_selection, to_device

pytestmark = pytest.mark.gpu


def _sample(inp):
    wl = inp.wl
    if wl.mode == "decode":
        return list(range(wl.n_q))
    picks = np.linspace(0, wl.n_q - 1, 32).astype(int).tolist() + [qi for (_, _, qi) in inp.needles]
    return sorted(set(picks))


def _ascending_valid(row, Li, k):
    got = row[row >= 0]
    assert np.all(np.diff(got) > 0)
    assert len(got) == min(k, Li) and np.all(row[len(got):] == -1)
    assert got.size == 0 or (got[0] >= 0 and got[-1] < Li)


@pytest.mark.parametrize("name", sorted(G.WORKLOADS))
def test_full_size_sampled(name):
    wl = G.WORKLOADS[name]
    inp = G.make_inputs(wl, 0)
    cache, qs = to_device(inp, torch)
    k_route = wl.k_prime or wl.k
    ties = {"heads": 0, "routed": 0, "dense": 0, "final": 0}

    if wl.k_prime:
        # the decode step as measured: the cache starts one token short and the
        # step appends each query's own key before routing
        cache.seq_len.copy_(torch.from_numpy(inp.seq_len - 1))
        M.pool_keys(cache)
        last = np.stack([inp.keys[s, inp.q_pos[s]:inp.q_pos[s] + 1] for s in range(wl.n_seq)])
        sc = np.stack([inp.scale[s, inp.q_pos[s]:inp.q_pos[s] + 1] for s in range(wl.n_seq)])
        step = M.MisaDaggerDecode(cache, qs, wl.h, wl.k_prime, wl.k, torch.from_numpy(last).cuda(),
                                  torch.from_numpy(sc).cuda(), torch.from_numpy(inp.q_pos.copy()).cuda())
        step.run()
        torch.cuda.synchronize()
        step_heads = step.heads.cpu().numpy()
        # restore the short cache and replay the captured step: same result
        first = step.topk.clone()
        cache.seq_len.copy_(torch.from_numpy(inp.seq_len - 1))
        step.capture()
        cache.seq_len.copy_(torch.from_numpy(inp.seq_len - 1))
        step.replay()
        torch.cuda.synchronize()
        assert torch.equal(cache.seq_len.cpu(), torch.from_numpy(inp.seq_len))
        final = step.topk.cpu().numpy()
        assert np.array_equal(final, first.cpu().numpy())
    else:
        M.pool_keys(cache)

    r_gpu = torch.empty(wl.n_q, wl.H, dtype=torch.float32, device="cuda")
    heads = M.route_heads(cache, qs, wl.h, router_scores=r_gpu)
    routed = torch.empty(wl.n_q, wl.L, dtype=torch.float32, device="cuda")
    top = M.score_topk(cache, qs, heads, k_route, scores_out=routed)
    # without scores_out (the call the throughput figures time) the scores
    # live in the workspace: every row's selection is the same
    top_ws = M.score_topk(cache, qs, heads, k_route)
    assert torch.equal(top_ws, top), f"{name}: routed top-k without scores_out differs"
    heads, r_gpu, top = heads.cpu().numpy(), r_gpu.cpu().numpy(), top.cpu().numpy()
    picks = _sample(inp)
    routed_rows = routed[picks].cpu().numpy()
    del routed
    dense = torch.empty(wl.n_q, wl.L, dtype=torch.float32, device="cuda")
    dtop_t = M.dense_score_topk(cache, qs, wl.k, scores_out=dense)
    assert torch.equal(M.dense_score_topk(cache, qs, wl.k), dtop_t), f"{name}: dense top-k without scores_out differs"
    dtop = dtop_t.cpu().numpy()
    dense_rows = dense[picks].cpu().numpy()
    del dense
    torch.cuda.synchronize()
    assert cache.device_status() == 0

    K_by_seq = {}
    for j, i in enumerate(picks):
        s = int(inp.q_seq[i])
        Li = int(inp.q_pos[i]) + 1
        if s not in K_by_seq:
            K_by_seq = {s: O.seq_keys(inp.keys, inp.scale, wl.key_dtype, s)}
        K = K_by_seq[s]
        q, w = O.query_arrays(inp.q, inp.w, i)
        tag = f"{name} q{i}"

        r, hs = O.route_query(q, w, K, Li, wl.B, wl.h)
        assert_close(r_gpu[i], r, f"{tag} router scores")
        assert np.all(np.diff(heads[i]) > 0)
        ties["heads"] += compare_selection(heads[i], hs, lambda t: r[t], wl.h, f"{tag} heads")
        if wl.k_prime:  # the decode step routes inside its scoring kernel
            assert np.all(np.diff(step_heads[i]) > 0)
            ties["heads"] += compare_selection(step_heads[i], hs, lambda t: r[t], wl.h, f"{tag} step heads")

        I = O.index_scores(q, w, K[:Li], heads[i])
        assert_close(routed_rows[j, :Li], I, f"{tag} routed scores")
        _ascending_valid(top[i], Li, k_route)
        ties["routed"] += compare_selection(top[i], O.top_k(I, k_route), lambda t: I[t], k_route,
                                            f"{tag} routed top-k")

        d = O.dense_query(q, w, K, Li, wl.k)
        assert_close(dense_rows[j, :Li], d["scores"], f"{tag} dense scores")
        _ascending_valid(dtop[i], Li, wl.k)
        ties["dense"] += compare_selection(dtop[i], d["topk"], lambda t: d["scores"][t], wl.k, f"{tag} dense top-k")

        if wl.k_prime and np.array_equal(step_heads[i], heads[i]):
            # the step's final top-k against the oracle's re-rank of the
            # candidates of the same heads (the separate call's)
            fine = O.rerank_query(q, w, K, top[i], wl.k)
            by_tok = dict(zip(fine["cand"].tolist(), fine["scores"].tolist()))
            _ascending_valid(final[i], Li, wl.k)
            assert set(final[i][final[i] >= 0].tolist()) <= set(top[i][top[i] >= 0].tolist())
            ties["final"] += compare_selection(final[i], fine["topk"], lambda t: by_tok[t], wl.k,
                                               f"{tag} MISA-dagger top-k")

    print(f"\n{name}: {len(picks)} queries checked against the oracle, boundary ties {ties}")
    n = len(picks)
    assert ties["heads"] <= n
    assert max(ties["routed"], ties["dense"], ties["final"]) <= 4 * n
    if wl.k_prime:  # near-tied head importances are rare: the step routed like the router
        assert sum(np.array_equal(step_heads[i], heads[i]) for i in picks) >= n - 1
