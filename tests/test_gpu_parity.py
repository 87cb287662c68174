"""GPU parity: every entry point of libmisa against the CPU oracle.

Inputs come from the seeded generator; expected values from the oracle only
(the oracle's head sets and candidate lists feed the GPU calls that take
them).  Sizes span several tiles with ragged tails; ragged sequence lengths,
tiny prefixes, k >= L and h = H_I are covered.
"""
import numpy as np
import pytest
import torch

from long_context_misa_b200 import inputs as G
from long_context_misa_b200 import misa as M
from oracle import misa_oracle as O
from tests.parity import assert_close, compare_selection, to_device

pytestmark = pytest.mark.gpu

W = G.WORKLOADS
CASES = {
    "bf16_normal": W["tiny_decode"].scaled(L=1000, k=50),
    "bf16_mixture": W["batched_decode"].scaled(n_seq=3, L=2500, B=64, k=100),
    "fp8_mixture": W["misa_dagger_decode_128k"].scaled(n_seq=3, L=3001, B=128, k=64, k_prime=300),
    "bf16_prefill": W["causal_prefill"].scaled(L=1500, n_q=70, k=64),
    "fp8_prefill_h32": W["long_prefill_128k"].scaled(L=2100, n_q=40, B=100, k=33),
    # few long rows: the top-k goes through the compact boundary-bin list
    "fp8_long": W["misa_dagger_decode_128k"].scaled(n_seq=2, L=40000, B=128, k=600, k_prime=4000),
    # 96 heads: dense decode on 128 tensor-core columns, 32 of them zero-weight
    # padding, one-tile chunks
    "fp8_h96": W["misa_dagger_decode_128k"].scaled(n_seq=2, L=2999, H=96, k=64, k_prime=300),
    # prefill chunks of >= 64 queries score on the tcgen05 tensor-core path
    "fp8_prefill_umma": W["long_prefill_128k"].scaled(L=3000, n_q=96, B=100, k=33),
    # query groups that span two sequences (two passes over different keys)
    "bf16_prefill_2seq": W["causal_prefill"].scaled(n_seq=2, L=1300, n_q=80, k=40),
    # score rows whose pitch is not a multiple of 16 bytes (plain stores, no
    # TMA store) and a last query group cut short by n_q
    "bf16_prefill_odd": W["causal_prefill"].scaled(L=1501, n_q=100, k=37),
}


def make(case, seed=0, ragged=True):
    """Inputs of a named case, or of a Workload given directly."""
    wl = CASES[case] if isinstance(case, str) else case
    inp = G.make_inputs(wl, seed)
    if isinstance(case, str) and case.endswith("_2seq"):  # blocks of 20 queries alternate between the sequences
        inp.q_seq = ((np.arange(wl.n_q) // 20) % 2).astype(np.int32)
    if ragged and wl.mode == "decode":
        inp.seq_len = (wl.L - 37 * np.arange(wl.n_seq)).astype(np.int32)
        inp.q_pos = (inp.seq_len - 1).astype(np.int32)
    return inp


class Ref:
    """Oracle views of one input set."""

    def __init__(self, inp):
        self.inp, self.wl = inp, inp.wl
        self.K = [O.seq_keys(inp.keys, inp.scale, self.wl.key_dtype, s) for s in range(self.wl.n_seq)]

    def query(self, i):
        q, w = O.query_arrays(self.inp.q, self.inp.w, i)
        s = int(self.inp.q_seq[i])
        return q, w, self.K[s], int(self.inp.q_pos[i]) + 1


def device_status(cache):
    torch.cuda.synchronize()
    return cache.device_status()


@pytest.mark.parametrize("case", sorted(CASES))
def test_pool_rebuild(case):
    inp = make(case)
    ref = Ref(inp)
    cache, _ = to_device(inp, torch)
    M.pool_keys(cache)
    pool = cache.pool.cpu().numpy()
    for s in range(inp.wl.n_seq):
        n = int(inp.seq_len[s])
        expect = O.pool_keys(ref.K[s], n, inp.wl.B)
        assert_close(pool[s, :expect.shape[0]], expect, f"pool seq {s}")
    assert device_status(cache) == 0


@pytest.mark.parametrize("case", ["bf16_mixture", "fp8_mixture"])
@pytest.mark.parametrize("count", [1, 37, 200])
def test_pool_append(case, count):
    inp = make(case)
    wl = inp.wl
    full_len = inp.seq_len.copy()
    start = (full_len - count).astype(np.int32)
    inp_short = make(case)
    inp_short.seq_len = start.copy()
    cache, _ = to_device(inp_short, torch)
    M.pool_keys(cache)                                    # pool of the shorter prefix
    new = np.stack([inp.keys[s, start[s]:start[s] + count] for s in range(wl.n_seq)])
    nk = torch.from_numpy(new.view(np.int16) if new.dtype == np.uint16 else new).cuda().contiguous()
    ns = None
    if inp.scale is not None:
        ns = torch.from_numpy(np.stack([inp.scale[s, start[s]:start[s] + count] for s in range(wl.n_seq)])).cuda()
    # overwrite the cache tail with garbage first so the append must write it
    for s in range(wl.n_seq):
        cache.keys[s, start[s]:start[s] + count] = 0
    pos = torch.from_numpy(start).cuda()
    M.pool_keys(cache, nk, ns, pos)
    M.pool_keys(cache, nk, ns, pos)                       # idempotent
    assert np.array_equal(cache.seq_len.cpu().numpy(), full_len)
    keys = cache.keys.cpu().numpy()
    ref = Ref(inp)
    for s in range(wl.n_seq):
        n = int(full_len[s])
        assert np.array_equal(keys[s, :n].view(inp.keys.dtype), inp.keys[s, :n])
        expect = O.pool_keys(ref.K[s], n, wl.B)
        assert_close(cache.pool[s, :expect.shape[0]].cpu().numpy(), expect, f"pool after append seq {s}")
    assert device_status(cache) == 0


@pytest.mark.parametrize("count", [1, 7, 64])
def test_append_keys_e4m3(count):
    # bf16 keys quantised to e4m3 with one scale per token on the way into the
    # cache: codes and scales bit-exact against the oracle's encoder, block
    # means within tolerance of the oracle's pool of the updated cache
    inp = make("fp8_mixture")
    wl = inp.wl
    rng = np.random.default_rng(11 + count)
    x = (rng.standard_normal((wl.n_seq, count, 128)) * rng.uniform(0.01, 100.0, (wl.n_seq, count, 1))).astype(np.float32)
    x[0, 0] = 0.0                                          # a zero row: scale 1, codes 0
    x[1, 0, :64] = -0.0                                    # negative zeros keep their sign
    x[1, 0, 64:] = rng.standard_normal(64).astype(np.float32) * 1e-3   # values that land in the subnormal range
    x[2, count - 1] *= 1e6                                 # large magnitudes
    bits = (x.view(np.uint32) >> 16).astype(np.uint16)
    L = inp.seq_len.astype(np.int64)
    pos = np.array([100, int(L[1]) - count, -1], dtype=np.int32)   # middle, the end, untouched
    cache, _ = to_device(inp, torch)
    M.pool_keys(cache)
    M.append_keys_e4m3(cache, torch.from_numpy(bits.view(np.int16)).cuda().contiguous(),
                       torch.from_numpy(pos).cuda())
    codes, scale = O.quantize_key_rows(bits)
    keys = cache.keys.cpu().numpy()
    sc = cache.scale.cpu().numpy()
    seq_len = cache.seq_len.cpu().numpy()
    new_keys, new_scale = inp.keys.copy(), inp.scale.copy()
    for s in range(wl.n_seq):
        if pos[s] < 0:
            assert seq_len[s] == L[s]
            assert np.array_equal(keys[s], inp.keys[s]) and np.array_equal(sc[s], inp.scale[s])
            continue
        p0 = int(pos[s])
        assert seq_len[s] == p0 + count
        np.testing.assert_array_equal(keys[s, p0:p0 + count], codes[s], err_msg=f"codes seq {s}")
        np.testing.assert_array_equal(sc[s, p0:p0 + count], scale[s], err_msg=f"scales seq {s}")
        new_keys[s, p0:p0 + count], new_scale[s, p0:p0 + count] = codes[s], scale[s]
    pool = cache.pool.cpu().numpy()
    for s in range(wl.n_seq):
        n = int(seq_len[s])
        expect = O.pool_keys(O.seq_keys(new_keys, new_scale, "fp8", s, n), n, wl.B)
        assert_close(pool[s, :expect.shape[0]], expect, f"pool after quantised append seq {s}")
    assert device_status(cache) == 0


def test_pool_append_past_capacity_is_flagged():
    inp = make("bf16_mixture")
    cache, _ = to_device(inp, torch)
    M.pool_keys(cache)
    before = cache.seq_len.clone()
    nk = torch.zeros(inp.wl.n_seq, 4, 128, dtype=torch.int16, device="cuda")
    pos = torch.full((inp.wl.n_seq,), inp.wl.L - 2, dtype=torch.int32, device="cuda")
    M.pool_keys(cache, nk, None, pos)
    assert device_status(cache) & M.DEV_APPEND_RANGE
    assert torch.equal(cache.seq_len, before)


@pytest.mark.parametrize("case", sorted(CASES))
@pytest.mark.parametrize("h", [1, 8, "H"])
def test_route_heads(case, h):
    inp = make(case)
    ref = Ref(inp)
    wl = inp.wl
    h = wl.H if h == "H" else h
    cache, qs = to_device(inp, torch)
    M.pool_keys(cache)
    r_gpu = torch.empty(wl.n_q, wl.H, dtype=torch.float32, device="cuda")
    heads = M.route_heads(cache, qs, h, router_scores=r_gpu).cpu().numpy()
    r_gpu = r_gpu.cpu().numpy()
    ties = 0
    for i in range(wl.n_q):
        q, w, K, Li = ref.query(i)
        r, hs = O.route_query(q, w, K, Li, wl.B, h)
        assert_close(r_gpu[i], r, f"router scores q{i}")
        assert np.all(np.diff(heads[i]) > 0)               # ascending, distinct
        ties += compare_selection(heads[i], hs, lambda j: r[j], h, f"heads q{i}")
    assert ties <= max(1, wl.n_q // 10), f"{ties} head boundary ties"
    assert device_status(cache) == 0


# routing cases for the aggregation variants: the decode router, the tcgen05
# router with its finish fused (64 and 32 heads, one and two sequences per
# group) and with the separate finishing kernel (24 heads do not divide 128)
AGG_CASES = {
    "bf16_mixture": None,
    "bf16_prefill": None,
    "fp8_prefill_umma": None,
    "bf16_prefill_2seq": None,
    "prefill_h24": W["causal_prefill"].scaled(L=1500, n_q=70, H=24, k=64),
}


@pytest.mark.parametrize("case", sorted(AGG_CASES))
@pytest.mark.parametrize("agg", [M.AGG_SIGNED_SUM, M.AGG_SUM, M.AGG_ABS_MAX])
def test_route_heads_aggregations(case, agg):
    inp = make(AGG_CASES[case] or case)
    ref = Ref(inp)
    wl = inp.wl
    cache, qs = to_device(inp, torch)
    M.pool_keys(cache)
    r_gpu = torch.empty(wl.n_q, wl.H, dtype=torch.float32, device="cuda")
    heads = M.route_heads(cache, qs, wl.h, router_scores=r_gpu, agg=agg).cpu().numpy()
    r_gpu = r_gpu.cpu().numpy()
    ties = 0
    for i in range(wl.n_q):
        q, w, K, Li = ref.query(i)
        r, hs = O.route_query(q, w, K, Li, wl.B, wl.h, agg=agg)
        assert_close(r_gpu[i], r, f"router scores q{i} agg {agg}")
        assert np.all(np.diff(heads[i]) > 0)
        ties += compare_selection(heads[i], hs, lambda j: r[j], wl.h, f"heads q{i} agg {agg}")
    assert ties <= max(1, wl.n_q // 10), f"{ties} head boundary ties"
    assert device_status(cache) == 0


def _score_case(case, kind, k=None, h=None, seed=0):
    inp = make(case, seed)
    ref = Ref(inp)
    wl = inp.wl
    k = wl.k if k is None else k
    h = wl.h if h is None else h
    cache, qs = to_device(inp, torch)
    scores = torch.full((wl.n_q, wl.L), float("nan"), dtype=torch.float32, device="cuda")
    exp = []
    if kind == "misa":
        heads_ref = []
        for i in range(wl.n_q):
            q, w, K, Li = ref.query(i)
            heads_ref.append(O.route_query(q, w, K, Li, wl.B, h)[1])
        heads_dev = torch.from_numpy(np.stack(heads_ref).astype(np.int32)).cuda()
        top = M.score_topk(cache, qs, heads_dev, k, scores_out=scores).cpu().numpy()
        for i in range(wl.n_q):
            q, w, K, Li = ref.query(i)
            I = O.index_scores(q, w, K[:Li], heads_ref[i])
            exp.append((I, O.top_k(I, k), Li))
    else:
        top = M.dense_score_topk(cache, qs, k, scores_out=scores).cpu().numpy()
        for i in range(wl.n_q):
            q, w, K, Li = ref.query(i)
            d = O.dense_query(q, w, K, Li, k)
            exp.append((d["scores"], d["topk"], Li))
    sc = scores.cpu().numpy()
    ties = 0
    for i, (I, tk, Li) in enumerate(exp):
        assert_close(sc[i, :Li], I, f"{kind} scores q{i}")
        ties += compare_selection(top[i], tk, lambda t: I[t], k, f"{kind} top-k q{i}")
        got = top[i][top[i] >= 0]
        assert np.all(np.diff(got) > 0)                    # ascending, distinct
        assert np.all(top[i][len(got):] == -1) and len(got) == min(k, Li)
    assert device_status(cache) == 0
    return ties


@pytest.mark.parametrize("case", sorted(CASES))
@pytest.mark.parametrize("kind", ["misa", "dense"])
def test_score_topk(case, kind):
    ties = _score_case(case, kind)
    assert ties <= 4, ties


@pytest.mark.parametrize("k", [1, 7, 999, 5000])
def test_score_topk_k_edges(k):
    _score_case("bf16_mixture", "misa", k=k)


@pytest.mark.parametrize("case", ["bf16_mixture", "fp8_mixture"])
def test_misa_all_heads_equals_dense(case):
    # structural reduction (h = H_I routes every head) holds on the GPU path too
    inp = make(case)
    wl = inp.wl
    cache, qs = to_device(inp, torch)
    heads = torch.arange(wl.H, dtype=torch.int32, device="cuda").repeat(wl.n_q, 1).contiguous()
    s1 = torch.empty(wl.n_q, wl.L, device="cuda")
    s2 = torch.empty(wl.n_q, wl.L, device="cuda")
    a = M.score_topk(cache, qs, heads, wl.k, scores_out=s1)
    b = M.dense_score_topk(cache, qs, wl.k, scores_out=s2)
    assert torch.equal(a, b)


@pytest.mark.parametrize("case", sorted(CASES))
def test_rerank(case):
    inp = make(case)
    ref = Ref(inp)
    wl = inp.wl
    kp = wl.k_prime or 4 * wl.k
    cache, qs = to_device(inp, torch)
    cands, fine = [], []
    for i in range(wl.n_q):
        q, w, K, Li = ref.query(i)
        c = O.misa_query(q, w, K, Li, wl.B, wl.h, kp)["topk"]
        cands.append(c)
        fine.append(O.rerank_query(q, w, K, c, wl.k))
    cand_dev = torch.from_numpy(np.stack(cands)).cuda()
    sc = torch.full((wl.n_q, kp), float("nan"), device="cuda")
    top = M.rerank_topk(cache, qs, cand_dev, wl.k, scores_out=sc).cpu().numpy()
    sc = sc.cpu().numpy()
    ties = 0
    for i in range(wl.n_q):
        valid = cands[i] >= 0
        assert_close(sc[i][valid], fine[i]["scores"], f"rerank scores q{i}")
        smap = dict(zip(fine[i]["cand"].tolist(), fine[i]["scores"].tolist()))
        ties += compare_selection(top[i], fine[i]["topk"], lambda t: smap[t], wl.k, f"rerank q{i}")
    assert ties <= 4
    assert device_status(cache) == 0


def _large_kprime_case():
    """Two queries re-ranking k' = 20000 candidates: rows too long to stage in
    shared memory, so the selection sweeps them from global memory."""
    wl = W["misa_dagger_decode_128k"].scaled(n_seq=2, L=40000, B=128, k=1500, k_prime=20000)
    inp = make(wl, seed=3)
    ref = Ref(inp)
    rng = np.random.default_rng(21)
    cands = []
    for i in range(wl.n_q):
        Li = int(inp.q_pos[i]) + 1
        c = rng.choice(Li, size=wl.k_prime, replace=False).astype(np.int32)
        c[:5] = -1                                         # ignored entries
        cands.append(c)
    return inp, ref, wl, np.stack(cands)


def check_rerank_against_oracle(ref, wl, cands, top, sc=None):
    ties = 0
    for i in range(wl.n_q):
        q, w, K, Li = ref.query(i)
        f = O.rerank_query(q, w, K, cands[i], wl.k)
        smap = dict(zip(f["cand"].tolist(), f["scores"].tolist()))
        if sc is not None:
            valid = cands[i] >= 0
            assert_close(sc[i][valid], f["scores"], f"rerank scores q{i}")
        ties += compare_selection(top[i], f["topk"], lambda t: smap[t], wl.k, f"rerank q{i}")
        got = top[i][top[i] >= 0]
        assert np.all(np.diff(got) > 0) and len(got) == min(wl.k, int((cands[i] >= 0).sum()))
    return ties


def test_rerank_k_prime_above_16k():
    inp, ref, wl, cands = _large_kprime_case()
    cache, qs = to_device(inp, torch)
    sc = torch.full((wl.n_q, wl.k_prime), float("nan"), device="cuda")
    top = M.rerank_topk(cache, qs, torch.from_numpy(cands).cuda(), wl.k, scores_out=sc).cpu().numpy()
    ties = check_rerank_against_oracle(ref, wl, cands, top, sc.cpu().numpy())
    top2 = M.rerank_topk(cache, qs, torch.from_numpy(cands).cuda(), wl.k).cpu().numpy()  # scores in the workspace
    np.testing.assert_array_equal(top, top2)
    print(f"\nrerank k'=20000: {ties} boundary ties")
    assert ties <= 2
    assert device_status(cache) == 0


def test_rerank_with_all_candidates_is_dense():
    inp = make("bf16_mixture")
    wl = inp.wl
    cache, qs = to_device(inp, torch)
    L = int(inp.seq_len.max())
    cand = np.full((wl.n_q, L), -1, dtype=np.int32)
    for i in range(wl.n_q):
        n = int(inp.q_pos[i]) + 1
        cand[i, :n] = np.arange(n)
    a = M.rerank_topk(cache, qs, torch.from_numpy(cand).cuda(), wl.k)
    b = M.dense_score_topk(cache, qs, wl.k)
    assert torch.equal(a, b)


def test_tiny_prefixes_and_bad_positions():
    wl = CASES["bf16_prefill"].scaled(L=300, n_q=8, B=64, k=70)
    inp = G.make_inputs(wl, 3)
    inp.q_pos = np.array([0, 1, 62, 63, 64, 65, 299, 299], dtype=np.int32)
    ref = Ref(inp)
    cache, qs = to_device(inp, torch)
    M.pool_keys(cache)
    heads = M.route_heads(cache, qs, 4)
    top = M.dense_score_topk(cache, qs, wl.k).cpu().numpy()
    for i in range(wl.n_q):
        q, w, K, Li = ref.query(i)
        d = O.dense_query(q, w, K, Li, wl.k)
        compare_selection(top[i], d["topk"], lambda t: d["scores"][t], wl.k, f"q{i}")
    assert device_status(cache) == 0
    # a query past its sequence is clamped and flagged
    qs.q_pos[0] = 10_000
    M.dense_score_topk(cache, qs, wl.k)
    assert device_status(cache) & M.DEV_BAD_POSITION


def test_empty_query_batch():
    inp = make("bf16_mixture")
    cache, _ = to_device(inp, torch)
    e = torch.empty(0, 64, 128, dtype=torch.int16, device="cuda")
    qs = M.Queries(e, torch.empty(0, 64, device="cuda"), torch.empty(0, dtype=torch.int32, device="cuda"),
                   torch.empty(0, dtype=torch.int32, device="cuda"))
    assert M.dense_score_topk(cache, qs, 16).shape == (0, 16)


def test_needles_selected_by_dense_gpu():
    inp = make("bf16_mixture", ragged=False)
    cache, qs = to_device(inp, torch)
    top = M.dense_score_topk(cache, qs, inp.wl.k).cpu().numpy()
    for s, p, qi in inp.needles:
        assert p in set(top[qi].tolist())


def _tied_case(L, pattern, k):
    """bf16 cache whose keys take two values (pattern[t] = 0 or 1), so that
    scores tie massively; expected top-k from the oracle (ties to the lower
    token index)."""
    wl = W["batched_decode"].scaled(n_seq=2, L=L, B=128, k=k)
    inp = G.make_inputs(wl, 4)
    a, b = inp.keys[0, 0].copy(), inp.keys[0, 1].copy()
    for s_ in range(wl.n_seq):
        inp.keys[s_] = np.where(pattern[:, None] == 1, b[None, :], a[None, :])
    ref = Ref(inp)
    cache, qs = to_device(inp, torch)
    top = M.dense_score_topk(cache, qs, k).cpu().numpy()
    for i in range(wl.n_q):
        q, w, K, Li = ref.query(i)
        d = O.dense_query(q, w, K, Li, k)
        np.testing.assert_array_equal(top[i], d["topk"], err_msg=f"q{i}")
    assert device_status(cache) == 0


@pytest.mark.parametrize("L", [3000, 40000])
@pytest.mark.parametrize("k", [1, 100, 2999])
def test_topk_all_scores_equal(L, k):
    # one boundary bin holds every element: ties decide (listed refinement for
    # short rows, whole-row passes when the bin is too large to list)
    _tied_case(L, np.zeros(L, dtype=np.int64), k)


@pytest.mark.parametrize("L", [3000, 40000])
def test_topk_two_score_levels(L):
    # half the tokens share one score, half another: k equal to one half takes
    # a whole bin; k a little larger cuts into the other half by index
    pat = (np.arange(L) % 2).astype(np.int64)
    for k in (L // 2, L // 2 + 37):
        _tied_case(L, pat, k)


# Prefill chunks over caches longer than 16K keys: tensor-core scoring, then
# a sampled lower bound of each row's boundary bin, the elements above it
# listed and selected; every query is checked.
LONG_PREFILL = {
    "bf16": W["causal_prefill"].scaled(L=20000, n_q=64, k=300),
    "fp8": W["long_prefill_128k"].scaled(L=24000, n_q=72, B=256, k=500),
}


@pytest.mark.parametrize("dt", sorted(LONG_PREFILL))
@pytest.mark.parametrize("kind", ["misa", "dense"])
def test_long_prefill_topk(dt, kind):
    ties = _score_case(LONG_PREFILL[dt], kind)
    assert ties <= 4, ties


def _tied_prefill(L, pattern, k):
    """Prefill chunk over a bf16 cache whose keys take two values: the sampled
    bound lists far more than a row holds, so every row falls back to counting
    its whole score row; expected top-k from the oracle (ties to the lower
    token index)."""
    wl = W["causal_prefill"].scaled(L=L, n_q=64, k=k)
    inp = G.make_inputs(wl, 5)
    a, b = inp.keys[0, 0].copy(), inp.keys[0, 1].copy()
    inp.keys[0] = np.where(pattern[:, None] == 1, b[None, :], a[None, :])
    ref = Ref(inp)
    cache, qs = to_device(inp, torch)
    top = M.dense_score_topk(cache, qs, k).cpu().numpy()
    for i in range(wl.n_q):
        q, w, K, Li = ref.query(i)
        d = O.dense_query(q, w, K, Li, k)
        np.testing.assert_array_equal(top[i], d["topk"], err_msg=f"q{i}")
    assert device_status(cache) == 0


@pytest.mark.parametrize("k", [1, 700])
def test_long_prefill_topk_all_scores_equal(k):
    _tied_prefill(20000, np.zeros(20000, dtype=np.int64), k)


def test_long_prefill_topk_two_score_levels():
    L = 20000
    pat = (np.arange(L) % 2).astype(np.int64)
    _tied_prefill(L, pat, 8000)  # inside the upper level: ties by index


def test_rerank_candidate_order_does_not_matter():
    # outputs are token indices in ascending order whatever the candidate
    # order, and the selection is the oracle's (ties to the lower token)
    inp = make("fp8_long")
    ref = Ref(inp)
    wl = inp.wl
    kp = wl.k_prime
    rng = np.random.default_rng(9)
    cache, qs = to_device(inp, torch)
    cands = []
    for i in range(wl.n_q):
        Li = int(inp.q_pos[i]) + 1
        cands.append(rng.choice(Li, size=kp, replace=False).astype(np.int32))
    c_sorted = torch.from_numpy(np.sort(np.stack(cands), axis=1)).cuda()
    c_shuf = torch.from_numpy(np.stack(cands)).cuda()
    a = M.rerank_topk(cache, qs, c_sorted, wl.k).cpu().numpy()
    b = M.rerank_topk(cache, qs, c_shuf, wl.k).cpu().numpy()
    np.testing.assert_array_equal(a, b)
    for i in range(wl.n_q):
        q, w, K, Li = ref.query(i)
        f = O.rerank_query(q, w, K, cands[i], wl.k)
        smap = dict(zip(f["cand"].tolist(), f["scores"].tolist()))
        compare_selection(b[i], f["topk"], lambda t: smap[t], wl.k, f"q{i}")
        got = b[i][b[i] >= 0]
        assert np.all(np.diff(got) > 0)


def _decode_step_inputs(inp):
    """The cache one token short of every sequence's length, and that token's
    key (and scale) to append at its position."""
    wl = inp.wl
    pos = (inp.seq_len - 1).astype(np.int32)
    last = np.stack([inp.keys[s, pos[s]:pos[s] + 1] for s in range(wl.n_seq)])
    nk = torch.from_numpy(last.view(np.int16) if last.dtype == np.uint16 else last).cuda().contiguous()
    ns = None
    if inp.scale is not None:
        ns = torch.from_numpy(np.stack([inp.scale[s, pos[s]:pos[s] + 1] for s in range(wl.n_seq)])).cuda()
    return nk, ns, torch.from_numpy(pos).cuda()


@pytest.mark.parametrize("case", ["fp8_mixture", "fp8_long", "bf16_mixture", "fp8_h96", "bf16_normal",
                                  "bf16_prefill", "fp8_prefill_umma"])
def test_dagger_decode_step(case):
    # append + route + MISA-dagger in one call: the appended cache and pool
    # are the oracle's, the heads are the oracle's up to boundary ties, and
    # the final top-k is what misa_dagger_topk returns with those heads (that
    # call is checked against the oracle by the composition and re-rank
    # tests).  Decode cases route inside the scoring kernel; prefill chunks
    # run the three calls in sequence.
    inp = make(case)
    ref = Ref(inp)
    wl = inp.wl
    kp = wl.k_prime or 4 * wl.k
    cache, qs = to_device(inp, torch)
    cache.seq_len.copy_(torch.from_numpy(inp.seq_len - 1))
    M.pool_keys(cache)
    nk, ns, pos = _decode_step_inputs(inp)
    heads = torch.full((wl.n_q, wl.h), -7, dtype=torch.int32, device="cuda")
    top = M.dagger_decode(cache, qs, nk, ns, pos, wl.h, kp, wl.k, heads=heads).cpu().numpy()
    assert np.array_equal(cache.seq_len.cpu().numpy(), inp.seq_len)
    pool = cache.pool.cpu().numpy()
    for s_ in range(wl.n_seq):
        expect = O.pool_keys(ref.K[s_], int(inp.seq_len[s_]), wl.B)
        assert_close(pool[s_, :expect.shape[0]], expect, f"pool seq {s_}")
    hd = heads.cpu().numpy()
    ties = 0
    for i in range(wl.n_q):
        q, w, K, Li = ref.query(i)
        r, hs = O.route_query(q, w, K, Li, wl.B, wl.h)
        assert np.all(np.diff(hd[i]) > 0), hd[i]
        ties += compare_selection(hd[i], hs, lambda j: r[j], wl.h, f"heads q{i}")
        got = top[i][top[i] >= 0]
        assert np.all(np.diff(got) > 0) and len(got) == min(wl.k, Li)
    assert ties <= max(1, wl.n_q // 10), f"{ties} head boundary ties"
    again = M.dagger_topk(cache, qs, heads, kp, wl.k).cpu().numpy()
    np.testing.assert_array_equal(top, again)
    # without the heads output, and a second step at the same positions
    top2 = M.dagger_decode(cache, qs, nk, ns, pos, wl.h, kp, wl.k).cpu().numpy()
    np.testing.assert_array_equal(top, top2)
    assert device_status(cache) == 0


@pytest.mark.parametrize("period,k_prime,k", [(37, 1000, 300), (5, 3000, 700)])
def test_dagger_decode_step_tied_scores(period, k_prime, k):
    # every sequence repeats `period` distinct keys, so scores come in tied
    # groups: the routed top-k' boundary falls inside a group that the
    # scoring kernel hands to the re-rank kernel (a few hundred to a few
    # thousand tokens), and the final top-k ties too.  Checked against the
    # oracle with the heads the step chose.
    wl = W["misa_dagger_decode_128k"].scaled(n_seq=3, L=20000, B=128, k=k, k_prime=k_prime)
    inp = G.make_inputs(wl, 5)
    t = np.arange(wl.L)
    inp.keys[:] = inp.keys[:, t % period]
    inp.scale[:] = inp.scale[:, t % period]
    ref = Ref(inp)
    cache, qs = to_device(inp, torch)
    cache.seq_len.copy_(torch.from_numpy(inp.seq_len - 1))
    M.pool_keys(cache)
    nk, ns, pos = _decode_step_inputs(inp)
    heads = torch.empty(wl.n_q, wl.h, dtype=torch.int32, device="cuda")
    top = M.dagger_decode(cache, qs, nk, ns, pos, wl.h, k_prime, k, heads=heads).cpu().numpy()
    hd = heads.cpu().numpy()
    for i in range(wl.n_q):
        q, w, K, Li = ref.query(i)
        cand = O.top_k(O.index_scores(q, w, K[:Li], hd[i]), k_prime)
        expect = O.rerank_query(q, w, K, cand, k)["topk"]
        np.testing.assert_array_equal(top[i], expect, err_msg=f"query {i}")
    again = M.dagger_topk(cache, qs, heads, k_prime, k).cpu().numpy()
    np.testing.assert_array_equal(top, again)
    assert device_status(cache) == 0


# Final sequence lengths, tokens appended per sequence, the sequences not
# appended to (new_pos -1), the query rows' sequences and (None: each row's
# last token) their positions, per layout.
APPEND_LAYOUTS = {
    "block_end": ([1024, 2432, 8960, 640], 1, (), (0, 1, 2, 3), None),      # the append completes a block
    "block_start": ([1025, 2433, 8961, 129], 1, (), (0, 1, 2, 3), None),    # the append opens a block
    "span": ([1025, 2434, 8962, 130], 3, (), (0, 1, 2, 3), None),           # three keys over a block boundary
    "skip": ([3000, 5000, 7000, 8999], 1, (1,), (0, 1, 2, 3), None),        # one sequence not appended to
    "permuted": ([4096, 3001, 6000, 8192], 1, (), (2, 0, 3, 1), None),      # rows on other rows' sequences
    # two rows per sequence: one at the appended token, one whose prefix ends
    # before it (in the same block, and at the end of the full block before)
    "shared": ([5000, 7681], 1, (), (0, 0, 1, 1), (4999, 4995, 7680, 7679)),
}


@pytest.mark.parametrize("dtype", ["fp8", "bf16"])
@pytest.mark.parametrize("layout", sorted(APPEND_LAYOUTS))
def test_dagger_decode_step_append_layouts(layout, dtype):
    # The routed pass routes while the append kernel may still run: the
    # appended keys of a query's last (cut) block come from the append's
    # input, and a CTA whose block means the append rewrites waits for it.
    # The cache rows the append fills hold zeros before the step, and each
    # appended key copies the query's best dense token, so a read of the
    # rows before the append lands changes the selection.  Checked against
    # the oracle with the heads the step chose; the pool and lengths after
    # the step against the oracle's.
    lens, count, skipped, rows, qpos = APPEND_LAYOUTS[layout]
    base = W["misa_dagger_decode_128k"] if dtype == "fp8" else W["batched_decode"]
    # a batch with rows != sequences is drawn as a prefill chunk, then laid out here
    wl = base.scaled(n_seq=len(lens), n_q=len(rows), L=9000, B=128, k=256, k_prime=2048,
                     mode=base.mode if len(rows) == len(lens) else "prefill")
    inp = G.make_inputs(wl, 21)
    lens = np.array(lens, dtype=np.int32)
    inp.seq_len[:] = lens
    inp.q_seq[:] = np.array(rows, dtype=np.int32)
    inp.q_pos[:] = lens[inp.q_seq] - 1 if qpos is None else np.array(qpos, dtype=np.int32)
    pos = np.where(np.isin(np.arange(wl.n_seq), skipped), -1, lens - count).astype(np.int32)
    ref0 = Ref(inp)
    for i in range(wl.n_q):  # the appended keys copy the query's best dense token before them
        s_ = int(inp.q_seq[i])
        if pos[s_] < 0:
            continue
        q, w, K, _ = ref0.query(i)
        best = int(np.argmax(O.index_scores(q, w, K[:pos[s_]], range(wl.H))))
        inp.keys[s_, pos[s_]:pos[s_] + count] = inp.keys[s_, best]
        if inp.scale is not None:
            inp.scale[s_, pos[s_]:pos[s_] + count] = inp.scale[s_, best]
    ref = Ref(inp)
    nk = np.stack([inp.keys[s_, max(p, 0):max(p, 0) + count] for s_, p in enumerate(pos)])
    nk = torch.from_numpy(nk.view(np.int16) if nk.dtype == np.uint16 else nk).cuda().contiguous()
    ns = None
    if inp.scale is not None:
        ns = torch.from_numpy(np.stack([inp.scale[s_, max(p, 0):max(p, 0) + count] for s_, p in enumerate(pos)])).cuda()
    cache, qs = to_device(inp, torch)
    short = np.where(pos >= 0, pos, lens).astype(np.int32)
    cache.seq_len.copy_(torch.from_numpy(short))
    for s_, p in enumerate(pos):  # the rows the append fills hold zeros until it does
        if p >= 0:
            cache.keys.view(torch.uint8)[s_, p:p + count] = 0
            if cache.scale is not None:
                cache.scale[s_, p:p + count] = 0
    M.pool_keys(cache)
    heads = torch.empty(wl.n_q, wl.h, dtype=torch.int32, device="cuda")
    top = M.dagger_decode(cache, qs, nk, ns, torch.from_numpy(pos).cuda(), wl.h, wl.k_prime, wl.k,
                          heads=heads).cpu().numpy()
    assert np.array_equal(cache.seq_len.cpu().numpy(), lens)
    pool = cache.pool.cpu().numpy()
    for s_ in range(wl.n_seq):
        expect = O.pool_keys(ref.K[s_], int(lens[s_]), wl.B)
        assert_close(pool[s_, :expect.shape[0]], expect, f"pool seq {s_}")
    hd = heads.cpu().numpy()
    ties = 0
    for i in range(wl.n_q):
        q, w, K, Li = ref.query(i)
        r, hs = O.route_query(q, w, K, Li, wl.B, wl.h)
        ties += compare_selection(hd[i], hs, lambda j: r[j], wl.h, f"heads q{i}")
        cand = O.top_k(O.index_scores(q, w, K[:Li], hd[i]), wl.k_prime)
        expect = O.rerank_query(q, w, K, cand, wl.k)["topk"]
        np.testing.assert_array_equal(top[i], expect, err_msg=f"query {i}")
    assert ties <= 1, f"{ties} head boundary ties"
    assert device_status(cache) == 0


@pytest.mark.parametrize("case", ["fp8_mixture", "fp8_long", "bf16_mixture", "bf16_prefill", "fp8_prefill_umma"])
def test_dagger_topk_equals_composition(case):
    # one call (its k' candidates stay unordered inside) returns exactly what
    # the coarse stage followed by the fine stage returns; both stages are
    # checked against the oracle by test_score_topk and test_rerank
    inp = make(case)
    wl = inp.wl
    kp = wl.k_prime or 4 * wl.k
    cache, qs = to_device(inp, torch)
    M.pool_keys(cache)
    heads = M.route_heads(cache, qs, wl.h)
    cand = M.score_topk(cache, qs, heads, kp)
    two = M.rerank_topk(cache, qs, cand, wl.k).cpu().numpy()
    one = M.dagger_topk(cache, qs, heads, kp, wl.k).cpu().numpy()
    np.testing.assert_array_equal(one, two)
    for i in range(wl.n_q):
        got = one[i][one[i] >= 0]
        assert np.all(np.diff(got) > 0)
    assert device_status(cache) == 0
