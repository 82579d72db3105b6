"""Pins for the CPU oracle: each check is fixed by something other than the
oracle itself (hand-worked values, a brute-force token-level formula, an
independent dense attention, invariants), chosen so that a dropped term, a
wrong sign or index, or a transposed operand in the oracle fails one of them.
"""
import json
import math
import os

import numpy as np
import pytest

from oracle import dhsa
from long_context_prefill_dhsa_b200 import inputs as I

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
D = 128


def _one_chunk_layout(n):
    off = np.array([[0, n]], dtype=np.int32)
    return off, np.array([1], dtype=np.int32)


# ------------------------------------------------------------ pooling
def _hand_rows(kind, n):
    X = np.zeros((n, D))
    if kind == "ones":
        X[:] = 1.0
    elif kind == "const3":
        X[:] = 3.0
    elif kind == "const_m05":
        X[:] = -0.5
    elif kind == "ramp_e0":
        X[:, 0] = np.arange(1, n + 1)
    elif kind == "single":
        X[0, :3] = [0.5, -1.25, 3.0]
    return X


def test_pool_hand_cases():
    cases = json.load(open(os.path.join(GOLDEN, "pool_hand_cases.json")))["cases"]
    for c in cases:
        X = _hand_rows(c["rows"], c["n"])[None, None]
        off, nc = _one_chunk_layout(c["n"])
        p = dhsa.chunk_pool(X, off, nc, 1)[0, 0, 0]
        if "expect_all" in c:
            np.testing.assert_allclose(p, c["expect_all"], rtol=0, atol=1e-12, err_msg=c["name"])
        if "expect_dim0" in c:
            assert abs(p[0] - c["expect_dim0"]) < 1e-12, c["name"]
            np.testing.assert_allclose(p[1:], c["expect_rest"], atol=1e-12)
        if "expect_row" in c:
            exp = np.zeros(D)
            exp[:3] = c["expect_row"]
            np.testing.assert_allclose(p, exp, atol=1e-12, err_msg=c["name"])


def test_pool_concat_two_equal_chunks():
    # pooling a chunk made of two equal-length halves = (p1 + p2) / sqrt(2)
    rng = np.random.default_rng(1)
    n = 7
    X = rng.standard_normal((1, 1, 2 * n, D))
    off2 = np.array([[0, n, 2 * n]], dtype=np.int32)
    p12 = dhsa.chunk_pool(X, off2, np.array([2], dtype=np.int32), 2)[0, 0]
    pall = dhsa.chunk_pool(X, np.array([[0, 2 * n]], dtype=np.int32), np.array([1], dtype=np.int32), 1)[0, 0, 0]
    np.testing.assert_allclose(pall, (p12[0] + p12[1]) / math.sqrt(2), rtol=1e-12, atol=1e-12)


def test_pool_padded_rows_zero_and_multi_batch():
    rng = np.random.default_rng(2)
    X = rng.standard_normal((2, 3, 10, D))
    off = np.array([[0, 3, 10, 10], [0, 1, 4, 10]], dtype=np.int32)
    nc = np.array([2, 3], dtype=np.int32)
    P = dhsa.chunk_pool(X, off, nc, 3)
    assert np.all(P[0, :, 2] == 0)
    # b=1, chunk 2 = rows 4..9 (6 rows), by hand: column sums / sqrt(6)
    np.testing.assert_allclose(P[1, 2, 2], X[1, 2, 4:10].sum(0) / math.sqrt(6), rtol=1e-12)


# ------------------------------------------------------------ selection
def _brute_block_select(Q, K, c, m, k):
    """Equal chunks of c rows: block score from token-level dot products
    sum_{t in i} sum_{s in j} q_t . k_s / c, ranked with Python's sort by
    (-score, j); returns a token-level causal keep mask."""
    T = Q @ K.T
    L = Q.shape[0]
    M = np.zeros((L, L), dtype=bool)
    for i in range(m):
        scores = []
        for j in range(i):
            blk = T[i * c:(i + 1) * c, j * c:(j + 1) * c].sum() / c
            scores.append((-blk, j))
        kept = [j for _, j in sorted(scores)[:k]] + [i]
        for j in kept:
            M[i * c:(i + 1) * c, j * c:(j + 1) * c] = True
    return M & np.tril(np.ones((L, L), dtype=bool))


@pytest.mark.parametrize("c,m,k,G", [(4, 12, 3, 1), (8, 9, 2, 2), (5, 16, 5, 4), (3, 10, 0, 1)])
def test_select_matches_bruteforce_block_mask(c, m, k, G):
    rng = np.random.default_rng(100 + c * m + k)
    L = c * m
    Hkv = 2
    Hq = Hkv * G
    Q = rng.standard_normal((1, Hq, L, D))
    K = rng.standard_normal((1, Hkv, L, D))
    off = (np.arange(m + 1, dtype=np.int32) * c)[None]
    nc = np.array([m], dtype=np.int32)
    _, _, S, sel = dhsa.routing(Q, K, off, nc, k)
    for hq in range(Hq):
        want = _brute_block_select(Q[0, hq], K[0, hq // G], c, m, k)
        got = dhsa.token_keep_mask(sel[0][hq], off[0], m, L)
        assert np.array_equal(got, want), (hq, c, m, k)


def test_select_ties_go_to_lower_index():
    # chunks 1 and 2 have identical K rows, so S[3,1] == S[3,2]; with k = 1
    # the lower index (1) must win. Chunk 0's keys are the negation, so its
    # score is the negative of the tied value.
    c = 4
    rng = np.random.default_rng(5)
    K = np.zeros((1, 1, 4 * c, D))
    base = rng.standard_normal((c, D))
    K[0, 0, 0:c] = -base
    K[0, 0, c:2 * c] = base
    K[0, 0, 2 * c:3 * c] = base
    K[0, 0, 3 * c:4 * c] = rng.standard_normal((c, D))
    Q = np.zeros((1, 1, 4 * c, D))
    Q[0, 0, 3 * c:] = base.sum(0) / 10.0          # makes S[3,1] = S[3,2] > 0
    off = (np.arange(5, dtype=np.int32) * c)[None]
    nc = np.array([4], dtype=np.int32)
    _, _, S, sel = dhsa.routing(Q, K, off, nc, 1)
    assert S[0, 0, 3, 1] == S[0, 0, 3, 2] and S[0, 0, 3, 1] > 0
    assert list(sel[0][0][3]) == [1, 3]
    _, _, S, sel = dhsa.routing(Q, K, off, nc, 2)
    assert list(sel[0][0][3]) == [1, 2, 3]


def test_select_edges():
    rng = np.random.default_rng(7)
    S = rng.standard_normal((1, 1, 10, 10))
    nc = np.array([10], dtype=np.int32)
    sel = dhsa.select(S, nc, 4)[0][0]
    for i in range(5):                       # i <= k: every earlier chunk kept
        assert list(sel[i]) == list(range(i + 1))
    sel0 = dhsa.select(S, nc, 0)[0][0]
    for i in range(10):                      # k = 0: diagonal only
        assert list(sel0[i]) == [i]
    # hand-ranked row: scores for j < 6, k = 2 -> j = 4 (9.0) and 1 (7.0)
    row = np.full(10, np.nan)
    row[:6] = [1.0, 7.0, -3.0, 2.0, 9.0, 7.0 - 1e-9]
    assert list(dhsa.select_row(row, 6, 2)) == [1, 4, 6]
    assert abs(dhsa.tie_gap(row, 6, 2) - 1e-9) < 1e-15
    assert dhsa.near_tie(row, 6, 2) and not dhsa.near_tie(row, 6, 1)


def test_csr_by_hand():
    off = np.array([[0, 2, 5, 6]], dtype=np.int32)      # lengths 2, 3, 1
    nc = np.array([3], dtype=np.int32)
    sel = [[[np.array([0]), np.array([0, 1]), np.array([1, 2])]]]
    rp, ci, cost = dhsa.block_csr(sel, off, nc, 4)
    assert list(rp) == [0, 1, 3, 5, 5]
    assert list(ci) == [0, 0, 1, 1, 2]
    # cost = n_i * sum n_j: 2*2, 3*(2+3), 1*(3+1), padded 0
    assert list(cost) == [4, 15, 4, 0]


def test_kept_pairs_by_hand():
    off = np.array([[0, 2, 5, 6]], dtype=np.int32)
    nc = np.array([3], dtype=np.int32)
    sel = [[[np.array([0]), np.array([0, 1]), np.array([1, 2])]]]
    # chunk 0: 2*3/2 = 3; chunk 1: 3*2 + 3*4/2 = 12; chunk 2: 1*3 + 1 = 4
    assert dhsa.kept_pairs(off, nc, sel)[0, 0] == 19
    M = dhsa.token_keep_mask(sel[0][0], off[0], 3, 6)
    assert M.sum() == 19


# ------------------------------------------------------------ attention
def _rand_qkv(rng, B, Hq, Hkv, L):
    return (rng.standard_normal((B, Hq, L, D)), rng.standard_normal((B, Hkv, L, D)),
            rng.standard_normal((B, Hkv, L, D)))


def test_attn_k_all_equals_dense():
    rng = np.random.default_rng(11)
    w = I.custom(B=2, Hq=4, Hkv=2, L=150, lo=1, hi=20, k=1000)
    off, nc = I.offsets(w)
    Q, K, V = _rand_qkv(rng, 2, 4, 2, 150)
    Q *= 2.0                                   # sharper softmax
    _, _, _, sel = dhsa.routing(Q, K, off, nc, 1000)
    O = dhsa.attn_sparse(Q, K, V, off, nc, sel)
    Od = dhsa.attn_dense(Q, K, V)
    assert np.max(np.abs(O - Od)) < 1e-10


def test_attn_k0_is_per_chunk_causal():
    rng = np.random.default_rng(12)
    w = I.custom(B=1, Hq=2, Hkv=1, L=90, lo=3, hi=17, k=0)
    off, nc = I.offsets(w)
    Q, K, V = _rand_qkv(rng, 1, 2, 1, 90)
    _, _, _, sel = dhsa.routing(Q, K, off, nc, 0)
    O = dhsa.attn_sparse(Q, K, V, off, nc, sel)
    for c in range(int(nc[0])):
        s, e = int(off[0, c]), int(off[0, c + 1])
        Oc = dhsa.attn_dense(Q[:, :, s:e], K[:, :, s:e], V[:, :, s:e])
        assert np.max(np.abs(O[:, :, s:e] - Oc)) < 1e-12


def test_attn_matches_explicit_token_mask():
    # textbook masked softmax over the explicit L x L keep mask
    rng = np.random.default_rng(13)
    w = I.custom(B=1, Hq=4, Hkv=2, L=200, lo=1, hi=30, k=3)
    off, nc = I.offsets(w)
    Q, K, V = _rand_qkv(rng, 1, 4, 2, 200)
    _, _, _, sel = dhsa.routing(Q, K, off, nc, 3)
    O = dhsa.attn_sparse(Q, K, V, off, nc, sel)
    n = int(nc[0])
    for hq in range(4):
        M = dhsa.token_keep_mask(sel[0][hq], off[0], n, 200)
        s = (Q[0, hq] @ K[0, hq // 2].T) / math.sqrt(D)
        s = np.where(M, s, -np.inf)
        p = np.exp(s - s.max(1, keepdims=True))
        ref = (p / p.sum(1, keepdims=True)) @ V[0, hq // 2]
        assert np.max(np.abs(O[0, hq] - ref)) < 1e-12


def test_attn_single_token_and_convexity():
    rng = np.random.default_rng(14)
    Q, K, V = _rand_qkv(rng, 1, 2, 1, 1)
    off = np.array([[0, 1]], dtype=np.int32)
    nc = np.array([1], dtype=np.int32)
    sel = [[[np.array([0])], [np.array([0])]]]
    O = dhsa.attn_sparse(Q, K, V, off, nc, sel)
    np.testing.assert_allclose(O[0, 0, 0], V[0, 0, 0], rtol=0, atol=1e-15)
    # each output row is a convex combination of the kept V rows
    w = I.custom(B=1, Hq=2, Hkv=1, L=120, lo=1, hi=25, k=2)
    off, nc = I.offsets(w)
    Q, K, V = _rand_qkv(rng, 1, 2, 1, 120)
    _, _, _, sel = dhsa.routing(Q, K, off, nc, 2)
    O = dhsa.attn_sparse(Q, K, V, off, nc, sel)
    for i in range(int(nc[0])):
        rows = np.concatenate([np.arange(off[0, j], off[0, j + 1]) for j in sel[0][0][i]])
        s, e = off[0, i], off[0, i + 1]
        for t in range(s, e):
            vis = rows[rows <= t]
            assert np.all(O[0, 0, t] <= V[0, 0, vis].max(0) + 1e-12)
            assert np.all(O[0, 0, t] >= V[0, 0, vis].min(0) - 1e-12)


# ------------------------------------------------------------ inputs + invariants
def test_inputs_layout():
    for name, w in I.WORKLOADS.items():
        off, nc = I.offsets(w)
        for b in range(w.B):
            n = int(nc[b])
            lens = np.diff(off[b, : n + 1])
            assert off[b, 0] == 0 and off[b, n] == w.L and lens.min() >= 1
            assert np.all(off[b, n:] == w.L)
            assert lens[:-1].min() >= w.length_lo and lens.max() <= w.length_hi


def test_bf16_rounding_recipe():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 3.140625], dtype=np.float32)
    # ties to even: 1 + 2^-8 -> 1.0; 1 + 3*2^-8 -> 1 + 2^-6 (= 1.015625)
    back = I.bf16_bits_to_f32(I.f32_to_bf16_bits(x))
    assert list(back) == [1.0, 1.0, 1.015625, -2.5, 3.140625]


def test_needles_recovered_small():
    # a planted K chunk mean 3x a later query chunk's mean must be selected
    w = I.custom(B=1, Hq=4, Hkv=2, L=6000, lo=16, hi=160, kind="uniform", k=6,
                 needles_per_head=4, wid=200)
    d = I.make_inputs(w, with_v=False)
    Q, K = dhsa.bf16_to_f64(d["Q"]), dhsa.bf16_to_f64(d["K"])
    _, _, _, sel = dhsa.routing(Q, K, d["off"], d["n_chunks"], w.k)
    for (hq, i, j) in d["needles"][0]:
        assert j in sel[0][hq][i], (hq, i, j)


@pytest.mark.slow
def test_needles_recovered_ragged_workload_sampled():
    # the ragged 64K workload, kv head 0 and its query heads, both batches
    w = I.WORKLOADS["ragged-64k"]
    heads = list(range(w.G))
    d = I.make_inputs(w, heads_q=heads, heads_kv=[0], with_v=False)
    off, nc = d["off"], d["n_chunks"]
    nmax = off.shape[1] - 1
    Qp = dhsa.chunk_pool(dhsa.bf16_to_f64(d["Q"][:, :w.G]), off, nc, nmax)
    Kp = dhsa.chunk_pool(dhsa.bf16_to_f64(d["K"][:, :1]), off, nc, nmax)
    S = dhsa.chunk_scores(Qp, Kp, nc)
    sel = dhsa.select(S, nc, w.k)
    total = hit = 0
    for b in range(w.B):
        for (hq, i, j) in d["needles"][b]:
            if hq < w.G:
                total += 1
                hit += j in sel[b][hq][i]
    assert total == w.G * w.needles_per_head * w.B
    assert hit == total, (hit, total)


@pytest.mark.slow
def test_frozen_k_for_8k_workload():
    from oracle import freeze_k
    w = I.WORKLOADS["qwen3b-8k"]
    off, nc, S = freeze_k.pooled_scores(w, I)
    assert freeze_k.density_for_k(S, off, nc, w.k, w.L) >= w.target_density
    assert freeze_k.density_for_k(S, off, nc, w.k - 1, w.L) < w.target_density


# ---------------------------------------------------------------- row budgets
def test_budget_hand_cases():
    g = json.load(open(os.path.join(GOLDEN, "budget_hand_cases.json")))
    S = np.array(g["row"]["S"])
    lens = np.array(g["row"]["lens"])
    i = g["row"]["i"]
    for c in g["cases"]:
        got = dhsa.select_budget_row(S, lens, i, c["budget"], c["recent"], c["k_max"])
        assert got.tolist() == c["expect"], c


@pytest.mark.parametrize("seed", range(4))
def test_budget_reduces_to_topk(seed):
    # a budget no row can fill, no window: the top-k_max rule (pinned above
    # against the brute-force token-level block score)
    rng = np.random.default_rng(seed)
    n = 40
    lens = rng.integers(1, 50, n)
    for i in range(n):
        S = rng.standard_normal(n)
        S[rng.integers(0, n, 5)] = 0.25          # a few exact ties
        for k_max in (0, 1, 3, 7, 50):
            got = dhsa.select_budget_row(S, lens, i, 10 ** 9, 0, k_max)
            assert got.tolist() == dhsa.select_row(S, i, k_max).tolist()


def test_budget_uniform_lengths_is_topk_of_budget_over_length():
    rng = np.random.default_rng(7)
    n, ln = 30, 16
    lens = np.full(n, ln)
    for i in range(n):
        S = rng.standard_normal(n)
        for m in range(0, 8):
            for extra in (0, 1, ln - 1):          # budgets m*ln - extra .. round up to m chunks
                budget = m * ln - extra if m > 0 else 0
                want = dhsa.select_row(S, i, m)
                got = dhsa.select_budget_row(S, lens, i, budget, 0, 100)
                assert got.tolist() == want.tolist(), (i, m, extra)


def test_budget_zero_keeps_recent_window_only():
    S = np.linspace(1.0, -1.0, 20)
    lens = np.arange(1, 21)
    for i in range(20):
        for r in (0, 1, 3, 25):
            got = dhsa.select_budget_row(S, lens, i, 0, r, 100)
            assert got.tolist() == list(range(max(0, i - r), i)) + [i]


def test_budget_invariants_random():
    rng = np.random.default_rng(11)
    n = 60
    for trial in range(30):
        lens = rng.integers(1, 80, n)
        S = rng.standard_normal(n)
        i = int(rng.integers(0, n))
        r = int(rng.integers(0, 5))
        k_max = int(rng.integers(0, 20))
        prev = None
        for budget in (0, 10, 50, 200, 800, 10 ** 6):
            kept = dhsa.select_budget_row(S, lens, i, budget, r, k_max)
            assert kept[-1] == i and np.all(np.diff(kept) > 0)
            earlier = kept[:-1]
            assert len(earlier) <= max(k_max, 0)
            rr = min(r, i, k_max)
            assert set(range(i - rr, i)) <= set(earlier.tolist())
            ranked = [j for j in earlier if j < i - rr]
            used = int(lens[i - rr:i].sum()) + int(sum(int(lens[j]) for j in ranked))
            # the ranked picks are a prefix of the (score desc, index asc) order
            order = np.argsort(-S[: i - rr], kind="stable")
            t = len(ranked)
            assert sorted(order[:t].tolist()) == ranked
            # stopping rule: below the budget before the last pick; when the fill
            # stopped early, the budget was met or the cap reached
            if t:
                assert used - int(lens[order[t - 1]]) < budget
            if t < i - rr and len(earlier) < k_max:
                assert used >= budget
            if prev is not None:                     # monotone in the budget
                assert set(prev.tolist()) <= set(kept.tolist())
            prev = kept


def test_budget_vector_matches_per_row_scalar():
    rng = np.random.default_rng(3)
    B, Hq, n = 2, 3, 12
    off = np.zeros((B, n + 1), dtype=np.int64)
    for b in range(B):
        off[b, 1:] = np.cumsum(rng.integers(1, 9, n))
    S = rng.standard_normal((B, Hq, n, n))
    budgets = rng.integers(0, 30, (B, Hq, n))
    sel = dhsa.select_budget(S, off, np.array([n, n]), budgets, 1, 5)
    for b in range(B):
        lens = np.diff(off[b])
        for hq in range(Hq):
            for i in range(n):
                want = dhsa.select_budget_row(S[b, hq, i], lens, i, int(budgets[b, hq, i]), 1, 5)
                assert sel[b][hq][i].tolist() == want.tolist()


def test_budget_near_tie_hand_cases():
    g = json.load(open(os.path.join(GOLDEN, "budget_near_tie_cases.json")))
    lens = np.array(g["lens"])
    for c in g["cases"]:
        got = dhsa.budget_near_tie(np.array(c["S"]), lens, g["i"], c["budget"], c["recent"], c["k_max"])
        assert got == c["expect"], c["name"]


# ------------------------------------------------------------ density, bf16 upcast
def test_density_by_hand():
    # the 6-token layout of test_kept_pairs_by_hand: causal pairs 6*7/2 = 21
    off = np.array([[0, 2, 5, 6]], dtype=np.int32)
    nc = np.array([3], dtype=np.int32)
    sel_a = [np.array([0]), np.array([0, 1]), np.array([1, 2])]        # 19 kept pairs
    sel_b = [np.array([0]), np.array([1]), np.array([2])]              # 3 + 6 + 1 = 10
    assert dhsa.density(off, nc, [[sel_a]], 6) == 19 / 21
    # two heads average: (19 + 10) / 2 over 21
    assert dhsa.density(off, nc, [[sel_a, sel_b]], 6) == 14.5 / 21


def test_bf16_upcast_bit_patterns():
    bits = np.array([0x3F80, 0xC020, 0x0001, 0xFF80, 0x7F80, 0x8000, 0x4049, 0x7F7F, 0x0080, 0x3F81],
                    dtype=np.uint16)
    want = [1.0, -2.5, 2.0 ** -133, -math.inf, math.inf, -0.0, 3.140625, (2 - 2 ** -7) * 2.0 ** 127,
            2.0 ** -126, 1 + 2 ** -7]
    got = dhsa.bf16_to_f64(bits)
    assert got.dtype == np.float64
    assert got.tolist() == want
    assert math.copysign(1.0, got[5]) == -1.0             # the sign of -0 survives
    # a quiet NaN pattern stays NaN
    assert math.isnan(dhsa.bf16_to_f64(np.array([0x7FC0], dtype=np.uint16))[0])
