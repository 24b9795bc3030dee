"""Pins of the fp64 oracle to facts that do not come from the oracle itself.

Each test names what fixes the expected value: a special case that reduces to
textbook attention, a closed form, an invariant, a moment generating function,
or exhaustive enumeration on tiny inputs.
"""

import itertools
import json
import math
import os

import numpy as np
import pytest

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(rng, T, d, G, scale_k=1.0):
    K = rng.standard_normal((T, d)) * scale_k
    V = rng.standard_normal((T, d))
    q = rng.standard_normal((G, d))
    return q, K, V


CASES = [  # (T, S, W, Bk)
    (300, 4, 16, 8), (301, 4, 16, 8), (97, 0, 5, 7), (97, 3, 0, 4), (64, 4, 60, 4),
    (65, 4, 60, 4), (200, 1, 1, 1), (513, 16, 33, 32),
]


@pytest.mark.parametrize("T,S,W,Bk", CASES)
def test_all_blocks_selected_equals_full_softmax(T, S, W, Bk):
    """Selecting every block leaves no linearised token: the operator must be
    plain softmax attention over [0, T) (the exact/approximate split of SPLA's
    abstract with an empty approximate part)."""
    rng = np.random.default_rng(T * 7 + S)
    q, K, V = _rand(rng, T, 16, 3)
    scale = 1 / math.sqrt(16)
    part = O.partition(T, S, W, Bk)
    sel = np.arange(part.nb)
    ref = O.full_softmax(q, K, V, T, scale)
    np.testing.assert_allclose(O.hybrid_subtract(q, K, V, part, sel, scale), ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(O.hybrid_direct(q, K, V, part, sel, scale), ref, rtol=0, atol=1e-12)
    # through the stateful unit with k >= nb
    u = O.OracleUnit(K, V, S, W, Bk, k=part.nb + 3, scale=scale)
    out, s, _ = u.decode(q)
    assert list(s) == list(range(part.nb))
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("T", [1, 2, 50, 333])
def test_empty_exact_set_equals_pure_taylor(T):
    """No sinks, no window, k = 0: every token goes through exp(s) ~ 1 + s
    (SLAKE, PTAA), i.e. first-order Taylor attention over [0, T)."""
    rng = np.random.default_rng(T)
    q, K, V = _rand(rng, T, 8, 2, scale_k=0.3)
    scale = 1 / math.sqrt(8)
    part = O.partition(T, 0, 0, 5)
    ref = O.pure_taylor(q, K, V, T, scale)
    np.testing.assert_allclose(O.hybrid_subtract(q, K, V, part, [], scale), ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(O.hybrid_direct(q, K, V, part, [], scale), ref, rtol=0, atol=1e-12)
    u = O.OracleUnit(K, V, 0, 0, 5, k=0, scale=scale)
    np.testing.assert_allclose(u.decode(q)[0], ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("T,S,W,Bk", CASES)
def test_subtraction_form_equals_direct_sum(T, S, W, Bk):
    """SPLA's subtraction formulation (global minus selected) must equal the
    explicit sum over the unselected evicted tokens, for any selection."""
    rng = np.random.default_rng(1000 + T)
    q, K, V = _rand(rng, T, 12, 4)
    scale = 0.37
    part = O.partition(T, S, W, Bk)
    for trial in range(6):
        k = int(rng.integers(0, part.nb + 1)) if part.nb else 0
        sel = np.sort(rng.choice(part.nb, size=k, replace=False)) if k else np.array([], int)
        a = O.hybrid_subtract(q, K, V, part, sel, scale)
        b = O.hybrid_direct(q, K, V, part, sel, scale)
        np.testing.assert_allclose(a, b, rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("T,S,W,Bk", CASES)
def test_zero_query_gives_mean_value(T, S, W, Bk):
    """q = 0 makes every score 0, so exact weights e^0 and Taylor weights 1 + 0
    are all 1: the output is the mean of V over [0, T) for ANY selection."""
    rng = np.random.default_rng(5)
    _, K, V = _rand(rng, T, 6, 2)
    q = np.zeros((2, 6))
    part = O.partition(T, S, W, Bk)
    ref = V[:T].mean(axis=0)
    for k in (0, 1, part.nb):
        sel = np.arange(min(k, part.nb))
        for f in (O.hybrid_subtract, O.hybrid_direct):
            out = f(q, K, V, part, sel, 0.5)
            np.testing.assert_allclose(out, np.broadcast_to(ref, out.shape), rtol=0, atol=1e-12)


def test_brute_force_token_loop_agrees():
    """Token-by-token definition (pure Python loops, tiny sizes) against both
    vectorised forms, for random tiny configurations and selections."""
    rng = np.random.default_rng(77)
    for trial in range(40):
        T = int(rng.integers(1, 40))
        S = int(rng.integers(0, 5))
        W = int(rng.integers(0, 8))
        Bk = int(rng.integers(1, 6))
        G = int(rng.integers(1, 4))
        d = int(rng.integers(1, 5))
        q, K, V = _rand(rng, T, d, G)
        scale = float(rng.uniform(0.2, 1.0))
        part = O.partition(T, S, W, Bk)
        k = int(rng.integers(0, part.nb + 1)) if part.nb else 0
        sel = np.sort(rng.choice(part.nb, size=k, replace=False)) if k else np.array([], int)
        bf = O.brute_force_hybrid(q, K, V, T, S, W, Bk, sel, scale)
        np.testing.assert_allclose(O.hybrid_direct(q, K, V, part, sel, scale), bf, rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(O.hybrid_subtract(q, K, V, part, sel, scale), bf, rtol=1e-10, atol=1e-12)


def test_partition_by_enumeration():
    """Every position falls in exactly one of sink / window / one block, and the
    block sizes are Bk except possibly the newest one."""
    for T in range(0, 40):
        for S in range(0, 4):
            for W in range(0, 6):
                for Bk in (1, 3, 4):
                    p = O.partition(T, S, W, Bk)
                    owner = [None] * T
                    for t in range(*p.sink):
                        owner[t] = "s"
                    for t in range(*p.window):
                        assert owner[t] is None
                        owner[t] = "w"
                    for j, (a, b) in enumerate(p.blocks):
                        assert a == S + j * Bk and 0 < b - a <= Bk
                        assert b - a == Bk or j == p.nb - 1
                        for t in range(a, b):
                            assert owner[t] is None
                            owner[t] = j
                    assert all(o is not None for o in owner)
                    assert p.nb == max(0, -(-(T - S - W) // Bk))


def test_golden_closed_forms():
    """Hand-derived outputs (tests/golden/closed_form_small.json): with
    scale = ln 2 and integer keys, exp(s) is a power of two and 1 + s is
    1 + k ln 2, so the outputs are closed forms in ln 2."""
    with open(os.path.join(GOLDEN, "closed_form_small.json")) as f:
        g = json.load(f)
    for case in g["cases"]:
        K = np.array(case["K"], dtype=float)
        V = np.array(case["V"], dtype=float)
        q = np.array(case["q"], dtype=float)
        S, W, Bk, k = case["S"], case["W"], case["Bk"], case["top_k"]
        scale = math.log(2.0)
        expect = np.array([[eval(e, {"ln2": math.log(2.0)}) for e in row] for row in case["expected"]])
        u = O.OracleUnit(K, V, S, W, Bk, k=k, scale=scale)
        out, sel, scores = u.decode(q)
        assert list(sel) == case["expected_selection"]
        np.testing.assert_allclose(out, expect, rtol=0, atol=1e-13)


# ----------------------------------------------------------------------------- score

def test_score_identical_keys_is_plain_dot():
    """A block of identical keys has zero variance, so its score is exactly the
    group-summed q'.k (the Taylor expansion has no second-order term)."""
    rng = np.random.default_rng(3)
    k = rng.standard_normal(10)
    Kb = np.tile(k, (7, 1))
    part = O.partition(7 + 2, 2, 0, 7)
    K = np.vstack([rng.standard_normal((2, 10)), Kb])
    mu, var = O.block_stats(K, part)
    assert np.all(var < 1e-25)
    q = rng.standard_normal((3, 10))
    sc = O.block_scores(q, mu, var, 0.25)
    assert sc[0] == pytest.approx(float((q * 0.25).sum(axis=0) @ k), abs=1e-12)


@pytest.mark.parametrize("G", [1, 3])
def test_score_matches_gaussian_mgf(G):
    """For keys k ~ N(mu, diag(sigma^2)), E[exp(q'.k)] = exp(q'.mu + 1/2
    q'^T diag(sigma^2) q') (Gaussian moment generating function).  So the
    per-head score equals log of the sample mean of exp(q'.k) up to Monte Carlo
    error; the group score is the sum over heads.  A dropped 1/2, a wrong sign or
    a missing square would be off by ~0.25 here."""
    rng = np.random.default_rng(11 + G)
    d, n = 8, 400_000
    mu = rng.standard_normal(d) * 0.5
    sig = rng.uniform(0.3, 1.2, d)
    keys = mu + sig * rng.standard_normal((n, d))
    part = O.partition(n + 1, 1, 0, n)
    K = np.vstack([np.zeros((1, d)), keys])
    m_hat, v_hat = O.block_stats(K, part)
    q = rng.standard_normal((G, d)) * 0.6
    scale = 0.5
    score = O.block_scores(q, m_hat, v_hat, scale)[0]
    qs = q * scale
    mc = sum(math.log(np.mean(np.exp(keys @ qs[i]))) for i in range(G))
    second = 0.5 * float(((qs ** 2) @ (sig ** 2)).sum())
    assert second > 0.2                 # the second-order term is not negligible
    assert score == pytest.approx(mc, abs=2e-3 * G)


def test_score_is_second_order_accurate():
    """Scaling the within-block spread by eps, the score's gap to the exact
    log-mean-exp of the block must shrink like eps^3 (the expansion keeps the
    first and second cumulants).  A wrong second-order coefficient leaves an
    eps^2 gap: halving eps would then cut the gap by ~4x instead of ~8x.  The
    block's channels are made exactly uncorrelated (orthogonal, zero-mean
    columns) so that its covariance is the diagonal the score uses."""
    rng = np.random.default_rng(21)
    d, c = 6, 64
    mu = rng.standard_normal(d)
    A = np.hstack([np.ones((c, 1)), rng.standard_normal((c, d))])
    Q, _ = np.linalg.qr(A)
    z = Q[:, 1:] * math.sqrt(c) * rng.uniform(0.5, 2.0, d)
    q = rng.standard_normal((1, d))
    gaps = []
    for eps in (0.2, 0.1, 0.05):
        keys = mu + eps * z
        part = O.partition(c, 0, 0, c)
        m_hat, v_hat = O.block_stats(keys, part)
        score = O.block_scores(q, m_hat, v_hat, 1.0)[0]
        exact = math.log(np.mean(np.exp(keys @ q[0])))
        gaps.append(abs(score - exact))
    r1, r2 = gaps[0] / gaps[1], gaps[1] / gaps[2]
    assert 6.0 < r1 < 10.5 and 6.5 < r2 < 9.5, gaps


# ----------------------------------------------------------------------------- top-k

def test_topk_against_exhaustive_search():
    """Among all k-subsets, the selection must maximise the score sum; among the
    maximisers (ties) it must be the lexicographically smallest index tuple,
    i.e. ties go to the lower block index (R5)."""
    rng = np.random.default_rng(9)
    for trial in range(60):
        nb = int(rng.integers(0, 9))
        scores = rng.integers(-3, 4, nb).astype(float)      # many ties
        for k in range(0, nb + 2):
            got = tuple(O.select_blocks(scores, k))
            kk = min(k, nb)
            best = None
            for sub in itertools.combinations(range(nb), kk):
                key = (-sum(scores[list(sub)]), sub)
                if best is None or key < best:
                    best = key
            assert got == best[1], (scores, k, got, best)


def test_strided_selection_by_exhaustive_search():
    """Strided block selection (R8, one reading of a heading the page leaves
    empty): the strided blocks are range(stride - 1, nb, stride); the rest of
    the selection is, among all subsets of the other blocks of the right
    size, the one with the largest score sum, ties to the lexicographically
    smallest index tuple."""
    rng = np.random.default_rng(21)
    for trial in range(50):
        nb = int(rng.integers(0, 10))
        scores = rng.integers(-3, 4, nb).astype(float)      # many ties
        for stride in range(1, nb + 3):
            fixed = list(range(stride - 1, nb, stride))
            assert list(O.strided_blocks(nb, stride)) == fixed
            others = [j for j in range(nb) if j not in fixed]
            for k in range(0, nb + 2):
                got = tuple(O.select_blocks_strided(scores, k, stride))
                kk = min(k, len(others))
                best = None
                for sub in itertools.combinations(others, kk):
                    key = (-sum(scores[list(sub)]), sub)
                    if best is None or key < best:
                        best = key
                assert got == tuple(sorted(fixed + list(best[1]))), (scores, k, stride, got)


def test_strided_selection_special_cases():
    """A stride past the block count is plain top-k; stride 1 selects every
    block, and the hybrid output then equals full softmax."""
    rng = np.random.default_rng(22)
    scores = rng.standard_normal(40)
    for k in (0, 3, 39, 50):
        assert list(O.select_blocks_strided(scores, k, 41)) == list(O.select_blocks(scores, k))
    T, S, W, Bk, d, G = 300, 4, 32, 16, 16, 2
    K = rng.standard_normal((T, d))
    V = rng.standard_normal((T, d))
    q = rng.standard_normal((G, d))
    part = O.partition(T, S, W, Bk)
    scale = 1 / math.sqrt(d)
    mu, var = O.block_stats(K, part)
    sc = O.block_scores(q, mu, var, scale)
    sel = O.select_blocks_strided(sc, 2, 1)
    assert list(sel) == list(range(part.nb))
    np.testing.assert_allclose(O.hybrid_subtract(q, K, V, part, sel, scale), O.full_softmax(q, K, V, T, scale),
                               rtol=1e-12, atol=1e-12)


# ----------------------------------------------------------------------------- state / recurrence

def test_linear_state_by_loops():
    """H[r][c] = sum_t k_t[r] v_t[c] by explicit loops (tiny), zk, zv, n by
    counting: pins the orientation of H and the evicted range."""
    rng = np.random.default_rng(4)
    T, S, W, d = 13, 2, 3, 3
    K = rng.standard_normal((T, d))
    V = rng.standard_normal((T, d))
    part = O.partition(T, S, W, 4)
    H, zk, zv, n = O.linear_state(K, V, part)
    Hl = [[0.0] * d for _ in range(d)]
    for t in range(S, T - W):
        for r in range(d):
            for c in range(d):
                Hl[r][c] += K[t, r] * V[t, c]
    np.testing.assert_allclose(H, np.array(Hl), atol=1e-14)
    np.testing.assert_allclose(zk, K[S:T - W].sum(0), atol=1e-14)
    assert n == T - W - S


@pytest.mark.parametrize("T0,S,W,Bk,n_app", [
    (100, 4, 16, 8, 40), (20, 4, 16, 8, 30), (3, 4, 16, 8, 40), (50, 0, 0, 5, 20),
    (50, 2, 0, 1, 9), (61, 4, 8, 16, 70),
])
def test_incremental_append_equals_fresh_state(T0, S, W, Bk, n_app):
    """The recurrence (rank-1 fold of the token leaving the window, running
    block sums) after n appends equals the state defined directly on the final
    history (SPLA "Recurrence": the RLA state is maintained token by token)."""
    rng = np.random.default_rng(T0 + n_app)
    d = 5
    Kall = rng.standard_normal((T0 + n_app, d))
    Vall = rng.standard_normal((T0 + n_app, d))
    u = O.OracleUnit(Kall[:T0], Vall[:T0], S, W, Bk, k=3, scale=0.4)
    for i in range(n_app):
        u.append(Kall[T0 + i], Vall[T0 + i])
        part = O.partition(u.T, S, W, Bk)
        H, zk, zv, n = O.linear_state(Kall, Vall, part)
        np.testing.assert_allclose(u.H, H, atol=1e-11)
        np.testing.assert_allclose(u.zk, zk, atol=1e-12)
        np.testing.assert_allclose(u.zv, zv, atol=1e-12)
        assert u.n == n
        mu, var = O.block_stats(Kall, part)
        mu2, var2 = u.stats()
        np.testing.assert_allclose(mu2, mu, atol=1e-12)
        np.testing.assert_allclose(var2, var, atol=1e-11)


def test_population_variance():
    """Block variance divides by the block's count (R2): for keys {0, 2} the
    variance is 1, not 2."""
    K = np.array([[0.0], [2.0]])
    mu, var = O.block_stats(K, O.partition(2, 0, 0, 2))
    assert mu[0, 0] == 1.0 and var[0, 0] == 1.0


# ----------------------------------------------------------------------------- token granularity

def test_block_size_one_is_token_granular_selection():
    """Token-granular exact set (the first-order Taylor kernel for every
    evicted token but the top ones by their own score, which keep the exact
    kernel): at block size 1 a block is one token, its mean is the key and its
    variance 0, so the block score is the group-summed s_t = sum_i q'_i . k_t,
    computed here by loops over the tokens; the selection is then the k evicted
    tokens of largest summed score (ties to the lower position), and the hybrid
    output is the token-by-token definition with exactly those tokens exact."""
    rng = np.random.default_rng(31)
    T, S, W, G, d, k = 90, 3, 7, 2, 6, 9
    q, K, V = _rand(rng, T, d, G)
    scale = 1 / math.sqrt(d)
    part = O.partition(T, S, W, 1)
    assert part.nb == T - S - W
    mu, var = O.block_stats(K, part)
    scores = O.block_scores(q, mu, var, scale)
    for j in range(part.nb):
        t = S + j
        st = 0.0
        for i in range(G):
            for c in range(d):
                st += q[i, c] * scale * K[t, c]
        assert abs(scores[j] - st) < 1e-12
        assert np.all(var[j] == 0.0)
    sel = O.select_blocks(scores, k)
    order = sorted(range(part.nb), key=lambda j: (-scores[j], j))[:k]
    assert list(sel) == sorted(order)
    got = O.hybrid_subtract(q, K, V, part, sel, scale)
    ref = O.brute_force_hybrid(q, K, V, T, S, W, 1, sel, scale)
    np.testing.assert_allclose(got, ref, rtol=1e-11, atol=1e-12)
