"""Pins for the float64 CPU oracle, each against something other than itself.

The AdaSplash pages print no numeric example and no formula, so the pins are
mathematical: hand-derived worked examples (tests/golden), brute-force support
enumeration, the KKT/variational characterisation solved by a library
optimiser, the sort-based closed forms at alpha = 2 and alpha = 1.5, the
softmax limit alpha -> 1, invariants, and central finite differences of the
backward.  Each is chosen so that a plausible mistake in the oracle (a dropped
term, a wrong sign or index, a transposed operand, a wrong scale) fails one.
"""
import itertools
import json
import os

import numpy as np
import pytest
from scipy.optimize import minimize

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "entmax_worked_examples.json")


def brute_force_tau(s, alpha):
    """tau and support by enumerating every support set (N <= 8).

    For each non-empty subset S, solve sum_S (x - t)^gamma = 1 for t below
    min_S x (bisection written here), then keep S only if the KKT conditions
    hold: x_j > t on S and x_j <= t off S.
    """
    x = (alpha - 1.0) * np.asarray(s, float)
    gamma = 1.0 / (alpha - 1.0)
    n = x.size
    found = []
    for r in range(1, n + 1):
        for S in itertools.combinations(range(n), r):
            xs = x[list(S)]
            lo, hi = xs.max() - 1.0, xs.min()
            h = lambda t: np.sum((xs - t) ** gamma) - 1.0
            if h(hi) >= 0.0:
                continue
            for _ in range(200):
                mid = 0.5 * (lo + hi)
                if h(mid) > 0:
                    lo = mid
                else:
                    hi = mid
            t = 0.5 * (lo + hi)
            out = [j for j in range(n) if j not in S]
            if np.all(xs > t) and np.all(x[out] <= t):
                found.append((t, set(S)))
    return found


def rows_for_tests(n_rows=40, max_n=8, seed=1):
    g = np.random.default_rng(seed)
    for _ in range(n_rows):
        n = int(g.integers(1, max_n + 1))
        yield g.normal(size=n) * float(g.choice([0.5, 1.0, 3.0]))


# ------------------------------------------------------------ worked examples
def test_golden_worked_examples(orc):
    g = json.load(open(GOLDEN))
    for c in g["cases"]:
        p, tau = orc.entmax_row(c["s"], c["alpha"])
        assert tau == pytest.approx(c["tau"], abs=1e-11), c
        np.testing.assert_allclose(p, c["p"], atol=1e-11)
    for a in g["attention"]:
        q, k, v = (np.array(a[key], float) for key in ("q_full", "k", "v"))
        o, tau, _ = orc.attn_fwd(q, k, v, a["alpha"], a["causal"])
        np.testing.assert_allclose(o, a["o"], atol=1e-11)
        np.testing.assert_allclose(tau, a["tau"], atol=1e-11)


# ------------------------------------------------------------ brute force
@pytest.mark.parametrize("alpha", [1.25, 1.5, 1.75, 2.0])
def test_brute_force_support(orc, alpha):
    for s in rows_for_tests(seed=int(alpha * 100)):
        found = brute_force_tau(s, alpha)
        assert len(found) == 1, (s, found)
        t_bf, S = found[0]
        p, tau = orc.entmax_row(s, alpha)
        assert abs(tau - t_bf) <= 1e-11
        assert set(np.nonzero(p > 0)[0]) == S


# ------------------------------------------------------------ closed forms
def test_sparsemax_sort_closed_form(orc):
    for s in rows_for_tests(200, 64, seed=7):
        assert abs(orc.sparsemax_tau_sort(s) - orc.entmax_tau(s, 2.0)) <= 1e-10


def test_entmax15_sort_closed_form(orc):
    for s in rows_for_tests(200, 64, seed=8):
        assert abs(orc.entmax15_tau_sort(s) - orc.entmax_tau(s, 1.5)) <= 1e-10


def _simplex_argmax(s, alpha):
    """argmax_{p in simplex} p.s + H_alpha(p) by SLSQP (library optimiser).

    H_alpha is the Tsallis entropy (sum_j p_j - p_j^alpha) / (alpha (alpha-1));
    alpha-entmax is its regularised argmax, and at alpha = 2 this is the
    Euclidean projection of s onto the simplex (sparsemax).
    """
    s = np.asarray(s, float)
    n = s.size

    def neg(p):
        p = np.clip(p, 0, None)
        return -(p @ s + np.sum(p - p ** alpha) / (alpha * (alpha - 1)))

    def grad(p):
        p = np.clip(p, 0, None)
        return -(s + (1 - alpha * p ** (alpha - 1)) / (alpha * (alpha - 1)))

    res = minimize(neg, np.full(n, 1.0 / n), jac=grad, method="SLSQP",
                   bounds=[(0, 1)] * n,
                   constraints=[{"type": "eq", "fun": lambda p: p.sum() - 1,
                                 "jac": lambda p: np.ones_like(p)}],
                   options={"ftol": 1e-15, "maxiter": 1000})
    return res.x


@pytest.mark.parametrize("alpha", [1.5, 2.0])
def test_variational_form_library_optimiser(orc, alpha):
    for s in rows_for_tests(15, 8, seed=11):
        p, _ = orc.entmax_row(s, alpha)
        np.testing.assert_allclose(p, _simplex_argmax(s, alpha), atol=2e-5)


def test_sparsemax_is_simplex_projection(orc):
    # Euclidean projection onto the simplex, by an independent library QP.
    for s in rows_for_tests(15, 8, seed=12):
        res = minimize(lambda p: np.sum((p - s) ** 2), np.full(s.size, 1.0 / s.size),
                       jac=lambda p: 2 * (p - s), method="SLSQP", bounds=[(0, None)] * s.size,
                       constraints=[{"type": "eq", "fun": lambda p: p.sum() - 1}],
                       options={"ftol": 1e-15, "maxiter": 1000})
        p, _ = orc.entmax_row(s, 2.0)
        np.testing.assert_allclose(p, res.x, atol=1e-6)


# ------------------------------------------------------------ softmax limit
def test_softmax_limit(orc):
    g = np.random.default_rng(3)
    s = g.normal(size=12)
    soft = np.exp(s - s.max())
    soft /= soft.sum()
    errs = []
    for eps in (1e-2, 1e-3, 1e-4):
        p, _ = orc.entmax_row(s, 1.0 + eps)
        errs.append(np.max(np.abs(p - soft)))
    # error falls roughly linearly in eps (ratio ~10 per decade)
    assert errs[0] < 0.05
    assert 4 < errs[0] / errs[1] < 25 and 4 < errs[1] / errs[2] < 25, errs


# ------------------------------------------------------------ invariants
@pytest.mark.parametrize("alpha", [1.25, 1.5, 2.0])
def test_invariants(orc, alpha):
    g = np.random.default_rng(5)
    for _ in range(20):
        n = int(g.integers(1, 300))
        s = g.normal(size=n) * 3
        p, tau = orc.entmax_row(s, alpha)
        assert np.all(p >= 0)
        assert abs(p.sum() - 1) <= 1e-10
        # permutation equivariance
        perm = g.permutation(n)
        p2, _ = orc.entmax_row(s[perm], alpha)
        np.testing.assert_allclose(p2, p[perm], atol=1e-12)
        # shift: s + c leaves p, moves tau by (alpha-1) c
        p3, tau3 = orc.entmax_row(s + 1.7, alpha)
        np.testing.assert_allclose(p3, p, atol=1e-10)
        assert tau3 - tau == pytest.approx((alpha - 1) * 1.7, abs=1e-10)
        # monotonicity: s_i >= s_j  =>  p_i >= p_j
        order = np.argsort(s)
        assert np.all(np.diff(p[order]) >= -1e-13)
    # constant row -> uniform; a single key -> 1
    p, _ = orc.entmax_row(np.full(7, 0.3), alpha)
    np.testing.assert_allclose(p, np.full(7, 1 / 7), atol=1e-12)
    p, tau = orc.entmax_row([2.5], alpha)
    assert p[0] == pytest.approx(1.0, abs=1e-12)
    assert tau == pytest.approx((alpha - 1) * 2.5 - 1.0, abs=1e-12)


# ------------------------------------------------------------ attention plumbing
def _brute_attention(q, k, v, alpha, causal):
    """O from numpy matmuls and brute-force tau per row (tiny sizes)."""
    B, H, N, d = q.shape
    o = np.zeros_like(q)
    tau = np.zeros((B, H, N))
    for b in range(B):
        for h in range(H):
            S = q[b, h] @ k[b, h].T / np.sqrt(d)
            for i in range(N):
                n = i + 1 if causal else N
                (t, _), = brute_force_tau(S[i, :n], alpha)
                tau[b, h, i] = t
                p = np.clip((alpha - 1) * S[i, :n] - t, 0, None) ** (1 / (alpha - 1))
                o[b, h, i] = p @ v[b, h, :n]
    return o, tau


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("alpha", [1.5, 2.0])
def test_attention_vs_brute_force(orc, causal, alpha):
    g = np.random.default_rng(21)
    q, k, v = (g.normal(size=(2, 2, 7, 3)) for _ in range(3))
    o, tau, marg = orc.attn_fwd(q, k, v, alpha, causal, blk=3)
    o_bf, tau_bf = _brute_attention(q, k, v, alpha, causal)
    np.testing.assert_allclose(tau, tau_bf, atol=1e-11)
    np.testing.assert_allclose(o, o_bf, atol=1e-10)
    # block margins from the brute-force tau
    S = np.einsum("bhid,bhjd->bhij", q, k) / np.sqrt(3)
    X = (alpha - 1) * S - tau_bf[..., None]
    if causal:
        X = np.where(np.tril(np.ones((7, 7), bool)), X, -np.inf)
    for t in range(3):
        for b in range(3):
            want = X[:, :, 3 * t:3 * t + 3, 3 * b:3 * b + 3].max(axis=(2, 3))
            np.testing.assert_allclose(marg[:, :, t, b], want, atol=1e-10)


def test_fwd_rows_matches_full(orc):
    g = np.random.default_rng(4)
    q, k, v = (g.normal(size=(2, 3, 40, 8)) for _ in range(3))
    o, tau, marg = orc.attn_fwd(q, k, v, 1.5, True, blk=16)
    rows = np.array([0, 5, 39, 40, 119, 200, 239])
    o_r, tau_r, bmax = orc.attn_fwd_rows(q, k, v, 1.5, True, rows, blk=16)
    np.testing.assert_array_equal(o_r, o.reshape(-1, 8)[rows])
    np.testing.assert_array_equal(tau_r, tau.reshape(-1)[rows])
    for r, flat in enumerate(rows):
        bh, i = divmod(flat, 40)
        assert np.all(bmax[r] <= marg.reshape(6, 3, 3)[bh, i // 16] + 0)


# ------------------------------------------------------------ backward
def _loss(orc, q, k, v, do, alpha, causal):
    o, _, _ = orc.attn_fwd(q, k, v, alpha, causal)
    return float(np.sum(o * do))


def _pick_seed(orc, alpha, causal, shape, margin=1e-4):
    """First seed whose scores stay clear of every support boundary."""
    for seed in range(100):
        g = np.random.default_rng(seed)
        q, k, v, do = (g.normal(size=shape) for _ in range(4))
        _, tau, _ = orc.attn_fwd(q, k, v, alpha, causal)
        X = (alpha - 1) * np.einsum("bhid,bhjd->bhij", q, k) / np.sqrt(shape[-1]) - tau[..., None]
        if causal:
            X = np.where(np.tril(np.ones(X.shape[-2:], bool)), X, 1.0)
        if np.min(np.abs(X)) > margin:
            return q, k, v, do
    raise RuntimeError("no seed clear of the support boundaries")


@pytest.mark.parametrize("alpha,causal", [(1.5, True), (2.0, False), (1.25, True), (1.75, False)])
def test_backward_finite_differences(orc, alpha, causal):
    shape = (1, 2, 10, 4)
    q, k, v, do = _pick_seed(orc, alpha, causal, shape)
    dq, dk, dv, _, _ = orc.attn_bwd(q, k, v, do, alpha, causal)
    h = 1e-5
    for X, dX in ((q, dq), (k, dk), (v, dv)):
        num = np.zeros_like(X)
        for idx in np.ndindex(X.shape):
            old = X[idx]
            X[idx] = old + h
            lp = _loss(orc, q, k, v, do, alpha, causal)
            X[idx] = old - h
            lm = _loss(orc, q, k, v, do, alpha, causal)
            X[idx] = old
            num[idx] = (lp - lm) / (2 * h)
        rel = np.linalg.norm(num - dX) / np.linalg.norm(num)
        assert rel <= 1e-6, rel


@pytest.mark.parametrize("alpha", [1.25, 1.5, 2.0])
def test_row_jacobian_properties(orc, alpha):
    """J = diag(g) - g g^T / sum g: symmetric, J 1 = 0, and the VJP agrees with
    finite differences of p(s) away from support changes."""
    g = np.random.default_rng(9)
    s = g.normal(size=9) * 2
    p, tau = orc.entmax_row(s, alpha)
    n = s.size
    J = np.zeros((n, n))
    for j in range(n):
        e = np.zeros(n)
        e[j] = 1.0
        J[j], _, _ = orc.entmax_vjp_row(s, alpha, tau, e)   # row j = e_j^T J
    np.testing.assert_allclose(J, J.T, atol=1e-13)
    np.testing.assert_allclose(J @ np.ones(n), 0, atol=1e-12)
    x = (alpha - 1) * s - tau
    assert np.min(np.abs(x)) > 1e-3
    h = 1e-6
    Jfd = np.zeros((n, n))
    for j in range(n):
        sp, sm = s.copy(), s.copy()
        sp[j] += h
        sm[j] -= h
        Jfd[:, j] = (orc.entmax_row(sp, alpha)[0] - orc.entmax_row(sm, alpha)[0]) / (2 * h)
    np.testing.assert_allclose(J, Jfd, atol=2e-6)


def test_backward_sampled_matches_full(orc):
    g = np.random.default_rng(12)
    q, k, v, do = (g.normal(size=(1, 1, 48, 8)) for _ in range(4))
    for causal in (True, False):
        dq, dk, dv, _, _ = orc.attn_bwd(q, k, v, do, 1.5, causal)
        rows, keys = np.array([0, 17, 47]), np.array([3, 30, 47])
        dq_r, dk_k, dv_k = orc.attn_bwd_head_sampled(q[0, 0], k[0, 0], v[0, 0], do[0, 0], 1.5,
                                                     causal, rows, keys)
        np.testing.assert_allclose(dq_r, dq[0, 0, rows], atol=1e-13)
        np.testing.assert_allclose(dk_k, dk[0, 0, keys], atol=1e-13)
        np.testing.assert_allclose(dv_k, dv[0, 0, keys], atol=1e-13)


def test_backward_sum_rules(orc):
    """sum_j dK_j = 0 (each row of dS sums to 0) and sum_j dV_j = sum_i dO_i
    (each row of P sums to 1)."""
    g = np.random.default_rng(13)
    q, k, v, do = (g.normal(size=(2, 2, 33, 8)) for _ in range(4))
    dq, dk, dv, _, _ = orc.attn_bwd(q, k, v, do, 1.5, True)
    np.testing.assert_allclose(dk.sum(axis=2), 0, atol=1e-11)
    np.testing.assert_allclose(dv.sum(axis=2), do.sum(axis=2), atol=1e-11)


# ------------------------------------------------------------ otilde (g-weighted value mean)
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("alpha", [1.25, 1.5, 2.0])
def test_otilde_vs_brute_force(orc, causal, alpha):
    """otilde_i = sum_j g_ij v_j / sum_j g_ij with g = (x - tau)_+^(gamma - 1), tau and the
    support from the brute-force enumeration."""
    g = np.random.default_rng(31)
    q, k, v = (g.normal(size=(1, 2, 7, 3)) for _ in range(3))
    rows = np.arange(14)
    ot = orc.attn_otilde_rows(q, k, v, alpha, causal, rows)
    S = np.einsum("bhid,bhjd->bhij", q, k) / np.sqrt(3)
    for flat in rows:
        h, i = divmod(int(flat), 7)
        n = i + 1 if causal else 7
        (t, supp), = brute_force_tau(S[0, h, i, :n], alpha)
        u = (alpha - 1) * S[0, h, i, :n] - t
        w = np.zeros(n)
        idx = sorted(supp)
        w[idx] = u[idx] ** (1 / (alpha - 1) - 1)
        np.testing.assert_allclose(ot[flat], w @ v[0, h, :n] / w.sum(), atol=1e-11)


def test_otilde_sparsemax_is_support_mean(orc):
    """At alpha = 2, g is the support indicator: otilde is the plain mean of the values
    on the support, which the sort-based closed form of tau fixes."""
    g = np.random.default_rng(32)
    q, k, v = (g.normal(size=(1, 1, 40, 8)) for _ in range(3))
    ot = orc.attn_otilde_rows(q, k, v, 2.0, False, np.arange(40))
    S = q[0, 0] @ k[0, 0].T / np.sqrt(8)
    for i in range(40):
        supp = S[i] > orc.sparsemax_tau_sort(S[i])
        np.testing.assert_allclose(ot[i], v[0, 0][supp].mean(axis=0), atol=1e-11)


def test_otilde_gives_backward_delta(orc):
    """dO_i . otilde_i equals the backward's delta_i = sum_j g_ij dP_ij / sum_j g_ij, which
    the backward computes through dP = dO V^T (another contraction order)."""
    g = np.random.default_rng(33)
    q, k, v, do = (g.normal(size=(2, 2, 33, 8)) for _ in range(4))
    for alpha, causal in ((1.5, True), (1.25, False), (2.0, True)):
        _, _, _, _, delta = orc.attn_bwd(q, k, v, do, alpha, causal)
        ot = orc.attn_otilde_rows(q, k, v, alpha, causal, np.arange(2 * 2 * 33))
        np.testing.assert_allclose(np.einsum("rd,rd->r", do.reshape(-1, 8), ot),
                                   delta.reshape(-1), atol=1e-11)


# ------------------------------------------------------------ iteration counts
def test_iterative_solvers_converge_and_counts(orc):
    """All three root-finders land on the bisection tau; pass counts follow the
    pages' claims: bisection over 20, Halley-bisection a few, the histogram
    start fewer still (soft checks on means)."""
    g = np.random.default_rng(17)
    counts = {0: [], 1: [], 2: []}
    for _ in range(60):
        s = g.normal(size=2048) * 4.0
        t_ref = orc.entmax_tau(s, 1.5)
        for m in (0, 1, 2):
            t, n = orc.entmax_tau_iterative(s, 1.5, m, nbins=64, ftol=1e-7, maxpass=64)
            assert abs(t - t_ref) <= 1e-6
            counts[m].append(n)
    mean = {m: np.mean(c) for m, c in counts.items()}
    assert mean[0] > 20
    assert mean[1] <= 6
    assert mean[2] <= mean[1]
    assert mean[0] / mean[1] >= 4
