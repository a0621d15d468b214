"""Pins for the CPU oracle: each check ties it to something other than itself.

Sources: EntmaxKV technical summary (gist.science) §2.A (page metadata and bound), §2.B
(top-k and Gaussian-aware selection), §2.C (exact sparse entmax attention), §3 (error bound
2*B*delta, support recovery). Pins are closed forms, hand-worked fixtures under tests/golden/,
library routines (numpy/scipy) on the defining equations, brute force on tiny inputs, and the
invariants the summary states.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest
from scipy import integrate, optimize, special, stats

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------------------- helpers
def rand_cache(rng, nb, H_kv, P, d, dist=None):
    if dist is None:
        return rng.standard_normal((nb, H_kv, P, d)).astype(np.float32)
    return dist(rng, (nb, H_kv, P, d)).astype(np.float32)


def parse_golden(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, val = (s.strip() for s in line.split("=", 1))
            rows = [[float(Fraction(x)) for x in r.split()] for r in val.split(";")]
            out[key] = np.array(rows if len(rows) > 1 else rows[0])
    return out


def page_cache_from_keys(keys, P=None):
    """One sequence, one KV head, one block holding `keys` [n, d]."""
    n, d = keys.shape
    P = P or n
    k = np.zeros((1, 1, P, d), dtype=np.float32)
    k[0, 0, :n] = keys
    return k


# ----------------------------------------------------------------------------- §2.A metadata
def test_meta_golden_fixture():
    g = parse_golden("bbox_page_example.txt")
    k = page_cache_from_keys(g["keys"])
    kmin, kmax, mean, var = O.page_meta_head(k, [0], 3, 0)
    np.testing.assert_array_equal(kmin[0], g["kmin"])
    np.testing.assert_array_equal(kmax[0], g["kmax"])
    np.testing.assert_allclose(mean[0], g["mean"], rtol=0, atol=1e-15)
    np.testing.assert_allclose(var[0], g["var"], rtol=1e-15, atol=1e-15)


@pytest.mark.parametrize("n,P", [(16, 16), (5, 16), (1, 8), (64, 64)])
def test_meta_arithmetic_progression_closed_form(n, P):
    # k_t = a_c + t * b_c: min/max at the ends, mean a + b(n-1)/2, variance b^2 (n^2-1)/12.
    d = 8
    a = np.array([-3.0, -1.5, 0.25, 2.0, -0.75, 1.0, 0.5, -2.0])  # dyadic: exact in float32
    b = np.array([0.5, -0.25, 1.0, -1.0, 0.125, 2.0, -0.5, 0.0])
    keys = a[None, :] + np.arange(n)[:, None] * b[None, :]
    k = page_cache_from_keys(keys, P)
    kmin, kmax, mean, var = O.page_meta_head(k, [0], n, 0)
    ends = np.stack([a, a + (n - 1) * b])
    np.testing.assert_array_equal(kmin[0], ends.min(0))
    np.testing.assert_array_equal(kmax[0], ends.max(0))
    np.testing.assert_allclose(mean[0], a + b * (n - 1) / 2, atol=1e-12)
    np.testing.assert_allclose(var[0], b * b * (n * n - 1) / 12.0, rtol=1e-12, atol=1e-12)


def test_meta_constant_page():
    keys = np.full((7, 4), 1.25)
    kmin, kmax, mean, var = O.page_meta_head(page_cache_from_keys(keys, 16), [0], 7, 0)
    assert np.all(kmin == 1.25) and np.all(kmax == 1.25) and np.all(mean == 1.25)
    assert np.all(var == 0.0)


def test_meta_paged_layout_against_numpy():
    # Several sequences, scattered blocks, partial last pages: numpy reductions over the
    # valid tokens of block page_table[b, j], head h, must agree.
    rng = np.random.default_rng(1)
    nb, H_kv, P, d = 40, 3, 8, 6
    k = rand_cache(rng, nb, H_kv, P, d)
    perm = rng.permutation(nb).astype(np.int32)
    seq_lens = [37, 8, 1]
    pt = np.full((3, 5), -1, np.int32)
    nxt = 0
    for b, L in enumerate(seq_lens):
        n = O.pages_of(L, P)
        pt[b, :n] = perm[nxt:nxt + n]
        nxt += n
    for b, L in enumerate(seq_lens):
        for h in range(H_kv):
            kmin, kmax, mean, var = O.page_meta_head(k, pt[b], L, h)
            for j in range(O.pages_of(L, P)):
                rows = k[pt[b, j], h, :min(P, L - j * P)].astype(np.float64)
                np.testing.assert_array_equal(kmin[j], rows.min(0))
                np.testing.assert_array_equal(kmax[j], rows.max(0))
                np.testing.assert_allclose(mean[j], rows.mean(0), atol=1e-14)
                np.testing.assert_allclose(var[j], rows.var(0), atol=1e-14)


def test_meta_bf16_widening_is_exact():
    # bf16 bit patterns widen to the float32 with the same upper half.
    rng = np.random.default_rng(2)
    f = rng.standard_normal((1, 1, 4, 8)).astype(np.float32)
    bits = (f.view(np.uint32) >> 16).astype(np.uint16)
    exact = (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    kmin, kmax, _, _ = O.page_meta_head(bits, [0], 4, 0)
    np.testing.assert_array_equal(kmin[0], exact[0, 0].min(0))
    np.testing.assert_array_equal(kmax[0], exact[0, 0].max(0))


def test_meta_rejects_bad_block():
    k = np.zeros((2, 1, 4, 2), np.float32)
    with pytest.raises(ValueError):
        O.page_meta_head(k, [0, 2], 8, 0)


# ----------------------------------------------------------------------------- §2.A bound
def test_bound_golden_fixture():
    g = parse_golden("bbox_page_example.txt")
    ub, S = O.score_head(g["q"], 1.0, g["kmin"][None], g["kmax"][None])
    np.testing.assert_array_equal(ub[:, 0], g["ub"])
    assert S[0] == g["S"]
    best = (g["q"] @ g["keys"].T).max(1)
    np.testing.assert_array_equal(best, g["best"])
    m, v = O.gauss_stats_head(g["q"], 1.0, g["mean"][None], g["var"][None])
    np.testing.assert_allclose(m[:, 0], g["m"], atol=1e-15)
    np.testing.assert_allclose(v[:, 0], g["v"], rtol=1e-15)


def test_bound_dominates_every_token_brute_force():
    # §2.A: the bound is an upper bound on the score of every token in the page.
    rng = np.random.default_rng(3)
    for trial in range(30):
        P, d, G = rng.choice([1, 3, 16]), rng.choice([2, 5, 64]), rng.choice([1, 4])
        n = rng.integers(1, P + 1)
        keys = rng.standard_normal((n, d)) * rng.choice([0.1, 1, 10])
        k = page_cache_from_keys(keys.astype(np.float32), P)
        kmin, kmax, _, _ = O.page_meta_head(k, [0], n, 0)
        q = rng.standard_normal((G, d))
        scale = float(rng.choice([1.0, 0.125, 3.0]))
        ub, S = O.score_head(q, scale, kmin, kmax)
        s = scale * q @ k[0, 0, :n].astype(np.float64).T
        assert np.all(ub[:, 0] >= s.max(1) - 1e-12 * np.abs(s).max())
        np.testing.assert_allclose(S[0], ub[:, 0].sum(), rtol=1e-14)


def test_bound_tight_for_single_token_page():
    rng = np.random.default_rng(4)
    keys = rng.standard_normal((1, 16))
    kmin, kmax, _, _ = O.page_meta_head(page_cache_from_keys(keys.astype(np.float32)), [0], 1, 0)
    q = rng.standard_normal((3, 16))
    ub, _ = O.score_head(q, 0.5, kmin, kmax)
    np.testing.assert_allclose(ub[:, 0], 0.5 * q @ keys.astype(np.float32).astype(np.float64)[0],
                               rtol=1e-13)


def test_bound_sign_split_closed_form():
    # For q >= 0 coordinate-wise the bound is q.kmax; for q <= 0 it is q.kmin.
    rng = np.random.default_rng(5)
    kmin = -np.abs(rng.standard_normal((3, 8)))
    kmax = np.abs(rng.standard_normal((3, 8)))
    qp = np.abs(rng.standard_normal((1, 8)))
    ub, _ = O.score_head(qp, 1.0, kmin, kmax)
    np.testing.assert_allclose(ub[0], kmax @ qp[0], rtol=1e-14)
    ub, _ = O.score_head(-qp, 1.0, kmin, kmax)
    np.testing.assert_allclose(ub[0], kmin @ -qp[0], rtol=1e-14)


@pytest.mark.parametrize("scale", [1.0, 0.37])
def test_gauss_stats_are_mean_and_variance_of_the_scores(scale):
    # m = scale q.mean and v = scale^2 sum_c q_c^2 var_c are the exact mean and variance of the
    # scores scale q.k over a page whose coordinates are independent: check on an outer-product
    # page where they are.
    rng = np.random.default_rng(6)
    d = 3
    vals = [rng.standard_normal(2) for _ in range(d)]
    import itertools
    keys = np.array(list(itertools.product(*vals)))  # every combination: coordinates independent
    k = page_cache_from_keys(keys.astype(np.float32))
    _, _, mean, var = O.page_meta_head(k, [0], len(keys), 0)
    q = rng.standard_normal((2, d))
    m, v = O.gauss_stats_head(q, scale, mean, var)
    s = scale * (q @ k[0, 0].astype(np.float64).T)
    np.testing.assert_allclose(m[:, 0], s.mean(1), atol=1e-13)
    np.testing.assert_allclose(v[:, 0], s.var(1), atol=1e-13)


# ----------------------------------------------------------------------------- §2.B.1 top-k
@pytest.mark.parametrize("seed", range(8))
def test_topk_matches_library_sort(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(1, 300))
    S = rng.integers(-5, 5, size=n).astype(np.float64) if seed % 2 else rng.standard_normal(n)
    for k in [1, 2, n // 3 + 1, n, n + 7]:
        ref = sorted(sorted(range(n), key=lambda j: (-S[j], j))[:k])
        np.testing.assert_array_equal(O.topk(S, k), ref)


def test_topk_tie_storm_prefers_lower_index():
    S = np.zeros(100)
    np.testing.assert_array_equal(O.topk(S, 10), np.arange(10))
    S[50:] = 1.0
    np.testing.assert_array_equal(O.topk(S, 55), np.r_[np.arange(5), np.arange(50, 100)])


# ----------------------------------------------------------------------------- §2.C entmax
def entmax_objective(p, z, alpha):
    # Peters et al. (2019): alpha-entmax(s) = argmax_p p.s + H_alpha(p) over the simplex, with
    # the Tsallis entropy H_alpha(p) = sum_j (p_j - p_j^alpha) / (alpha (alpha - 1)). The
    # oracle works in the z = (alpha - 1) s domain, so the logits here are s = z / (alpha - 1).
    s = np.asarray(z) / (alpha - 1.0)
    return p @ s + np.sum(p - p ** alpha) / (alpha * (alpha - 1.0))


@pytest.mark.parametrize("alpha", [1.5, 2.0])
def test_entmax_closed_forms(alpha):
    np.testing.assert_allclose(O.entmax([3.7], alpha), [1.0])
    np.testing.assert_allclose(O.entmax(np.zeros(5), alpha), np.full(5, 0.2), atol=1e-15)
    np.testing.assert_allclose(O.entmax([1.0, 0.0], alpha), [1.0, 0.0])       # gap >= 1
    np.testing.assert_allclose(O.entmax([2.0, 0.5, -3.0], alpha), [1.0, 0.0, 0.0])
    d = 0.5
    if alpha == 2.0:
        ref = [(1 + d) / 2, (1 - d) / 2]
    else:
        x = (d + math.sqrt(2 - d * d)) / 2  # x^2 + (x - d)^2 = 1, both positive for d < 1
        ref = [x * x, (x - d) ** 2]
    np.testing.assert_allclose(O.entmax([d, 0.0], alpha), ref, atol=1e-15)


@pytest.mark.parametrize("alpha", [1.5, 2.0])
def test_entmax_tau_solves_the_normalisation_equation(alpha):
    # tau is the root of sum_i [z_i - tau]_+^(1/(alpha-1)) = 1, found here by scipy's brentq.
    rng = np.random.default_rng(7)
    for n in [1, 2, 3, 10, 100, 2000]:
        z = rng.standard_normal(n) * rng.choice([0.1, 1.0, 5.0])
        pw = 1.0 / (alpha - 1.0)
        f = lambda t: np.sum(np.maximum(z - t, 0.0) ** pw) - 1.0
        ref = optimize.brentq(f, z.max() - 1.0, z.max(), xtol=1e-15, rtol=1e-15)
        tau = O.entmax_tau(z, alpha)
        assert abs(tau - ref) <= 1e-12 * max(1.0, abs(ref))
        p = O.entmax(z, alpha)
        assert abs(p.sum() - 1.0) <= 1e-12
        assert np.all(p >= 0)


@pytest.mark.parametrize("alpha", [1.5, 2.0])
def test_entmax_is_the_variational_maximiser(alpha):
    rng = np.random.default_rng(8)
    for _ in range(10):
        n = int(rng.integers(2, 7))
        z = rng.standard_normal(n)
        p = O.entmax(z, alpha)
        best = entmax_objective(p, z, alpha)
        res = optimize.minimize(lambda x: -entmax_objective(x, z, alpha),
                                np.full(n, 1.0 / n), method="SLSQP", bounds=[(0.0, 1.0)] * n,
                                constraints=[{"type": "eq", "fun": lambda x: x.sum() - 1}],
                                options={"ftol": 1e-14, "maxiter": 500})
        x = np.maximum(res.x, 0.0)
        x /= x.sum()  # a feasible simplex point near the optimiser's answer
        assert best >= entmax_objective(x, z, alpha) - 1e-12
        assert np.abs(x - p).max() < 1e-4  # and the optimiser lands on the same distribution
        for _ in range(200):
            r = rng.dirichlet(np.ones(n) * rng.choice([0.2, 1.0, 5.0]))
            assert best >= entmax_objective(r, z, alpha) - 1e-12


@pytest.mark.parametrize("alpha", [1.5, 2.0])
def test_entmax_shift_invariance_and_kkt(alpha):
    rng = np.random.default_rng(9)
    z = rng.standard_normal(64) * 2
    tau = O.entmax_tau(z, alpha)
    assert abs(O.entmax_tau(z + 3.25, alpha) - (tau + 3.25)) <= 1e-12
    p = O.entmax(z, alpha)
    on = p > 0
    # KKT: in the support z_i - tau = p_i^(alpha-1); outside it z_i <= tau.
    np.testing.assert_allclose(z[on] - tau, p[on] ** (alpha - 1.0), rtol=1e-12)
    assert np.all(z[~on] <= tau)


# ----------------------------------------------------------------------------- §2.B.2 Gaussian
@pytest.mark.parametrize("alpha", [1.5, 2.0])
def test_trunc_moment_against_quadrature(alpha):
    pw = 1.0 / (alpha - 1.0)
    for a, b, tau in [(0.3, 1.0, 0.0), (-2.0, 0.5, 1.0), (1.0, 0.01, 0.5), (4.0, 3.0, 9.0),
                      (0.0, 2.0, -5.0)]:
        f = lambda x: (x - tau) ** pw * stats.norm.pdf(x, loc=a, scale=b)
        ref, _ = integrate.quad(f, tau, np.inf, epsabs=1e-14, epsrel=1e-12)
        assert abs(O.trunc_moment(a, b, tau, alpha) - ref) <= 1e-10 * max(1.0, ref)
    assert O.trunc_moment(1.0, 0.0, 0.25, alpha) == 0.75 ** pw
    assert O.trunc_moment(1.0, 0.0, 1.5, alpha) == 0.0


@pytest.mark.parametrize("alpha", [1.5, 2.0])
def test_gauss_tau_zero_variance_reduces_to_exact_entmax(alpha):
    # With all page variances zero, page j is n_j copies of one score: F(tau) = 1 is exactly
    # the entmax normalisation over that multiset, so tau-hat is the exact entmax threshold.
    rng = np.random.default_rng(10)
    for _ in range(5):
        n = int(rng.integers(1, 40))
        m = rng.standard_normal(n) * 2
        cnt = rng.integers(1, 17, size=n).astype(np.int32)
        th = O.gauss_tau(m, np.zeros(n), cnt, alpha)
        z = np.repeat((alpha - 1.0) * m, cnt)
        pw = 1.0 / (alpha - 1.0)
        ref = optimize.brentq(lambda t: np.sum(np.maximum(z - t, 0) ** pw) - 1.0,
                              z.max() - 1, z.max(), xtol=1e-15, rtol=1e-15)
        assert abs(th - ref) <= 1e-11 * max(1.0, abs(ref))
        assert abs(th - O.entmax_tau(z, alpha)) <= 1e-11 * max(1.0, abs(ref))


@pytest.mark.parametrize("alpha", [1.5, 2.0])
def test_gauss_tau_monte_carlo(alpha):
    # F(tau-hat) = 1 in expectation: draw n_j iid N(m_j, v_j) scores per page and average the
    # entmax mass sum_i [(alpha-1) s_i - tau-hat]_+^(1/(alpha-1)) over many draws.
    rng = np.random.default_rng(11)
    n = 12
    m = rng.standard_normal(n)
    v = rng.uniform(0.05, 1.0, n)
    cnt = rng.integers(1, 33, size=n).astype(np.int32)
    th = O.gauss_tau(m, v, cnt, alpha)
    assert abs(O.gauss_F(m, v, cnt, alpha, th) - 1.0) <= 1e-10
    draws = 20000
    tot = np.zeros(draws)
    pw = 1.0 / (alpha - 1.0)
    for j in range(n):
        s = rng.normal(m[j], math.sqrt(v[j]), size=(draws, cnt[j]))
        tot += np.sum(np.maximum((alpha - 1.0) * s - th, 0.0) ** pw, axis=1)
    se = tot.std() / math.sqrt(draws)
    assert abs(tot.mean() - 1.0) <= 5 * se


def test_gauss_F_is_decreasing():
    rng = np.random.default_rng(12)
    m, v = rng.standard_normal(20), rng.uniform(0, 1, 20)
    cnt = np.full(20, 16, np.int32)
    taus = np.linspace(-5, 5, 200)
    F = [O.gauss_F(m, v, cnt, 1.5, t) for t in taus]
    assert np.all(np.diff(F) <= 0)


def test_gauss_select_rule():
    # keep j iff some query g has (alpha - 1) UB_gj > tau_hat_g - delta (strict)
    ub = np.array([[1.0, 2.0, 3.0, 0.0], [0.0, 0.0, 0.0, 2.1]])
    tau_hat = np.array([1.1, 1.0])
    # alpha 1.5: thresholds 1.0 / 0.9; page 1 gives 0.5*2 = 1.0, not strictly above -> dropped
    np.testing.assert_array_equal(O.gauss_select(ub, tau_hat, 1.5, 0.1), [2, 3])
    np.testing.assert_array_equal(O.gauss_select(ub, tau_hat, 2.0, 0.1), [1, 2, 3])
    np.testing.assert_array_equal(O.gauss_select(ub, tau_hat, 2.0, 0.0), [1, 2, 3])
    np.testing.assert_array_equal(O.gauss_select(ub, np.array([2.0, 1.0]), 2.0, 0.0), [2, 3])


def test_est_max_bounds_the_expected_page_maximum():
    # second reading of the "estimated maximum" (EntmaxKV §2.B): for n iid N(m, v) token scores
    # the expected maximum lies below m + sqrt(2 ln n) sqrt(v) (the classical bound on the
    # expected maximum of n standard normals) and not far below it; the bbox cap is exact
    rng = np.random.default_rng(21)
    for n, m, sd in [(16, 0.3, 1.0), (64, -1.0, 0.5), (2, 2.0, 2.0)]:
        draws = m + sd * rng.standard_normal((40000, n))
        mc = draws.max(axis=1).mean()
        est = O.est_max(np.inf, m, sd * sd, n)
        assert mc <= est + 0.01 * sd
        assert est - mc <= 0.8 * sd
    assert O.est_max(1.5, 1.0, 4.0, 16) == 1.5           # capped by the bound
    assert O.est_max(9.0, 1.0, 0.0, 16) == 1.0           # zero variance: the common score


def test_est_max_of_a_one_token_page_is_its_score():
    rng = np.random.default_rng(22)
    k = rng.standard_normal((3, 1, 4, 8)).astype(np.float32)
    pt = np.array([2, 0], dtype=np.int32)
    q = rng.standard_normal((1, 8))
    kmin, kmax, mean, var = O.page_meta_head(k, pt, 5, 0)   # the second page holds one token
    ub, _ = O.score_head(q, 1.0, kmin, kmax)
    m, v = O.gauss_stats_head(q, 1.0, mean, var)
    s_tok = float(q[0] @ k[0, 0, 0].astype(np.float64))
    assert abs(O.est_max(ub[0, 1], m[0, 1], v[0, 1], 1) - s_tok) < 1e-12


def test_gauss_select_est_rule_and_subset():
    # hand-worked: alpha 2 (factor 1), delta 0.1, tau_hat 1.0 -> keep iff est > 0.9
    ub = np.array([[2.0, 2.0, 0.5, 2.0]])
    m = np.array([[0.5, 0.95, 0.4, 0.1]])
    v = np.array([[0.0, 0.0, 1.0, 0.04]])
    cnt = np.array([16, 16, 16, 1], dtype=np.int32)
    # est: 0.5 | 0.95 | min(0.5, 0.4 + 2.355) = 0.5 | 0.1 (one token) -> only page 1
    np.testing.assert_array_equal(O.gauss_select_est(ub, m, v, cnt, np.array([1.0]), 2.0, 0.1), [1])
    # est <= UB, so the estimate keeps a subset of what the bound keeps
    rng = np.random.default_rng(23)
    G, n = 4, 300
    ub = rng.normal(3, 1, (G, n))
    m = ub - rng.uniform(0, 3, (G, n))
    v = rng.uniform(0, 1, (G, n))
    cnt = rng.integers(1, 33, n).astype(np.int32)
    tau = rng.normal(2, 0.5, G)
    for alpha in (1.5, 2.0):
        a = set(O.gauss_select_est(ub, m, v, cnt, tau, alpha, 0.1).tolist())
        b = set(O.gauss_select(ub, tau, alpha, 0.1).tolist())
        assert a <= b and len(a) < len(b)


# ----------------------------------------------------------------------------- §2.C / §3 attention
def make_seq(rng, P=8, d=16, H_kv=2, L=61, nb=20, dist_scale=1.0):
    k = (rng.standard_normal((nb, H_kv, P, d)) * dist_scale).astype(np.float32)
    v = rng.standard_normal((nb, H_kv, P, d)).astype(np.float32)
    pt = rng.permutation(nb)[:O.pages_of(L, P)].astype(np.int32)
    return k, v, pt


def dense_tokens(cache, pt, L, h):
    P = cache.shape[2]
    rows = [cache[pt[j], h, t] for j in range(O.pages_of(L, P)) for t in range(min(P, L - j * P))]
    return np.array(rows, dtype=np.float64)


def test_softmax_all_pages_equals_dense_attention():
    rng = np.random.default_rng(13)
    k, v, pt = make_seq(rng)
    L, h, scale = 61, 1, 0.3
    q = rng.standard_normal((3, 16))
    allp = np.arange(O.pages_of(L, 8))
    out, stat, _ = O.attend_head(k, v, pt, L, h, q, scale, O.SOFTMAX, allp)
    K, V = dense_tokens(k, pt, L, h), dense_tokens(v, pt, L, h)
    s = scale * q @ K.T
    ref = special.softmax(s, axis=1) @ V
    np.testing.assert_allclose(out, ref, atol=1e-13)
    np.testing.assert_allclose(stat, special.logsumexp(s, axis=1), atol=1e-13)


@pytest.mark.parametrize("mode", [O.ENTMAX15, O.SPARSEMAX])
def test_entmax_all_pages_equals_dense_entmax(mode):
    rng = np.random.default_rng(14)
    k, v, pt = make_seq(rng, dist_scale=3.0)
    L, h, scale = 61, 0, 0.5
    alpha = O.ALPHA_OF_MODE[mode]
    q = rng.standard_normal((2, 16))
    out, stat, _ = O.attend_head(k, v, pt, L, h, q, scale, mode, np.arange(8))
    K, V = dense_tokens(k, pt, L, h), dense_tokens(v, pt, L, h)
    pw = 1.0 / (alpha - 1.0)
    for g in range(2):
        z = (alpha - 1.0) * scale * K @ q[g]
        tau = optimize.brentq(lambda t: np.sum(np.maximum(z - t, 0) ** pw) - 1.0,
                              z.max() - 1, z.max(), xtol=1e-15, rtol=1e-15)
        p = np.maximum(z - tau, 0) ** pw
        np.testing.assert_allclose(out[g], p @ V, atol=1e-11)
        assert abs(stat[g] - tau) <= 1e-12 * max(1, abs(tau))


def full_support_pages(k, v, pt, L, h, q, scale, mode):
    P = k.shape[2]
    allp = np.arange(O.pages_of(L, P))
    out, _, w = O.attend_head(k, v, pt, L, h, q, scale, mode, allp, want_weights=True)
    tok_page = np.concatenate([[j] * min(P, L - j * P) for j in allp])
    support = sorted(set(tok_page[np.any(w > 0, axis=0)]))
    return out, w, support, tok_page


@pytest.mark.parametrize("mode", [O.ENTMAX15, O.SPARSEMAX])
def test_support_superset_gives_the_full_cache_output(mode):
    # §3 support recovery: if the kept pages contain the whole entmax support, delta = 0 and
    # the sparse output equals the full-cache output.
    rng = np.random.default_rng(15)
    for trial in range(10):
        k, v, pt = make_seq(rng, L=int(rng.integers(20, 160)), nb=24, dist_scale=3.0)
        L = int(rng.integers(20, 160))
        pt = rng.permutation(24)[:O.pages_of(L, 8)].astype(np.int32)
        q = rng.standard_normal((2, 16))
        full, _, support, _ = full_support_pages(k, v, pt, L, 1, q, 0.7, mode)
        n = O.pages_of(L, 8)
        extra = rng.choice(n, size=int(rng.integers(0, n)), replace=False)
        keep = np.array(sorted(set(support) | set(extra.tolist())), dtype=np.int32)
        out, _, _ = O.attend_head(k, v, pt, L, 1, q, 0.7, mode, keep)
        np.testing.assert_allclose(out, full, atol=1e-12)
        if len(keep) < n and len(support) > 0:
            # dropping a support page changes the output
            drop = np.array([j for j in keep if j != support[0]], dtype=np.int32)
            o2, _, _ = O.attend_head(k, v, pt, L, 1, q, 0.7, mode, drop)
            assert np.abs(o2 - full).max() > 0


@pytest.mark.parametrize("mode", [O.SOFTMAX, O.ENTMAX15, O.SPARSEMAX])
def test_error_bound_two_B_delta(mode):
    # §3: ||o - o_sparse|| <= 2 B delta, B = max ||v_i||, delta = full-cache mass of the
    # dropped tokens.
    rng = np.random.default_rng(16)
    for trial in range(20):
        L = int(rng.integers(9, 120))
        k, v, pt = make_seq(rng, L=L, nb=16, dist_scale=float(rng.choice([0.5, 2.0])))
        pt = rng.permutation(16)[:O.pages_of(L, 8)].astype(np.int32)
        q = rng.standard_normal((2, 16))
        full, w, _, tok_page = full_support_pages(k, v, pt, L, 0, q, 0.5, mode)
        n = O.pages_of(L, 8)
        keep = np.sort(rng.choice(n, size=int(rng.integers(1, n + 1)), replace=False))
        out, _, _ = O.attend_head(k, v, pt, L, 0, q, 0.5, mode, keep.astype(np.int32))
        B = np.linalg.norm(dense_tokens(v, pt, L, 0), axis=1).max()
        kept_tok = np.isin(tok_page, keep)
        for g in range(2):
            delta = w[g, ~kept_tok].sum()
            err = np.linalg.norm(out[g] - full[g])
            assert err <= 2 * B * delta + 1e-12


def test_entmax_drops_less_mass_than_softmax_on_needle_heads():
    # §3/§4 comparison, on a planted-needle head: for the same kept set (the needle pages)
    # the entmax full-cache mass outside it is below softmax's.
    rng = np.random.default_rng(17)
    P, d, nb, L = 16, 64, 64, 1024
    k = rng.standard_normal((nb, 1, P, d)).astype(np.float32)
    v = rng.standard_normal((nb, 1, P, d)).astype(np.float32)
    pt = np.arange(nb, dtype=np.int32)
    q = rng.standard_normal((1, d)) / 8
    qh = q[0] / np.linalg.norm(q[0])
    for blk in [3, 17, 40]:
        k[blk, 0, 5] = (math.sqrt(d) * qh).astype(np.float32)
    keep = np.array([3, 17, 40], np.int32)
    masses = {}
    for mode in [O.SOFTMAX, O.ENTMAX15]:
        _, w, _, tok_page = full_support_pages(k, v, pt, L, 0, q, 1.0, mode)
        masses[mode] = w[0, ~np.isin(tok_page, keep)].sum()
    assert masses[O.ENTMAX15] < masses[O.SOFTMAX]


def test_empty_selection():
    rng = np.random.default_rng(18)
    k, v, pt = make_seq(rng)
    out, stat, _ = O.attend_head(k, v, pt, 61, 0, rng.standard_normal((2, 16)), 1.0,
                                 O.ENTMAX15, np.zeros(0, np.int32))
    assert np.all(out == 0) and np.all(np.isneginf(stat))


def test_partial_last_page_only_reads_valid_tokens():
    # Tokens at positions >= seq_len must not count: poison them and compare.
    rng = np.random.default_rng(19)
    k, v, pt = make_seq(rng, L=61)
    q = rng.standard_normal((2, 16))
    sel = np.arange(8, dtype=np.int32)
    a = O.attend_head(k, v, pt, 61, 0, q, 1.0, O.SOFTMAX, sel)[0]
    k2, v2 = k.copy(), v.copy()
    k2[pt[7], 0, 5:] = 1e6
    v2[pt[7], 0, 5:] = 1e6
    b = O.attend_head(k2, v2, pt, 61, 0, q, 1.0, O.SOFTMAX, sel)[0]
    np.testing.assert_array_equal(a, b)
    m1 = O.page_meta_head(k, pt, 61, 0)
    m2 = O.page_meta_head(k2, pt, 61, 0)
    for x, y in zip(m1, m2):
        np.testing.assert_array_equal(x, y)


# ----------------------------------------------------------------------------- MomentKV correction
# MomentKV technical summary (gist.science), Methodology §1 (compact moments of the evicted
# set), §2 (first-order estimate of the evicted output), §4 (Jensen-weighted mix).
def test_moment_correction_golden_fixture():
    g = parse_golden("moment_correction_example.txt")
    k = np.zeros((2, 1, 2, 2), dtype=np.float32)
    v = np.zeros((2, 1, 2, 2), dtype=np.float32)
    k[0, 0], v[0, 0] = g["keys_page0"], g["vals_page0"]
    k[1, 0], v[1, 0] = g["keys_page1"], g["vals_page1"]
    out, stat, n_e = O.moment_corrected_head(k, v, np.array([0, 1], np.int32), 4, 0,
                                             g["q"][None, :], float(g["scale"][0]), [0])
    assert n_e == int(g["n_e"][0])
    e = math.e
    zr, ze = math.exp(0.5) + e, int(g["n_e"][0]) * math.exp(float(g["sbar"][0]))
    ref = (math.exp(0.5) * np.array([1.0, 1.0]) + e * np.array([-1.0, 3.0]) + ze * g["fE"]) / (zr + ze)
    np.testing.assert_allclose(out[0], ref, rtol=0, atol=1e-14)
    np.testing.assert_allclose(out[0], [(math.exp(0.5) + 2 * e) / (math.exp(0.5) + 3 * e),
                                        (math.exp(0.5) + 5 * e) / (math.exp(0.5) + 3 * e)],
                               rtol=0, atol=1e-14)
    assert abs(stat[0] - math.log(zr + ze)) < 1e-14


@pytest.mark.parametrize("sel", [[1, 4], [], [0, 2, 5, 7]])
def test_moment_correction_exact_when_skipped_keys_coincide(sel):
    # All skipped tokens share one key: their softmax is uniform (output = their mean value) and
    # Jensen's bound on their partition sum is an equality, so the corrected output is the
    # full-cache softmax.
    rng = np.random.default_rng(31)
    L, P, d, h, scale = 61, 8, 16, 1, 0.4
    k, v, pt = make_seq(rng, P=P, d=d, L=L)
    common = rng.standard_normal(d).astype(np.float32)
    for j in range(O.pages_of(L, P)):
        if j not in sel:
            k[pt[j], h] = common
    q = rng.standard_normal((3, d))
    out, stat, n_e = O.moment_corrected_head(k, v, pt, L, h, q, scale, sel)
    full, fstat, _ = O.attend_head(k, v, pt, L, h, q, scale, O.SOFTMAX, np.arange(O.pages_of(L, P)))
    assert n_e == L - sum(min(P, L - j * P) for j in sel)
    np.testing.assert_allclose(out, full, rtol=0, atol=1e-12)
    np.testing.assert_allclose(stat, fstat, rtol=0, atol=1e-12)


def test_moment_correction_error_is_second_order_in_the_logit_scale():
    # For logits scale * q.k with small scale, expanding the skipped tokens' softmax to first
    # order leaves an O(scale^2) error in the output and in the partition sum, while dropping
    # the skipped tokens (plain renormalisation) leaves an O(1) error.
    rng = np.random.default_rng(32)
    L, P, d, h = 61, 8, 16, 0
    k, v, pt = make_seq(rng, P=P, d=d, L=L)
    q = rng.standard_normal((2, d))
    sel = [1, 3, 6]
    allp = np.arange(O.pages_of(L, P))
    errs, stat_errs, plain = [], [], []
    for scale in (0.04, 0.02, 0.01):
        out, stat, _ = O.moment_corrected_head(k, v, pt, L, h, q, scale, sel)
        full, fstat, _ = O.attend_head(k, v, pt, L, h, q, scale, O.SOFTMAX, allp)
        sparse, _, _ = O.attend_head(k, v, pt, L, h, q, scale, O.SOFTMAX, sel)
        errs.append(np.abs(out - full).max())
        stat_errs.append(np.abs(stat - fstat).max())
        plain.append(np.abs(sparse - full).max())
    for e in (errs, stat_errs):
        for a, b in zip(e, e[1:]):
            assert 3.4 < a / b < 4.6, e
    assert errs[-1] < 1e-2 * plain[-1]


def test_moment_correction_without_skipped_tokens_is_the_plain_softmax():
    rng = np.random.default_rng(33)
    L, P = 61, 8
    k, v, pt = make_seq(rng, P=P, L=L)
    q = rng.standard_normal((2, 16))
    allp = np.arange(O.pages_of(L, P))
    out, stat, n_e = O.moment_corrected_head(k, v, pt, L, 0, q, 0.7, allp)
    ref, rstat, _ = O.attend_head(k, v, pt, L, 0, q, 0.7, O.SOFTMAX, allp)
    assert n_e == 0
    np.testing.assert_array_equal(out, ref)
    np.testing.assert_array_equal(stat, rstat)


# ----------------------------------------------------------------------------- token-level selection
# JSSA abstract (ai.info): token-granular selection, one selection per KV head, attention indexed
# into the standard GQA cache layout.
def candidate_rows(cache, pt, L, h, sel):
    P = cache.shape[2]
    idx = [(j, t) for j in sel for t in range(min(P, L - j * P))]
    rows = np.array([cache[pt[j], h, t] for j, t in idx], dtype=np.float64)
    return idx, rows


@pytest.mark.parametrize("T", [1, 5, 17, 1000])
def test_token_topk_matches_library_sort(T):
    rng = np.random.default_rng(41)
    L, P, d, h, scale = 61, 8, 16, 1, 0.3
    k, v, pt = make_seq(rng, P=P, d=d, L=L)
    q = rng.standard_normal((3, d))
    sel = [0, 2, 5, 7]  # page 7 holds the five valid tokens of the partial last page
    pages, pos = O.token_topk_head(k, pt, L, h, q, scale, sel, T)
    idx, K = candidate_rows(k, pt, L, h, sel)
    score = (scale * (q @ K.T)).sum(axis=0)
    order = np.lexsort((np.arange(len(idx)), -score))  # score descending, earlier first on ties
    keep = np.sort(order[:T])
    assert list(zip(pages.tolist(), pos.tolist())) == [idx[i] for i in keep]


def test_token_topk_ties_prefer_earlier_candidates():
    rng = np.random.default_rng(42)
    L, P, d = 61, 8, 16
    k, v, pt = make_seq(rng, P=P, d=d, L=L)
    k[:, 0] = 0.5  # every key of head 0 equal: every candidate ties
    pages, pos = O.token_topk_head(k, pt, L, 0, rng.standard_normal((2, d)), 1.0, [3, 1, 6], 11)
    assert pages.tolist() == [3] * 8 + [1] * 3 and pos.tolist() == list(range(8)) + [0, 1, 2]


@pytest.mark.parametrize("mode", [O.SOFTMAX, O.ENTMAX15, O.SPARSEMAX])
def test_attention_over_every_candidate_is_the_page_attention(mode):
    rng = np.random.default_rng(43)
    L, P, d, h = 61, 8, 16, 0
    k, v, pt = make_seq(rng, P=P, d=d, L=L, dist_scale=2.0)
    q = rng.standard_normal((4, d))
    sel = [1, 4, 7]
    pages, pos = O.token_topk_head(k, pt, L, h, q, 0.5, sel, 10 ** 6)
    out, stat = O.attend_tokens_head(k, v, pt, L, h, q, 0.5, mode, pages, pos)
    ref, rstat, _ = O.attend_head(k, v, pt, L, h, q, 0.5, mode, sel)
    np.testing.assert_array_equal(out, ref)
    np.testing.assert_array_equal(stat, rstat)


@pytest.mark.parametrize("mode", [O.SOFTMAX, O.ENTMAX15, O.SPARSEMAX])
def test_attention_over_one_token_is_its_value(mode):
    # one token: softmax weight 1 with log-partition = its logit; entmax tau = z - 1, weight 1
    rng = np.random.default_rng(44)
    k, v, pt = make_seq(rng, P=8, d=16, L=61)
    q = rng.standard_normal((2, 16))
    out, stat = O.attend_tokens_head(k, v, pt, 61, 1, q, 0.7, mode, [6], [3])
    row_k, row_v = k[pt[6], 1, 3].astype(np.float64), v[pt[6], 1, 3].astype(np.float64)
    np.testing.assert_allclose(out, np.tile(row_v, (2, 1)), rtol=0, atol=1e-15)
    s = 0.7 * q @ row_k
    want = s if mode == O.SOFTMAX else (O.ALPHA_OF_MODE[mode] - 1.0) * s - 1.0
    np.testing.assert_allclose(stat, want, rtol=0, atol=1e-13)


@pytest.mark.parametrize("mode", [O.ENTMAX15, O.SPARSEMAX])
def test_token_selection_holding_the_support_gives_the_page_output(mode):
    # EntmaxKV §3 at token granularity: entmax over any superset of its support has the same
    # threshold and output, because the extra tokens sit at or below tau.
    rng = np.random.default_rng(45)
    L, P, d, h, scale = 61, 8, 16, 1, 0.8
    k, v, pt = make_seq(rng, P=P, d=d, L=L, dist_scale=3.0)
    q = rng.standard_normal((2, d))
    sel = list(range(O.pages_of(L, P)))
    ref, rstat, w = O.attend_head(k, v, pt, L, h, q, scale, mode, sel, want_weights=True)
    idx, _ = candidate_rows(k, pt, L, h, sel)
    support = {idx[i] for i in np.nonzero((w > 0).any(axis=0))[0]}
    assert 0 < len(support) < len(idx) // 2
    for T in range(1, len(idx) + 1):
        pages, pos = O.token_topk_head(k, pt, L, h, q, scale, sel, T)
        if support <= set(zip(pages.tolist(), pos.tolist())):
            break
    assert T < len(idx)
    out, stat = O.attend_tokens_head(k, v, pt, L, h, q, scale, mode, pages, pos)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(stat, rstat, rtol=0, atol=1e-12)


def test_indexed_attention_reads_only_the_listed_rows():
    rng = np.random.default_rng(46)
    L, P, d = 61, 8, 16
    k, v, pt = make_seq(rng, P=P, d=d, L=L)
    q = rng.standard_normal((2, d))
    pages, pos = [0, 0, 3, 7], [1, 6, 2, 4]
    a = O.attend_tokens_head(k, v, pt, L, 0, q, 1.0, O.SOFTMAX, pages, pos)
    k2, v2 = np.full_like(k, 1e6), np.full_like(v, 1e6)
    for j, t in zip(pages, pos):
        k2[pt[j], 0, t], v2[pt[j], 0, t] = k[pt[j], 0, t], v[pt[j], 0, t]
    b = O.attend_tokens_head(k2, v2, pt, L, 0, q, 1.0, O.SOFTMAX, pages, pos)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])
    with pytest.raises(ValueError):  # position 5 of page 7 is past the sequence end (61 tokens)
        O.attend_tokens_head(k, v, pt, L, 0, q, 1.0, O.SOFTMAX, [7], [5])


def test_moment_sums_golden_fixture_and_additivity():
    g = parse_golden("moment_correction_example.txt")
    k = np.zeros((2, 1, 2, 2), dtype=np.float32)
    v = np.zeros((2, 1, 2, 2), dtype=np.float32)
    k[0, 0], v[0, 0] = g["keys_page0"], g["vals_page0"]
    k[1, 0], v[1, 0] = g["keys_page1"], g["vals_page1"]
    pt = np.array([0, 1], np.int32)
    n, sk, sv, S = O.moment_sums_head(k, v, pt, 4, 0, [1])
    assert n == 2
    np.testing.assert_array_equal(sk, g["sums_page1_k"])
    np.testing.assert_array_equal(sv, g["sums_page1_v"])
    np.testing.assert_array_equal(S, g["sums_page1_vk"])
    # sums over disjoint page sets add up (the running sums less the selected ones are the
    # skipped ones), checked on a random paged sequence with a partial last page
    rng = np.random.default_rng(47)
    k, v, pt = make_seq(rng, P=8, d=16, L=61)
    whole = O.moment_sums_head(k, v, pt, 61, 1)
    a = O.moment_sums_head(k, v, pt, 61, 1, [0, 3, 7])
    b = O.moment_sums_head(k, v, pt, 61, 1, [1, 2, 4, 5, 6])
    assert whole[0] == 61 and a[0] + b[0] == 61
    for x, y, z in zip(whole[1:], a[1:], b[1:]):
        np.testing.assert_allclose(x, y + z, rtol=0, atol=1e-12)


# ----------------------------------------------------------------------------- §3 selection quality
def dense_full_cache_weights(k, pt, L, h, qg, scale, mode):
    """Full-cache weights of one query from a dense evaluation: scipy softmax, or entmax with
    tau from brentq on its normalisation equation; also the support mask and min |z - tau|."""
    s = scale * dense_tokens(k, pt, L, h) @ qg
    if mode == O.SOFTMAX:
        return special.softmax(s), np.ones(len(s), bool), np.inf
    alpha = O.ALPHA_OF_MODE[mode]
    pw = 1.0 / (alpha - 1.0)
    z = (alpha - 1.0) * s
    tau = optimize.brentq(lambda t: np.sum(np.maximum(z - t, 0) ** pw) - 1.0, z.max() - 1,
                          z.max(), xtol=1e-15, rtol=1e-15)
    return np.maximum(z - tau, 0) ** pw, z > tau, np.abs(z - tau).min()


@pytest.mark.parametrize("mode", [O.SOFTMAX, O.ENTMAX15, O.SPARSEMAX])
def test_selection_quality_against_dense_weights(mode):
    # delta = the full-cache weight outside the kept pages, and the support counts, against a
    # dense scipy evaluation of the full-cache weights
    rng = np.random.default_rng(40)
    for trial in range(8):
        L = int(rng.integers(9, 140))
        k, v, pt = make_seq(rng, L=L, nb=20, dist_scale=2.0)
        n = O.pages_of(L, 8)
        q = rng.standard_normal((3, 16))
        keep = np.sort(rng.choice(n, size=int(rng.integers(0, n + 1)), replace=False)).astype(np.int32)
        dropped, n_sup, n_kept = O.selection_quality_head(k, v, pt, L, 1, q, 0.6, mode, keep)
        in_sel = np.isin(np.arange(L) // 8, keep)
        for g in range(3):
            p, sup, gap = dense_full_cache_weights(k, pt, L, 1, q[g], 0.6, mode)
            assert gap > 1e-9  # no token sits on the threshold
            assert abs(dropped[g] - p[~in_sel].sum()) <= 1e-12
            assert n_sup[g] == sup.sum() and n_kept[g] == (sup & in_sel).sum()


@pytest.mark.parametrize("mode", [O.SOFTMAX, O.ENTMAX15, O.SPARSEMAX])
def test_selection_quality_extremes_and_complement(mode):
    # every page kept drops nothing and keeps the whole support; no page kept drops all the
    # mass; a selection and its complement drop masses that add up to one
    rng = np.random.default_rng(41)
    L = 77
    k, v, pt = make_seq(rng, L=L, nb=20, dist_scale=2.0)
    n = O.pages_of(L, 8)
    q = rng.standard_normal((2, 16))
    d_all, s_all, k_all = O.selection_quality_head(k, v, pt, L, 0, q, 0.8, mode, np.arange(n))
    assert np.all(d_all == 0) and np.array_equal(s_all, k_all) and np.all(s_all > 0)
    d_none, s_none, k_none = O.selection_quality_head(k, v, pt, L, 0, q, 0.8, mode, [])
    np.testing.assert_allclose(d_none, 1.0, atol=1e-12)
    assert np.all(k_none == 0) and np.array_equal(s_none, s_all)
    a = np.array([0, 3, 4, 9], np.int32)
    c = np.setdiff1d(np.arange(n), a).astype(np.int32)
    d_a, _, k_a = O.selection_quality_head(k, v, pt, L, 0, q, 0.8, mode, a)
    d_c, _, k_c = O.selection_quality_head(k, v, pt, L, 0, q, 0.8, mode, c)
    np.testing.assert_allclose(d_a + d_c, 1.0, atol=1e-12)
    np.testing.assert_array_equal(k_a + k_c, s_all)


@pytest.mark.parametrize("mode", [O.SOFTMAX, O.ENTMAX15, O.SPARSEMAX])
def test_selection_quality_given_stat_reproduces_the_full_cache_weights(mode):
    # the full-cache statistic (log-partition or tau) of the attention over every page defines
    # the same weights as that attention; a statistic shifted by 0.05 changes delta
    rng = np.random.default_rng(42)
    L = 100
    k, v, pt = make_seq(rng, L=L, nb=20, dist_scale=2.0)
    n = O.pages_of(L, 8)
    q = rng.standard_normal((2, 16))
    _, stat, _ = O.attend_head(k, v, pt, L, 1, q, 0.7, mode, np.arange(n))
    keep = np.array([1, 2, 7, 11], np.int32)
    own = O.selection_quality_head(k, v, pt, L, 1, q, 0.7, mode, keep)
    given = O.selection_quality_head(k, v, pt, L, 1, q, 0.7, mode, keep, stat=stat)
    np.testing.assert_allclose(given[0], own[0], atol=1e-12)
    np.testing.assert_array_equal(given[1], own[1])
    np.testing.assert_array_equal(given[2], own[2])
    moved = O.selection_quality_head(k, v, pt, L, 1, q, 0.7, mode, keep, stat=stat + 0.05)
    assert np.all(np.abs(moved[0] - own[0]) > 1e-6)


@pytest.mark.parametrize("mode", [O.SOFTMAX, O.ENTMAX15, O.SPARSEMAX])
def test_selection_quality_delta_bounds_the_output_error(mode):
    # §3 with this function's delta: ||o_selected - o_full|| <= 2 B delta, B = max ||v_i||
    rng = np.random.default_rng(43)
    for trial in range(10):
        L = int(rng.integers(9, 120))
        k, v, pt = make_seq(rng, L=L, nb=16, dist_scale=float(rng.choice([0.5, 2.0])))
        n = O.pages_of(L, 8)
        q = rng.standard_normal((2, 16))
        full, _, _ = O.attend_head(k, v, pt, L, 0, q, 0.5, mode, np.arange(n))
        keep = np.sort(rng.choice(n, size=int(rng.integers(1, n + 1)), replace=False)).astype(np.int32)
        out, _, _ = O.attend_head(k, v, pt, L, 0, q, 0.5, mode, keep)
        dropped, _, _ = O.selection_quality_head(k, v, pt, L, 0, q, 0.5, mode, keep)
        B = np.linalg.norm(dense_tokens(v, pt, L, 0), axis=1).max()
        for g in range(2):
            assert np.linalg.norm(out[g] - full[g]) <= 2 * B * dropped[g] + 1e-12
