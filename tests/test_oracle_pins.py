"""Pins for the fp64 oracle: checks against what the pages and the mathematics
fix, never against the oracle itself.

Sources of truth used here:
  * the operator and its constraint, Technical Summary section 2.1 of
    "Fast LapSum: Exact Differentiable Top-k at Million Scale"
    (p_i = F((r_i - b)/t), sum_i p_i = k, F the Laplace CDF);
  * the claim that DFTopK is LapSum's zero-temperature limit (section 2.3);
  * closed forms for one score, all-equal scores and a symmetric pair;
  * independent bisection on the directly summed memberships;
  * finite differences for the backward pass (section 2.1's analytic VJP);
  * published splitmix64 vectors and the Laplace distribution for the
    localization step (section 2.2).
"""
import math
import os

import numpy as np
import pytest

from differentiable_soft_top_b200.workloads import WORKLOADS, make_grad, make_scores

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------------------
# independent helpers (no oracle code): Laplace CDF, its inverse, direct S(b)
# ---------------------------------------------------------------------------
def lap_cdf(z):
    z = np.asarray(z, dtype=np.float64)
    return np.where(z < 0, 0.5 * np.exp(np.minimum(z, 0)), 1.0 - 0.5 * np.exp(-np.maximum(z, 0)))


def lap_icdf(q):
    return math.log(2 * q) if q < 0.5 else -math.log(2 - 2 * q)


def direct_S(r, b, alpha):
    """sum_i F((r_i - b)/alpha), exactly rounded summation of fp64 terms."""
    return math.fsum(lap_cdf((np.asarray(r, np.float64) - b) / alpha).tolist())


def bisect_b(r, k, alpha, iters=200):
    r = np.asarray(r, np.float64)
    n = r.size
    lo = r.min() - alpha * (math.log(n / (2.0 * (n - k))) + 40.0)
    hi = r.max() + alpha * (math.log(n / (2.0 * k)) + 40.0)
    assert direct_S(r, lo, alpha) > k > direct_S(r, hi, alpha)
    for _ in range(iters):
        mid = 0.5 * (lo + hi)
        if mid == lo or mid == hi:
            break
        if direct_S(r, mid, alpha) > k:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


# ---------------------------------------------------------------------------
# random number generator (localization step): published vectors
# ---------------------------------------------------------------------------
def test_splitmix64_published_vectors(orc):
    rows = [ln.split() for ln in open(os.path.join(GOLDEN, "splitmix64_vectors.txt"))
            if ln.strip() and not ln.startswith("#")]
    assert len(rows) == 6
    for seed, idx, out in rows:
        assert orc.sm64_out(int(seed), int(idx)) == int(out)


# ---------------------------------------------------------------------------
# closed forms
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("k", [1e-6, 0.1, 0.5, 0.73, 0.999999])
@pytest.mark.parametrize("alpha", [1e-3, 1.0, 37.0])
def test_single_score_closed_form(orc, k, alpha):
    # n = 1: F((r - b)/alpha) = k  =>  b = r - alpha F^{-1}(k)
    r = np.array([0.8125], np.float64)
    b = orc.threshold(r, k, alpha)
    assert b == pytest.approx(0.8125 - alpha * lap_icdf(k), rel=1e-13, abs=1e-13 * alpha)


@pytest.mark.parametrize("n,k", [(2, 1.0), (5, 0.3), (64, 17.5), (1000, 999.0), (4096, 64.0)])
def test_all_equal_closed_form(orc, n, k):
    # n copies of v: n F((v - b)/alpha) = k  =>  b = v - alpha F^{-1}(k/n)
    v, alpha = -1.375, 0.25
    r = np.full(n, v, np.float64)
    b = orc.threshold(r, k, alpha)
    assert b == pytest.approx(v - alpha * lap_icdf(k / n), rel=1e-12, abs=1e-12)
    p, _, _ = orc.forward(r, k, alpha)
    assert np.allclose(p, k / n, rtol=1e-12, atol=0)


@pytest.mark.parametrize("a,alpha", [(0.5, 1.0), (3.0, 0.01), (1e3, 1.0)])
def test_symmetric_pair(orc, a, alpha):
    # {-a, a} with k = 1: by symmetry b = 0, p = (1 - F(-a/alpha), F(-a/alpha)) swapped
    r = np.array([-a, a], np.float64)
    b = orc.threshold(r, 1.0, alpha)
    assert abs(b) <= 1e-12 * max(1.0, a)
    p, _, _ = orc.forward(r, 1.0, alpha)
    assert p[0] + p[1] == pytest.approx(1.0, abs=1e-15)
    assert p[1] == pytest.approx(1.0 - 0.5 * math.exp(-a / alpha), abs=1e-15)


def test_pair_huge_gap_midpoint(orc):
    # gap of 2000 alpha: every exponential underflows in the plain form; the
    # root is still the midpoint by symmetry
    r = np.array([0.0, 2000.0])
    assert orc.threshold(r, 1.0, 1.0) == pytest.approx(1000.0, abs=1e-9)


# ---------------------------------------------------------------------------
# brute force on tiny rows: exhaustive interval search + bisection
# ---------------------------------------------------------------------------
def brute_force_b(r, k, alpha):
    """Try every one of the n+1 intervals between sorted scores; inside each,
    S is continuous and strictly decreasing, so bisect there if it brackets k.
    Exactly one interval must hold the root."""
    x = np.sort(np.asarray(r, np.float64))
    n = x.size
    edges = [x[0] - alpha * 60.0] + list(x) + [x[-1] + alpha * 60.0]
    roots = []
    for j in range(n + 1):
        lo, hi = edges[j], edges[j + 1]
        slo, shi = direct_S(x, lo, alpha), direct_S(x, hi, alpha)
        if slo >= k >= shi and (j == n or shi < k or lo == hi):
            for _ in range(200):
                mid = 0.5 * (lo + hi)
                if mid in (lo, hi):
                    break
                if direct_S(x, mid, alpha) > k:
                    lo = mid
                else:
                    hi = mid
            roots.append(0.5 * (lo + hi))
    return roots


@pytest.mark.parametrize("seed", range(40))
def test_brute_force_tiny(orc, seed):
    rng = np.random.default_rng(1000 + seed)
    n = int(rng.integers(1, 9))
    scale = [1e-3, 0.1, 1.0, 10.0][seed % 4]
    r = rng.standard_normal(n) * scale
    if seed % 5 == 0 and n > 2:
        r[1] = r[0]  # a tie
    alpha = float(10 ** rng.uniform(-3, 1))
    k = float(rng.uniform(0.02, n - 0.02)) if seed % 3 else float(rng.integers(1, n + 1)) - 0.5
    roots = brute_force_b(r, k, alpha)
    assert len(roots) >= 1
    b = orc.threshold(r, k, alpha)
    assert min(abs(b - t) for t in roots) <= 1e-10 * max(1.0, abs(b)) + 1e-12 * alpha
    assert direct_S(r, b, alpha) == pytest.approx(k, rel=1e-11, abs=1e-11)


# ---------------------------------------------------------------------------
# bisection / direct check on the five workloads (scaled where needed)
# ---------------------------------------------------------------------------
CASES = [
    ("c1", None),
    ("c2", None),
    ("c3", 1_000_000),
    ("c4", 1_000_000),
]


@pytest.mark.parametrize("name,n", CASES)
def test_threshold_matches_direct_sum(orc, name, n):
    w = WORKLOADS[name] if n is None else WORKLOADS[name].scaled(n=n)
    r = make_scores(w)[0].astype(np.float64)
    b = orc.threshold(r, w.k, w.alpha)
    S = direct_S(r, b, w.alpha)
    # the root is exact up to rounding: |S(b) - k| tiny relative to k
    assert abs(S - w.k) <= 1e-9 * w.k
    # and b is pinned: moving it by 1e-9 relative crosses the budget both ways
    d = 1e-9 * max(1.0, abs(b))
    assert direct_S(r, b - d, w.alpha) > w.k > direct_S(r, b + d, w.alpha)


def test_threshold_c1_bisection(orc):
    w = WORKLOADS["c1"]
    r = make_scores(w)[0].astype(np.float64)
    b = orc.threshold(r, w.k, w.alpha)
    assert b == pytest.approx(bisect_b(r, w.k, w.alpha), rel=1e-12)
    assert b > r.max()  # the edge interval beyond every score


def test_tied_batch_rows(orc):
    w = WORKLOADS["c5"]
    x = make_scores("tied_batch", rows=8, n=w.n)
    for i in (0, 3, 7):
        r = x[i].astype(np.float64)
        b = orc.threshold(r, w.k, w.alpha)
        assert abs(direct_S(r, b, w.alpha) - w.k) <= 1e-10 * w.k
    assert len(np.unique(x[3])) <= 16


# ---------------------------------------------------------------------------
# invariants
# ---------------------------------------------------------------------------
def _rand_row(seed, n=777):
    rng = np.random.default_rng(seed)
    return rng.standard_normal(n) * 2.0


def test_budget_sum(orc):
    for seed in range(5):
        r = _rand_row(seed)
        for k in (0.5, 3.0, 100.25, 700.0):
            p, b, _ = orc.forward(r, k, 0.3)
            assert math.fsum(p.tolist()) == pytest.approx(k, rel=1e-12)
            # pages section 4.1: budget relative error below 1e-5
            assert abs(math.fsum(p.tolist()) - k) / k < 1e-5


def test_shift_scale_permutation(orc):
    r = _rand_row(11)
    k, alpha = 42.5, 0.2
    p, b, _ = orc.forward(r, k, alpha)
    c = 1024.0
    p2, b2, _ = orc.forward(r + c, k, alpha)
    assert b2 == pytest.approx(b + c, abs=1e-9)
    assert np.max(np.abs(p2 - p)) < 1e-9
    s = 4.0
    p3, b3, _ = orc.forward(r * s, k, alpha * s)
    assert b3 == pytest.approx(b * s, rel=1e-12, abs=1e-12)
    assert np.max(np.abs(p3 - p)) < 1e-12
    perm = np.random.default_rng(3).permutation(r.size)
    p4, b4, _ = orc.forward(r[perm], k, alpha)
    assert b4 == b
    assert np.array_equal(p4, p[perm])


def test_backward_invariants(orc):
    r = _rand_row(5)
    k, alpha = 50.0, 0.4
    _, b, sf = orc.forward(r, k, alpha)
    g = np.full(r.size, 3.25)
    grad, lam, sf2 = orc.backward(r, g, b, alpha)
    assert lam == pytest.approx(3.25, rel=1e-14)
    assert np.max(np.abs(grad)) < 1e-12
    assert sf2 == pytest.approx(sf, rel=1e-14)
    g = np.random.default_rng(9).standard_normal(r.size)
    grad, lam, _ = orc.backward(r, g, b, alpha)
    assert abs(math.fsum(grad.tolist())) <= 1e-12 * np.sum(np.abs(grad))


# ---------------------------------------------------------------------------
# zero-temperature limit (section 2.3): DFTopK midpoint and hard top-k mask
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("n,k", [(10, 3), (257, 64), (1000, 500), (1000, 1)])
def test_zero_temperature_limit(orc, n, k):
    rng = np.random.default_rng(n + k)
    r = rng.permutation(np.arange(n, dtype=np.float64)) * 1e-3  # distinct, spacing 1e-3
    alpha = 1e-6 * 1e-3
    b = orc.threshold(r, float(k), alpha)
    xs = np.sort(r)[::-1]
    mid = 0.5 * (xs[k - 1] + xs[k])
    assert abs(b - mid) <= 1e-6 * 1e-3
    p, _, _ = orc.forward(r, float(k), alpha)
    mask = (r >= xs[k - 1]).astype(np.float64)
    assert np.max(np.abs(p - mask)) <= 1e-6


# DFTopK (section 2.3): midpoint threshold, no budget; the mass drifts
def test_dftopk_limits(orc):
    rng = np.random.default_rng(11)
    r = rng.standard_normal(3000).astype(np.float32)
    k = 40
    xs = np.sort(r.astype(np.float64))[::-1]
    p, b, mass = orc.dftopk_forward(r, k, 1e-9)
    assert b == 0.5 * (xs[k - 1] + xs[k])
    assert mass == pytest.approx(k, abs=1e-6)           # zero temperature: the hard top-k
    assert np.array_equal(p >= 0.5, r.astype(np.float64) > b)
    _, _, mass_hot = orc.dftopk_forward(r, k, 1e9)
    assert mass_hot == pytest.approx(r.size / 2, rel=1e-6)  # infinite temperature: every p -> 1/2
    _, _, mass_mid = orc.dftopk_forward(r, k, 0.5)
    assert mass_mid > k                                  # the drift the pages cite: mass above k here
    # the LapSum threshold at the same alpha keeps the budget the midpoint loses
    _, b_lap, _ = orc.forward(r, float(k), 0.5)
    assert orc.S(r, b_lap, 0.5) == pytest.approx(k, rel=1e-12)


def test_dftopk_symmetric_pair(orc):
    """r = (-d, d), k = 1: b = 0, p = (e^{-d/a}/2, 1 - e^{-d/a}/2), mass 1."""
    d, a = 0.8, 0.25
    p, b, mass = orc.dftopk_forward(np.array([-d, d], np.float32), 1, a)
    e = 0.5 * math.exp(-float(np.float32(d)) / a)
    assert b == 0.0
    assert p[0] == pytest.approx(e, rel=1e-14) and p[1] == pytest.approx(1 - e, rel=1e-14)
    assert mass == pytest.approx(1.0, rel=1e-15)


# ---------------------------------------------------------------------------
# finite differences for the analytic VJP (section 2.1)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("seed", range(6))
def test_vjp_finite_differences(orc, seed):
    rng = np.random.default_rng(200 + seed)
    n = int(rng.integers(3, 65))
    r = rng.standard_normal(n)
    g = rng.standard_normal(n)
    alpha = float(10 ** rng.uniform(-1, 0.5))
    k = float(rng.uniform(0.5, n - 0.5))
    _, b, _ = orc.forward(r, k, alpha)
    grad, lam, _ = orc.backward(r, g, b, alpha)

    def L(rr, kk=k):
        p, _, _ = orc.forward(rr, kk, alpha)
        return float(np.dot(g, p))

    h = 1e-6
    fd = np.empty(n)
    for j in range(n):
        e = np.zeros(n)
        e[j] = h
        fd[j] = (L(r + e) - L(r - e)) / (2 * h)
    assert np.linalg.norm(fd - grad) <= 1e-6 * max(1e-12, np.linalg.norm(grad)) + 1e-9
    fdk = (L(r, k + h) - L(r, k - h)) / (2 * h)
    assert fdk == pytest.approx(lam, rel=1e-6, abs=1e-9)


# dL/dalpha: the threshold moves with alpha (section 2.1's constraint)
@pytest.mark.parametrize("seed", range(6))
def test_alpha_gradient_finite_differences(orc, seed):
    rng = np.random.default_rng(300 + seed)
    n = int(rng.integers(3, 65))
    r = rng.standard_normal(n)
    g = rng.standard_normal(n)
    alpha = float(10 ** rng.uniform(-1, 0.5))
    k = float(rng.uniform(0.5, n - 0.5))
    _, b, _ = orc.forward(r, k, alpha)
    da = orc.backward_alpha(r, g, b, alpha)

    def L(a):
        p, _, _ = orc.forward(r, k, a)
        return float(np.dot(g, p))

    h = 1e-6 * alpha
    fd = (L(alpha + h) - L(alpha - h)) / (2 * h)
    assert da == pytest.approx(fd, rel=1e-6, abs=1e-9)


def test_alpha_gradient_symmetric_pair(orc):
    """r = (-d, d), k = 1: b = 0 for every alpha, so p_1 = e^{-d/a}/2 and
    p_2 = 1 - e^{-d/a}/2, and dL/da = (g_1 - g_2) e^{-d/a} d / (2 a^2)."""
    d, a = 0.7, 0.3
    r = np.array([-d, d])
    g = np.array([1.3, -0.4])
    _, b, _ = orc.forward(r, 1.0, a)
    assert abs(b) < 1e-15
    expect = (g[0] - g[1]) * math.exp(-d / a) * d / (2 * a * a)
    assert orc.backward_alpha(r, g, b, a) == pytest.approx(expect, rel=1e-12)


def test_alpha_gradient_constant_upstream_is_zero(orc):
    """g = c: L = c * k does not depend on alpha."""
    rng = np.random.default_rng(7)
    r = rng.standard_normal(50)
    _, b, _ = orc.forward(r, 12.5, 0.4)
    assert abs(orc.backward_alpha(r, np.full(50, 2.5), b, 0.4)) < 1e-12


# ---------------------------------------------------------------------------
# localization step (section 2.2): samples, ranks, tails, coverage
# ---------------------------------------------------------------------------
def test_laplace_noise_distribution(orc):
    r = np.zeros(16, np.float32)
    m, alpha = 200_000, 0.7
    Y, idx, eps = orc.sample(r, alpha, 12345, 0, m)
    z = np.sort(eps / alpha)
    F = lap_cdf(z)
    ecdf_hi = np.arange(1, m + 1) / m
    ecdf_lo = np.arange(0, m) / m
    D = max(np.max(ecdf_hi - F), np.max(F - ecdf_lo))
    assert D < 1.63 / math.sqrt(m)  # KS test at the 1% level
    counts = np.bincount(idx, minlength=16)
    chi2 = np.sum((counts - m / 16) ** 2 / (m / 16))
    assert chi2 < 37.7  # chi-square, 15 dof, 0.1% level
    assert np.array_equal(Y, (r[idx].astype(np.float64) + eps).astype(np.float32))


# ---------------------------------------------------------------------------
# the bracket's ranks against the binomial law they must follow
# ---------------------------------------------------------------------------
# Technical summary section 2.2, step 1: with Laplace noise at the scale alpha,
# P(Y_j > b) = (1/n) sum_i F((r_i - b)/alpha) = k/n exactly, so the number of
# samples above b is X ~ Binomial(m, q = k/n).  The bracket edges are order
# statistics at ranks placed z standard deviations either side of the mean,
# so each edge misses b with probability close to Phi(-z):
#   b >= a_R  <=>  X <= c_lo - 1,        b < a_L  <=>  X >= c_hi + 1.
# Normal approximation with the Berry-Esseen bound for a binomial
# (|P(X <= x) - Phi((x - mq)/s)| <= 0.4748 (q^2 + (1-q)^2) / s, s = sqrt(mq(1-q))),
# and the rounding of the ranks to integers (at most one unit, 1/s in z):
#   Phi(-z - 2/s) - BE  <=  P(miss on either side)  <=  Phi(-z) + BE.
def _phi(x):
    return 0.5 * math.erfc(-x / math.sqrt(2.0))


def _miss_band(m, q, z):
    s = math.sqrt(m * q * (1.0 - q))
    be = 0.4748 * (q * q + (1.0 - q) ** 2) / s
    return max(0.0, _phi(-z - 2.0 / s) - be), min(1.0, _phi(-z) + be)


RANK_CASES = [  # (n, k, m): q = 1/64 (c1), 1/100 (c2), 1/2 and 9/10, where the (1 - q) factor matters
    (4096, 64.0, 1 << 16), (10**6, 1e4, 1 << 17), (10**5, 5e4, 1 << 16), (10**5, 9e4, 1 << 16),
]


def check_rank_miss_probabilities(o):
    from scipy.stats import binom
    for n, k, m in RANK_CASES:
        q = k / n
        for z in (1.0, 2.0, 4.0):
            lo, hi = o.sample_ranks(n, k, m, z)
            p_right = float(binom.cdf(lo - 1, m, q))  # P(X <= c_lo - 1): b at or above a_R
            p_left = float(binom.sf(hi, m, q))        # P(X >= c_hi + 1): b below a_L
            band = _miss_band(m, q, z)
            assert band[0] <= p_right <= band[1], (n, k, m, z, lo, p_right, band)
            assert band[0] <= p_left <= band[1], (n, k, m, z, hi, p_left, band)


def test_sample_ranks_reach_the_binomial_miss_probability(orc):
    """Exact binomial tails at the oracle's ranks (scipy's binomial, not the
    oracle's arithmetic) against the miss probability Phi(-z) the ranks are
    meant to give; a variance without its (1 - q) factor, or a half-width on
    one side only, lands far outside the band at q = 1/2 and 9/10."""
    check_rank_miss_probabilities(orc)


MISS_CASES = [  # (name, n, k, alpha, m): c1 as is, c2 scaled to 1e5, and a budget of half the row
    ("c1", 4096, 64.0, 1.0, 8192), ("c2", 100_000, 1000.0, 0.1, 8192), ("half", 100_000, 50_000.0, 0.1, 8192),
]


def check_bracket_miss_rates(o, trials=1000, cases=MISS_CASES):
    """Draw the bracket with `trials` seeds and count how often each edge
    misses the oracle's threshold; each count must lie in the 99.9% binomial
    range of `trials` draws at the miss probability band above."""
    from scipy.stats import binom
    for name, n, k, alpha, m in cases:
        dist = "uniform" if name == "half" else ("normal" if name != "c3" else "mixture")
        r = make_scores(dist, 1, n, seed=0)[0]
        b = o.threshold(r, k, alpha)
        for z in (1.0, 2.0):
            miss_r = miss_l = 0
            for seed in range(trials):
                aL, aR, _, _ = o.bracket(r, k, alpha, m, z, seed)
                miss_r += int(b >= aR)
                miss_l += int(b < aL)
            lo_p, hi_p = _miss_band(m, k / n, z)
            lo_c, hi_c = binom.ppf(0.0005, trials, lo_p), binom.ppf(0.9995, trials, hi_p)
            assert lo_c <= miss_r <= hi_c, (name, z, "right edge", miss_r, (lo_c, hi_c))
            assert lo_c <= miss_l <= hi_c, (name, z, "left edge", miss_l, (lo_c, hi_c))


def test_bracket_miss_rates_follow_the_binomial(orc):
    """The sampled bracket (noise, indices, order statistics) misses b on
    each side at the rate the binomial law of section 2.2 fixes."""
    check_bracket_miss_rates(orc)


@pytest.mark.parametrize("name,n", [("c1", None), ("c2", None), ("c3", 1_000_000), ("c4", 2_000_000)])
def test_tails_certify_identity(orc, name, n):
    """S at the bracket edges from the tail aggregates alone equals the direct sum."""
    w = WORKLOADS[name] if n is None else WORKLOADS[name].scaled(n=n)
    r32 = make_scores(w)[0]
    r = r32.astype(np.float64)
    m = min(w.n, 1 << 16)
    aL, aR, _, _ = orc.bracket(r32, w.k, w.alpha, m, 5.0, 0)
    nL, SL, nR, SR, M = orc.tails(r32, aL, aR, w.alpha)
    assert nL + nR + M == w.n
    assert nL == int(np.sum(r < aL)) and nR == int(np.sum(r >= aR))
    band = r[(r >= aL) & (r < aR)]
    for e in (aL, aR):
        if not np.isfinite(e):
            continue
        left = 0.5 * SL * math.exp((aL - e) / w.alpha) if np.isfinite(aL) else 0.0
        right = nR - 0.5 * SR * math.exp((e - aR) / w.alpha) if np.isfinite(aR) else 0.0
        S_tails = left + math.fsum(lap_cdf((band - e) / w.alpha).tolist()) + right
        assert S_tails == pytest.approx(direct_S(r, e, w.alpha), rel=1e-10, abs=1e-9)


@pytest.mark.parametrize("name", ["c1", "c2"])
def test_bracket_coverage(orc, name):
    w = WORKLOADS[name]
    r = make_scores(w)[0]
    b = orc.threshold(r, w.k, w.alpha)
    m = min(w.n, 1 << 15)
    for seed in range(20):
        aL, aR, lo, hi = orc.bracket(r, w.k, w.alpha, m, 5.0, seed)
        assert aL <= b < aR


def test_bracket_order_statistics(orc):
    r = make_scores("normal", 1, 5000, seed=4)[0]
    m = 1000
    Y, _, _ = orc.sample(r, 0.5, 77, 3, m)
    aL, aR, lo, hi = orc.bracket(r, 500.0, 0.5, m, 5.0, 77, 3)
    Ys = np.sort(Y)
    assert 1 <= lo and hi + 1 <= m
    assert aR == Ys[m - lo] and aL == Ys[m - hi - 1]
    assert np.sum(Y >= aR) >= lo and np.sum(Y > aL) <= hi
    # a small budget leaves the bracket open above: c_lo < 1 gives a_R = +inf
    aL2, aR2, lo2, hi2 = orc.bracket(r, 5.0, 0.5, m, 5.0, 77, 3)
    assert lo2 < 1 and aR2 == np.inf and aL2 == Ys[m - hi2 - 1]
