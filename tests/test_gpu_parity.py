"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Tolerances (fp32 outputs):
  max |p_gpu - p_ref|                          <= 1e-5
  |sum p_gpu - k|                              <= 1e-3 max(1,k) sqrt(n/1e6)
  ||grad_gpu - grad_ref||_2 / ||grad_ref||_2   <= 1e-4
and, as a diagnostic of the threshold itself, |b_gpu - b_ref| small against
alpha (the fp64 b must agree far below the p tolerance: dp/db <= 1/(2 alpha)).
Every input is seeded and synthetic (differentiable_soft_top_b200.workloads).
"""
import math

import numpy as np
import pytest

import differentiable_soft_top_b200 as lt
from differentiable_soft_top_b200.workloads import WORKLOADS, make_grad, make_scores

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)


def tol_sum(k, n):
    return 1e-3 * max(1.0, k) * math.sqrt(n / 1e6)


def gpu_run(x_np, g_np, k, alpha, params=None, stats=False):
    x = torch.from_numpy(np.ascontiguousarray(x_np)).cuda()
    g = torch.from_numpy(np.ascontiguousarray(g_np)).cuda()
    res = lt.forward(x, k, alpha, params=params, stats=stats)
    grad, gk = lt.backward(x, g, res.b, alpha)
    torch.cuda.synchronize()
    return dict(p=res.p.cpu().numpy(), b=res.b.cpu().numpy(), sumf=res.sumf.cpu().numpy(),
                status=res.status.cpu().numpy().astype(np.uint32), stats=res.stats,
                grad=grad.cpu().numpy(), gk=gk.cpu().numpy())


def check_row(orc, r, g, p, grad, b, gk, k, alpha, label="", pure=False):
    """The GPU outputs of one row against the oracle.  The gradient must meet
    the relative L2 bound 1e-4 up to the floor an fp32 result cannot beat
    (terms f g rounded to fp32 before g - lambda cancels; values flushed below
    the smallest normal fp32 number); with `pure`, the plain relative error
    ||grad - grad_ref|| / ||grad_ref|| <= 1e-4 must hold as well, with no
    floor."""
    r = np.asarray(r, np.float32).reshape(-1)
    gg = np.asarray(g, np.float32).reshape(-1)
    n = r.size
    p_ref, b_ref, sumf_ref = orc.forward(r, k, alpha)
    grad_ref, lam, _ = orc.backward(r, gg, b_ref, alpha)
    p = np.asarray(p, np.float64).reshape(-1)
    grad = np.asarray(grad, np.float64).reshape(-1)
    dp = float(np.max(np.abs(p - p_ref)))
    assert dp <= 1e-5, f"{label} max|dp|={dp:.3e} b_gpu={b!r} b_ref={b_ref!r}"
    sp = math.fsum(p.tolist())
    assert abs(sp - k) <= tol_sum(k, n), f"{label} sum p={sp} k={k}"
    # relative L2 error of the gradient, with the floor an fp32 output cannot
    # beat: rounding of the terms f g (6e-8 each, 16x margin) and values below
    # the smallest normal fp32 number
    f = 0.5 * np.exp(-np.abs(r.astype(np.float64) - b_ref) / alpha) / alpha
    err = float(np.linalg.norm(grad - grad_ref))
    ref_norm = float(np.linalg.norm(grad_ref))
    rel = err / ref_norm if ref_norm > 0 else (0.0 if err == 0 else math.inf)
    bound = 1e-4 * ref_norm + 1e-6 * float(np.linalg.norm(f * gg)) + 1.2e-38 * math.sqrt(n)
    assert err <= bound, f"{label} grad err {err:.3e} > {bound:.3e} (ref norm {ref_norm:.3e}, relative {rel:.3e})"
    if pure:
        assert rel <= 1e-4, f"{label} relative gradient error {rel:.3e} > 1e-4"
    # b: far inside the p tolerance (dp/db <= 1/(2 alpha)); fp32 tail sums allow ~1e-6 alpha
    assert abs(b - b_ref) <= 2e-6 * alpha + 1e-12 * abs(b_ref), f"{label} b {b!r} vs {b_ref!r}"
    assert gk == pytest.approx(lam, rel=1e-4, abs=1e-6 * (1 + abs(lam)))
    return b_ref


def case(name, n=None, rows=None):
    w = WORKLOADS[name]
    if n is not None or rows is not None:
        w = w.scaled(n=n, rows=rows)
    return w, make_scores(w), make_grad(w.rows, w.n)


# ---------------------------------------------------------------------------
# the five workloads
# ---------------------------------------------------------------------------
def test_c1_single_row_4096(orc):
    w, x, g = case("c1")
    out = gpu_run(x, g, w.k, w.alpha, stats=True)
    check_row(orc, x[0], g[0], out["p"], out["grad"], out["b"][0], out["gk"][0], w.k, w.alpha, "c1", pure=True)
    assert out["status"][0] & lt.ROW_CERTIFIED


def test_c5_tied_batch(orc):
    w, x, g = case("c5")
    out = gpu_run(x, g, w.k, w.alpha)
    assert np.all(out["status"] & lt.ROW_CERTIFIED)
    for i in range(w.rows):
        check_row(orc, x[i], g[i], out["p"][i], out["grad"][i], out["b"][i], out["gk"][i], w.k, w.alpha,
                  f"c5 row {i}", pure=True)


def test_c2_1e6(orc):
    w, x, g = case("c2")
    out = gpu_run(x, g, w.k, w.alpha, stats=True)
    check_row(orc, x[0], g[0], out["p"], out["grad"], out["b"][0], out["gk"][0], w.k, w.alpha, "c2", pure=True)
    assert out["status"][0] == lt.ROW_CERTIFIED


def test_c3_1e7_mixture(orc):
    w, x, g = case("c3")
    out = gpu_run(x, g, w.k, w.alpha, stats=True)
    check_row(orc, x[0], g[0], out["p"], out["grad"], out["b"][0], out["gk"][0], w.k, w.alpha, "c3", pure=True)
    assert out["status"][0] == lt.ROW_CERTIFIED


@pytest.mark.slow
def test_c4_1e8_uniform(orc):
    """Full size, same launch configuration as bench.py; every output compared."""
    w, x, g = case("c4")
    out = gpu_run(x, g, w.k, w.alpha, stats=True)
    assert out["status"][0] == lt.ROW_CERTIFIED
    check_row(orc, x[0], g[0], out["p"], out["grad"], out["b"][0], out["gk"][0], w.k, w.alpha, "c4", pure=True)


# ---------------------------------------------------------------------------
# sizes spanning several tiles with ragged tails, strides, several rows
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("n", [4097, 16383, 16385, 100_003, 1_000_001])
def test_ragged_sizes(orc, n):
    x = make_scores("normal", 1, n, seed=n)
    g = make_grad(1, n, seed=n + 1)
    k, alpha = n / 37.0, 0.3
    out = gpu_run(x, g, k, alpha)
    check_row(orc, x[0], g[0], out["p"], out["grad"], out["b"][0], out["gk"][0], k, alpha, f"n={n}")


@pytest.mark.parametrize("n,force", [(3000, lt.FORCE_NONE), (5000, lt.FORCE_NONE), (5000, lt.FORCE_STREAMING),
                                     (12001, lt.FORCE_NONE), (70001, lt.FORCE_NONE)])
def test_strided_unaligned_rows(orc, n, force):
    # scores start 4 bytes past the 16-byte grid, row stride n + 3; the
    # binding places p and grad at the same address mod 16
    rows, stride = 3, n + 3
    base = make_scores("mixture", rows, stride, seed=7)
    gb = make_grad(rows, stride, seed=8)
    xt = torch.from_numpy(base).cuda()[:, 1:n + 1]  # 4-byte aligned only, row stride n+3
    gt = torch.from_numpy(gb).cuda()[:, 1:n + 1]
    k, alpha = 123.5, 0.07
    params = lt.Params(force_path=force)
    res = lt.forward(xt, k, alpha, params=params)
    grad, gk = lt.backward(xt, gt, res.b, alpha)
    torch.cuda.synchronize()
    p, b = res.p.cpu().numpy(), res.b.cpu().numpy()
    for i in range(rows):
        check_row(orc, base[i, 1:n + 1], gb[i, 1:n + 1], p[i], grad.cpu().numpy()[i], b[i], gk.cpu().numpy()[i],
                  k, alpha, f"strided row {i}")


@pytest.mark.parametrize("n", [3000, 70001])
def test_one_row_with_any_row_stride(orc, n):
    # a single row whose row stride is 0 (numpy's [None, :] view) or short
    x = make_scores("normal", 1, n, seed=9)
    g = make_grad(1, n, seed=10)
    k, alpha = 77.0, 0.1
    dense = gpu_run(x, g, k, alpha)
    for s0 in (0, 1):
        xt = torch.from_numpy(x).cuda().as_strided((1, n), (s0, 1))
        gt = torch.from_numpy(g).cuda().as_strided((1, n), (s0, 1))
        res = lt.forward(xt, k, alpha)
        grad, gk = lt.backward(xt, gt, res.b, alpha)
        assert np.array_equal(res.p.cpu().numpy(), dense["p"]) and np.array_equal(grad.cpu().numpy(), dense["grad"])
    check_row(orc, x[0], g[0], dense["p"], dense["grad"], dense["b"][0], dense["gk"][0], k, alpha, f"one row n={n}")


@pytest.mark.parametrize("n,force", [(3000, lt.FORCE_NONE), (12001, lt.FORCE_NONE), (70001, lt.FORCE_NONE)])
def test_outputs_off_the_scores_phase(orc, n, force):
    # p and grad given by the caller 4 bytes further along the 16-byte grid
    # than the scores: the passes that write take every score one at a time
    rows, stride = 3, n + 3
    base = make_scores("mixture", rows, stride, seed=9)
    gb = make_grad(rows, stride, seed=10)
    xt = torch.from_numpy(base).cuda()[:, 1:n + 1]
    gt = torch.from_numpy(gb).cuda()[:, 1:n + 1]
    p_out = torch.empty(rows * stride + 4, device="cuda").as_strided((rows, n), (stride, 1), storage_offset=2)
    g_out = torch.empty(rows * stride + 4, device="cuda").as_strided((rows, n), (stride, 1), storage_offset=2)
    assert (p_out.data_ptr() - xt.data_ptr()) % 16 != 0
    k, alpha = 97.5, 0.07
    res = lt.forward(xt, k, alpha, params=lt.Params(force_path=force), p_out=p_out)
    grad, gk = lt.backward(xt, gt, res.b, alpha, grad_out=g_out)
    torch.cuda.synchronize()
    p, b = p_out.cpu().numpy(), res.b.cpu().numpy()
    for i in range(rows):
        check_row(orc, base[i, 1:n + 1], gb[i, 1:n + 1], p[i], g_out.cpu().numpy()[i], b[i],
                  gk.cpu().numpy()[i], k, alpha, f"outputs off phase, row {i}")


@pytest.mark.parametrize("n,force", [(3001, lt.FORCE_NONE), (4095, lt.FORCE_NONE), (5001, lt.FORCE_NONE),
                                     (12001, lt.FORCE_NONE), (16383, lt.FORCE_NONE), (5001, lt.FORCE_STREAMING),
                                     (70001, lt.FORCE_NONE)])
def test_odd_n_rows_start_off_the_16_byte_grid(orc, n, force):
    # contiguous rows of odd length start at every address mod 16 in turn
    # (head of 0-3 scores before the float4 body); one-block rows copied to
    # shared memory (n <= 4096) and read from global memory, and streaming rows
    rows = 5
    x = make_scores("mixture", rows, n, seed=n + 11)
    g = make_grad(rows, n, seed=n + 12)
    k, alpha = n / 41.0, 0.05
    out = gpu_run(x, g, k, alpha, params=lt.Params(force_path=force))
    for i in range(rows):
        check_row(orc, x[i], g[i], out["p"][i], out["grad"][i], out["b"][i], out["gk"][i], k, alpha,
                  f"n={n} row {i}")


def test_many_rows_streaming(orc):
    rows, n = 5, 40_000
    x = make_scores("normal", rows, n, seed=3)
    g = make_grad(rows, n, seed=4)
    out = gpu_run(x, g, 400.0, 0.2)
    for i in range(rows):
        check_row(orc, x[i], g[i], out["p"][i], out["grad"][i], out["b"][i], out["gk"][i], 400.0, 0.2, f"row {i}")


# ---------------------------------------------------------------------------
# edge cases and degenerate inputs
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("n,k,alpha", [
    (1, 0.5, 1.0), (1, 1e-6, 0.01), (2, 1.0, 0.5), (3, 2.999, 0.1), (7, 1e-4, 2.0),
    (4096, 1e-3, 0.5), (4096, 4095.9, 0.5), (4096, 2048.0, 1e-6), (4096, 64.0, 1e6),
    (100_000, 1.5, 1e-4), (100_000, 99_990.0, 0.3), (100_000, 50_000.0, 10.0),
])
def test_edge_budgets_and_temperatures(orc, n, k, alpha):
    x = make_scores("normal", 1, n, seed=n + 17)
    g = make_grad(1, n, seed=n + 18)
    out = gpu_run(x, g, k, alpha)
    check_row(orc, x[0], g[0], out["p"], out["grad"], out["b"][0], out["gk"][0], k, alpha, f"n={n} k={k}")


@pytest.mark.parametrize("n", [5000, 300_000])
def test_all_equal_scores(orc, n):
    x = np.full((1, n), 0.25, np.float32)
    g = make_grad(1, n, seed=2)
    out = gpu_run(x, g, n / 3.0, 0.5)
    check_row(orc, x[0], g[0], out["p"], out["grad"], out["b"][0], out["gk"][0], n / 3.0, 0.5, "all-equal")


@pytest.mark.parametrize("n", [6000, 200_000])
def test_signed_zeros_and_large_magnitudes(orc, n):
    x = make_scores("normal", 1, n, seed=5)
    x[0, ::7] = 0.0
    x[0, 3::7] = -0.0
    x[0, 5::97] = 3e30
    x[0, 6::97] = -3e30
    g = make_grad(1, n, seed=6)
    k = n / 10.0
    out = gpu_run(x, g, k, 0.05)
    check_row(orc, x[0], g[0], out["p"], out["grad"], out["b"][0], out["gk"][0], k, 0.05, "zeros/large")


@pytest.mark.parametrize("n", [3000, 50_000])
def test_nonfinite_rows_flagged(orc, n):
    x = make_scores("normal", 3, n, seed=9)
    g = make_grad(3, n, seed=10)
    x[1, n // 2] = np.nan
    x[2, 7] = np.inf
    out = gpu_run(x, g, 30.0, 0.5)
    assert out["status"][1] & lt.ROW_NONFINITE
    assert out["status"][2] & lt.ROW_NONFINITE
    assert not (out["status"][0] & lt.ROW_NONFINITE)
    check_row(orc, x[0], g[0], out["p"][0], out["grad"][0], out["b"][0], out["gk"][0], 30.0, 0.5, "finite row")


# ---------------------------------------------------------------------------
# the rare branches: widening, band overflow, full-sort fallback
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("name,n", [("c1", None), ("c2", None), ("c5", 2048)])
@pytest.mark.parametrize("force", [lt.FORCE_NONE, lt.FORCE_STREAMING])
def test_forced_paths_give_the_same_threshold(orc, name, n, force):
    w, x, g = case(name, n=n) if name != "c5" else case("c5", rows=8)
    x, g = x[:2], g[:2]
    base = gpu_run(x, g, w.k, w.alpha, params=lt.Params(force_path=force))
    runs = [base]
    fb = gpu_run(x, g, w.k, w.alpha, params=lt.Params(force_path=force | lt.FORCE_FALLBACK))
    assert np.all(fb["status"] & lt.ROW_FALLBACK)
    runs.append(fb)
    ovf = gpu_run(x, g, w.k, w.alpha, params=lt.Params(force_path=force, band_capacity=8))
    # a row whose band outgrows 8 slots must take the fallback
    assert np.all(((ovf["status"] & lt.ROW_OVERFLOW) == 0) | ((ovf["status"] & lt.ROW_FALLBACK) != 0))
    runs.append(ovf)
    # a very narrow bracket (z = 0.02) misses b for many seeds: find one whose
    # miss is repaired by the widening, and one whose miss goes straight to the
    # full sort when widening is switched off
    widened = nowiden = None
    for seed in range(24):
        o = gpu_run(x, g, w.k, w.alpha, params=lt.Params(force_path=force, z=0.02, seed=seed))
        if widened is None and np.any(o["status"] & lt.ROW_WIDENED):
            widened = o
        o2 = gpu_run(x, g, w.k, w.alpha, params=lt.Params(force_path=force, z=0.02, seed=seed, max_widen=0))
        assert not np.any(o2["status"] & lt.ROW_WIDENED)
        if nowiden is None and np.any(o2["status"] & lt.ROW_FALLBACK):
            nowiden = o2
        if widened is not None and nowiden is not None:
            break
    assert widened is not None and nowiden is not None
    runs += [widened, nowiden]
    for o in runs:
        assert np.all(o["status"] & lt.ROW_CERTIFIED)
        for i in range(x.shape[0]):
            check_row(orc, x[i], g[i], o["p"][i], o["grad"][i], o["b"][i], o["gk"][i], w.k, w.alpha, name)
            # paths differ only in which sums use fp32 exp (tails) or fp64 (band, fallback)
            assert abs(o["b"][i] - base["b"][i]) <= 4e-6 * w.alpha + 1e-12 * abs(base["b"][i])


@pytest.mark.parametrize("name,rows", [("c2", None), ("c5", 4)])
def test_band_overflow_takes_the_fallback(orc, name, rows):
    w, x, g = case(name, rows=rows)
    # z = 5: a bracket wide enough that every row's band holds more than 8
    # scores (at z = 4 a tied row's bracket can open above all its scores,
    # with an empty band that certifies)
    o = gpu_run(x, g, w.k, w.alpha, params=lt.Params(band_capacity=8, z=5.0))
    assert np.all(o["status"] & lt.ROW_OVERFLOW) and np.all(o["status"] & lt.ROW_FALLBACK)
    for i in range(x.shape[0]):
        check_row(orc, x[i], g[i], o["p"][i], o["grad"][i], o["b"][i], o["gk"][i], w.k, w.alpha, f"{name} row {i}")


def test_widened_rows_report_it(orc):
    w, x, g = case("c2")
    seen = 0
    for seed in range(6):
        o = gpu_run(x, g, w.k, w.alpha, params=lt.Params(z=0.3, seed=seed))
        check_row(orc, x[0], g[0], o["p"], o["grad"], o["b"][0], o["gk"][0], w.k, w.alpha, f"z=0.3 seed {seed}")
        seen |= int(o["status"][0])
    assert seen & (lt.ROW_WIDENED | lt.ROW_FALLBACK)


@pytest.mark.parametrize("n", [3000, 16384])
def test_widened_one_block_rows(orc, n):
    # a narrow bracket (z = 0.3) misses often: the one-block path then sorts
    # its sample and widens; rows in shared and in global memory
    w, x, g = case("c5", n=n, rows=24)
    o = gpu_run(x, g, w.k, w.alpha, params=lt.Params(z=0.3, seed=5))
    for i in range(w.rows):
        check_row(orc, x[i], g[i], o["p"][i], o["grad"][i], o["b"][i], o["gk"][i], w.k, w.alpha,
                  f"n={n} z=0.3 row {i}")
    assert np.any(o["status"] & lt.ROW_WIDENED)


# ---------------------------------------------------------------------------
# the localization step against the oracle's own sample (same splitmix64)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("name,n", [("c1", None), ("c2", None), ("c3", 2_000_000), ("c5", None)])
def test_bracket_and_tails_match_oracle(orc, name, n):
    w, x, g = case(name, n=n) if name != "c5" else case("c5", rows=4)
    out = gpu_run(x, g, w.k, w.alpha, stats=True, params=lt.Params(seed=123))  # z: the library default
    for i in range(x.shape[0]):
        st = out["stats"][i]
        assert st["status"] == lt.ROW_CERTIFIED  # the first bracket held (checked with the oracle at z = 4)
        aL, aR, _, _ = orc.bracket(x[i], w.k, w.alpha, int(st["sample_m"]), lt.DEFAULT_Z, 123, i)
        assert np.float32(st["a_L"]) == np.float32(aL) and np.float32(st["a_R"]) == np.float32(aR)
        nL, SL, nR, SR, M = orc.tails(x[i], aL, aR, w.alpha)
        assert (st["n_L"], st["n_R"], st["band"]) == (nL, nR, M)
        assert st["S_L"] == pytest.approx(SL, rel=2e-6, abs=1e-30)
        assert st["S_R"] == pytest.approx(SR, rel=2e-6, abs=1e-30)
        assert st["sum_p"] == pytest.approx(w.k, abs=tol_sum(w.k, w.n))
        assert st["sum_f"] == pytest.approx(out["sumf"][i])


@pytest.mark.parametrize("dist,n,k", [
    ("normal", 4096, 64.0),       # the two ranks in different first-level bins (~60 keys and 1)
    ("uniform", 16384, 256.0),    # both ranks in one first-level bin of ~200 keys
    ("uniform", 16384, 8192.0),   # ranks near the median, bins of ~370 and ~510 keys
])
def test_one_block_bracket_selection_matches_oracle(orc, dist, n, k):
    """The one-block path selects the bracket's two sample ranks by a radix
    selection in the block (no sort of the sample): the oracle's order
    statistics exactly, whether the two ranks share first-level bins or not."""
    rows, alpha = 3, 0.05
    x = make_scores(dist, rows, n, seed=21)
    g = make_grad(rows, n, seed=22)
    out = gpu_run(x, g, k, alpha, stats=True, params=lt.Params(seed=7))
    for i in range(rows):
        st = out["stats"][i]
        aL, aR, _, _ = orc.bracket(x[i], k, alpha, int(st["sample_m"]), lt.DEFAULT_Z, 7, i)
        assert np.float32(st["a_L"]) == np.float32(aL) and np.float32(st["a_R"]) == np.float32(aR), f"row {i}"
        check_row(orc, x[i], g[i], out["p"][i], out["grad"][i], out["b"][i], out["gk"][i], k, alpha, f"row {i}")


def test_deterministic():
    w, x, g = case("c3", n=3_000_000)
    a = gpu_run(x, g, w.k, w.alpha)
    b = gpu_run(x, g, w.k, w.alpha)
    assert np.array_equal(a["p"], b["p"]) and np.array_equal(a["b"], b["b"])
    assert np.array_equal(a["grad"], b["grad"])


def test_deterministic_with_a_band_cluster():
    """A band split over a cluster of CTAs (the 1e8 workload's regime): the
    band arrives in a different order each call and is sliced differently,
    yet the bin sums are exact integers anchored at the cluster's extremes,
    so every result is bit-identical."""
    n = 30_000_000
    x = make_scores("uniform", 1, n, seed=3)
    g = make_grad(1, n, seed=4)
    k, alpha = 3e5, 1e-3
    runs = [gpu_run(x, g, k, alpha) for _ in range(3)]
    st = runs[0]["stats"]
    for r in runs[1:]:
        assert np.array_equal(runs[0]["b"], r["b"]) and np.array_equal(runs[0]["sumf"], r["sumf"])
        assert np.array_equal(runs[0]["p"], r["p"]) and np.array_equal(runs[0]["grad"], r["grad"])
    res = lt.forward(torch.from_numpy(x).cuda(), k, alpha, stats=True)
    assert int(res.stats[0]["band"]) > 2 * 16384  # more than one CTA of the cluster bins it


def test_small_band_sorted_whole_or_binned(orc):
    """A lone band CTA sorts a band of at most 4096 values whole and solves
    it as one run (no key bins); a band whose ties crowd one bucket of the
    bucket pass is binned instead.  Both give the oracle's result."""
    n, k, alpha = 200_000, 2000.0, 0.05
    rng = np.random.default_rng(11)
    smooth = rng.standard_normal((1, n)).astype(np.float32)
    tied = (np.round(smooth.astype(np.float64) * 64) / 64).astype(np.float32)  # ~80 ties a level at b
    g = rng.standard_normal((1, n)).astype(np.float32)
    for x, run in ((smooth, True), (tied, False)):
        out = gpu_run(x, g, k, alpha, stats=True)
        st = out["stats"][0]
        assert 0 < int(st["band"]) <= 4096
        assert (int(st["buckets"]) == 0) == run, f"buckets {int(st['buckets'])}, band {int(st['band'])}"
        assert out["status"][0] & lt.ROW_CERTIFIED
        check_row(orc, x[0], g[0], out["p"], out["grad"], out["b"][0], out["gk"][0], k, alpha, f"run={run}")


def test_autograd_wrapper(orc):
    w, x, g = case("c1")
    xt = torch.from_numpy(x[0]).cuda().requires_grad_(True)
    p = lt.soft_topk(xt, w.k, w.alpha)
    p.backward(torch.from_numpy(g[0]).cuda())
    res = lt.forward(xt.detach(), w.k, w.alpha)
    g1, _ = lt.backward(xt.detach(), torch.from_numpy(g[0]).cuda(), res.b, w.alpha)
    assert torch.equal(xt.grad, g1)
    assert lt.launch_count() > 0


def test_sumf_matches_oracle(orc):
    for name, n in (("c1", None), ("c2", None), ("c5", None)):
        w, x, g = case(name, n=n) if name != "c5" else case("c5", rows=4)
        out = gpu_run(x, g, w.k, w.alpha)
        for i in range(x.shape[0]):
            _, _, sf = orc.forward(x[i], w.k, w.alpha)
            assert out["sumf"][i] == pytest.approx(sf, rel=1e-5)


def test_deep_underflow_gradient_stays_finite(orc):
    """alpha far below the score spacing: every f is below the fp32 range, yet
    lambda (= dL/dk) is finite and the gradient is zero, not NaN."""
    n = 4096
    x = (np.arange(n, dtype=np.float64) * 1e-2).astype(np.float32).reshape(1, n)
    g = make_grad(1, n, seed=3)
    out = gpu_run(x, g, 100.0, 1e-5)  # integer k: b at the midpoint of two scores, 500 alpha from each
    _, b_ref, _ = orc.forward(x[0], 100.0, 1e-5)
    _, lam, _ = orc.backward(x[0], g[0], b_ref, 1e-5)
    assert np.isfinite(out["gk"][0]) and out["gk"][0] == pytest.approx(lam, rel=1e-4, abs=1e-6)
    assert np.all(np.isfinite(out["grad"]))


# ---------------------------------------------------------------------------
# dL/dalpha (the threshold moves with alpha): both paths, several rows, and
# through autograd with k and alpha as tensors
# ---------------------------------------------------------------------------
def alpha_tol(r, g, b, alpha):
    z = r.astype(np.float64) - b
    f = 0.5 * np.exp(-np.abs(z) / alpha) / alpha
    return 1e-6 * float(np.sum(np.abs(z) * f * np.abs(g.astype(np.float64)))) / alpha


@pytest.mark.parametrize("name,n,rows,force", [
    ("c1", None, None, 0),
    ("c1", 4096, 3, lt.FORCE_STREAMING),
    ("c2", None, None, 0),
    ("c3", 2_000_003, None, 0),
    ("c5", 16384, 4, 0),
    ("c5", 5001, 4, 0),
    ("c5", 12001, 4, 0),
    ("c2", 100_003, 3, 0),
])
def test_alpha_gradient_matches_oracle(orc, name, n, rows, force):
    w, x, g = case(name, n=n, rows=rows)
    xt = torch.from_numpy(np.ascontiguousarray(x)).cuda()
    gt = torch.from_numpy(np.ascontiguousarray(g)).cuda()
    params = lt.Params(force_path=force) if force else None
    res = lt.forward(xt, w.k, w.alpha, params=params)
    gs, gk, ga = lt.backward(xt, gt, res.b, w.alpha, want_alpha=True)
    gs0, gk0 = lt.backward(xt, gt, res.b, w.alpha)
    torch.cuda.synchronize()
    # asking for dL/dalpha changes nothing else
    assert torch.equal(gs, gs0) and torch.equal(gk, gk0)
    ga = ga.cpu().numpy()
    for i in range(x.shape[0]):
        _, b_ref, _ = orc.forward(x[i], w.k, w.alpha)
        ref = orc.backward_alpha(x[i], g[i], b_ref, w.alpha)
        tol = 1e-4 * abs(ref) + alpha_tol(x[i], g[i], b_ref, w.alpha)
        assert abs(ga[i] - ref) <= tol, f"{name} row {i}: {ga[i]!r} vs {ref!r} (tol {tol:.3e})"


def test_autograd_k_and_alpha_tensors(orc):
    w, x, g = case("c1")
    xt = torch.from_numpy(x.copy()).cuda().requires_grad_(True)
    kt = torch.tensor(w.k, dtype=torch.float64, device="cuda", requires_grad=True)
    at = torch.tensor(w.alpha, dtype=torch.float32, device="cuda", requires_grad=True)
    p = lt.soft_topk(xt, kt, at)
    (p * torch.from_numpy(g).cuda()).sum().backward()
    _, b_ref, _ = orc.forward(x[0], w.k, w.alpha)
    _, lam, _ = orc.backward(x[0], g[0], b_ref, w.alpha)
    ref_a = orc.backward_alpha(x[0], g[0], b_ref, w.alpha)
    assert kt.grad.shape == kt.shape and at.grad.shape == at.shape and at.grad.dtype == torch.float32
    assert float(kt.grad) == pytest.approx(lam, rel=1e-4, abs=1e-6 * (1 + abs(lam)))
    assert float(at.grad) == pytest.approx(ref_a, rel=1e-4, abs=alpha_tol(x[0], g[0], b_ref, w.alpha) + 1e-6)
    assert xt.grad is not None and torch.isfinite(xt.grad).all()


# ---------------------------------------------------------------------------
# sparse forward: the entries with p >= eps as (index, p) pairs
# ---------------------------------------------------------------------------
EPS = 2.0 ** -24


@pytest.mark.parametrize("name,n,rows,force", [
    ("c1", None, None, 0),
    ("c1", 4096, 3, lt.FORCE_STREAMING),
    ("c2", None, None, 0),
    ("c3", 2_000_003, None, 0),
    ("c5", 16384, 4, 0),
    ("c2", 100_003, 2, 0),
    ("c5", 12001, 4, 0),
])
def test_sparse_forward_matches_dense_and_oracle(orc, name, n, rows, force):
    w, x, _ = case(name, n=n, rows=rows)
    xt = torch.from_numpy(np.ascontiguousarray(x)).cuda()
    params = lt.Params(force_path=force) if force else None
    dense = lt.forward(xt, w.k, w.alpha, params=params)
    sp = lt.forward_sparse(xt, w.k, w.alpha, EPS, capacity=x.shape[1], params=params)
    torch.cuda.synchronize()
    assert torch.equal(sp.b, dense.b) and torch.equal(sp.status, dense.status)
    p_dense = dense.p.view(x.shape).cpu().numpy()
    resident = x.shape[1] <= 16384 and not force
    for i in range(x.shape[0]):
        idx, val = (t.cpu().numpy() for t in sp.row(i))
        want = np.nonzero(p_dense[i] >= EPS)[0]
        assert int(sp.count[i]) == want.size
        assert np.array_equal(np.sort(idx), want), f"{name} row {i}: index sets differ"
        assert np.array_equal(val, p_dense[i][idx])  # same arithmetic as the dense pass
        if resident:
            assert np.all(np.diff(idx) > 0)  # index order on the one-block path
        p_ref, _, _ = orc.forward(x[i], w.k, w.alpha)
        assert np.max(np.abs(val - p_ref[idx])) <= 1e-5
        sure = np.nonzero(p_ref >= EPS * (1 + 1e-3) + 1e-5)[0]
        assert np.all(np.isin(sure, idx))


@pytest.mark.parametrize("name,n", [("c1", None), ("c2", None)])
def test_sparse_forward_truncates_and_reports(orc, name, n):
    w, x, _ = case(name, n=n)
    xt = torch.from_numpy(np.ascontiguousarray(x)).cuda()
    full = lt.forward_sparse(xt, w.k, w.alpha, EPS, capacity=x.shape[1])
    torch.cuda.synchronize()
    total = int(full.count[0])
    cap = total // 3
    part = lt.forward_sparse(xt, w.k, w.alpha, EPS, capacity=cap)
    torch.cuda.synchronize()
    assert int(part.count[0]) == total
    assert int(part.status[0]) & lt.ROW_TRUNCATED
    assert not int(full.status[0]) & lt.ROW_TRUNCATED
    idx, val = (t.cpu().numpy() for t in part.row(0))
    assert idx.size == cap and np.unique(idx).size == cap
    fi, fv = (t.cpu().numpy() for t in full.row(0))
    ref = dict(zip(fi.tolist(), fv.tolist()))
    assert all(ref[int(j)] == v for j, v in zip(idx, val))


def test_sparse_forward_default_capacity_retries(orc):
    """The binding's default capacity (2k + 4096) is too small for a wide
    transition; it then repeats the call with the exact count."""
    rng = np.random.default_rng(5)
    x = rng.standard_normal((1, 200_000)).astype(np.float32)
    xt = torch.from_numpy(x).cuda()
    sp = lt.forward_sparse(xt, 10.0, 5.0, EPS)  # alpha 5: most entries are non-negligible
    torch.cuda.synchronize()
    assert sp.idx.shape[1] == int(sp.count[0]) > 2 * 10 + 4096
    assert not int(sp.status[0]) & lt.ROW_TRUNCATED


# ---------------------------------------------------------------------------
# DFTopK relaxation (Fast LapSum technical summary, section 2.3): threshold at
# the midpoint of the k-th and (k+1)-th largest, memberships at alpha
# ---------------------------------------------------------------------------
def dftopk_check(orc, r, k, alpha, res, i, label):
    r = np.asarray(r, np.float32).reshape(-1)
    p_ref, b_ref, mass_ref = orc.dftopk_forward(r, k, alpha)
    b = float(res.b[i])
    # the solve at alpha = 1e-30 lands on the midpoint up to fp64 rounding of
    # b = x_k - (x_k - x_k+1)/2 + O(1e-30)
    gap = float(np.max(np.abs(r))) if r.size else 1.0
    assert abs(b - b_ref) <= 8 * np.finfo(np.float64).eps * max(abs(b_ref), gap), f"{label} b {b!r} vs {b_ref!r}"
    p = res.p.view(-1, r.size)[i].cpu().numpy().astype(np.float64)
    dp = float(np.max(np.abs(p - p_ref)))
    assert dp <= 1e-5, f"{label} max|dp|={dp:.3e}"
    # the mass: sums of the same fp32 memberships (partial sums of up to 16 in
    # fp32 on the streaming path, each rounded to 2^-24 relative; fp64 above)
    mass = float(res.mass[i])
    assert abs(mass - math.fsum(p.tolist())) <= 1e-6 * max(1.0, mass)
    assert abs(mass - mass_ref) <= 1e-5 * max(1.0, k) * max(1.0, math.sqrt(r.size / 1e6)), f"{label} mass"
    x = r.astype(np.float64)
    sumf_ref = math.fsum((0.5 * np.exp(-np.abs(x - b_ref) / alpha) / alpha).tolist())
    assert float(res.sumf[i]) == pytest.approx(sumf_ref, rel=1e-5, abs=1e-300)
    return mass_ref


@pytest.mark.parametrize("name,n,rows,force", [
    ("c1", None, None, 0),
    ("c1", 4096, 3, lt.FORCE_STREAMING),
    ("c2", None, None, 0),
    ("c3", 2_000_003, None, 0),
    ("c5", 16384, 4, 0),
    ("c2", 100_003, 2, 0),
    ("c5", 5001, 4, 0),
    ("c5", 12001, 4, 0),
])
def test_dftopk_matches_oracle(orc, name, n, rows, force):
    w, x, _ = case(name, n=n, rows=rows)
    k = int(round(w.k))
    xt = torch.from_numpy(np.ascontiguousarray(x)).cuda()
    params = lt.Params(force_path=force) if force else None
    res = lt.dftopk_forward(xt, k, w.alpha, params=params)
    torch.cuda.synchronize()
    assert np.all(res.status.cpu().numpy() & lt.ROW_NONFINITE == 0)
    for i in range(x.shape[0]):
        dftopk_check(orc, x[i], k, w.alpha, res, i, f"{name} row {i}")


@pytest.mark.parametrize("n,k,alpha", [
    (2, 1, 0.5), (3, 1, 1e-3), (3, 2, 10.0), (4096, 1, 0.01), (4096, 4095, 0.01),
    (100_000, 1, 1e-4), (100_000, 99_999, 0.3), (100_000, 50_000, 10.0), (300_001, 7, 1e-6),
    # half-gap / alpha of a few hundred: sum f far below fp32 range, still in fp64
    (5000, 2500, 5e-7), (300_001, 150_000, 1e-8),
])
def test_dftopk_edge_budgets(orc, n, k, alpha):
    x = make_scores("normal", 1, n, seed=n + 29)
    res = lt.dftopk_forward(torch.from_numpy(x).cuda(), k, alpha)
    torch.cuda.synchronize()
    dftopk_check(orc, x[0], k, alpha, res, 0, f"n={n} k={k}")


def test_dftopk_sumf_mixes_near_and_far_blocks(orc):
    """Uniform scores with alpha far below the typical spacing of a block:
    the block holding the scores next to b sums its fp32 terms, the others
    (every term below 2^-64) recount relative to their nearest score."""
    n, k, alpha = 1_000_000, 500_000, 3e-8
    x = make_scores("uniform", 1, n, seed=77)
    res = lt.dftopk_forward(torch.from_numpy(x).cuda(), k, alpha)
    torch.cuda.synchronize()
    dftopk_check(orc, x[0], k, alpha, res, 0, "mixed blocks")


@pytest.mark.parametrize("n", [5000, 300_000])
def test_dftopk_ties_at_the_boundary(orc, n):
    """k-th and (k+1)-th largest equal: the midpoint is that value."""
    rng = np.random.default_rng(n)
    x = np.round(rng.standard_normal((1, n)) * 4).astype(np.float32)  # heavy ties
    k = n // 3
    res = lt.dftopk_forward(torch.from_numpy(x).cuda(), k, 0.05)
    torch.cuda.synchronize()
    s = np.sort(x[0].astype(np.float64))[::-1]
    assert s[k - 1] == s[k] and float(res.b[0]) == s[k]
    dftopk_check(orc, x[0], k, 0.05, res, 0, f"ties n={n}")


def test_dftopk_is_the_zero_temperature_limit_of_lapsum(orc):
    """The midpoint equals the LapSum threshold at alpha = 1e-30, and at a
    finite alpha the LapSum mass is k while the DFTopK mass drifts."""
    w, x, _ = case("c2")
    k = int(round(w.k))
    xt = torch.from_numpy(x).cuda()
    cold = lt.forward(xt, float(k), 1e-30)
    d = lt.dftopk_forward(xt, k, w.alpha)
    exact = lt.forward(xt, float(k), w.alpha)
    torch.cuda.synchronize()
    assert float(cold.b[0]) == float(d.b[0])
    mass_exact = math.fsum(exact.p.view(-1).double().cpu().numpy().tolist())
    assert abs(mass_exact - k) <= tol_sum(k, x.shape[1])
    mass_ref = orc.dftopk_forward(x[0], k, w.alpha)[2]
    assert float(d.mass[0]) == pytest.approx(mass_ref, rel=1e-6)


# ---------------------------------------------------------------------------
# per-row k and alpha (one budget and one scale per row of a batch)
# ---------------------------------------------------------------------------
def per_row_values(rows, n, seed):
    rng = np.random.default_rng(seed)
    k = np.round(rng.uniform(0.5, n - 0.5, rows), 3)
    k[0], k[-1] = 0.25, n - 0.75  # near both ends of (0, n)
    alpha = 10.0 ** rng.uniform(-3, 0.5, rows)
    return k, alpha


@pytest.mark.parametrize("rows,n,force", [
    (6, 4096, 0), (5, 16384, 0), (3, 4096, lt.FORCE_STREAMING), (3, 200_003, 0), (2, 1_000_000, 0),
])
def test_per_row_k_and_alpha_match_oracle(orc, rows, n, force):
    x = make_scores("normal", rows, n, seed=rows * 1000 + n)
    g = make_grad(rows, n, seed=rows + n)
    k, alpha = per_row_values(rows, n, seed=n)
    xt, gt = torch.from_numpy(x).cuda(), torch.from_numpy(g).cuda()
    kt, at = torch.from_numpy(k).cuda(), torch.from_numpy(alpha).cuda()
    params = lt.Params(force_path=force) if force else None
    res = lt.forward(xt, kt, at, params=params)
    gs, gk, ga = lt.backward(xt, gt, res.b, at, want_alpha=True)
    torch.cuda.synchronize()
    p, b, grad = res.p.cpu().numpy(), res.b.cpu().numpy(), gs.cpu().numpy()
    gk, ga = gk.cpu().numpy(), ga.cpu().numpy()
    assert np.all(res.status.cpu().numpy() & lt.ROW_CERTIFIED)
    for i in range(rows):
        b_ref = check_row(orc, x[i], g[i], p[i], grad[i], b[i], gk[i], float(k[i]), float(alpha[i]), f"row {i}")
        ref = orc.backward_alpha(x[i], g[i], b_ref, float(alpha[i]))
        tol = 1e-4 * abs(ref) + alpha_tol(x[i], g[i], b_ref, float(alpha[i]))
        assert abs(ga[i] - ref) <= tol, f"row {i}: dL/dalpha {ga[i]!r} vs {ref!r}"


@pytest.mark.parametrize("n", [3000, 100_000])
def test_per_row_call_agrees_with_scalar_calls(orc, n):
    """Each row of a per-row call against a scalar call with that row's k and
    alpha: the same threshold to fp64 rounding (the streaming path draws the
    same sample and ranks; the one-block path a larger sample)."""
    rows = 4
    x = make_scores("normal", rows, n, seed=n + 3)
    k, alpha = per_row_values(rows, n, seed=n + 4)
    xt = torch.from_numpy(x).cuda()
    res = lt.forward(xt, torch.from_numpy(k).cuda(), torch.from_numpy(alpha).cuda())
    torch.cuda.synchronize()
    for i in range(rows):
        one = lt.forward(xt[i:i + 1].contiguous(), float(k[i]), float(alpha[i]))
        torch.cuda.synchronize()
        bi, b1 = float(res.b[i]), float(one.b[0])
        assert abs(bi - b1) <= 2e-6 * alpha[i] + 1e-12 * abs(b1), f"row {i}: {bi!r} vs {b1!r}"


@pytest.mark.parametrize("n", [2048, 50_000])
def test_per_row_bad_values_mark_only_their_rows(orc, n):
    rows = 6
    x = make_scores("normal", rows, n, seed=n + 5)
    g = make_grad(rows, n, seed=n + 6)
    k = np.array([0.0, n, 10.0, np.nan, 20.0, 5.0])
    alpha = np.array([0.5, 0.5, 0.0, 0.5, np.inf, 0.2])
    good = [5]
    xt, gt = torch.from_numpy(x).cuda(), torch.from_numpy(g).cuda()
    at = torch.from_numpy(alpha).cuda()
    res = lt.forward(xt, torch.from_numpy(k).cuda(), at)
    gs, gk, ga = lt.backward(xt, gt, res.b, at, want_alpha=True)
    torch.cuda.synchronize()
    st = res.status.cpu().numpy().astype(np.uint32)
    b, p, grad = res.b.cpu().numpy(), res.p.cpu().numpy(), gs.cpu().numpy()
    for i in range(rows):
        if i in good:
            assert not st[i] & lt.ROW_BADARG
            check_row(orc, x[i], g[i], p[i], grad[i], b[i], float(gk[i]), float(k[i]), float(alpha[i]), f"row {i}")
        else:
            assert st[i] & lt.ROW_BADARG, f"row {i} status {st[i]:#x}"
            assert np.isnan(b[i]) and np.all(np.isnan(p[i]))
    # the backward flags only a bad alpha (it has no k)
    for i in (2, 4):
        assert np.all(np.isnan(grad[i])) and np.isnan(float(gk[i])) and np.isnan(float(ga[i]))


def test_autograd_per_row_k_and_alpha(orc):
    rows, n = 3, 5000
    x = make_scores("normal", rows, n, seed=11)
    g = make_grad(rows, n, seed=12)
    k, alpha = per_row_values(rows, n, seed=13)
    xt = torch.from_numpy(x).cuda().requires_grad_(True)
    kt = torch.from_numpy(k).cuda().requires_grad_(True)
    at = torch.from_numpy(alpha).float().cuda().requires_grad_(True)
    p = lt.soft_topk(xt, kt, at)
    (p * torch.from_numpy(g).cuda()).sum().backward()
    assert kt.grad.shape == (rows,) and at.grad.shape == (rows,) and at.grad.dtype == torch.float32
    for i in range(rows):
        a = float(at[i].detach())  # the fp32 value the operator saw
        _, b_ref, _ = orc.forward(x[i], float(k[i]), a)
        _, lam, _ = orc.backward(x[i], g[i], b_ref, a)
        ref_a = orc.backward_alpha(x[i], g[i], b_ref, a)
        assert float(kt.grad[i]) == pytest.approx(lam, rel=1e-4, abs=1e-6 * (1 + abs(lam)))
        assert float(at.grad[i]) == pytest.approx(ref_a, rel=1e-4, abs=alpha_tol(x[i], g[i], b_ref, a) + 1e-6)


@pytest.mark.parametrize("name,n,rows", [("c3", 2_000_000, None), ("c5", 16384, 8)])
def test_capture_in_a_cuda_graph(name, n, rows):
    """forward_into / backward_into make no host synchronisation, so a step
    captures into a CUDA graph; its replays give the eager results bit for bit."""
    w, x, g = case(name, n=n, rows=rows)
    xt, gt = torch.from_numpy(x).cuda(), torch.from_numpy(g).cuda()
    rws, nn = x.shape
    p, grad = torch.empty_like(xt), torch.empty_like(xt)
    b = torch.empty(rws, dtype=torch.float64, device="cuda")
    sumf, gk = torch.empty_like(b), torch.empty_like(b)
    st = torch.empty(rws, dtype=torch.int32, device="cuda")
    ws = torch.empty(lt.workspace_size(rws, nn), dtype=torch.uint8, device="cuda")

    def step():
        lt.forward_into(xt, w.k, w.alpha, p, b, sumf, st, ws)
        lt.backward_into(xt, gt, b, w.alpha, grad, ws, grad_k=gk)

    step()
    torch.cuda.synchronize()
    ref = [t.clone() for t in (p, b, sumf, grad, gk)]
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    for t in (p, b, grad):
        t.zero_()
    for _ in range(2):
        graph.replay()
    torch.cuda.synchronize()
    for a, r in zip((p, b, sumf, grad, gk), ref):
        assert torch.equal(a, r)
