"""The allocation-free forward, lapsum_topk_fwd_noalloc.

It serves callers that cannot allocate device memory while the operator runs:
an inference engine that gives each plugin a fixed arena, a host that has
reserved all device memory for its own pool, or a framework that must not risk
cudaMalloc's implicit synchronisation in the middle of a step.  Its scratch is
a static device array inside the library, shared by every call on a device, so
the GPU test below makes two calls in a row -- the second one must not see the
first one's leftovers -- and compares each with lapsum_topk_fwd (which takes a
caller workspace) within the parity tolerances of the other GPU tests.

This file is named to be collected last: a run that stops at its first
failure has then already run every other test.
"""
import ctypes

import numpy as np
import pytest

import differentiable_soft_top_b200 as lt
from differentiable_soft_top_b200.workloads import WORKLOADS, make_scores

FAKE = 1 << 20  # aligned non-null placeholder; validation fails before any use


@pytest.fixture(scope="module")
def lib():
    return lt._load()


def noalloc(lib, scores=FAKE, rows=1, n=16, stride=16, k=4.0, alpha=0.5, p=FAKE * 4, b=FAKE * 8, params=None):
    return lib.lapsum_topk_fwd_noalloc(scores, rows, n, stride, k, alpha, p, b, None, None, None, params, None)


def test_noalloc_rejects_sizes_beyond_its_limits(lib):
    """Checked on the host before any CUDA work, so this runs without a GPU."""
    big_rows = lt.NOALLOC_MAX_ROWS + 1
    assert noalloc(lib, rows=big_rows, n=16, stride=16) == lt.LAPSUM_ETOOLARGE
    n = lt.NOALLOC_MAX_N + 1
    assert noalloc(lib, n=n, stride=n, p=FAKE * 64) == lt.LAPSUM_ETOOLARGE
    assert "NOALLOC" in lt.status_string(lt.LAPSUM_ETOOLARGE)
    streaming = lt.Params(force_path=lt.FORCE_STREAMING)._c()
    assert noalloc(lib, params=ctypes.byref(streaming)) == lt.LAPSUM_EINVAL
    assert noalloc(lib, k=16.0) == lt.LAPSUM_EBADK
    assert noalloc(lib, alpha=0.0) == lt.LAPSUM_EBADALPHA
    assert noalloc(lib, scores=None) == lt.LAPSUM_EINVAL


@pytest.mark.gpu
def test_noalloc_matches_workspace_forward_on_two_calls_in_a_row(lib):
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dev = torch.device("cuda:0")
    stream = torch.cuda.current_stream(dev).cuda_stream

    # call 1: 300 rows of 16384 scores (a quarter of them on 16 levels),
    #         every row through the full-sort fallback, which fills the
    #         fallback row list in the static scratch array;
    # call 2: fewer, shorter rows on the default path -- a stale fallback
    #         counter or list from call 1 would rewrite rows that are not there.
    w5 = WORKLOADS["c5"].scaled(n=16384, rows=300)
    w1 = WORKLOADS["c1"].scaled(n=4096, rows=64)
    calls = [
        (w5, lt.Params(force_path=lt.FORCE_FALLBACK)),
        (w1, None),
    ]
    inputs = [torch.from_numpy(make_scores(w, seed=0)).to(dev) for w, _ in calls]
    refs = []
    for (w, params), x in zip(calls, inputs):
        rows, n = x.shape
        ws = torch.empty(lt.workspace_size(rows, n, params), dtype=torch.uint8, device=dev)
        ref = dict(p=torch.empty_like(x), b=torch.empty(rows, dtype=torch.float64, device=dev),
                   sumf=torch.empty(rows, dtype=torch.float64, device=dev),
                   status=torch.empty(rows, dtype=torch.int32, device=dev))
        lt.forward_into(x, w.k, w.alpha, ref["p"], ref["b"], ref["sumf"], ref["status"], ws, params=params)
        refs.append(ref)
    torch.cuda.synchronize()

    outs = []
    for (w, params), x in zip(calls, inputs):
        rows, n = x.shape
        outs.append(dict(p=torch.full_like(x, float("nan")),
                         b=torch.full((rows,), float("nan"), dtype=torch.float64, device=dev),
                         sumf=torch.full((rows,), float("nan"), dtype=torch.float64, device=dev),
                         status=torch.zeros(rows, dtype=torch.int32, device=dev)))
    torch.cuda.synchronize()
    before = torch.cuda.memory_stats(dev).get("allocation.all.allocated", 0)
    for ((w, params), x, o) in zip(calls, inputs, outs):  # two calls in a row, no sync between them
        rows, n = x.shape
        c = params._c() if params is not None else None
        rc = lib.lapsum_topk_fwd_noalloc(x.data_ptr(), rows, n, x.stride(0), float(w.k), float(w.alpha),
                                         o["p"].data_ptr(), o["b"].data_ptr(), o["sumf"].data_ptr(),
                                         o["status"].data_ptr(), None,
                                         ctypes.byref(c) if c is not None else None, stream)
        assert rc == lt.LAPSUM_OK, lt.status_string(rc)
    torch.cuda.synchronize()
    assert torch.cuda.memory_stats(dev).get("allocation.all.allocated", 0) == before

    for (w, params), o, ref in zip(calls, outs, refs):
        p, p_ref = o["p"].double().cpu().numpy(), ref["p"].double().cpu().numpy()
        assert np.isfinite(p).all()
        assert float(np.max(np.abs(p - p_ref))) <= 1e-5
        b, b_ref = o["b"].cpu().numpy(), ref["b"].cpu().numpy()
        assert np.all(np.abs(b - b_ref) <= 2e-6 * w.alpha + 1e-12 * np.abs(b_ref))
        sf, sf_ref = o["sumf"].cpu().numpy(), ref["sumf"].cpu().numpy()
        np.testing.assert_allclose(sf, sf_ref, rtol=1e-6)
        st = o["status"].cpu().numpy().astype(np.uint32)
        np.testing.assert_array_equal(st, ref["status"].cpu().numpy().astype(np.uint32))
        assert np.all(st & lt.ROW_CERTIFIED)
        if params is not None:
            assert np.all(st & lt.ROW_FALLBACK)

    # the binding's wrapper takes the same route
    w, x = calls[1][0], inputs[1]
    p2 = torch.empty_like(x)
    b2 = torch.empty(x.shape[0], dtype=torch.float64, device=dev)
    lt.forward_noalloc_into(x, w.k, w.alpha, p2, b2)
    torch.cuda.synchronize()
    assert float((p2.double() - refs[1]["p"].double()).abs().max()) <= 1e-5
