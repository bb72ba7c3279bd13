"""Bounded device waits that run out (failure detection without a GPU fault).

Every wait in the library's kernels -- the bulk-copy barrier of a one-block
row copied into shared memory, the barriers of the filter's ring of bulk
copies, the grid barrier of the cooperative recovery kernel -- gives up
after a fixed number of polls, marks the row
LAPSUM_ROW_TIMEOUT and returns (the pages' solver widens its bracket and falls
back to a full sort, technical summary section 2.2 step 4; a wait that never
ends would hang the GPU instead).  The LAPSUM_FORCE_TIMEOUT test knob makes
the wait of every odd-numbered row run out: the one-block row waits on a
barrier that no copy targets, so does each filter block of a streaming row
numbered 1 mod 4 (for its first chunk), and the recovery barrier of a
streaming row numbered 3 mod 4 waits for one block more than the grid holds.  Nothing faults or waits for good; a short
spin_limit keeps each wait to a fraction of a millisecond.

Checked: the forced rows report the timeout and carry NaN outputs, the other
rows are certified and equal to the oracle, and the next call on the same
stream (no knob) is correct for every row.
"""
import numpy as np
import pytest

import differentiable_soft_top_b200 as lt
from differentiable_soft_top_b200.workloads import make_grad, make_scores

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

from tests.test_gpu_parity import check_row, gpu_run  # noqa: E402


@pytest.mark.parametrize("n,force,rows", [
    (4096, 0, 5),                       # one-block rows copied into shared memory
    (3001, 0, 4),                       # the same with rows off the 16-byte grid
    (100_003, 0, 5),                    # streaming rows: the recovery kernel's barrier
    (4096, lt.FORCE_STREAMING, 3),      # short rows forced onto the streaming path
])
def test_forced_waits_time_out_and_the_rest_is_solved(orc, n, force, rows):
    x = make_scores("normal", rows, n, seed=n + 31)
    g = make_grad(rows, n, seed=n + 32)
    k, alpha = n / 50.0, 0.2
    params = lt.Params(force_path=force | lt.FORCE_TIMEOUT, spin_limit=2000)
    out = gpu_run(x, g, k, alpha, params=params, stats=True)
    for i in range(rows):
        st = int(out["status"][i])
        if i % 2:
            assert st & lt.ROW_TIMEOUT, f"row {i} status {st:#x}"
            assert not (st & lt.ROW_CERTIFIED)
            assert np.isnan(out["p"][i]).all() and np.isnan(out["b"][i]) and np.isnan(out["sumf"][i])
            assert int(out["stats"][i]["status"]) & lt.ROW_TIMEOUT
        else:
            assert st == lt.ROW_CERTIFIED, f"row {i} status {st:#x}"
            check_row(orc, x[i], g[i], out["p"][i], out["grad"][i], out["b"][i], out["gk"][i], k, alpha,
                      f"row {i} beside timed-out rows")
    # the next call on the same stream starts afresh
    again = gpu_run(x, g, k, alpha, params=lt.Params(force_path=force))
    for i in range(rows):
        assert int(again["status"][i]) & lt.ROW_CERTIFIED
        check_row(orc, x[i], g[i], again["p"][i], again["grad"][i], again["b"][i], again["gk"][i], k, alpha,
                  f"row {i} after the timed-out call")


def test_timeout_with_the_fallback_forced_on_every_row(orc):
    """FORCE_FALLBACK sends every row to the recovery kernel, except row 1,
    whose filter wait already ran out (a row that timed out is not
    recovered).  The full sorts of rows 0 and 2 run first and are certified,
    row 3's barrier runs out, and the rows after it that still need recovery
    are marked too (row 4, an even row); row 5 times out in its filter."""
    rows, n = 6, 50_001
    x = make_scores("mixture", rows, n, seed=5)
    g = make_grad(rows, n, seed=6)
    k, alpha = 200.0, 0.05
    params = lt.Params(force_path=lt.FORCE_FALLBACK | lt.FORCE_TIMEOUT, spin_limit=2000)
    out = gpu_run(x, g, k, alpha, params=params)
    st = out["status"].astype(np.uint32)
    for i in (0, 2):
        assert st[i] & lt.ROW_FALLBACK and st[i] & lt.ROW_CERTIFIED, f"row {i} status {st[i]:#x}"
        check_row(orc, x[i], g[i], out["p"][i], out["grad"][i], out["b"][i], out["gk"][i], k, alpha, f"row {i}")
    for i in (1, 3, 4, 5):
        assert st[i] & lt.ROW_TIMEOUT and not (st[i] & lt.ROW_CERTIFIED), f"row {i} status {st[i]:#x}"
        assert np.isnan(out["p"][i]).all() and np.isnan(out["b"][i])
