"""CPU-only checks of the C-ABI boundary: the library builds and loads, it
exports every entry point include/lapsum_topk.h declares, host-side argument
validation rejects bad calls before any CUDA work, and the CUDA path shares no
code with the oracle.  No kernel is launched here."""
import ctypes
import os
import re

import pytest

import differentiable_soft_top_b200 as lt

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lapsum_topk.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"LAPSUM_API\s+[\w\s\*]+?\b(lapsum_\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    return lt._load()


def test_header_declares_the_boundary():
    names = declared_functions()
    assert names == sorted([
        "lapsum_default_params", "lapsum_dftopk_fwd", "lapsum_last_cuda_error", "lapsum_launch_count",
        "lapsum_status_string", "lapsum_topk_bwd", "lapsum_topk_bwd_rows", "lapsum_topk_fwd", "lapsum_topk_fwd_noalloc",
        "lapsum_topk_fwd_rows", "lapsum_topk_fwd_sparse", "lapsum_shard_bwd_finish", "lapsum_shard_bwd_partials",
        "lapsum_shard_fwd_filter", "lapsum_shard_fwd_finish", "lapsum_shard_fwd_sample", "lapsum_shard_layout_get",
        "lapsum_topk_sparse_workspace_size", "lapsum_topk_workspace_size",
        "lapsum_trace_collect", "lapsum_trace_enable",
    ])


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    # nothing else leaks out of the library
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", lt.library_path()], capture_output=True, text=True).stdout
    exported = sorted(ln.split()[-1] for ln in out.splitlines() if " T " in ln)
    assert exported == declared_functions()


def test_params_struct_layout(lib):
    assert ctypes.sizeof(lt._CParams) == 40
    c = lt._CParams()
    lib.lapsum_default_params(ctypes.byref(c))
    assert c.z == 4.0 == lt.DEFAULT_Z and c.max_widen == -1 and c.sample_m == 0 and c.seed == 0
    assert lt.STATS_DTYPE.itemsize == 88


def test_trace_collect_without_launches(lib):
    lt.trace_enable(True)
    assert lt.trace_collect() == {}
    lt.trace_enable(False)


def test_status_strings(lib):
    for code in range(7):
        assert len(lt.status_string(code)) >= 2 and lt.status_string(code) != "unknown status"
    assert lt.status_string(99) == "unknown status"


def test_workspace_size(lib):
    assert lt.workspace_size(0, 10) == 0
    assert lt.workspace_size(1, 0) == 0
    small = lt.workspace_size(1, 4096)
    assert 0 < small < 1 << 20
    assert lt.workspace_size(2048, 16384) >= lt.workspace_size(1024, 16384)
    big = lt.workspace_size(1, 10**8)
    assert 4 * 10**8 <= big < 2 * 10**9  # holds the fallback key buffer
    forced = lt.workspace_size(1, 4096, lt.Params(force_path=lt.FORCE_STREAMING))
    assert forced > small


FAKE = 1 << 20  # aligned non-null placeholder; validation fails before any use


def fwd(lib, scores=FAKE, rows=1, n=16, stride=16, k=4.0, alpha=0.5, p=FAKE * 4, b=FAKE * 8,
        ws=FAKE * 16, wsb=1 << 30, params=None):
    return lib.lapsum_topk_fwd(scores, rows, n, stride, k, alpha, p, b, None, None, None, ws, wsb, params, None)


@pytest.mark.parametrize("kw,code", [
    (dict(scores=None), lt.LAPSUM_EINVAL),
    (dict(p=None), lt.LAPSUM_EINVAL),
    (dict(b=None), lt.LAPSUM_EINVAL),
    (dict(rows=0), lt.LAPSUM_EINVAL),
    (dict(n=0), lt.LAPSUM_EINVAL),
    (dict(stride=15), lt.LAPSUM_EINVAL),
    (dict(scores=FAKE + 2), lt.LAPSUM_EINVAL),
    (dict(p=FAKE + 8), lt.LAPSUM_EINVAL),  # overlaps the scores
    (dict(k=0.0), lt.LAPSUM_EBADK),
    (dict(k=-1.0), lt.LAPSUM_EBADK),
    (dict(k=16.0), lt.LAPSUM_EBADK),
    (dict(k=float("nan")), lt.LAPSUM_EBADK),
    (dict(k=float("inf")), lt.LAPSUM_EBADK),
    (dict(alpha=0.0), lt.LAPSUM_EBADALPHA),
    (dict(alpha=-1.0), lt.LAPSUM_EBADALPHA),
    (dict(alpha=1e-31), lt.LAPSUM_EBADALPHA),
    (dict(alpha=float("nan")), lt.LAPSUM_EBADALPHA),
    (dict(ws=None), lt.LAPSUM_EWORKSPACE),
    (dict(wsb=8), lt.LAPSUM_EWORKSPACE),
    (dict(ws=FAKE * 16 + 128), lt.LAPSUM_EWORKSPACE),
])
def test_fwd_rejects_bad_arguments(lib, kw, code):
    assert fwd(lib, **kw) == code


def test_bwd_rejects_bad_arguments(lib):
    B = lib.lapsum_topk_bwd
    ok = dict(s=FAKE, g=FAKE * 2, b=FAKE * 3, rows=1, n=100000, stride=100000, a=0.5, out=FAKE * 4,
              gk=None, ga=None, ws=FAKE * 8, wsb=1 << 30)

    def call(**kw):
        d = dict(ok, **kw)
        return B(d["s"], d["g"], d["b"], d["rows"], d["n"], d["stride"], d["a"], d["out"], d["gk"], d["ga"],
                 d["ws"], d["wsb"], None)

    assert call(s=None) == lt.LAPSUM_EINVAL
    assert call(out=None) == lt.LAPSUM_EINVAL
    assert call(b=FAKE * 3 + 4) == lt.LAPSUM_EINVAL
    assert call(n=0) == lt.LAPSUM_EINVAL
    assert call(a=0.0) == lt.LAPSUM_EBADALPHA
    assert call(out=FAKE + 64) == lt.LAPSUM_EINVAL  # overlaps the scores
    assert call(wsb=16) == lt.LAPSUM_EWORKSPACE
    assert call(ga=FAKE * 5 + 4) == lt.LAPSUM_EINVAL  # misaligned dL/dalpha output


def test_sparse_fwd_rejects_bad_arguments(lib):
    F = lib.lapsum_topk_fwd_sparse
    ok = dict(s=FAKE, rows=1, n=100000, stride=100000, k=40.0, a=0.5, eps=2.0 ** -24, idx=FAKE * 64,
              val=FAKE * 128, cap=1000, cnt=FAKE * 192, b=FAKE * 200, ws=FAKE * 256, wsb=1 << 31)

    def call(**kw):
        d = dict(ok, **kw)
        return F(d["s"], d["rows"], d["n"], d["stride"], d["k"], d["a"], d["eps"], d["idx"], d["val"], d["cap"],
                 d["cnt"], d["b"], None, None, None, d["ws"], d["wsb"], None, None)

    assert call(idx=None) == lt.LAPSUM_EINVAL
    assert call(cnt=None) == lt.LAPSUM_EINVAL
    assert call(cnt=FAKE * 192 + 4) == lt.LAPSUM_EINVAL
    assert call(eps=0.0) == lt.LAPSUM_EINVAL
    assert call(eps=1.5) == lt.LAPSUM_EINVAL
    assert call(eps=float("nan")) == lt.LAPSUM_EINVAL
    assert call(cap=-1) == lt.LAPSUM_EINVAL
    assert call(idx=FAKE + 16) == lt.LAPSUM_EINVAL  # overlaps the scores
    assert call(k=0.0) == lt.LAPSUM_EBADK
    # the dense forward's workspace is too small: the fallback needs 4n more
    assert call(wsb=lt.workspace_size(1, 100000)) == lt.LAPSUM_EWORKSPACE
    assert lt.sparse_workspace_size(1, 100000) == lt.workspace_size(1, 100000) + 400128
    assert lt.sparse_workspace_size(4, 4096) == lt.workspace_size(4, 4096)


def test_dftopk_fwd_rejects_bad_arguments(lib):
    """Argument checks of the DFTopK forward (integer 1 <= k <= n-1, alpha in
    range, the dense forward's pointer rules); none of them reaches a GPU."""
    F = lib.lapsum_dftopk_fwd
    ok = dict(s=FAKE, rows=1, n=100000, stride=100000, k=40, a=0.5, out=FAKE * 64, b=FAKE * 128, mass=FAKE * 192,
              ws=FAKE * 256, wsb=1 << 31)

    def call(**kw):
        d = dict(ok, **kw)
        return F(d["s"], d["rows"], d["n"], d["stride"], d["k"], d["a"], d["out"], d["b"], None, d["mass"], None,
                 None, d["ws"], d["wsb"], None, None)

    assert call(k=0) == lt.LAPSUM_EBADK
    assert call(k=100000) == lt.LAPSUM_EBADK
    assert call(k=-3) == lt.LAPSUM_EBADK
    assert call(a=0.0) == lt.LAPSUM_EBADALPHA
    assert call(a=float("inf")) == lt.LAPSUM_EBADALPHA
    assert call(a=1e-31) == lt.LAPSUM_EBADALPHA
    assert call(out=None) == lt.LAPSUM_EINVAL
    assert call(mass=FAKE * 192 + 4) == lt.LAPSUM_EINVAL  # misaligned mass output
    assert call(out=FAKE + 64) == lt.LAPSUM_EINVAL  # overlaps the scores
    assert call(wsb=16) == lt.LAPSUM_EWORKSPACE
    with pytest.raises(ValueError):
        lt.dftopk_forward(None, 2.5, 1.0)


def test_per_row_entry_points_reject_bad_arguments(lib):
    """The *_rows entry points check pointers on the host (the values
    themselves are checked per row on the device)."""
    F = lib.lapsum_topk_fwd_rows
    ok = dict(s=FAKE, rows=4, n=100000, stride=100000, k=FAKE * 128, a=FAKE * 130, out=FAKE * 64, b=FAKE * 132,
              ws=FAKE * 256, wsb=1 << 31)

    def call(**kw):
        d = dict(ok, **kw)
        return F(d["s"], d["rows"], d["n"], d["stride"], d["k"], d["a"], d["out"], d["b"], None, None, None,
                 d["ws"], d["wsb"], None, None)

    assert call(k=None) == lt.LAPSUM_EINVAL
    assert call(a=None) == lt.LAPSUM_EINVAL
    assert call(k=FAKE * 128 + 4) == lt.LAPSUM_EINVAL  # misaligned fp64 vector
    assert call(a=FAKE * 130 + 2) == lt.LAPSUM_EINVAL
    assert call(out=FAKE + 64) == lt.LAPSUM_EINVAL
    assert call(wsb=16) == lt.LAPSUM_EWORKSPACE
    B = lib.lapsum_topk_bwd_rows
    bok = dict(s=FAKE, g=FAKE * 64, b=FAKE * 128, rows=4, n=100000, stride=100000, a=FAKE * 130, out=FAKE * 192,
               ws=FAKE * 256, wsb=1 << 31)

    def bcall(**kw):
        d = dict(bok, **kw)
        return B(d["s"], d["g"], d["b"], d["rows"], d["n"], d["stride"], d["a"], d["out"], None, None, d["ws"],
                 d["wsb"], None)

    assert bcall(a=None) == lt.LAPSUM_EINVAL
    assert bcall(a=FAKE * 130 + 4) == lt.LAPSUM_EINVAL
    assert bcall(out=FAKE + 8) == lt.LAPSUM_EINVAL  # overlaps the scores
    assert bcall(wsb=16) == lt.LAPSUM_EWORKSPACE


def test_binding_rejects_a_misshaped_per_row_vector():
    torch = pytest.importorskip("torch")
    with pytest.raises(ValueError):
        lt._rows_pair(torch.ones(3), 1.0, 4, "cpu")
    assert lt._rows_pair(2.0, torch.tensor(1.0), 4, "cpu") is None


@pytest.mark.parametrize("rows,n,stride,off", [(3, 5000, 5003, 1), (1, 7, 7, 0), (5, 12001, 12001, 0),
                                             (2, 10, 13, 3), (4, 9, 11, 2), (0, 5, 5, 0)])
def test_outputs_start_at_the_scores_address_mod_16(rows, n, stride, off):
    """Outputs the binding allocates share the scores' row stride and their
    address mod 16 (the kernels then move both 16 bytes at a time)."""
    torch = pytest.importorskip("torch")
    base = torch.zeros(rows * stride + 8)
    x = base.as_strided((rows, n), (stride, 1), storage_offset=off)
    p = lt._like_rows(x)
    assert p.shape == x.shape and p.stride() == x.stride()
    if rows:
        assert (p.data_ptr() - x.data_ptr()) % 16 == 0
        assert p.storage_offset() + (rows - 1) * stride + n <= p.untyped_storage().nbytes() // 4
        p.fill_(1.0)


def test_caller_outputs_must_match_the_scores_layout():
    """A caller-given output is written with the scores' row stride for every
    row: a smaller, reshaped or differently strided buffer would be written
    past its end, so the binding rejects it before any call."""
    torch = pytest.importorskip("torch")
    x = torch.zeros(4, 1000)
    lt._check_like(x, torch.zeros(4, 1000), "p")  # the natural case passes
    with pytest.raises(ValueError, match="shape"):
        lt._check_like(x, torch.zeros(1, 1000), "p")  # a 1-D p_out viewed as one row
    with pytest.raises(ValueError, match="shape"):
        lt._check_like(x, torch.zeros(4, 999), "p")
    # strided scores (a column slice) beside a contiguous output of that shape
    xs = torch.zeros(4, 1001)[:, 1:]
    with pytest.raises(ValueError, match="row stride"):
        lt._check_like(xs, torch.zeros(4, 1000), "p")
    lt._check_like(xs, torch.zeros(4, 1001)[:, :1000], "p")
    # one row: its stride is never used
    lt._check_like(torch.zeros(1, 10), torch.zeros(1, 16)[:, :10], "p")
    with pytest.raises(ValueError, match="device"):
        lt._check_like(x, torch.zeros(4, 1000, device="meta"), "p")


def test_per_row_outputs_must_hold_a_value_per_row():
    torch = pytest.importorskip("torch")
    lt._check_vec(torch.zeros(3, dtype=torch.float64), "b", 3, torch.float64, torch.device("cpu"))
    with pytest.raises(TypeError):  # float32 b would be written as float64 past its end
        lt._check_vec(torch.zeros(3), "b", 3, torch.float64, torch.device("cpu"))
    with pytest.raises(ValueError):
        lt._check_vec(torch.zeros(2, dtype=torch.float64), "b", 3, torch.float64, torch.device("cpu"))
    with pytest.raises(ValueError):
        lt._check_vec(torch.zeros(6, dtype=torch.float64)[::2], "b", 3, torch.float64, torch.device("cpu"))
    lt._check_vec(None, "sumf", 3, torch.float64, torch.device("cpu"), optional=True)
    with pytest.raises(ValueError):
        lt._check_vec(None, "b", 3, torch.float64, torch.device("cpu"))


def test_preallocated_entry_points_reject_cpu_tensors():
    torch = pytest.importorskip("torch")
    x = torch.zeros(2, 8)
    b = torch.zeros(2, dtype=torch.float64)
    with pytest.raises(TypeError):
        lt.forward_noalloc_into(x, 2.0, 1.0, torch.zeros(2, 8), b)
    with pytest.raises(TypeError):
        lt.forward_into(x, 2.0, 1.0, torch.zeros(2, 8), b, None, None, torch.zeros(16, dtype=torch.uint8))
    with pytest.raises(TypeError):
        lt.backward_into(x, x, b, 1.0, torch.zeros(2, 8), torch.zeros(16, dtype=torch.uint8))


def test_binding_rejects_cpu_tensors():
    torch = pytest.importorskip("torch")
    with pytest.raises(TypeError):
        lt.forward(torch.zeros(8), 2.0, 1.0)


def test_cuda_path_and_oracle_share_no_code():
    """The oracle and the CUDA path neither include nor import each other; the
    input generators (workloads.py) are the only module both sides use."""
    csrc = os.path.join(ROOT, "differentiable_soft_top_b200", "csrc")
    for f in os.listdir(csrc):
        text = open(os.path.join(csrc, f)).read()
        assert "oracle" not in text.lower(), f
    imp = re.compile(r"^\s*(from|import)\s+(\S+)", re.M)
    pkg = os.path.join(ROOT, "differentiable_soft_top_b200")
    for f in os.listdir(pkg):
        if f.endswith(".py"):
            mods = [m[1] for m in imp.findall(open(os.path.join(pkg, f)).read())]
            assert not any(m.startswith("oracle") for m in mods), f
    text = open(os.path.join(ROOT, "oracle", "lapsum_oracle.c")).read()
    assert '#include "' not in text
    mods = [m[1] for m in imp.findall(open(os.path.join(ROOT, "oracle", "__init__.py")).read())]
    assert not any(m.startswith("differentiable_soft_top_b200") for m in mods)
