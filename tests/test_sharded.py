"""Sharded rows: one row split over GPUs in contiguous shards.

On CPU: the shard bounds, the lockstep driver, and the torch.distributed
driver with two gloo ranks (the exchanges the GPU ranks would make with
NCCL), both on a toy program and on the real forward and backward programs
with the library's buffer layout and the kernel calls stubbed.  On a GPU: the sharded forward and backward, run as 2-4 ranks in
lockstep on one device, against the one-GPU operator and the oracle."""
import math
import os
import socket

import numpy as np
import pytest

import differentiable_soft_top_b200 as lt
from differentiable_soft_top_b200 import sharded as sh
from differentiable_soft_top_b200.workloads import WORKLOADS, make_grad, make_scores

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402


@pytest.mark.parametrize("n,world", [(16, 2), (17, 4), (1001, 3), (1_000_003, 8), (4096, 1)])
def test_shard_bounds_tile_the_row(n, world):
    b = [sh.shard_bounds(n, world, r) for r in range(world)]
    assert b[0][0] == 0 and b[-1][1] == n
    for (lo, hi), (lo2, _) in zip(b, b[1:]):
        assert hi == lo2
    assert all(hi > lo and lo % 4 == 0 for lo, hi in b)
    sizes = [hi - lo for lo, hi in b[:-1]]
    assert not sizes or max(sizes) - min(sizes) <= 4
    with pytest.raises(ValueError):
        sh.shard_bounds(4 * world - 1, world, 0)


def _fake_program(rank, world):
    """A rank's program with CPU tensors standing in for the exchange buffers."""
    s = torch.full((6,), 0, dtype=torch.int32)
    s[rank::world] = rank + 10  # every slot non-zero on one rank only, as the sample keys
    h = torch.arange(4, dtype=torch.int32) * (rank + 1)
    yield ("sum", [s, h])
    mine = torch.full((3,), float(rank), dtype=torch.float32)
    out = torch.empty(3 * world, dtype=torch.float32)
    yield ("gather", [(out, mine)])
    return s.tolist(), h.tolist(), out.tolist()


def _expected(world):
    s = [10 + (i % world) for i in range(6)]
    h = [i * sum(r + 1 for r in range(world)) for i in range(4)]
    g = [float(r) for r in range(world) for _ in range(3)]
    return s, h, g


def test_lockstep_driver_makes_the_exchanges():
    world = 3
    res = sh.run_lockstep([_fake_program(r, world) for r in range(world)])
    assert all(tuple(x) == _expected(world) for x in res)


def test_lockstep_driver_rejects_diverging_programs():
    def prog(kind):
        yield (kind, [])
    with pytest.raises(RuntimeError):
        sh.run_lockstep([prog("sum"), prog("gather")])


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _gloo_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        q.put((rank, sh.run_distributed(_fake_program(rank, world))))
    finally:
        dist.destroy_process_group()


def test_distributed_driver_with_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_gloo_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for _, r in res:
        assert tuple(r) == _expected(world)


class _HostShard(sh.ShardedTopK):
    """The real per-rank object (layout from the C library, exchange buffers
    on the CPU) with its kernel calls replaced by rank-stamped fills: the real
    forward and backward programs then make the real exchanges, and the
    finish calls check what arrived."""

    def _check_shard(self, x):
        return x

    def fwd_sample(self, x):
        self.x_sample.zero_()
        self.x_sample[self.rank::self.world] = self.rank + 1  # disjoint slots, as the sample keys
        self.x_hist.fill_(self.rank + 1)

    def fwd_filter(self, x):
        self.x_meta.fill_(100 + self.rank)
        self.x_fpart.fill_(50 + self.rank)
        self.x_band.fill_(self.rank + 0.5)

    def _ranks_of(self, t):
        return [t.view(self.world, -1)[w] for w in range(self.world)]

    def fwd_finish(self, x):
        W = self.world
        assert all(int(v) == (i % W) + 1 for i, v in enumerate(self.x_sample.tolist()))
        assert bool((self.x_hist == W * (W + 1) // 2).all())
        for w, (m, f, b) in enumerate(zip(self._ranks_of(self.g_meta), self._ranks_of(self.g_fpart),
                                          self._ranks_of(self.g_band))):
            assert bool((m == 100 + w).all()) and bool((f == 50 + w).all()) and bool((b == w + 0.5).all())
        rows = self.rows
        return sh.ShardResult(torch.zeros_like(x), torch.zeros(rows, dtype=torch.float64),
                              torch.zeros(rows, dtype=torch.float64),
                              torch.full((rows,), lt.ROW_CERTIFIED, dtype=torch.int32))

    def bwd_partials(self, x, g, b, with_alpha):
        self.x_parts.fill_(7 + self.rank)

    def bwd_finish(self, x, g, b, with_alpha):
        for w, t in enumerate(self._ranks_of(self.g_parts)):
            assert bool((t == 7 + w).all())
        return torch.zeros_like(x), torch.zeros(self.rows, dtype=torch.float64), None


def _real_program_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        rows, n_total = 2, 200_003
        obj = _HostShard(rows, n_total, world, rank, 1000.0, 0.1, torch.device("cpu"))
        x = torch.zeros(rows, obj.n)
        res = sh.run_distributed(sh.forward_program(obj, x))
        grad, gk, ga = sh.run_distributed(sh.backward_program(obj, x, x, res.b))
        q.put((rank, bool((res.status == lt.ROW_CERTIFIED).all()), tuple(grad.shape)))
    except Exception as e:  # the parent reports it
        q.put((rank, repr(e), None))
    finally:
        dist.destroy_process_group()


def test_real_programs_exchange_over_two_gloo_ranks():
    """The sharded forward and backward programs, with the library's own
    layout and buffers, make their exchanges over torch.distributed (gloo
    here, NCCL on GPUs): sums and rank-major gathers arrive as the kernels of
    every rank wrote them."""
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_real_program_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ok, shape in res:
        assert ok is True, f"rank {rank}: {ok}"
        lo, hi = sh.shard_bounds(200_003, world, rank)
        assert shape == (2, hi - lo)


# ---------------------------------------------------------------------------
# GPU: ranks in lockstep on one device
# ---------------------------------------------------------------------------
gpu = pytest.mark.gpu


def _shards(x, world):
    return [x[:, lo:hi].contiguous() for lo, hi in (sh.shard_bounds(x.shape[1], world, r) for r in range(world))]


def _sharded_forward(xt, k, alpha, world, params=None):
    objs = [sh.ShardedTopK(xt.shape[0], xt.shape[1], world, r, k, alpha, xt.device, params) for r in range(world)]
    parts = _shards(xt, world)
    res = sh.run_lockstep([sh.forward_program(o, s) for o, s in zip(objs, parts)])
    return objs, parts, res


@gpu
@pytest.mark.parametrize("name,n,rows,world", [
    ("c2", None, None, 2),
    ("c2", 1_000_003, 2, 3),
    ("c3", 2_000_000, None, 4),
    ("c1", 40_000, 3, 2),
])
def test_sharded_forward_and_backward_match_one_gpu(orc, name, n, rows, world):
    w = WORKLOADS[name].scaled(n=n, rows=rows) if (n or rows) else WORKLOADS[name]
    x = make_scores(w)
    g = make_grad(w.rows, w.n)
    xt, gt = torch.from_numpy(x).cuda(), torch.from_numpy(g).cuda()
    one = lt.forward(xt, w.k, w.alpha)
    gs1, gk1, ga1 = lt.backward(xt, gt, one.b, w.alpha, want_alpha=True)
    objs, parts, res = _sharded_forward(xt, w.k, w.alpha, world)
    gparts = _shards(gt, world)
    bwd = sh.run_lockstep([sh.backward_program(o, s, gs, r.b, True) for o, s, gs, r in zip(objs, parts, gparts, res)])
    torch.cuda.synchronize()
    b1 = one.b.cpu().numpy()
    for r in res:
        assert not r.resolved
        assert torch.equal(r.b, res[0].b)  # every rank solved the same band
        assert np.all(r.status.cpu().numpy() & lt.ROW_CERTIFIED)
        # the same sample and band as one GPU; the tail sums group their fp32
        # terms by other chunks (each shard starts its own), ~1e-7 relative
        assert np.allclose(r.b.cpu().numpy(), b1, rtol=0, atol=1e-6 * w.alpha)
        assert np.allclose(r.sumf.cpu().numpy(), one.sumf.cpu().numpy(), rtol=1e-6)
    p = torch.cat([r.p for r in res], dim=1).cpu().numpy()
    assert np.max(np.abs(p - one.p.cpu().numpy())) <= 1e-6
    grad = torch.cat([q[0] for q in bwd], dim=1).cpu().numpy()
    gref = gs1.cpu().numpy()
    assert np.linalg.norm(grad - gref) <= 1e-6 * np.linalg.norm(gref) + 1e-30
    # lambda and dL/dalpha: the same terms, partial sums (fp32 over 16 scores,
    # then fp64) grouped by another block partition; both are differences of
    # sums, so the error scales with the sums of the absolute terms
    for i in range(w.rows):
        z = x[i].astype(np.float64) - b1[i]
        f = 0.5 * np.exp(-np.abs(z) / w.alpha) / w.alpha
        ag = np.abs(g[i].astype(np.float64))
        lam_scale = float(np.sum(f * ag) / np.sum(f))
        a_scale = float(np.sum(np.abs(z) * f * ag)) / w.alpha
        for q in bwd:
            assert abs(float(q[1][i]) - float(gk1[i])) <= 1e-6 * lam_scale
            assert abs(float(q[2][i]) - float(ga1[i])) <= 1e-6 * a_scale
    # and against the oracle, row by row
    for i in range(w.rows):
        p_ref, b_ref, _ = orc.forward(x[i], w.k, w.alpha)
        assert abs(float(res[0].b[i]) - b_ref) <= 2e-6 * w.alpha + 1e-12 * abs(b_ref)
        assert np.max(np.abs(p[i] - p_ref)) <= 1e-5
        assert abs(math.fsum(p[i].astype(np.float64).tolist()) - w.k) <= 1e-3 * max(1.0, w.k) * math.sqrt(w.n / 1e6)


@gpu
def test_sharded_row_the_band_does_not_certify_is_solved_again(orc):
    w = WORKLOADS["c2"]
    x = make_scores(w)
    xt = torch.from_numpy(x).cuda()
    params = lt.Params(force_path=lt.FORCE_FALLBACK)
    objs, parts, res = _sharded_forward(xt, w.k, w.alpha, 2, params)
    one = lt.forward(xt, w.k, w.alpha, params=params)
    torch.cuda.synchronize()
    assert all(r.resolved for r in res)
    assert torch.equal(res[0].b, one.b)
    assert torch.equal(torch.cat([r.p for r in res], dim=1), one.p)


@gpu
def test_sharded_rejects_a_misshaped_shard():
    o = sh.ShardedTopK(1, 100_000, 2, 0, 10.0, 0.1, torch.device("cuda"))
    with pytest.raises(ValueError):
        o.fwd_sample(torch.zeros(1, 10, device="cuda"))
