"""Sharded rows: one long row split over GPUs in contiguous shards.

The probabilistic bracketing of the Fast LapSum technical summary (section
2.2) only ever needs small summaries of the whole row: the localization
sample, the filter's tail sums and counts, and the band of scores inside the
bracket.  So a row too long for one GPU (or one that should be streamed by
several) runs the same kernels per GPU on its shard, joined by three
exchanges that the caller makes with NCCL:

    sample + level-1 histogram   summed over the GPUs     (~0.5 MB per row)
    filter partials, band stats,
    band values                  gathered from the GPUs   (the band: ~1 MB per row)
    backward partials            gathered from the GPUs   (~0.2 MB per row)

Every GPU then solves the same band for the same threshold b and writes the
memberships (and, backward, dL/dr) of its own shard.  The C calls never wait
on another GPU; the exchanges happen between them, on the host's order.

The per-rank program is written once, as a generator that yields each
exchange it needs (`forward_program`, `backward_program`).  `run_distributed`
executes it with torch.distributed collectives (one process per GPU);
`run_lockstep` executes several ranks' programs in one process, making the
exchanges itself, which is how the sharded path is checked on a single GPU.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass

from . import (LAPSUM_OK, LapsumError, Params, ROW_CERTIFIED, _load, _params_ptr, _torch)

SHARD_META = 8          # uint32 words of band statistics per row and GPU
FPART_SLOTS = 4096      # filter / backward partial slots per row and GPU
FPART_BYTES = 32
BPART_BYTES = 48


class _Layout(ctypes.Structure):
    _fields_ = [("sample_m", ctypes.c_int32), ("reserved", ctypes.c_int32), ("band_cap", ctypes.c_int64),
                ("sample_bytes", ctypes.c_size_t), ("hist_bytes", ctypes.c_size_t),
                ("meta_bytes", ctypes.c_size_t), ("fpart_bytes", ctypes.c_size_t),
                ("band_bytes", ctypes.c_size_t), ("parts_bytes", ctypes.c_size_t),
                ("workspace_bytes", ctypes.c_size_t)]


_bound = False


def _lib():
    global _bound
    lib = _load()
    if not _bound:
        P, i64, dbl, sz, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_double, ctypes.c_size_t, ctypes.c_int
        lib.lapsum_shard_layout_get.argtypes = [i64, i64, P, ctypes.POINTER(_Layout)]
        lib.lapsum_shard_layout_get.restype = None
        lib.lapsum_shard_fwd_sample.argtypes = [P, i64, i64, i64, i64, i64, dbl, dbl, P, P, P, sz, P, P]
        lib.lapsum_shard_fwd_filter.argtypes = [P, i64, i64, i64, i64, i64, dbl, dbl, P, P, P, P, P, P, sz, P, P]
        lib.lapsum_shard_fwd_finish.argtypes = [P, i64, i64, i64, i64, i64, dbl, dbl, i32, P, P, P, P, P, P, P,
                                                P, sz, P, P]
        lib.lapsum_shard_bwd_partials.argtypes = [P, P, P, i64, i64, i64, dbl, i32, P, P]
        lib.lapsum_shard_bwd_finish.argtypes = [P, P, P, i64, i64, i64, dbl, i32, P, P, P, P, P, sz, P]
        for f in (lib.lapsum_shard_fwd_sample, lib.lapsum_shard_fwd_filter, lib.lapsum_shard_fwd_finish,
                  lib.lapsum_shard_bwd_partials, lib.lapsum_shard_bwd_finish):
            f.restype = ctypes.c_int
        _bound = True
    return lib


def shard_bounds(n_total: int, world: int, rank: int) -> tuple[int, int]:
    """[lo, hi) of `rank`'s shard: contiguous and non-empty, the groups of 4
    scores split as evenly as possible (every shard starts on a multiple of 4,
    so 16-byte vector loads stay aligned); the last shard also takes the
    n_total % 4 scores left over."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank must lie in [0, world)")
    if n_total < 4 * world:
        raise ValueError(f"a row of {n_total} scores is too short for {world} shards")
    q, extra = divmod(n_total // 4, world)
    lo = 4 * (rank * q + min(rank, extra))
    hi = 4 * ((rank + 1) * q + min(rank + 1, extra))
    return lo, (n_total if rank == world - 1 else hi)


@dataclass
class ShardLayout:
    sample_m: int
    band_cap: int
    sample_bytes: int
    hist_bytes: int
    meta_bytes: int
    fpart_bytes: int
    band_bytes: int
    parts_bytes: int
    workspace_bytes: int


def shard_layout(rows: int, n_total: int, params: Params | None = None) -> ShardLayout:
    lib = _lib()
    out = _Layout()
    c, pptr = _params_ptr(params)
    lib.lapsum_shard_layout_get(int(rows), int(n_total), pptr, ctypes.byref(out))
    if out.workspace_bytes == 0:
        raise ValueError("invalid shape for a sharded row")
    return ShardLayout(out.sample_m, out.band_cap, out.sample_bytes, out.hist_bytes, out.meta_bytes,
                       out.fpart_bytes, out.band_bytes, out.parts_bytes, out.workspace_bytes)


@dataclass
class ShardResult:
    p: object        # torch.Tensor float32 [rows, n]: this shard's memberships
    b: object        # torch.Tensor float64 [rows]: the threshold (the same on every GPU)
    sumf: object     # torch.Tensor float64 [rows]
    status: object   # torch.Tensor int32 [rows]
    resolved: bool = False  # some row was solved again from the whole row


class ShardedTopK:
    """One GPU's part of a sharded soft top-k over rows of n_total scores.

    Holds the workspace and the exchange buffers (int32 views of the uint32
    sample keys and counts, so that NCCL sums them as integers).  Every rank
    constructs it with the same rows, n_total, world, k, alpha and params."""

    def __init__(self, rows: int, n_total: int, world: int, rank: int, k: float, alpha: float, device,
                 params: Params | None = None):
        torch = _torch()
        self.rows, self.n_total, self.world, self.rank = int(rows), int(n_total), int(world), int(rank)
        self.k, self.alpha, self.params = float(k), float(alpha), params
        self.lo, self.hi = shard_bounds(self.n_total, self.world, self.rank)
        self.n = self.hi - self.lo
        self.device = device
        L = shard_layout(self.rows, self.n_total, params)
        self.layout = L
        u8 = torch.uint8

        def buf(nbytes, dtype=u8, copies=1):
            itemsize = torch.empty(0, dtype=dtype).element_size()
            return torch.empty(copies * nbytes // itemsize, dtype=dtype, device=device)

        self.ws = buf(L.workspace_bytes)
        self.x_sample = buf(L.sample_bytes, torch.int32)
        self.x_hist = buf(L.hist_bytes, torch.int32)
        self.x_meta = buf(L.meta_bytes, torch.int32)
        self.x_fpart = buf(L.fpart_bytes)
        self.x_band = buf(L.band_bytes, torch.float32)
        self.g_meta = buf(L.meta_bytes, torch.int32, self.world)
        self.g_fpart = buf(L.fpart_bytes, u8, self.world)
        self.g_band = buf(L.band_bytes, torch.float32, self.world)
        self.x_parts = buf(L.parts_bytes)
        self.g_parts = buf(L.parts_bytes, u8, self.world)

    # -- the C calls ---------------------------------------------------------
    def _check_shard(self, x):
        torch = _torch()
        if not isinstance(x, torch.Tensor) or not x.is_cuda or x.dtype != torch.float32:
            raise TypeError("the shard must be a CUDA float32 tensor (this library has no CPU path)")
        x = x.view(1, -1) if x.dim() == 1 else x
        if x.shape != (self.rows, self.n):
            raise ValueError(f"shard of shape {tuple(x.shape)}, expected {(self.rows, self.n)}")
        return x if x.stride(1) == 1 else x.contiguous()

    def _stream(self):
        return _torch().cuda.current_stream(self.device).cuda_stream

    def _args(self, x):
        c, pptr = _params_ptr(self.params)
        self._keep = c
        return (x.data_ptr(), self.rows, self.n, x.stride(0), self.lo, self.n_total, self.k, self.alpha), pptr

    def fwd_sample(self, x):
        x = self._check_shard(x)
        a, pptr = self._args(x)
        rc = _lib().lapsum_shard_fwd_sample(*a, self.x_sample.data_ptr(), self.x_hist.data_ptr(),
                                            self.ws.data_ptr(), self.ws.numel(), pptr, self._stream())
        if rc != LAPSUM_OK:
            raise LapsumError(rc, "lapsum_shard_fwd_sample")

    def fwd_filter(self, x):
        x = self._check_shard(x)
        a, pptr = self._args(x)
        rc = _lib().lapsum_shard_fwd_filter(*a, self.x_sample.data_ptr(), self.x_hist.data_ptr(),
                                            self.x_meta.data_ptr(), self.x_fpart.data_ptr(),
                                            self.x_band.data_ptr(), self.ws.data_ptr(), self.ws.numel(), pptr,
                                            self._stream())
        if rc != LAPSUM_OK:
            raise LapsumError(rc, "lapsum_shard_fwd_filter")

    def fwd_finish(self, x) -> ShardResult:
        torch = _torch()
        x = self._check_shard(x)
        a, pptr = self._args(x)
        p = torch.empty_like(x)
        b = torch.empty(self.rows, dtype=torch.float64, device=self.device)
        sumf = torch.empty_like(b)
        status = torch.empty(self.rows, dtype=torch.int32, device=self.device)
        rc = _lib().lapsum_shard_fwd_finish(*a, self.world, self.g_meta.data_ptr(), self.g_fpart.data_ptr(),
                                            self.g_band.data_ptr(), p.data_ptr(), b.data_ptr(), sumf.data_ptr(),
                                            status.data_ptr(), self.ws.data_ptr(), self.ws.numel(), pptr,
                                            self._stream())
        if rc != LAPSUM_OK:
            raise LapsumError(rc, "lapsum_shard_fwd_finish")
        return ShardResult(p, b, sumf, status)

    def bwd_partials(self, x, g, b, with_alpha: bool):
        x, g = self._check_shard(x), self._check_shard(g)
        if g.stride(0) != x.stride(0):
            raise ValueError("grad_p must have the row stride of the scores")
        bb = b.to(device=self.device, dtype=_torch().float64).contiguous()
        rc = _lib().lapsum_shard_bwd_partials(x.data_ptr(), g.data_ptr(), bb.data_ptr(), self.rows, self.n,
                                              x.stride(0), self.alpha, 1 if with_alpha else 0,
                                              self.x_parts.data_ptr(), self._stream())
        if rc != LAPSUM_OK:
            raise LapsumError(rc, "lapsum_shard_bwd_partials")

    def bwd_finish(self, x, g, b, with_alpha: bool):
        torch = _torch()
        x, g = self._check_shard(x), self._check_shard(g)
        bb = b.to(device=self.device, dtype=torch.float64).contiguous()
        grad = torch.empty_like(x)
        gk = torch.empty(self.rows, dtype=torch.float64, device=self.device)
        ga = torch.empty_like(gk) if with_alpha else None
        rc = _lib().lapsum_shard_bwd_finish(x.data_ptr(), g.data_ptr(), bb.data_ptr(), self.rows, self.n,
                                            x.stride(0), self.alpha, self.world, self.g_parts.data_ptr(),
                                            grad.data_ptr(), gk.data_ptr(), ga.data_ptr() if ga is not None else None,
                                            self.ws.data_ptr(), self.ws.numel(), self._stream())
        if rc != LAPSUM_OK:
            raise LapsumError(rc, "lapsum_shard_bwd_finish")
        return grad, gk, ga


# ---------------------------------------------------------------------------
# the per-rank programs: generators that yield the exchanges they need
#   ("sum", [t, ...])            every t summed over the ranks, in place
#   ("gather", [(out, t), ...])  out = the ranks' t, rank-major
# ---------------------------------------------------------------------------
def forward_program(obj: ShardedTopK, x):
    """Forward of one rank; returns its ShardResult.  A row the band does not
    certify is solved again from the whole row (one more gather)."""
    torch = _torch()
    obj.fwd_sample(x)
    yield ("sum", [obj.x_sample, obj.x_hist])
    obj.fwd_filter(x)
    yield ("gather", [(obj.g_meta, obj.x_meta), (obj.g_fpart, obj.x_fpart), (obj.g_band, obj.x_band)])
    res = obj.fwd_finish(x)
    # every rank sees the same status (the same band, the same solve)
    if bool(((res.status & ROW_CERTIFIED) == 0).any()):
        from . import forward
        width = max(hi - lo for lo, hi in (shard_bounds(obj.n_total, obj.world, w) for w in range(obj.world)))
        mine = torch.zeros((obj.rows, width), dtype=torch.float32, device=obj.device)
        mine[:, :obj.n] = obj._check_shard(x)
        full = torch.empty((obj.world, obj.rows, width), dtype=torch.float32, device=obj.device)
        yield ("gather", [(full, mine)])
        whole = torch.cat([full[w, :, :shard_bounds(obj.n_total, obj.world, w)[1] -
                                shard_bounds(obj.n_total, obj.world, w)[0]] for w in range(obj.world)], dim=1)
        one = forward(whole.contiguous(), obj.k, obj.alpha, params=obj.params)
        res = ShardResult(one.p[:, obj.lo:obj.hi].contiguous(), one.b, one.sumf, one.status, resolved=True)
    return res


def backward_program(obj: ShardedTopK, x, g, b, want_alpha: bool = False):
    """Backward of one rank for the thresholds b: returns (dL/dr of its shard,
    dL/dk per row, dL/dalpha per row or None)."""
    obj.bwd_partials(x, g, b, want_alpha)
    yield ("gather", [(obj.g_parts, obj.x_parts)])
    return obj.bwd_finish(x, g, b, want_alpha)


def run_distributed(program, group=None):
    """Runs one rank's program, making each exchange with torch.distributed
    (NCCL for CUDA tensors; any backend whose all_reduce / all_gather take the
    tensors).  Every rank must run the same program."""
    import torch.distributed as dist
    try:
        req = next(program)
        while True:
            kind, items = req
            if kind == "sum":
                for t in items:
                    dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)
            elif kind == "gather":
                for out, t in items:
                    dist.all_gather_into_tensor(out.view(-1), t.contiguous().view(-1), group=group)
            else:
                raise ValueError(f"unknown exchange {kind!r}")
            req = program.send(None)
    except StopIteration as stop:
        return stop.value


def run_lockstep(programs):
    """Runs the programs of all ranks in one process, in lockstep: each
    exchange is made once every rank has reached it.  Returns their results,
    rank order."""
    torch = _torch()
    results = [None] * len(programs)
    reqs = []
    for p in programs:
        reqs.append(next(p))
    while True:
        kinds = {r[0] for r in reqs if r is not None}
        if not kinds:
            return results
        if len(kinds) != 1 or any(r is None for r in reqs):
            raise RuntimeError("the ranks' programs diverged")
        kind = kinds.pop()
        if kind == "sum":
            for j in range(len(reqs[0][1])):
                total = torch.stack([r[1][j] for r in reqs]).sum(dim=0).to(reqs[0][1][j].dtype)
                for r in reqs:
                    r[1][j].copy_(total)
        elif kind == "gather":
            for j in range(len(reqs[0][1])):
                cat = torch.cat([r[1][j][1].contiguous().view(-1) for r in reqs])
                for r in reqs:
                    r[1][j][0].view(-1).copy_(cat)
        else:
            raise ValueError(f"unknown exchange {kind!r}")
        nxt = []
        for i, p in enumerate(programs):
            try:
                nxt.append(p.send(None))
            except StopIteration as stop:
                results[i] = stop.value
                nxt.append(None)
        reqs = nxt
