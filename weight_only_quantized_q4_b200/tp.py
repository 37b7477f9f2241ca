"""Row-split (tensor-parallel) int4 layers over several GPUs, one process each.

Every rank keeps the rows [n0, n1) of W (``wq_tp_rows``, whole 16-row bands),
repacked alone into the B200_V1 stream, and computes those outputs with
``gemv_int4_tp``.  The all-gather of y is fused into that GEMV: its epilogue
stores the rank's outputs into every rank's copy of y, the peers' copies
mapped into this process through CUDA IPC (``PeerOutputs``).  After a barrier
every GPU holds the whole y.  ``gather_rows`` is the unfused alternative: each
rank writes its own slice, then an all-gather collective (NCCL on GPUs, gloo
on CPU) assembles y.

torch.distributed is only the plumbing here (handle exchange, barriers, the
unfused collective); the arithmetic runs in libwq.
"""
from __future__ import annotations

from . import api


def shard_rows(N: int, world: int, rank: int, align: int = 16):
    """Rows (n0, n1) of this rank."""
    return api.wq_tp_rows(N, world, rank, align)


def shard_int4(w_packed, scales, zeros, n0: int, n1: int):
    """The canonical int4 arrays of rows [n0, n1) (codes [N][K/2], scales
    [N][nb], zero-points [N][ceil(nb/2)] or None): row slices, contiguous."""
    cut = lambda a: None if a is None else a[n0:n1].contiguous() if hasattr(a, "contiguous") else a[n0:n1].copy()  # noqa: E731
    return cut(w_packed), cut(scales), cut(zeros)


class PeerOutputs:
    """Every rank's full y buffer, mapped into this process.

    ``y`` is this rank's own [M][N] fp16 output; the buffers of the other
    ranks of ``group`` are opened from their CUDA IPC handles.  ``ptrs`` lists
    the destinations for ``gemv_int4_tp``: this rank's buffer first."""

    def __init__(self, y, group=None):
        import torch.distributed as dist

        self.y = y
        world = dist.get_world_size(group)
        me = dist.get_rank(group)
        handles = [None] * world
        dist.all_gather_object(handles, api.wq_ipc_handle(y), group=group)
        self._opened = []
        self.ptrs = [y.data_ptr()]
        for r in range(world):
            if r != me:
                h, off = handles[r]
                p = api.wq_ipc_open(h, off)
                self._opened.append((p, off))
                self.ptrs.append(p)

    def close(self):
        for p, off in self._opened:
            api.wq_ipc_close(p, off)
        self._opened = []


def gemv_int4_rows(x, w_shard, peers: PeerOutputs, M: int, K: int, block_size: int, N: int, n0: int, n1: int,
                   stream=None):
    """This rank's rows of y, stored into every rank's y (the fused all-gather)."""
    if n1 > n0:
        api.gemv_int4_tp(x, w_shard, peers.ptrs, M, n1 - n0, K, block_size, N, n0, stream=stream)


def gather_rows(y_local, y_full, rows, group=None):
    """Unfused all-gather: y_local [M][n1 - n0] of every rank into y_full [M][N]
    (rows[r] = (n0, n1) of rank r); one all_gather of equal-size padded slices."""
    import torch
    import torch.distributed as dist

    M = y_full.shape[0]
    width = max(n1 - n0 for n0, n1 in rows)
    me = dist.get_rank(group)
    pad = torch.zeros((M, width), dtype=y_local.dtype, device=y_local.device)
    pad[:, :y_local.shape[1]] = y_local
    parts = [torch.empty_like(pad) for _ in rows]
    dist.all_gather(parts, pad, group=group)
    for r, (n0, n1) in enumerate(rows):
        y_full[:, n0:n1] = parts[r][:, :n1 - n0] if r != me else y_local
    return y_full
