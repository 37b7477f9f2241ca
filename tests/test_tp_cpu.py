"""Host-side logic of the row-split (tensor-parallel) layers, on CPU: the row
planner covers N exactly in whole bands, and the unfused all-gather assembles
the ranks' slices (computed here by the oracle) into the full y under two and
three gloo ranks."""
from __future__ import annotations

import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import weight_only_quantized_q4_b200 as wq  # noqa: E402


@pytest.mark.parametrize("align", [1, 16, 128])
def test_tp_rows_cover_n_exactly(align):
    for N in (1, 15, 16, 17, 100, 4096, 14336, 32000, 151936):
        for world in (1, 2, 3, 4, 7, 8):
            rows = [wq.wq_tp_rows(N, world, r, align) for r in range(world)]
            assert rows[0][0] == 0 and rows[-1][1] == N
            for (a0, a1), (b0, b1) in zip(rows, rows[1:]):
                assert a1 == b0  # contiguous, disjoint
            sizes = [n1 - n0 for n0, n1 in rows]
            assert all(s >= 0 for s in sizes)
            assert all(n0 % align == 0 for n0, n1 in rows if n1 > n0)  # a rank with rows starts on a unit
            full = [s for s, (n0, n1) in zip(sizes, rows) if n1 < N]
            assert not full or max(full) - min(full) <= align  # as even as the unit allows


def test_tp_rows_rejects_bad_arguments():
    for args in ((0, 2, 0, 16), (16, 0, 0, 16), (16, 2, 2, 16), (16, 2, -1, 16), (16, 2, 0, 0)):
        with pytest.raises(wq.WQError) as e:
            wq.wq_tp_rows(*args)
        assert e.value.code == wq.WQ_ERR_ARG


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, q) -> None:
    import datetime

    import torch
    import torch.distributed as dist

    import oracle
    from weight_only_quantized_q4_b200 import synth, tp

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        M, N, K, bs = 3, 100, 256, 128
        t = synth.int4_weights(N, K, bs, scale_lo=0.002, scale_hi=0.01, with_zeros=True, workload=140)
        x = synth.activations_f16(M, K, workload=140)
        rows = [tp.shard_rows(N, world, r) for r in range(world)]
        n0, n1 = rows[rank]
        w, s, z = tp.shard_int4(t["w_packed"], t["scales"], t["zeros"], n0, n1)
        # this rank's slice of y (the oracle stands in for the GPU kernel here)
        y_loc = oracle.gemv(oracle.dequant_int4(w, s, z, n1 - n0, K, bs), x.astype(np.float64))
        y_full = torch.full((M, N), float("nan"), dtype=torch.float64)
        tp.gather_rows(torch.from_numpy(y_loc), y_full, rows)
        q.put((rank, y_full.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_unfused_gather_assembles_every_ranks_rows(world):
    import oracle
    from weight_only_quantized_q4_b200 import synth

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    M, N, K, bs = 3, 100, 256, 128
    t = synth.int4_weights(N, K, bs, scale_lo=0.002, scale_hi=0.01, with_zeros=True, workload=140)
    x = synth.activations_f16(M, K, workload=140)
    ref = oracle.gemv(oracle.dequant_int4(t["w_packed"], t["scales"], t["zeros"], N, K, bs), x.astype(np.float64))
    for _, y in got:
        assert np.array_equal(y, ref)
