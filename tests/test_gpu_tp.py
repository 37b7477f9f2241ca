"""Row-split int4 layers through the C ABI (needs a B200): gemv_int4_tp stores
a shard's outputs into several full-size destinations (the fused all-gather),
checked against the oracle; and two processes on one GPU exchange their y
buffers by CUDA IPC and each ends with the whole y.

The kernels of the two processes never wait on one another: each only
stores into the other's buffer, and the host orders the check after both
(stream synchronize, then a gloo barrier)."""
from __future__ import annotations

import os
import socket

import numpy as np
import pytest

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover - CPU-only container
    pytestmark = pytest.mark.skip(reason="needs a CUDA GPU")
else:
    pytestmark = pytest.mark.gpu

import oracle  # noqa: E402
import weight_only_quantized_q4_b200 as wq  # noqa: E402
from _gpu import Guarded, check, dev  # noqa: E402
from weight_only_quantized_q4_b200 import synth, tp  # noqa: E402

gpu = pytest.mark.gpu
V1 = wq.WQ_LAYOUT_B200_V1


def _shard_v1(t, n0, n1, K, bs):
    w, s, z = tp.shard_int4(t["w_packed"], t["scales"], t["zeros"], n0, n1)
    out = torch.empty(wq.wq_int4_packed_bytes(n1 - n0, K, bs, V1), dtype=torch.uint8, device="cuda:0")
    wq.wq_repack_int4(dev(w), dev(s), dev(z) if z is not None else None, out, n1 - n0, K, bs, V1)
    return out


@gpu
@pytest.mark.parametrize("M", [1, 4, 8, 11])
@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("N,K,bs", [(300, 2048, 128), (4096, 4096, 128), (100, 896, 256)])
def test_row_split_into_several_destinations(M, world, N, K, bs):
    """Every shard is stored into three destinations; after all shards each
    destination holds the whole y (within the GEMV bound of the oracle's), the
    three are identical, and nothing outside them is written."""
    t = synth.int4_weights(N, K, bs, scale_lo=0.002, scale_hi=0.01, with_zeros=True, workload=141)
    x = synth.activations_f16(M, K, workload=141)
    dx = dev(x)
    dsts = [Guarded((M, N), torch.float16) for _ in range(3)]
    for g in dsts:
        g.t.fill_(float("nan"))
    for r in range(world):
        n0, n1 = tp.shard_rows(N, world, r)
        if n1 == n0:
            continue
        ws = _shard_v1(t, n0, n1, K, bs)
        wq.gemv_int4_tp(dx, ws, [g.t for g in dsts], M, n1 - n0, K, bs, N, n0)
        assert wq.last_kernel().startswith("int4.gemv.v1s.tp."), wq.last_kernel()
    torch.cuda.synchronize()
    ys = []
    for i, g in enumerate(dsts):
        g.check(f"destination {i}")
        ys.append(g.t.cpu().numpy().astype(np.float64))
    assert all(np.array_equal(ys[0], y) for y in ys[1:])
    W = oracle.dequant_int4(t["w_packed"], t["scales"], t["zeros"], N, K, bs)
    check(ys[0], W, x, f"row split world={world} M={M} N={N} K={K}")


@gpu
def test_row_split_argument_errors():
    t = synth.int4_weights(32, 256, 128, scale_lo=0.002, scale_hi=0.01, with_zeros=True, workload=142)
    ws = _shard_v1(t, 0, 32, 256, 128)
    x = dev(synth.activations_f16(1, 256, workload=142))
    y = torch.empty((1, 64), dtype=torch.float16, device="cuda:0")
    for args in ((x, ws, [y], 1, 32, 256, 128, 64, 40),   # rows past the output
                 (x, ws, [], 1, 32, 256, 128, 64, 0),     # no destination
                 (x, ws, [y] * 9, 1, 32, 256, 128, 64, 0)):  # more than eight
        with pytest.raises(wq.WQError) as e:
            wq.gemv_int4_tp(*args)
        assert e.value.code == wq.WQ_ERR_ARG


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _ipc_rank(rank: int, world: int, port: int, q) -> None:
    import datetime

    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    peers = None
    try:
        torch.cuda.set_device(0)
        M, N, K, bs = 4, 1000, 2048, 128
        t = synth.int4_weights(N, K, bs, scale_lo=0.002, scale_hi=0.01, with_zeros=True, workload=143)
        x = synth.activations_f16(M, K, workload=143)
        n0, n1 = tp.shard_rows(N, world, rank)
        ws = _shard_v1(t, n0, n1, K, bs)
        y = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda:0")
        torch.cuda.synchronize()
        peers = tp.PeerOutputs(y)
        dist.barrier()  # every y is initialised before anyone stores into it
        tp.gemv_int4_rows(dev(x), ws, peers, M, K, bs, N, n0, n1)
        torch.cuda.synchronize()
        dist.barrier()  # every rank's stores have completed
        got = y.cpu().numpy().astype(np.float64)
        W = oracle.dequant_int4(t["w_packed"], t["scales"], t["zeros"], N, K, bs)
        check(got, W, x, f"ipc row split rank={rank}")
        q.put((rank, "ok", len(peers.ptrs)))
        dist.barrier()  # nobody releases a mapping another rank may still use
    except Exception as e:  # noqa: BLE001
        q.put((rank, repr(e), 0))
        raise
    finally:
        if peers is not None:
            peers.close()
        dist.destroy_process_group()


@gpu
def test_two_processes_gather_through_ipc():
    import torch.multiprocessing as mp

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_ipc_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=180) for _ in range(2))
    for p in procs:
        p.join(timeout=120)
    assert [g[1] for g in got] == ["ok", "ok"], got
    assert all(g[2] == 2 for g in got)
    assert all(p.exitcode == 0 for p in procs)
