"""Back-to-back dependent calls: the output of one GEMV is the activation of
the next, and one intermediate buffer is reused by every pair.  The kernels
start early under programmatic dependent launch and must wait for the
previous kernel before reading x and before writing y; any missing wait shows
up as a result that differs from the same calls run one at a time (the
kernels are deterministic, so the comparison is bitwise)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import weight_only_quantized_q4_b200 as wq
from weight_only_quantized_q4_b200 import synth

gpu = pytest.mark.gpu
DEV = "cuda:0"


def _int4_v1(N, K, workload):
    t = synth.int4_weights(N, K, 128, scale_lo=0.002, scale_hi=0.01, with_zeros=True, workload=workload)
    dw, ds, dz = (torch.from_numpy(t[k]).to(DEV) for k in ("w_packed", "scales", "zeros"))
    packed = torch.empty((wq.wq_int4_packed_bytes(N, K, 128, wq.WQ_LAYOUT_B200_V1),), dtype=torch.uint8, device=DEV)
    wq.wq_repack_int4(dw, ds, dz, packed, N, K, 128, wq.WQ_LAYOUT_B200_V1)

    def run(x, y):
        wq.gemv_int4_blockwise(x, packed, None, None, y, 1, N, K, 128, layout=wq.WQ_LAYOUT_B200_V1)
    return run


def _int4_canonical(N, K, workload):
    t = synth.int4_weights(N, K, 128, scale_lo=0.002, scale_hi=0.01, with_zeros=True, workload=workload)
    dw, ds, dz = (torch.from_numpy(t[k]).to(DEV) for k in ("w_packed", "scales", "zeros"))

    def run(x, y):
        wq.gemv_int4_blockwise(x, dw, ds, dz, y, 1, N, K, 128)
    return run


def _q4k(N, K, workload):
    raw = torch.from_numpy(synth.q4k_weights(N, K, workload=workload)).to(DEV)

    def run(x, y):
        wq.gemv_q4k(x, raw, y, 1, N, K)
    return run


MAKERS = {"int4_v1": _int4_v1, "int4_canonical": _int4_canonical, "q4k": _q4k}


@gpu
@pytest.mark.parametrize("first,second", [("int4_v1", "int4_v1"), ("int4_v1", "q4k"), ("q4k", "int4_canonical"),
                                          ("int4_canonical", "int4_v1")])
@pytest.mark.parametrize("graph", [False, True])
def test_chained_calls_match_isolated_calls(first, second, graph):
    torch.cuda.set_device(DEV)
    K1, N1, N2 = 4096, 2048, 1024  # y of the first call (N1 wide) is x of the second (K2 = N1)
    f = MAKERS[first](N1, K1, 41)
    g = MAKERS[second](N2, N1, 42)
    reps = 12
    xs = [torch.from_numpy(synth.activations_f16(1, K1, workload=50 + i)).to(DEV) for i in range(reps)]
    # one at a time (synchronised after every call)
    want = []
    for x in xs:
        y1 = torch.empty((1, N1), dtype=torch.float16, device=DEV)
        f(x, y1)
        torch.cuda.synchronize()
        y2 = torch.empty((1, N2), dtype=torch.float16, device=DEV)
        g(y1, y2)
        torch.cuda.synchronize()
        want.append(y2.cpu())
    # back to back, one shared intermediate buffer
    y1 = torch.empty((1, N1), dtype=torch.float16, device=DEV)
    outs = [torch.empty((1, N2), dtype=torch.float16, device=DEV) for _ in range(reps)]

    def chain():
        for x, y2 in zip(xs, outs):
            f(x, y1)
            g(y1, y2)

    if graph:
        s = torch.cuda.Stream()
        with torch.cuda.stream(s):
            chain()  # configure every kernel outside capture
        torch.cuda.synchronize()
        for y2 in outs:
            y2.zero_()
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=s):
            chain()
        for _ in range(3):
            gr.replay()
    else:
        chain()
    torch.cuda.synchronize()
    wq.wq_device_status()
    for i, (y2, w) in enumerate(zip(outs, want)):
        assert np.array_equal(y2.cpu().view(torch.int16).numpy(), w.view(torch.int16).numpy()), (first, second, i)
