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


def _kernel_copy(dst, src):
    """dst = src through an elementwise torch kernel (not a memcpy), so the
    write comes from a kernel the GEMV may overlap with."""
    it = torch.int16 if src.element_size() == 2 else torch.uint8
    torch.bitwise_or(src.view(it), 0, out=dst.view(it))


@gpu
@pytest.mark.parametrize("case", ["int4_v1_repack", "int4_canonical_torch_kernel", "q4k_torch_kernel"])
def test_weights_written_by_the_kernel_right_before(case):
    """The kernel right before a GEMV on the same stream writes that GEMV's
    weights (the load-time repack, or a torch elementwise kernel), with no
    synchronization in between: the GEMV must read the new weights.  Weights
    alternate between two seeded sets, so stale data would show."""
    import oracle

    torch.cuda.set_device(DEV)
    N, K = 2048, 4096
    s = torch.cuda.Stream()
    x = synth.activations_f16(1, K, workload=61)
    dx = torch.from_numpy(x).to(DEV)
    sets, refs = [], []
    for wl in (62, 63):
        if case.startswith("int4"):
            t = synth.int4_weights(N, K, 128, scale_lo=0.002, scale_hi=0.01, with_zeros=True, workload=wl)
            sets.append([torch.from_numpy(t[k]).to(DEV) for k in ("w_packed", "scales", "zeros")])
            W = oracle.dequant_int4(t["w_packed"], t["scales"], t["zeros"], N, K, 128)
        else:
            raw = synth.q4k_weights(N, K, workload=wl)
            sets.append([torch.from_numpy(raw).to(DEV)])
            W = oracle.dequant_q4k(raw, N, K)
        refs.append((oracle.gemv(W, x), oracle.bound(W, x)))
    if case == "int4_v1_repack":
        live = torch.empty((wq.wq_int4_packed_bytes(N, K, 128, wq.WQ_LAYOUT_B200_V1),), dtype=torch.uint8, device=DEV)
    else:
        live = [torch.empty_like(t) for t in sets[0]]
    torch.cuda.synchronize()
    outs = [torch.empty((1, N), dtype=torch.float16, device=DEV) for _ in range(8)]
    with torch.cuda.stream(s):
        for i, y in enumerate(outs):
            src = sets[i % 2]
            if case == "int4_v1_repack":
                wq.wq_repack_int4(src[0], src[1], src[2], live, N, K, 128, wq.WQ_LAYOUT_B200_V1, stream=s)
                wq.gemv_int4_blockwise(dx, live, None, None, y, 1, N, K, 128, layout=wq.WQ_LAYOUT_B200_V1, stream=s)
            elif case == "int4_canonical_torch_kernel":
                for dst, t in zip(live, src):
                    _kernel_copy(dst, t)
                wq.gemv_int4_blockwise(dx, live[0], live[1], live[2], y, 1, N, K, 128, stream=s)
            else:
                _kernel_copy(live[0], src[0])
                wq.gemv_q4k(dx, live[0], y, 1, N, K, stream=s)
    torch.cuda.synchronize()
    wq.wq_device_status()
    for i, y in enumerate(outs):
        y_ref, B = refs[i % 2]
        bad = oracle.violations(y.cpu().numpy().astype(np.float64), y_ref, B)
        assert not bad.any(), (case, i, int(bad.sum()))
