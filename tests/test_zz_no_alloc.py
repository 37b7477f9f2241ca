"""gemv_q4k_noalloc, the q4_K GEMV for callers that must not allocate device
memory (programs that own all device memory through their own pool or a
fixed budget, or that must not let a library call block or synchronize the
device as cudaMalloc can), checked against the ordinary gemv_q4k on the same
B200_V1 weights.

The allocation-free call keeps its scratch in one fixed array of the
library's device memory shared by every call; two calls in a row must both
give the ordinary call's result within the tolerance used throughout the
tests (|y - y_ref| <= 2e-3·Σ|w·x| + 1e-3).  This file is collected last, so a
run that stops at the first failure has run every other test first; it also
passes when run alone in a fresh process."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover - CPU-only container
    pytestmark = pytest.mark.skip(reason="needs a CUDA GPU")
else:
    pytestmark = pytest.mark.gpu

import oracle  # noqa: E402
import weight_only_quantized_q4_b200 as wq  # noqa: E402
from weight_only_quantized_q4_b200 import synth  # noqa: E402

gpu = pytest.mark.gpu
DEV = "cuda:0"


@gpu
@pytest.mark.parametrize("M,N,K", [(1, 4096, 11008), (3, 300, 2048), (8, 1000, 4096), (2, 37, 256)])
def test_noalloc_matches_the_ordinary_call_twice(M, N, K):
    torch.cuda.set_device(DEV)
    raw = synth.q4k_weights(N, K, workload=95)
    x = synth.activations_f16(M, K, workload=95)
    packed = torch.empty((wq.wq_q4k_packed_bytes(N, K),), dtype=torch.uint8, device=DEV)
    wq.wq_repack_q4k(torch.from_numpy(raw).to(DEV), packed, N, K)
    dx = torch.from_numpy(x).to(DEV)
    y_ref = torch.empty((M, N), dtype=torch.float16, device=DEV)
    wq.gemv_q4k(dx, packed, y_ref, M, N, K, layout=wq.WQ_LAYOUT_B200_V1)
    torch.cuda.synchronize()
    ref = y_ref.cpu().numpy().astype(np.float64)
    W = oracle.dequant_q4k(raw, N, K)
    B = oracle.bound(W, x)
    for call in range(2):  # the shared array keeps the previous call's contents
        y = torch.full((M, N), float("nan"), dtype=torch.float16, device=DEV)
        wq.gemv_q4k_noalloc(dx, packed, y, M, N, K)
        torch.cuda.synchronize()
        assert "noalloc" in wq.last_kernel(), wq.last_kernel()
        got = y.cpu().numpy().astype(np.float64)
        bad = oracle.violations(got, ref, B)
        assert not bad.any(), f"call {call}: {int(bad.sum())} of {bad.size} outside the tolerance"
    wq.wq_device_status()


@gpu
def test_noalloc_rejects_sizes_beyond_its_fixed_scratch():
    torch.cuda.set_device(DEV)
    N, K = 65537, 256
    z = torch.zeros(16, dtype=torch.uint8, device=DEV)
    with pytest.raises(wq.WQError) as e:
        wq.gemv_q4k_noalloc(z, z, z, 1, N, K)
    assert e.value.code == wq.WQ_ERR_ARG and "65536" in str(e.value)
