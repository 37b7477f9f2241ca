"""mxfp4 blockwise weights (E2M1 codes, E8M0 block scales of 32 along K)
through the C ABI against the oracle's dequant_mxfp4 (needs a B200).

The dequant export is compared bit for bit with the oracle's fp64 values
rounded to fp32 (exact unless past the fp32 range, where both give ±inf);
the GEMV per element against 2e-3·Σ|w·x| + 1e-3, with guard bands around
every output and two calls in a row compared bit for bit."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover - CPU-only container
    pytestmark = pytest.mark.skip(reason="needs a CUDA GPU")
else:
    pytestmark = pytest.mark.gpu

import oracle  # noqa: E402
import weight_only_quantized_q4_b200 as wq  # noqa: E402
from _gpu import Guarded, check, dev, sample_rows  # noqa: E402
from weight_only_quantized_q4_b200 import synth  # noqa: E402

gpu = pytest.mark.gpu


def _run(x, t, M, N, K):
    g = Guarded((M, N), torch.float16)
    wq.gemv_mxfp4(dev(x), dev(t["w_packed"]), dev(t["scales"]), g.t, M, N, K)
    torch.cuda.synchronize()
    g.check(f"mxfp4 y M={M} N={N} K={K}")
    return g.t.cpu().numpy().astype(np.float64)


@gpu
@pytest.mark.parametrize("N,K", [(37, 96), (300, 2048), (64, 32)])
def test_dequant_mxfp4_bit_exact(N, K):
    t = synth.mxfp4_weights(N, K, workload=60)
    s = t["scales"].copy()
    s[0, 0], s[1 % N, -1], s[2 % N, 0] = 0, 254, 255  # 2^-127 (subnormal), 2^127 (overflows at |e2m1| >= 2), NaN
    g = Guarded((N, K), torch.float32)
    wq.dequant_mxfp4(dev(t["w_packed"]), dev(s), g.t, N, K)
    torch.cuda.synchronize()
    g.check("mxfp4 dequant export")
    got = g.t.cpu().numpy()
    with np.errstate(over="ignore", invalid="ignore"):
        ref = oracle.dequant_mxfp4(t["w_packed"], s, N, K).astype(np.float32)
    assert np.array_equal(got.view(np.uint32)[~np.isnan(ref)], ref.view(np.uint32)[~np.isnan(ref)])
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    assert wq.last_kernel() == "mxfp4.dequant"


@gpu
@pytest.mark.parametrize("M", [1, 2, 3, 5, 8, 11])
@pytest.mark.parametrize("N,K", [(37, 96), (300, 2048), (1000, 4128)])
def test_gemv_mxfp4(M, N, K):
    """Ragged bands (N = 37, 300, 1000), K with a block count that is not a
    multiple of the warps' stride (96, 4128), batches past 8 in chunks."""
    t = synth.mxfp4_weights(N, K, workload=61)
    x = synth.activations_f16(M, K, workload=61)
    y = _run(x, t, M, N, K)
    assert wq.last_kernel().startswith("mxfp4.gemv.mx"), wq.last_kernel()
    check(y, oracle.dequant_mxfp4(t["w_packed"], t["scales"], N, K), x, f"mxfp4 M={M} N={N} K={K}")
    assert np.array_equal(y, _run(x, t, M, N, K))


@gpu
@pytest.mark.parametrize("N,K", [(4096, 14336), (14336, 4096)])
def test_gemv_mxfp4_full_size_sampled(N, K):
    t = synth.mxfp4_weights(N, K, workload=62)
    rows = sample_rows(N)
    Wr = oracle.dequant_mxfp4(t["w_packed"][rows], t["scales"][rows], len(rows), K)
    for M in (1, 4, 8):
        x = synth.activations_f16(M, K, workload=62)
        y = _run(x, t, M, N, K)
        check(y[:, rows], Wr, x, f"mxfp4 full {N}x{K} M={M}")


@gpu
def test_gemv_mxfp4_special_scales():
    """A NaN scale (E = 255) makes its row NaN; E = 0 (2^-127) rows stay
    within the bound (absolute term); the other rows are unaffected."""
    N, K, M = 48, 256, 2
    t = synth.mxfp4_weights(N, K, workload=63)
    t["scales"][5, 3] = 255
    t["scales"][9, :] = 0
    x = synth.activations_f16(M, K, workload=63)
    y = _run(x, t, M, N, K)
    assert np.isnan(y[:, 5]).all()
    keep = np.array([n for n in range(N) if n != 5])
    W = oracle.dequant_mxfp4(t["w_packed"][keep], t["scales"][keep], len(keep), K)
    check(y[:, keep], W, x, "mxfp4 special scales")


@gpu
def test_gemv_mxfp4_argument_errors(monkeypatch):
    t = synth.mxfp4_weights(16, 64, workload=64)
    x, w, s = dev(synth.activations_f16(1, 64, workload=64)), dev(t["w_packed"]), dev(t["scales"])
    y = torch.empty((1, 16), dtype=torch.float16, device="cuda:0")
    with pytest.raises(wq.WQError) as e:
        wq.gemv_mxfp4(x, w, s, y, 1, 16, 48)
    assert e.value.code == wq.WQ_ERR_ARG
    monkeypatch.setenv("WQ_FORCE_KERNEL", "tc")
    with pytest.raises(wq.WQError) as e:
        wq.gemv_mxfp4(x, w, s, y, 1, 16, 64)
    assert e.value.code == wq.WQ_ERR_UNSUPPORTED
    monkeypatch.setenv("WQ_FORCE_KERNEL", "mx")
    wq.gemv_mxfp4(x, w, s, y, 1, 16, 64)
    torch.cuda.synchronize()
