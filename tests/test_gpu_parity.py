"""CUDA path vs the CPU oracle, through the C ABI (needs a B200).

Dequantization exports must match the oracle bit for bit; GEMV outputs must
satisfy |y − y_ref| ≤ 2e-3·Σ|w·x| + 1e-3 element by element.  Small cases
are compared whole; the full workload sizes, in the launch configuration the
benchmark uses, are compared on sampled rows.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover - CPU-only container
    pytestmark = pytest.mark.skip(reason="needs a CUDA GPU")
else:
    pytestmark = pytest.mark.gpu

import oracle  # noqa: E402
import weight_only_quantized_q4_b200 as wq  # noqa: E402
from _gpu import DEV, BF16Case, Int4Case, Q4KCase, check, dev, sample_rows  # noqa: E402
from weight_only_quantized_q4_b200 import synth  # noqa: E402

gpu = pytest.mark.gpu


# ----------------------------------------------------------- dequant exports

@gpu
@pytest.mark.parametrize("bs,zeros,N,K", [(32, False, 5, 1024), (128, True, 7, 1024), (16, True, 3, 80),
                                          (64, True, 9, 192), (256, False, 2, 512), (128, True, 4, 384)])
def test_dequant_int4_bit_exact(bs, zeros, N, K):
    c = Int4Case(1, N, K, bs, zeros, workload=11)
    out = torch.empty((N, K), dtype=torch.float32, device=DEV)
    wq.dequant_int4_blockwise(c.dw, c.ds, c.dz, out, N, K, bs)
    torch.cuda.synchronize()
    ref = c.W().astype(np.float32)
    got = out.cpu().numpy()
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))


@gpu
@pytest.mark.parametrize("N,K", [(3, 256), (5, 768), (8, 4096)])
@pytest.mark.parametrize("dsc", [False, True])
def test_dequant_q4k_bit_exact(N, K, dsc):
    c = Q4KCase(1, N, K, workload=12)
    out = torch.empty((N, K), dtype=torch.float32, device=DEV)
    wq.dequant_q4k(c.draw, c.plane_dev() if dsc else None, out, N, K)
    torch.cuda.synchronize()
    ref = c.W().astype(np.float32)
    assert np.array_equal(out.cpu().numpy().view(np.uint32), ref.view(np.uint32))


@gpu
@pytest.mark.parametrize("N,K", [(1, 256), (7, 512), (33, 2048)])
def test_plane_device_host_oracle_identical(N, K):
    raw = synth.q4k_weights(N, K, workload=13)
    P = torch.empty((K // 32, N, 2), dtype=torch.float32, device=DEV)
    wq.wq_build_q4k_dsc_device(dev(raw), P, N, K)
    torch.cuda.synchronize()
    host = wq.wq_build_q4k_dsc(raw, N, K)
    ref = oracle.q4k_plane(raw, N, K)
    assert np.array_equal(P.cpu().numpy().view(np.uint32), ref.view(np.uint32))
    assert np.array_equal(host.view(np.uint32), ref.view(np.uint32))


# ----------------------------------------------------------- GEMV, whole outputs

@gpu
@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 8])
@pytest.mark.parametrize("N,K,bs,zeros", [(256, 1024, 32, False), (37, 2048, 128, True), (301, 512, 16, True),
                                          (64, 4096, 64, True), (1000, 1536, 256, False)])
def test_gemv_int4_small(M, N, K, bs, zeros):
    c = Int4Case(M, N, K, bs, zeros, workload=21)
    check(c.run(), c.W(), c.x, f"int4 M={M} N={N} K={K} bs={bs} zp={zeros}")


@gpu
@pytest.mark.parametrize("M", [1, 2, 3, 4, 6, 8])
@pytest.mark.parametrize("N,K", [(3, 256), (129, 1024), (250, 2816), (64, 11008)])
@pytest.mark.parametrize("dsc", [False, True])
def test_gemv_q4k_small(M, N, K, dsc):
    c = Q4KCase(M, N, K, workload=22)
    check(c.run(dsc), c.W(), c.x, f"q4k dsc={dsc} M={M} N={N} K={K}")


@gpu
@pytest.mark.parametrize("M", [1, 2, 3, 4, 7, 8])
@pytest.mark.parametrize("N,K", [(256, 1536), (77, 6912), (300, 64)])
def test_gemv_bf16_small(M, N, K):
    c = BF16Case(M, N, K, workload=23)
    check(c.run(), c.W(), c.X(), f"bf16 M={M} N={N} K={K}")


@gpu
@pytest.mark.parametrize("K", [7, 12, 100, 1534])
@pytest.mark.parametrize("M", [1, 3])
@pytest.mark.parametrize("N", [256, 1536])
@pytest.mark.parametrize("offset", [0, 1])
def test_gemv_bf16_odd_k_and_offsets(K, M, N, offset):
    c = BF16Case(M, N, K, offset=offset, workload=24)
    check(c.run(), c.W(), c.X(), f"bf16 odd-K M={M} N={N} K={K} offset={offset}")


@gpu
@pytest.mark.parametrize("M", [9, 16, 17])
def test_gemv_larger_batches(M):
    c = Int4Case(M, 96, 1024, 128, True, workload=25)
    check(c.run(), c.W(), c.x, f"int4 M={M}")
    q = Q4KCase(M, 40, 512, workload=25)
    check(q.run(False), q.W(), q.x, f"q4k M={M}")
    b = BF16Case(M, 50, 256, workload=25)
    check(b.run(), b.W(), b.X(), f"bf16 M={M}")


# ----------------------------------------------------------- closed forms on the device

@gpu
def test_int4_zero_equals_code_gives_zero():
    """Every code equal to its block's zero-point: y must be exactly 0 (|y| ≤ 1e-3 is the bar)."""
    N, K, bs, M = 64, 1024, 128, 4
    codes = np.random.default_rng(5).integers(0, 16, (N, K // bs))
    w = np.repeat(codes, bs // 2, axis=1).astype(np.uint8)
    w = (w | (w << 4)).astype(np.uint8)
    z = np.zeros((N, (K // bs + 1) // 2), dtype=np.uint8)
    for b in range(K // bs):
        z[:, b // 2] |= (codes[:, b] << (4 * (b % 2))).astype(np.uint8)
    s = np.full((N, K // bs), 0.01, dtype=np.float16)
    x = synth.activations_f16(M, K, workload=26)
    y = torch.empty((M, N), dtype=torch.float16, device=DEV)
    wq.gemv_int4_blockwise(dev(x), dev(w), dev(s), dev(z), y, M, N, K, bs)
    torch.cuda.synchronize()
    W = oracle.dequant_int4(w, s, z, N, K, bs)
    assert np.all(W == 0)
    check(y.cpu().numpy().astype(np.float64), W, x, "int4 z=q")


@gpu
def test_one_hot_activation_reads_a_column():
    c = Q4KCase(1, 200, 1024, workload=27)
    x = np.zeros((1, 1024), dtype=np.float16)
    x[0, 517] = 1.0
    c.x = x
    c.dx = dev(x)
    y = c.run(False)
    ref = c.W()[:, 517].astype(np.float16).astype(np.float64)  # RN16 of the exact weight
    assert np.array_equal(y[0], ref)


# ----------------------------------------------------------- stream, liveness, status

@gpu
def test_uses_given_stream_and_labels():
    c = Int4Case(1, 4096, 4096, 128, True, workload=28)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        y = c.run()
    assert "int4.gemv.cc" in wq.last_kernel()
    check(y, c.W(), c.x, "int4 on a side stream")
    wq.wq_device_status()


# ----------------------------------------------------------- full workload sizes, sampled rows

FULL_INT4 = [(4096, 4096), (14336, 4096), (4096, 14336)]
FULL_Q4K = [(4096, 4096), (11008, 4096), (4096, 11008)]
FULL_BF16 = [(1536, 1536), (256, 1536), (1536, 6912), (151936, 1536)]


@gpu
@pytest.mark.parametrize("M", [1, 4])
@pytest.mark.parametrize("N,K", FULL_INT4)
def test_full_int4_b128_sampled(M, N, K):
    c = Int4Case(M, N, K, 128, True, workload=3)
    y = c.run()
    assert ".gemv." in wq.last_kernel()
    rows = sample_rows(N)
    check(y[:, rows], c.W(rows), c.x, f"int4 full {N}x{K} M={M}")


@gpu
def test_full_int4_b32_config():
    c = Int4Case(1, 256, 1024, 32, False, workload=1, s_lo=0.005, s_hi=0.02)
    check(c.run(), c.W(), c.x, "int4 b32 256x1024")


@gpu
@pytest.mark.parametrize("M", [1, 2, 4, 8])
@pytest.mark.parametrize("N,K", FULL_Q4K)
@pytest.mark.parametrize("dsc", [False, True])
def test_full_q4k_sampled(M, N, K, dsc):
    c = Q4KCase(M, N, K, workload=4)
    y = c.run(dsc)
    rows = sample_rows(N)
    check(y[:, rows], c.W(rows), c.x, f"q4k dsc={dsc} full {N}x{K} M={M}")


@gpu
@pytest.mark.parametrize("M", [1, 3, 8])
@pytest.mark.parametrize("N,K", FULL_BF16)
def test_full_bf16_sampled(M, N, K):
    c = BF16Case(M, N, K, workload=2)
    y = c.run()
    rows = sample_rows(N)
    check(y[:, rows], c.W(rows), c.X(), f"bf16 full {N}x{K} M={M}")
