"""int4 with a ragged last block (K not a multiple of the block size: the last
block of each row covers the remaining codes) through the C ABI against the
oracle (needs a B200).

Canonical layout: K % 16 == 0 with any block size; the B200_V1 layout keeps
K % 128 == 0, so there the ragged case is block 256 with K = 128 mod 256.
Every GEMV family that can run a shape is forced in turn; exports are
compared bit for bit; outputs sit between guard bands."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover - CPU-only container
    pytestmark = pytest.mark.skip(reason="needs a CUDA GPU")
else:
    pytestmark = pytest.mark.gpu

import weight_only_quantized_q4_b200 as wq  # noqa: E402
from _gpu import Guarded, Int4Case, check, each_variant, sample_rows  # noqa: E402
from test_gpu_swiglu import SwiGLUCase  # noqa: E402

gpu = pytest.mark.gpu
V1 = wq.WQ_LAYOUT_B200_V1

# (N, K, block, zero-points): last blocks of 128, 16, 80, 128, 16 and 64 codes
CANONICAL = [(37, 896, 256, True), (300, 1040, 128, True), (64, 1008, 32, False), (129, 4224, 256, True),
             (1000, 2000, 128, False), (5, 4160, 128, True)]
V1_SHAPES = [(37, 896, 256, True), (300, 4224, 256, False), (16, 1152, 256, True), (1000, 2432, 256, True)]


@gpu
@pytest.mark.parametrize("N,K,bs,zeros", CANONICAL)
def test_dequant_int4_ragged_bit_exact(N, K, bs, zeros):
    c = Int4Case(1, N, K, bs, zeros, workload=101)
    assert c.s.shape == (N, -(-K // bs))
    go = Guarded((N, K), torch.float32)
    wq.dequant_int4_blockwise(c.dw, c.ds, c.dz, go.t, N, K, bs)
    torch.cuda.synchronize()
    go.check("ragged int4 dequant export")
    ref = c.W().astype(np.float32)
    assert np.array_equal(go.t.cpu().numpy().view(np.uint32), ref.view(np.uint32))


@gpu
@pytest.mark.parametrize("N,K,bs,zeros", V1_SHAPES)
def test_dequant_int4_ragged_v1_layout_bit_exact(N, K, bs, zeros):
    """The repack puts the short last block's scale and zero-point in the band's last tile."""
    c = Int4Case(1, N, K, bs, zeros, workload=102, layout=V1)
    assert wq.wq_int4_packed_bytes(N, K, bs, V1) == ((N + 15) // 16) * (K // 128) * 1072
    go = Guarded((N, K), torch.float32)
    wq.dequant_int4_blockwise(c.dw, c.ds, c.dz, go.t, N, K, bs, layout=V1)
    torch.cuda.synchronize()
    go.check("ragged int4 B200_V1 dequant export")
    assert np.array_equal(go.t.cpu().numpy().view(np.uint32), c.W().astype(np.float32).view(np.uint32))


@gpu
@pytest.mark.parametrize("M", [1, 2, 3, 5, 8, 11])
@pytest.mark.parametrize("N,K,bs,zeros", CANONICAL)
def test_gemv_int4_ragged(M, N, K, bs, zeros):
    c = Int4Case(M, N, K, bs, zeros, workload=103)
    labels = each_variant(c.run, c.W(), c.x, f"ragged int4 M={M} N={N} K={K} bs={bs} zp={zeros}")
    if K % 128 == 0 and M <= 8:
        assert ".tc." in labels["tc"], labels
    assert ".simple." in labels["simple"], labels


@gpu
@pytest.mark.parametrize("M", [1, 2, 3, 4, 8, 11, 33])
@pytest.mark.parametrize("N,K,bs,zeros", V1_SHAPES)
def test_gemv_int4_ragged_v1_layout(M, N, K, bs, zeros):
    """Every B200_V1 family (band ring, stream-K, register stream, warp MMA,
    and tcgen05 past M = 8) on the short last block; repeat calls agree bit for bit."""
    c = Int4Case(M, N, K, bs, zeros, workload=104, layout=V1)
    labels = each_variant(c.run, c.W(), c.x, f"ragged int4 v1 M={M} N={N} K={K} zp={zeros}")
    if M <= 8:
        assert ".v1" in labels["v1s"] and ".v1k." in labels["v1k"] and ".v1r." in labels["v1r"], labels
    else:
        assert ".v1tc." in labels["v1tc"], labels
        fills = 2 * -(-N // 128) > torch.cuda.get_device_properties(0).multi_processor_count
        assert (".v1tc." in labels["default"]) if (M > 24 or fills) else (".v1w." in labels["default"]), labels
    assert np.array_equal(c.run(), c.run())


@gpu
@pytest.mark.parametrize("M", [1, 4])
def test_gemv_int4_ragged_full_size_sampled(M):
    """A decode-sized shape with a ragged block: 4864 rows, K = 896 with block 256
    (three full blocks and one of 128), both layouts."""
    for layout in (0, V1):
        c = Int4Case(M, 4864, 896, 256, True, workload=105, layout=layout)
        rows = sample_rows(4864)
        y = c.run()
        check(y[:, rows], c.W(rows), c.x, f"ragged 4864x896 layout={layout} M={M}")


@gpu
@pytest.mark.parametrize("M", [1, 3, 8])
@pytest.mark.parametrize("N,K", [(37, 896), (300, 4224)])
def test_swiglu_ragged(M, N, K):
    c = SwiGLUCase(M, N, K, 256, True, workload=106)
    y = c.run()
    assert "int4.swiglu.v1k" in wq.last_kernel(), wq.last_kernel()
    c.check(y)


@gpu
def test_ragged_needs_k_multiple_of_16():
    c = Int4Case(1, 16, 1024, 128, True, workload=107)
    with pytest.raises(wq.WQError) as e:
        wq.gemv_int4_blockwise(c.dx, c.dw, c.ds, c.dz, torch.empty((1, 16), dtype=torch.float16, device="cuda:0"),
                               1, 16, 1000, 128)
    assert e.value.code == wq.WQ_ERR_ARG
    with pytest.raises(wq.WQError) as e:
        wq.wq_repack_int4(c.dw, c.ds, c.dz, torch.empty(1 << 16, dtype=torch.uint8, device="cuda:0"), 16, 1040, 256, V1)
    assert e.value.code == wq.WQ_ERR_ARG
