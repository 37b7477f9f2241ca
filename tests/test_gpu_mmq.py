"""int8-activation batched q4_K through the C ABI (needs a B200): the q8
prepass against the oracle's quantize_q8 bit for bit, and the tcgen05
kind::i8 GEMM against the oracle's mmq_q4k within 2e-3·Σ|w·x̂| + 1e-3 per
element (x̂ = d·q, the activations the path multiplies by).

Every output lives between guard bands; repeat calls agree bit for bit; the
W_dsc-plane form gives the same bits as the in-kernel coefficients."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover - CPU-only container
    pytestmark = pytest.mark.skip(reason="needs a CUDA GPU")
else:
    pytestmark = pytest.mark.gpu

import oracle  # noqa: E402
import weight_only_quantized_q4_b200 as wq  # noqa: E402
from _gpu import Guarded, dev, sample_rows  # noqa: E402
from weight_only_quantized_q4_b200 import synth  # noqa: E402

gpu = pytest.mark.gpu


def _q8_dev(x, M, K):
    gq = Guarded((M, K), torch.int8)
    gs = Guarded((wq.wq_q8_scale_bytes(M, K) // 4,), torch.float32)
    wq.quantize_q8(dev(x), gq.t, gs.t, M, K)
    torch.cuda.synchronize()
    gq.check("q8 codes")
    gs.check("q8 scales")
    return gq, gs


def _sda_host(gs, M, K):
    Mp = (M + 15) // 16 * 16
    a = gs.t.cpu().numpy().reshape(K // 32, Mp, 2)
    return a[:, :M, 0].T.copy(), a[:, :M, 1].T.copy(), a[:, M:, :]


class MMQCase:
    def __init__(self, M, N, K, workload, x=None):
        self.M, self.N, self.K = M, N, K
        self.raw = synth.q4k_weights(N, K, workload=workload)
        self.x = synth.activations_f16(M, K, workload=workload) if x is None else x
        self.qa, self.d, self.s = oracle.quantize_q8(self.x, M, K)
        self.gq, self.gs = _q8_dev(self.x, M, K)
        self.draw = dev(self.raw)
        self._plane = None

    def plane(self):
        if self._plane is None:
            g = Guarded((self.K // 32, self.N, 2), torch.float32)
            wq.wq_build_q4k_dsc_device(self.draw, g.t, self.N, self.K)
            torch.cuda.synchronize()
            g.check("W_dsc plane")
            self._plane = g
        return self._plane.t

    def run(self, dsc=False, stream=None):
        g = Guarded((self.M, self.N), torch.float16)
        wq.gemm_q4k_q8(self.gq.t, self.gs.t, self.draw, self.plane() if dsc else None, g.t, self.M, self.N, self.K,
                       stream=stream)
        torch.cuda.synchronize()
        g.check(f"mmq y M={self.M} N={self.N} K={self.K}")
        return g.t.cpu().numpy().astype(np.float64)

    def check(self, y, rows=None):
        r = np.arange(self.N) if rows is None else np.asarray(rows)
        raw = self.raw[r]
        ref = oracle.mmq_q4k(raw, self.qa, self.d, self.s, self.M, len(r), self.K)
        W = oracle.dequant_q4k(raw, len(r), self.K)
        xd = oracle.dequant_q8(self.qa, self.d, self.M, self.K)
        B = oracle.bound(W, xd)
        bad = oracle.violations(y[:, r], ref, B)
        if bad.any():
            i = np.argwhere(bad)[:4]
            raise AssertionError(f"mmq M={self.M} N={self.N} K={self.K}: {int(bad.sum())} of {bad.size} outside; "
                                 f"first {[(tuple(t), y[:, r][tuple(t)], ref[tuple(t)], B[tuple(t)]) for t in i]}")


# ----------------------------------------------------------------- prepass

@gpu
@pytest.mark.parametrize("M,K", [(1, 32), (3, 96), (5, 1024), (17, 4096), (40, 2048)])
def test_quantize_q8_bit_exact(M, K):
    x = synth.activations_f16(M, K, workload=120)
    if M >= 3:
        x[1, 32:64] = 0                                                   # a zero chunk
        x[2] = (x[2].astype(np.float64) * 1e-6).astype(np.float16)        # fp16 subnormals
    if M >= 5:
        x[4] = (x[4].astype(np.float64) * 1e4).astype(np.float16)         # large values (finite)
        x[3, :8] = [0.5, 1.5, 2.5, -0.5, -1.5, 127.0, 3.25, -2.5]          # ties, amax 127 (d = 1)
    gq, gs = _q8_dev(x, M, K)
    qa, d, s = oracle.quantize_q8(x, M, K)
    assert np.array_equal(gq.t.cpu().numpy(), qa)
    dd, ss, pad = _sda_host(gs, M, K)
    assert np.array_equal(dd.view(np.uint32), d.view(np.uint32))
    assert np.array_equal(ss.view(np.uint32), s.view(np.uint32))
    assert not pad.any()
    assert wq.last_kernel() == "q8.quantize"


# ----------------------------------------------------------------- GEMM

@gpu
@pytest.mark.parametrize("M", [1, 9, 16, 17, 33, 64, 100, 128, 200])
@pytest.mark.parametrize("N,K", [(37, 256), (300, 1024), (129, 2048), (1000, 4096)])
def test_gemm_q4k_q8(M, N, K):
    c = MMQCase(M, N, K, workload=121)
    y = c.run()
    assert wq.last_kernel().startswith("q4k.mmq."), wq.last_kernel()
    c.check(y)
    assert np.array_equal(y, c.run())


@gpu
@pytest.mark.parametrize("M", [16, 64, 128])
@pytest.mark.parametrize("N,K", [(300, 1024), (1000, 4096)])
def test_gemm_q4k_q8_plane_is_bit_identical(M, N, K):
    """The coefficients read from the W_dsc plane equal the in-kernel products
    (one fp32 multiply each, no contraction), so y is the same to the bit."""
    c = MMQCase(M, N, K, workload=122)
    y0 = c.run()
    y1 = c.run(dsc=True)
    assert wq.last_kernel().endswith(".dsc"), wq.last_kernel()
    assert np.array_equal(y0, y1)


@gpu
@pytest.mark.parametrize("S", [1, 2, 4, 8])
@pytest.mark.parametrize("M", [16, 40, 128])
@pytest.mark.parametrize("K", [2048, 2816])
def test_gemm_q4k_q8_cluster_split(S, M, K, monkeypatch):
    """K split over clusters of S CTAs (K = 2816: eleven super-blocks, uneven
    runs per rank), partials added over distributed shared memory in rank order."""
    monkeypatch.setenv("WQ_MMQ_S", str(S))
    c = MMQCase(M, 300, K, workload=123)
    y = c.run()
    assert wq.last_kernel().endswith(f".s{S}"), wq.last_kernel()
    c.check(y)
    assert np.array_equal(y, c.run())


@gpu
@pytest.mark.parametrize("NS", [2, 3])
@pytest.mark.parametrize("NA", [2, 3])
@pytest.mark.parametrize("M", [33, 128])
def test_gemm_q4k_q8_ring_depths(NS, NA, M, monkeypatch):
    """Shallower stage rings and A-slot rings than the planner picks (the
    planner's choice is capped by shared memory, so a forced depth may come
    out smaller: the label tells)."""
    monkeypatch.setenv("WQ_MMQ_NS", str(NS))
    monkeypatch.setenv("WQ_MMQ_NA", str(NA))
    monkeypatch.setenv("WQ_MMQ_S", "1")
    c = MMQCase(M, 256, 4096, workload=124)
    y = c.run()
    assert ".ns" in wq.last_kernel() and ".na" in wq.last_kernel(), wq.last_kernel()
    c.check(y)


@gpu
@pytest.mark.parametrize("M", [16, 64, 128])
@pytest.mark.parametrize("N,K", [(4096, 4096), (11008, 4096), (4096, 11008), (32000, 4096)])
def test_gemm_q4k_q8_full_size_sampled(M, N, K):
    c = MMQCase(M, N, K, workload=125)
    y = c.run()
    c.check(y, sample_rows(N))


@gpu
def test_gemm_q4k_q8_special_activations():
    """A token of zeros gives y = 0 for that token; a one-hot token (the only
    non-zero value 1.0 at k) gives d = 1/127, q = 127 there, so y = w[:, k]·d·127."""
    M, N, K = 3, 64, 512
    x = synth.activations_f16(M, K, workload=126)
    x[0] = 0
    x[1] = 0
    x[1, 300] = 1.0
    c = MMQCase(M, N, K, workload=126, x=x)
    y = c.run()
    assert not y[0].any()
    c.check(y)


@gpu
def test_gemm_q4k_q8_argument_errors(monkeypatch):
    c = MMQCase(16, 32, 256, workload=127)
    y = torch.empty((16, 32), dtype=torch.float16, device="cuda:0")
    with pytest.raises(wq.WQError) as e:
        wq.gemm_q4k_q8(c.gq.t, c.gs.t, c.draw, None, y, 16, 32, 128)
    assert e.value.code == wq.WQ_ERR_ARG
    with pytest.raises(wq.WQError) as e:
        wq.quantize_q8(dev(c.x), c.gq.t, c.gs.t, 16, 48)
    assert e.value.code == wq.WQ_ERR_ARG
    monkeypatch.setenv("WQ_FORCE_KERNEL", "tc5")
    with pytest.raises(wq.WQError) as e:
        wq.gemm_q4k_q8(c.gq.t, c.gs.t, c.draw, None, y, 16, 32, 256)
    assert e.value.code == wq.WQ_ERR_UNSUPPORTED
    monkeypatch.setenv("WQ_FORCE_KERNEL", "mmq")
    wq.gemm_q4k_q8(c.gq.t, c.gs.t, c.draw, None, y, 16, 32, 256)
    torch.cuda.synchronize()
    monkeypatch.delenv("WQ_FORCE_KERNEL")
    monkeypatch.setenv("WQ_MMQ_S", "8")
    with pytest.raises(wq.WQError) as e:  # one super-block cannot be split eight ways
        wq.gemm_q4k_q8(c.gq.t, c.gs.t, c.draw, None, y, 16, 32, 256)
    assert e.value.code == wq.WQ_ERR_ARG


@gpu
def test_prepass_and_gemm_on_a_side_stream():
    """The two calls chained on one non-default stream, no host sync between them."""
    M, N, K = 33, 500, 2048
    raw = synth.q4k_weights(N, K, workload=128)
    x = synth.activations_f16(M, K, workload=128)
    s = torch.cuda.Stream()
    qa = torch.empty((M, K), dtype=torch.int8, device="cuda:0")
    sd = torch.empty(wq.wq_q8_scale_bytes(M, K) // 4, dtype=torch.float32, device="cuda:0")
    y = torch.empty((M, N), dtype=torch.float16, device="cuda:0")
    dx, dr = dev(x), dev(raw)
    torch.cuda.synchronize()
    wq.quantize_q8(dx, qa, sd, M, K, stream=s)
    wq.gemm_q4k_q8(qa, sd, dr, None, y, M, N, K, stream=s)
    s.synchronize()
    q, d, ss = oracle.quantize_q8(x, M, K)
    ref = oracle.mmq_q4k(raw, q, d, ss, M, N, K)
    B = oracle.bound(oracle.dequant_q4k(raw, N, K), oracle.dequant_q8(q, d, M, K))
    assert not oracle.violations(y.cpu().numpy().astype(np.float64), ref, B).any()
