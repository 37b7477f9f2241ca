"""Fused gate / up projection with the SiLU·mul epilogue (gemv_int4_swiglu)
against the oracle's swiglu_gemv, through the C ABI (needs a B200).

The acceptance bound is the oracle's swiglu_tolerance: each projection held to
the GEMV bound 2e-3·Σ|w·x| + 1e-3, carried through silu(a)·b, plus the fp16
rounding of y.  Guard bands surround every output; two calls in a row agree
bit for bit (the split-band fix-up adds pieces in a fixed order)."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover - CPU-only container
    pytestmark = pytest.mark.skip(reason="needs a CUDA GPU")
else:
    pytestmark = pytest.mark.gpu

import oracle  # noqa: E402
import weight_only_quantized_q4_b200 as wq  # noqa: E402
from _gpu import DEV, Guarded, dev, sample_rows  # noqa: E402
from weight_only_quantized_q4_b200 import synth  # noqa: E402

gpu = pytest.mark.gpu


class SwiGLUCase:
    def __init__(self, M, N, K, bs, zeros, workload):
        self.M, self.N, self.K, self.bs = M, N, K, bs
        self.gate = synth.int4_weights(N, K, bs, scale_lo=0.002, scale_hi=0.01, with_zeros=zeros, workload=workload)
        self.up = synth.int4_weights(N, K, bs, scale_lo=0.002, scale_hi=0.01, with_zeros=zeros, workload=workload + 50)
        self.x = synth.activations_f16(M, K, workload=workload)
        d = {h: [dev(t[k]) if t[k] is not None else None for k in ("w_packed", "scales", "zeros")]
             for h, t in (("g", self.gate), ("u", self.up))}
        self.guard = Guarded((wq.wq_int4_gate_up_packed_bytes(N, K, bs),), torch.uint8)
        wq.wq_repack_int4_gate_up(*d["g"], *d["u"], self.guard.t, N, K, bs)
        torch.cuda.synchronize()
        self.guard.check("fused gate-up repack output")
        self.dw, self.dx, self.dev_parts = self.guard.t, dev(self.x), d

    def run(self):
        g = Guarded((self.M, self.N), torch.float16)
        wq.gemv_int4_swiglu(self.dx, self.dw, g.t, self.M, self.N, self.K, self.bs)
        torch.cuda.synchronize()
        g.check(f"swiglu y M={self.M} N={self.N} K={self.K}")
        return g.t.cpu().numpy().astype(np.float64)

    def W(self, t, rows=None):
        r = slice(None) if rows is None else rows
        n = self.N if rows is None else len(rows)
        z = None if t["zeros"] is None else t["zeros"][r]
        return oracle.dequant_int4(t["w_packed"][r], t["scales"][r], z, n, self.K, self.bs)

    def check(self, y, rows=None):
        Wg, Wu = self.W(self.gate, rows), self.W(self.up, rows)
        a, b = oracle.gemv(Wg, self.x), oracle.gemv(Wu, self.x)
        ref = oracle.swiglu_gemv(Wg, Wu, self.x)
        tol = oracle.swiglu_tolerance(a, b, oracle.bound(Wg, self.x), oracle.bound(Wu, self.x))
        yy = y if rows is None else y[:, rows]
        bad = ~(np.abs(yy - ref) <= tol)
        assert not bad.any(), f"{int(bad.sum())} of {bad.size} outside the fused bound; first {np.argwhere(bad)[:3].tolist()}"


@gpu
@pytest.mark.parametrize("M", [1, 2, 3, 4, 8, 11])
@pytest.mark.parametrize("N,K,bs,zeros", [(37, 2048, 128, True), (300, 512, 128, False), (1000, 1536, 256, True),
                                          (16, 4096, 128, True)])
def test_swiglu_whole(M, N, K, bs, zeros):
    c = SwiGLUCase(M, N, K, bs, zeros, workload=81)
    y = c.run()
    assert "int4.swiglu.v1k" in wq.last_kernel(), wq.last_kernel()
    c.check(y)
    assert np.array_equal(y, c.run())


@gpu
@pytest.mark.parametrize("M", [1, 2, 4, 8])
def test_swiglu_full_size_sampled(M):
    """The decode feed-forward shape: gate and up 14336 × 4096."""
    c = SwiGLUCase(M, 14336, 4096, 128, True, workload=82)
    y = c.run()
    c.check(y, sample_rows(14336))


@gpu
def test_swiglu_equals_separate_gemvs_combined():
    """The fused result against the two projections run as separate B200_V1
    GEMVs through the library and combined by the oracle's silu on the host:
    the only extra error of the unfused path is its two fp16 roundings."""
    c = SwiGLUCase(2, 300, 1024, 128, True, workload=83)
    y = c.run()
    outs = []
    for h in ("g", "u"):
        w, s, z = c.dev_parts[h]
        p = torch.empty((wq.wq_int4_packed_bytes(300, 1024, 128),), dtype=torch.uint8, device=DEV)
        wq.wq_repack_int4(w, s, z, p, 300, 1024, 128)
        yy = torch.empty((2, 300), dtype=torch.float16, device=DEV)
        wq.gemv_int4_blockwise(c.dx, p, None, None, yy, 2, 300, 1024, 128, layout=wq.WQ_LAYOUT_B200_V1)
        torch.cuda.synchronize()
        outs.append(yy.cpu().numpy().astype(np.float64))
    unfused = oracle.silu(outs[0]) * outs[1]
    assert np.max(np.abs(y - unfused)) <= 4e-3 * np.max(np.abs(unfused)) + 1e-3


@gpu
def test_fused_stream_interleaves_the_two_v1_streams():
    N, K, bs = 21, 256, 128
    c = SwiGLUCase(1, N, K, bs, True, workload=84)
    fused = c.dw.cpu().numpy()
    tb = wq.wq_int4_packed_bytes(N, K, bs) // (((N + 15) // 16) * (K // 128))
    for i, h in enumerate(("g", "u")):
        w, s, z = c.dev_parts[h]
        p = torch.empty((wq.wq_int4_packed_bytes(N, K, bs),), dtype=torch.uint8, device=DEV)
        wq.wq_repack_int4(w, s, z, p, N, K, bs)
        torch.cuda.synchronize()
        single = p.cpu().numpy().reshape(-1, tb)
        assert np.array_equal(fused.reshape(-1, tb)[i::2], single)
