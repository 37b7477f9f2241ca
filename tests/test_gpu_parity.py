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
from _gpu import DEV, BF16Case, Guarded, Int4Case, Q4KCase, check, dev, each_variant, sample_rows  # noqa: E402
from weight_only_quantized_q4_b200 import synth  # noqa: E402

gpu = pytest.mark.gpu


# ----------------------------------------------------------- dequant exports

@gpu
@pytest.mark.parametrize("bs,zeros,N,K", [(32, False, 5, 1024), (128, True, 7, 1024), (16, True, 3, 80),
                                          (64, True, 9, 192), (256, False, 2, 512), (128, True, 4, 384)])
def test_dequant_int4_bit_exact(bs, zeros, N, K):
    c = Int4Case(1, N, K, bs, zeros, workload=11)
    go = Guarded((N, K), torch.float32)
    out = go.t
    wq.dequant_int4_blockwise(c.dw, c.ds, c.dz, out, N, K, bs)
    torch.cuda.synchronize()
    go.check("int4 dequant export")
    ref = c.W().astype(np.float32)
    got = out.cpu().numpy()
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))


@gpu
@pytest.mark.parametrize("N,K", [(3, 256), (5, 768), (8, 4096)])
@pytest.mark.parametrize("dsc", [False, True])
def test_dequant_q4k_bit_exact(N, K, dsc):
    c = Q4KCase(1, N, K, workload=12)
    go = Guarded((N, K), torch.float32)
    out = go.t
    wq.dequant_q4k(c.draw, c.plane_dev() if dsc else None, out, N, K)
    torch.cuda.synchronize()
    go.check("q4k dequant export")
    ref = c.W().astype(np.float32)
    assert np.array_equal(out.cpu().numpy().view(np.uint32), ref.view(np.uint32))


@gpu
@pytest.mark.parametrize("N,K", [(1, 256), (7, 512), (33, 2048)])
def test_plane_device_host_oracle_identical(N, K):
    raw = synth.q4k_weights(N, K, workload=13)
    gp = Guarded((K // 32, N, 2), torch.float32)
    P = gp.t
    wq.wq_build_q4k_dsc_device(dev(raw), P, N, K)
    torch.cuda.synchronize()
    gp.check("device W_dsc plane")
    host = wq.wq_build_q4k_dsc(raw, N, K)
    ref = oracle.q4k_plane(raw, N, K)
    assert np.array_equal(P.cpu().numpy().view(np.uint32), ref.view(np.uint32))
    assert np.array_equal(host.view(np.uint32), ref.view(np.uint32))


@gpu
@pytest.mark.parametrize("bs,zeros,N,K", [(32, False, 5, 1024), (128, True, 23, 1024), (64, True, 16, 384),
                                          (256, True, 33, 512)])
def test_dequant_int4_v1_layout_bit_exact(bs, zeros, N, K):
    """Codes repacked to B200_V1 read back (through the layout's addressing) bit-exactly."""
    c = Int4Case(1, N, K, bs, zeros, workload=14, layout=wq.WQ_LAYOUT_B200_V1)
    go = Guarded((N, K), torch.float32)
    out = go.t
    wq.dequant_int4_blockwise(c.dw, c.ds, c.dz, out, N, K, bs, layout=wq.WQ_LAYOUT_B200_V1)
    torch.cuda.synchronize()
    go.check("int4 B200_V1 dequant export")
    assert wq.last_kernel() == "int4.dequant.v1"
    ref = c.W().astype(np.float32)
    assert np.array_equal(out.cpu().numpy().view(np.uint32), ref.view(np.uint32))


def decode_v1(buf, N, K, bs):
    """Read a B200_V1 int4 stream back into (q, s, z) per the layout the header
    documents (pure Python/numpy, independent of the device code)."""
    bpt = 1 if bs >= 128 else 128 // bs
    tb = (1024 + bpt * 40 + 15) // 16 * 16
    nbands = (N + 15) // 16
    q = np.zeros((nbands * 16, K), dtype=np.int64)
    sc = np.zeros((nbands * 16, K // bs), dtype=np.float64)
    zp = np.zeros((nbands * 16, K // bs), dtype=np.int64)
    for band in range(nbands):
        for s_ in range(K // 128):
            tile = buf[(band * (K // 128) + s_) * tb:(band * (K // 128) + s_ + 1) * tb]
            for h in range(2):
                for lane in range(32):
                    g, t = lane // 4, lane % 4
                    for j in range(4):
                        gi, r8 = 2 * h + j // 2, j % 2
                        word = int(tile[h * 512 + lane * 16 + 4 * j:h * 512 + lane * 16 + 4 * j + 4].view(np.uint32)[0])
                        row = band * 16 + g + 8 * r8
                        for e in range(8):
                            pos = (e >> 1) | ((e & 1) << 2)
                            q[row, 128 * s_ + 32 * gi + 8 * t + e] = (word >> (4 * pos)) & 15
            for bt in range(bpt):
                blk = (128 * s_ + bt * bs) // bs if bs < 128 else (128 * s_) // bs
                svals = tile[1024 + bt * 32:1024 + bt * 32 + 32].view(np.float16).astype(np.float64)
                zbytes = tile[1024 + 32 * bpt + bt * 8:1024 + 32 * bpt + bt * 8 + 8]
                for r in range(16):
                    sc[band * 16 + r, blk] = svals[r]
                    zp[band * 16 + r, blk] = (int(zbytes[r // 2]) >> (4 * (r % 2))) & 15
    return q, sc, zp


@gpu
@pytest.mark.parametrize("bs", [32, 64, 128, 256])
def test_repack_v1_layout_matches_header(bs):
    """The repacked bytes, decoded by a plain reading of the documented layout,
    give the oracle's weights; pad rows hold codes 0, scale 0, zero-point 8."""
    N, K = 21, 256
    t = synth.int4_weights(N, K, bs, scale_lo=0.01, scale_hi=0.02, with_zeros=True, workload=15)
    gp = Guarded((wq.wq_int4_packed_bytes(N, K, bs),), torch.uint8)
    packed = gp.t
    wq.wq_repack_int4(dev(t["w_packed"]), dev(t["scales"]), dev(t["zeros"]), packed, N, K, bs)
    torch.cuda.synchronize()
    gp.check("B200_V1 repack output")
    q, sc, zp = decode_v1(packed.cpu().numpy(), N, K, bs)
    blk = np.arange(K) // bs
    W = (q[:N] - zp[:N][:, blk]).astype(np.float64) * sc[:N][:, blk]
    assert np.array_equal(W, oracle.dequant_int4(t["w_packed"], t["scales"], t["zeros"], N, K, bs))
    assert np.all(q[N:] == 0) and np.all(sc[N:] == 0) and np.all(zp[N:] == 8)


def decode_q4k_v1(buf, N, K):
    """Read a B200_V1 q4_K stream back into (q, d, dmin, sc, m) per the layout
    the header documents (plain numpy, independent of the device code)."""
    nb, tpb = (N + 15) // 16, K // 256
    q = np.zeros((nb * 16, K), dtype=np.int64)
    d = np.zeros((nb * 16, tpb), dtype=np.float64)
    dm = np.zeros((nb * 16, tpb), dtype=np.float64)
    sc = np.zeros((nb * 16, tpb, 8), dtype=np.int64)
    mn = np.zeros((nb * 16, tpb, 8), dtype=np.int64)
    for band in range(nb):
        for s_ in range(tpb):
            tile = buf[(band * tpb + s_) * 2304:(band * tpb + s_ + 1) * 2304]
            words = tile[:2048].view(np.uint32)
            for h in range(4):
                for lane in range(32):
                    g, t = lane // 4, lane % 4
                    for j in range(4):
                        gi, r8 = 2 * h + j // 2, j % 2
                        word = int(words[(h * 512 + lane * 16 + 4 * j) // 4])
                        row = band * 16 + g + 8 * r8
                        for e in range(8):
                            pos = (e >> 1) | ((e & 1) << 2)
                            q[row, 256 * s_ + 32 * gi + 8 * t + e] = (word >> (4 * pos)) & 15
            dd = tile[2048:2112].view(np.float16).astype(np.float64).reshape(16, 2)
            for r in range(16):
                row = band * 16 + r
                d[row, s_], dm[row, s_] = dd[r, 0], dd[r, 1]
                for p in range(4):
                    o = 2112 + 3 * (16 * p + r)
                    ent = int(tile[o]) | (int(tile[o + 1]) << 8) | (int(tile[o + 2]) << 16)
                    sc[row, s_, 2 * p], sc[row, s_, 2 * p + 1] = ent & 63, (ent >> 6) & 63
                    mn[row, s_, 2 * p], mn[row, s_, 2 * p + 1] = (ent >> 12) & 63, (ent >> 18) & 63
    return q, d, dm, sc, mn


@gpu
@pytest.mark.parametrize("N,K", [(21, 256), (16, 512), (5, 768)])
def test_repack_q4k_v1_layout_matches_header(N, K):
    """The q4_K band stream, decoded by a plain reading of the documented
    layout, gives the oracle's weights; pad rows are all zero."""
    raw = synth.q4k_weights(N, K, workload=17)
    gp = Guarded((wq.wq_q4k_packed_bytes(N, K),), torch.uint8)
    wq.wq_repack_q4k(dev(raw), gp.t, N, K)
    torch.cuda.synchronize()
    gp.check("q4_K B200_V1 repack output")
    q, d, dm, sc, mn = decode_q4k_v1(gp.t.cpu().numpy(), N, K)
    chunk = (np.arange(K) % 256) // 32
    sbk = np.arange(K) // 256
    W = d[:, sbk] * sc[:, sbk, chunk] * q - dm[:, sbk] * mn[:, sbk, chunk]
    assert np.array_equal(W[:N], oracle.dequant_q4k(raw, N, K))
    assert np.all(q[N:] == 0) and np.all(d[N:] == 0) and np.all(sc[N:] == 0) and np.all(mn[N:] == 0)


@gpu
@pytest.mark.parametrize("N,K", [(3, 256), (17, 768), (40, 4096)])
def test_dequant_q4k_v1_layout_bit_exact(N, K):
    raw = synth.q4k_weights(N, K, workload=18)
    packed = torch.empty((wq.wq_q4k_packed_bytes(N, K),), dtype=torch.uint8, device=DEV)
    wq.wq_repack_q4k(dev(raw), packed, N, K)
    go = Guarded((N, K), torch.float32)
    wq.dequant_q4k(packed, None, go.t, N, K, layout=wq.WQ_LAYOUT_B200_V1)
    torch.cuda.synchronize()
    go.check("q4_K B200_V1 dequant export")
    assert wq.last_kernel() == "q4k.dequant.v1"
    ref = oracle.dequant_q4k(raw, N, K).astype(np.float32)
    assert np.array_equal(go.t.cpu().numpy().view(np.uint32), ref.view(np.uint32))


# ----------------------------------------------------------- GEMV, whole outputs

@gpu
@pytest.mark.parametrize("M", [1, 2, 3, 4, 8, 11])
@pytest.mark.parametrize("N,K,bs,zeros", [(256, 1024, 32, False), (37, 2048, 128, True), (64, 4096, 64, True),
                                          (1000, 1536, 256, False), (5, 128, 128, True)])
def test_gemv_int4_v1_layout(M, N, K, bs, zeros):
    c = Int4Case(M, N, K, bs, zeros, workload=16, layout=wq.WQ_LAYOUT_B200_V1)
    labels = each_variant(c.run, c.W(), c.x, f"int4 v1 M={M} N={N} K={K} bs={bs} zp={zeros}")
    assert ".tc." in labels["tc"] and ".v1" in labels["tc"], labels
    assert labels["cc"] == "unsupported" and ".simple." in labels["simple"], labels

@gpu
@pytest.mark.parametrize("zq", [0, 1])
@pytest.mark.parametrize("C", [1, 2, 4])
@pytest.mark.parametrize("M", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("N,K,bs,zeros", [(37, 2048, 128, True), (1000, 1536, 256, False), (300, 512, 128, True),
                                          (4100, 1024, 128, True), (16, 4096, 256, True)])
def test_gemv_int4_v1_cluster_split(zq, C, M, N, K, bs, zeros, monkeypatch):
    """The B200_V1 band kernel, both tile forms (zq=1: exact q − z in the MMA
    operand; zq=0: subnormal codes with a per-tile Σx zero-point term), with
    the k-tiles of every band split over clusters of C CTAs (partials added
    through distributed shared memory).  Two calls in a row must agree bit for bit."""
    monkeypatch.setenv("WQ_FORCE_KERNEL", "v1s")
    monkeypatch.setenv("WQ_V1_ZQ", str(zq))
    monkeypatch.setenv("WQ_V1_C", str(C))
    c = Int4Case(M, N, K, bs, zeros, workload=23, layout=wq.WQ_LAYOUT_B200_V1)
    y1 = c.run()
    label = wq.last_kernel()
    assert ".gemv.v1s." in label and label.endswith(f".c{C}"), label
    check(y1, c.W(), c.x, f"v1s C={C} M={M} N={N} K={K} bs={bs} zp={zeros}")
    y2 = c.run()
    assert np.array_equal(y1, y2)


@gpu
@pytest.mark.parametrize("zq", [0, 1])
@pytest.mark.parametrize("ctas", [1, 4])
@pytest.mark.parametrize("M", [1, 2, 3, 4])
@pytest.mark.parametrize("N,K,bs,zeros", [(37, 2048, 128, True), (1000, 1536, 256, False), (300, 512, 128, True),
                                          (4100, 1024, 128, True), (16, 4096, 256, True), (5, 128, 128, True),
                                          (2368, 14336, 128, True)])
def test_gemv_int4_v1_stream_k(zq, ctas, M, N, K, bs, zeros, monkeypatch):
    """The stream-K B200_V1 kernel: every CTA takes an equal run of tiles, so
    bands are cut between CTAs (a band over up to 16 CTAs when N is small)
    and finished by the fix-up through the split-band workspace.  The fix-up
    adds the pieces in CTA order: two calls in a row agree bit for bit, and
    so does a third call after other shapes have used the workspace."""
    if ctas == 4 and 2 * M * K > 24 * 1024:
        pytest.skip("four CTAs per SM leave no room for these resident activations")
    monkeypatch.setenv("WQ_FORCE_KERNEL", "v1k")
    monkeypatch.setenv("WQ_V1K_ZQ", str(zq))
    monkeypatch.setenv("WQ_V1K_CTAS", str(ctas))
    monkeypatch.setenv("WQ_V1K_W", "16" if ctas == 1 else "4")  # four CTAs per SM leave room for 4 warps' stages
    c = Int4Case(M, N, K, bs, zeros, workload=25, layout=wq.WQ_LAYOUT_B200_V1)
    y1 = c.run()
    label = wq.last_kernel()
    assert ".gemv.v1k." in label, label
    check(y1, c.W(), c.x, f"v1k ctas={ctas} M={M} N={N} K={K} bs={bs} zp={zeros}")
    assert np.array_equal(y1, c.run())
    other = Int4Case(1, 77, 1024, 128, True, workload=26, layout=wq.WQ_LAYOUT_B200_V1)
    other.run()
    assert np.array_equal(y1, c.run())
    wq.wq_device_status()


@gpu
@pytest.mark.parametrize("P", [2, 3, 4])
@pytest.mark.parametrize("M", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("N,K,bs,zeros", [(37, 2048, 128, True), (1000, 1536, 256, False), (300, 512, 128, True),
                                          (4100, 1024, 128, True), (16, 4096, 256, True), (5, 128, 128, True)])
def test_gemv_int4_v1_register_stream(P, M, N, K, bs, zeros, monkeypatch):
    """The B200_V1 kernel that streams tiles straight into registers, P tiles
    ahead per warp.  Two calls in a row must agree bit for bit."""
    monkeypatch.setenv("WQ_FORCE_KERNEL", "v1r")
    monkeypatch.setenv("WQ_V1R_P", str(P))
    c = Int4Case(M, N, K, bs, zeros, workload=24, layout=wq.WQ_LAYOUT_B200_V1)
    y1 = c.run()
    label = wq.last_kernel()
    assert ".gemv.v1r." in label and f".p{P}" in label, label
    check(y1, c.W(), c.x, f"v1r P={P} M={M} N={N} K={K} bs={bs} zp={zeros}")
    assert np.array_equal(y1, c.run())


@gpu
def test_gemv_int4_v1_default_kernel_full_size():
    c = Int4Case(1, 4096, 14336, 128, True, workload=3, layout=wq.WQ_LAYOUT_B200_V1)
    rows = sample_rows(4096)
    y = c.run()
    assert ".gemv.v1s." in wq.last_kernel(), wq.last_kernel()
    W = oracle.dequant_int4(c.w[rows], c.s[rows], c.z[rows], len(rows), 14336, 128)
    check(y[:, rows], W, c.x, "B200_V1 4096x14336 sampled rows")


@gpu
@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 8])
@pytest.mark.parametrize("N,K,bs,zeros", [(256, 1024, 32, False), (37, 2048, 128, True), (301, 512, 16, True),
                                          (64, 4096, 64, True), (1000, 1536, 256, False)])
def test_gemv_int4_small(M, N, K, bs, zeros):
    c = Int4Case(M, N, K, bs, zeros, workload=21)
    labels = each_variant(c.run, c.W(), c.x, f"int4 M={M} N={N} K={K} bs={bs} zp={zeros}")
    if bs >= 32:
        assert ".tc." in labels["tc"], labels
    assert (".cc." in labels["cc"] or labels["cc"] == "unsupported") and ".simple." in labels["simple"], labels


@gpu
@pytest.mark.parametrize("M", [1, 2, 3, 4, 6, 8])
@pytest.mark.parametrize("N,K", [(3, 256), (129, 1024), (250, 2816), (64, 11008)])
@pytest.mark.parametrize("dsc", [False, True])
def test_gemv_q4k_small(M, N, K, dsc):
    c = Q4KCase(M, N, K, workload=22)
    labels = each_variant(lambda: c.run(dsc), c.W(), c.x, f"q4k dsc={dsc} M={M} N={N} K={K}")
    assert ".tc." in labels["tc"] and (".cc." in labels["cc"] or labels["cc"] == "unsupported"), labels


@gpu
@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 8, 11])
@pytest.mark.parametrize("N,K", [(3, 256), (129, 1024), (250, 2816), (64, 11008), (16, 4096)])
def test_gemv_q4k_v1_layout(M, N, K):
    """q4_K in the B200_V1 band stream: the stream-K kernel (MMA columns carrying
    chunks at M < 8) and the scalar kernel, against the oracle; two calls in a
    row agree bit for bit."""
    c = Q4KCase(M, N, K, workload=27, layout=wq.WQ_LAYOUT_B200_V1)
    labels = each_variant(lambda: c.run(False), c.W(), c.x, f"q4k v1 M={M} N={N} K={K}")
    assert ".simple." in labels["simple"] and labels["tc"] == "unsupported" and labels["tc5"] == "unsupported", labels
    if 2 * M * K <= 120 * 1024:
        assert ".gemv.v1k." in labels["default"], labels
        assert np.array_equal(c.run(False), c.run(False))


@gpu
@pytest.mark.parametrize("M", [1, 2, 3, 4, 7, 8])
@pytest.mark.parametrize("N,K", [(256, 1536), (77, 6912), (300, 64)])
def test_gemv_bf16_small(M, N, K):
    c = BF16Case(M, N, K, workload=23)
    labels = each_variant(c.run, c.W(), c.X(), f"bf16 M={M} N={N} K={K}")
    assert ".tc." in labels["tc"] and (".cc." in labels["cc"] or labels["cc"] == "unsupported"), labels


@gpu
@pytest.mark.parametrize("K", [7, 12, 100, 1534])
@pytest.mark.parametrize("M", [1, 3])
@pytest.mark.parametrize("N", [256, 1536])
@pytest.mark.parametrize("offset", [0, 1])
def test_gemv_bf16_odd_k_and_offsets(K, M, N, offset):
    c = BF16Case(M, N, K, offset=offset, workload=24)
    each_variant(c.run, c.W(), c.X(), f"bf16 odd-K M={M} N={N} K={K} offset={offset}")


@gpu
@pytest.mark.parametrize("M", [9, 16, 17])
def test_gemv_larger_batches(M):
    c = Int4Case(M, 96, 1024, 128, True, workload=25)
    each_variant(c.run, c.W(), c.x, f"int4 M={M}")
    q = Q4KCase(M, 40, 512, workload=25)
    each_variant(lambda: q.run(False), q.W(), q.x, f"q4k M={M}")
    each_variant(lambda: q.run(True), q.W(), q.x, f"q4k dsc M={M}")
    b = BF16Case(M, 50, 256, workload=25)
    each_variant(b.run, b.W(), b.X(), f"bf16 M={M}")


TC5_A = [pytest.param("1", id="A_tmem"), pytest.param("0", id="A_smem")]


def _tc5_a_placement(label, ta, M):
    """TMEM-A runs for batch tiles of at most 128 columns unless turned off."""
    assert (".tc5.ta." in label) == (ta == "1" and M <= 128), label


@gpu
@pytest.mark.parametrize("ta", TC5_A)
@pytest.mark.parametrize("M", [9, 16, 32, 64, 128, 200, 300])
@pytest.mark.parametrize("fmt", ["int4", "q4k"])
def test_gemm_tcgen05_batched(M, fmt, ta, monkeypatch):
    """The tcgen05 dequant-then-MMA path (default for M >= 9) on ragged row
    tiles (N = 300) and batches that span one or two N tiles of the MMA, with
    the fp16 A rows in tensor memory (batch tiles up to 128) or in shared
    memory."""
    monkeypatch.setenv("WQ_TC5_TA", ta)
    if fmt == "int4":
        c = Int4Case(M, 300, 1024, 128, True, workload=29)
        y = c.run()
        W, x = c.W(), c.x
    else:
        c = Q4KCase(M, 300, 1024, workload=29)
        y = c.run(False)
        W, x = c.W(), c.x
    assert ".gemm.tc5." in wq.last_kernel(), wq.last_kernel()
    _tc5_a_placement(wq.last_kernel(), ta, M)
    check(y, W, x, f"tcgen05 {fmt} M={M}")


@gpu
@pytest.mark.parametrize("M", [9, 16, 33, 128])
@pytest.mark.parametrize("N,K", [(300, 1536), (1536, 6912), (77, 136)])
def test_gemm_tcgen05_bf16(M, N, K):
    """bf16 batches of 9 and more run the tcgen05 kernel with the weights
    TMA-loaded straight into the MMA's A slots (K = 136: a partial last 64-k
    stage, zero-filled by the tensor-map bounds)."""
    c = BF16Case(M, N, K, workload=30)
    y = c.run()
    assert ".gemm.tc5." in wq.last_kernel() and wq.last_kernel().startswith("bf16"), wq.last_kernel()
    check(y, c.W(), c.X(), f"tcgen05 bf16 M={M} N={N} K={K}")
    assert np.array_equal(y, c.run())


@gpu
@pytest.mark.parametrize("ta", TC5_A)
@pytest.mark.parametrize("S", [1, 2, 4, 8])
@pytest.mark.parametrize("M", [16, 33, 128])
@pytest.mark.parametrize("fmt", ["int4", "q4k"])
def test_gemm_tcgen05_cluster_split_k(S, M, fmt, ta, monkeypatch):
    """The tcgen05 batched path with K split over a cluster of S CTAs whose fp32
    accumulators are added through distributed shared memory (ragged N tiles,
    batch tiles of 16..128 columns).  Two calls in a row agree bit for bit."""
    monkeypatch.setenv("WQ_TC5_TA", ta)
    monkeypatch.setenv("WQ_TC5_S", str(S))
    if fmt == "int4":
        c = Int4Case(M, 300, 4096, 128, True, workload=31)
        run = c.run
    else:
        c = Q4KCase(M, 300, 4096, workload=31)
        run = lambda: c.run(False)  # noqa: E731
    y = run()
    label = wq.last_kernel()
    assert ".gemm.tc5." in label and label.endswith(f".s{S}"), label
    check(y, c.W(), c.x, f"tcgen05 {fmt} M={M} S={S}")
    assert np.array_equal(y, run())


@gpu
@pytest.mark.parametrize("ta", TC5_A)
@pytest.mark.parametrize("S", [1, 4])
@pytest.mark.parametrize("fmt", ["int4", "q4k"])
def test_gemm_tcgen05_weights_beyond_fp16_range(fmt, S, ta, monkeypatch):
    """Half the rows dequantize beyond the fp16 range (int4 scales up to 9000,
    |w| up to 135000; q4_K d up to 100, |w| up to about 95000) beside ordinary
    rows.  The tcgen05 path forms such rows as w·2^-e and rescales their fp32
    result, so every output stays finite and within the tolerance (small
    activations keep y itself inside fp16)."""
    monkeypatch.setenv("WQ_TC5_TA", ta)
    monkeypatch.setenv("WQ_TC5_S", str(S))
    M, N, K = 16, 300, 2048
    rng = np.random.default_rng(32)
    big = rng.random(N) < 0.5
    if fmt == "int4":
        c = Int4Case(M, N, K, 128, True, workload=32)
        c.s[big] = rng.uniform(5000, 9000, (int(big.sum()), K // 128)).astype(np.float16)
        c.ds = dev(c.s)
        run = c.run
    else:
        c = Q4KCase(M, N, K, workload=32)
        d = rng.uniform(50, 100, (int(big.sum()), K // 256)).astype(np.float16)
        c.raw[big, :, 0:2] = d.view(np.uint8).reshape(int(big.sum()), K // 256, 2)
        c.draw = c.dw = dev(c.raw)
        run = lambda: c.run(False)  # noqa: E731
    c.x = (c.x.astype(np.float32) * 1e-4).astype(np.float16)
    c.dx = dev(c.x)
    y = run()
    label = wq.last_kernel()
    assert ".gemm.tc5." in label and label.endswith(f".s{S}"), label
    assert np.isfinite(y).all()
    check(y, c.W(), c.x, f"tcgen05 {fmt} beyond fp16 range S={S}")


@gpu
def test_gemm_tcgen05_forced_split_follows_the_automatic_rule(monkeypatch):
    """A forced cluster split must give every CTA an even number of 256-k raw
    slots (the rule of the automatic choice); K = 2048 with S = 8 gives one."""
    monkeypatch.setenv("WQ_TC5_S", "8")
    c = Q4KCase(16, 300, 2048, workload=31)
    with pytest.raises(wq.WQError) as e:
        c.run(False)
    assert e.value.code == wq.WQ_ERR_ARG


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
    gy = Guarded((M, N), torch.float16)
    y = gy.t
    wq.gemv_int4_blockwise(dev(x), dev(w), dev(s), dev(z), y, M, N, K, bs)
    torch.cuda.synchronize()
    gy.check("int4 z=q output")
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
def test_device_wait_timeout_is_reported_once_and_clears():
    """A bounded device wait that runs out (a test kernel waits on an mbarrier
    nothing arrives at, 2 ms limit, no copy in flight) is reported by
    wq_device_status() as WQ_ERR_TIMEOUT exactly once; the context stays
    usable and the next GEMV is correct."""
    wq.wq_device_status()  # start from a clear error word
    wq.wq_test_expire_wait(2_000_000)
    assert wq.last_kernel() == "test.expire_wait"
    with pytest.raises(wq.WQError) as e:
        wq.wq_device_status()
    assert e.value.code == wq.WQ_ERR_TIMEOUT
    wq.wq_device_status()  # read-and-clear: the second read is clean
    c = Int4Case(2, 300, 1024, 128, True, workload=44, layout=wq.WQ_LAYOUT_B200_V1)
    check(c.run(), c.W(), c.x, "GEMV after an expired wait")
    wq.wq_device_status()


@gpu
def test_uses_given_stream_and_labels():
    c = Int4Case(1, 4096, 4096, 128, True, workload=28)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        y = c.run()
    assert "int4.gemv.tc" in wq.last_kernel()
    check(y, c.W(), c.x, "int4 on a side stream")
    wq.wq_device_status()


# ----------------------------------------------------------- full workload sizes, sampled rows

FULL_INT4 = [(4096, 4096), (14336, 4096), (4096, 14336)]
FULL_Q4K = [(4096, 4096), (11008, 4096), (4096, 11008)]
FULL_BF16 = [(1536, 1536), (256, 1536), (1536, 6912), (151936, 1536)]


@gpu
@pytest.mark.parametrize("M", [1, 4])
@pytest.mark.parametrize("N,K", FULL_INT4)
@pytest.mark.parametrize("layout", [0, 1])
def test_full_int4_b128_sampled(M, N, K, layout):
    c = Int4Case(M, N, K, 128, True, workload=3, layout=layout)
    rows = sample_rows(N)
    Wr = c.W(rows)
    each_variant(lambda: c.run()[:, rows], Wr, c.x, f"int4 full {N}x{K} M={M}")


@gpu
def test_full_int4_b32_config():
    c = Int4Case(1, 256, 1024, 32, False, workload=1, s_lo=0.005, s_hi=0.02)
    check(c.run(), c.W(), c.x, "int4 b32 256x1024")


@gpu
@pytest.mark.parametrize("M", [1, 2, 4, 8])
@pytest.mark.parametrize("N,K", FULL_Q4K)
def test_full_q4k_v1_sampled(M, N, K):
    c = Q4KCase(M, N, K, workload=4, layout=wq.WQ_LAYOUT_B200_V1)
    rows = sample_rows(N)
    y = c.run(False)
    check(y[:, rows], c.W(rows), c.x, f"q4k B200_V1 full {N}x{K} M={M} [{wq.last_kernel()}]")


@gpu
@pytest.mark.parametrize("M", [1, 2, 4, 8])
@pytest.mark.parametrize("N,K", FULL_Q4K)
@pytest.mark.parametrize("dsc", [False, True])
def test_full_q4k_sampled(M, N, K, dsc):
    c = Q4KCase(M, N, K, workload=4)
    rows = sample_rows(N)
    Wr = c.W(rows)
    each_variant(lambda: c.run(dsc)[:, rows], Wr, c.x, f"q4k dsc={dsc} full {N}x{K} M={M}")


@gpu
@pytest.mark.parametrize("M", [1, 3, 8])
@pytest.mark.parametrize("N,K", FULL_BF16)
def test_full_bf16_sampled(M, N, K):
    c = BF16Case(M, N, K, workload=2)
    rows = sample_rows(N)
    Wr = c.W(rows)
    each_variant(lambda: c.run()[:, rows], Wr, c.X(), f"bf16 full {N}x{K} M={M}")


FULL_BATCHED = [(4096, 4096), (14336, 4096), (4096, 14336), (32000, 4096)]


@gpu
@pytest.mark.parametrize("N,K", FULL_BATCHED)
@pytest.mark.parametrize("fmt", ["int4", "q4k"])
def test_full_batched_sampled(fmt, N, K):
    """The batched workload at its full sizes (M = 16, 32, 64, 128), in the
    default launch configuration the benchmark times: multi-wave grids at
    N = 32000, the K = 14336 stage / split plan.  Sampled rows vs the oracle;
    guard bands around every output."""
    if fmt == "int4":
        t = synth.int4_weights(N, K, 128, scale_lo=0.002, scale_hi=0.01, with_zeros=True, workload=5)
        dw, ds, dz = dev(t["w_packed"]), dev(t["scales"]), dev(t["zeros"])
    else:
        raw = synth.q4k_weights(N, K, workload=5)
        draw = dev(raw)
    rows = sample_rows(N)
    if fmt == "int4":
        Wr = oracle.dequant_int4(t["w_packed"][rows], t["scales"][rows], t["zeros"][rows], len(rows), K, 128)
    else:
        Wr = oracle.dequant_q4k(raw[rows], len(rows), K)
    for M in (16, 32, 64, 128):
        x = synth.activations_f16(M, K, workload=5)
        g = Guarded((M, N), torch.float16)
        if fmt == "int4":
            wq.gemv_int4_blockwise(dev(x), dw, ds, dz, g.t, M, N, K, 128)
        else:
            wq.gemv_q4k(dev(x), draw, g.t, M, N, K)
        torch.cuda.synchronize()
        label = wq.last_kernel()
        g.check(f"batched {fmt} {N}x{K} M={M}")
        y = g.t.cpu().numpy().astype(np.float64)
        check(y[:, rows], Wr, x, f"batched {fmt} {N}x{K} M={M} [{label}]")


# ----------------------------------------------------- tcgen05 over the B200_V1 stream

V1TC_A = [pytest.param("1", id="A_tmem"), pytest.param("0", id="A_smem")]


@gpu
@pytest.mark.parametrize("ta", V1TC_A)
@pytest.mark.parametrize("M", [9, 16, 33, 64, 128, 200])
@pytest.mark.parametrize("N,K,bs", [(300, 1024, 128), (37, 4096, 256), (1000, 384, 128), (16, 128, 128)])
def test_gemm_v1tc_batched(M, N, K, bs, ta, monkeypatch):
    """The tcgen05 kernel that reads the B200_V1 band stream (forced: below 25
    rows the default is the warp-MMA GEMM), with the fp16 A rows in tensor
    memory (default) or in shared memory: ragged row tiles (N = 300, 37,
    1000), an odd number of 128-k steps (K = 384), a single step (K = 128),
    two batch tiles (M = 200).  Guard bands around every output; two calls
    agree bit for bit."""
    monkeypatch.setenv("WQ_FORCE_KERNEL", "v1tc")
    monkeypatch.setenv("WQ_V1TC_TA", ta)
    c = Int4Case(M, N, K, bs, True, workload=40, layout=wq.WQ_LAYOUT_B200_V1)
    y = c.run()
    assert ".gemm.v1tc." in wq.last_kernel(), wq.last_kernel()
    assert (".v1tc.ta." in wq.last_kernel()) == (ta == "1"), wq.last_kernel()
    check(y, c.W(), c.x, f"v1tc M={M} N={N} K={K} bs={bs}")
    assert np.array_equal(y, c.run())


@gpu
@pytest.mark.parametrize("ta", V1TC_A)
@pytest.mark.parametrize("S", [1, 2, 4, 8])
@pytest.mark.parametrize("M", [16, 48, 128])
def test_gemm_v1tc_cluster_split_k(S, M, ta, monkeypatch):
    """K split over a cluster of S CTAs whose fp32 accumulators are added
    through distributed shared memory in rank order."""
    monkeypatch.setenv("WQ_V1TC_TA", ta)
    monkeypatch.setenv("WQ_V1TC_S", str(S))
    monkeypatch.setenv("WQ_FORCE_KERNEL", "v1tc")
    c = Int4Case(M, 300, 4096, 128, True, workload=41, layout=wq.WQ_LAYOUT_B200_V1)
    y = c.run()
    label = wq.last_kernel()
    assert ".gemm.v1tc." in label and label.endswith(f".s{S}"), label
    check(y, c.W(), c.x, f"v1tc M={M} S={S}")
    assert np.array_equal(y, c.run())


@gpu
@pytest.mark.parametrize("T,ta", [(T, ta) for T in (1, 2, 3, 4) for ta in ("1", "0")] + [(5, "1"), (6, "1")])
def test_gemm_v1tc_raw_slot_sizes(T, ta, monkeypatch):
    """Raw slots of T steps per band: odd and even T (the band stride inside a
    slot is padded to an odd number of 16-byte units when T·1072 is not).
    With A in shared memory at most 4 steps per raw slot fit at this M."""
    monkeypatch.setenv("WQ_FORCE_KERNEL", "v1tc")
    monkeypatch.setenv("WQ_V1TC_TA", ta)
    monkeypatch.setenv("WQ_V1TC_T", str(T))
    monkeypatch.setenv("WQ_V1TC_S", "1")  # all 16 steps in one CTA, so T is not cut by the split
    monkeypatch.setenv("WQ_V1TC_NX", "2")  # a short activation ring leaves room for six steps per raw slot
    c = Int4Case(40, 260, 2048, 128, True, workload=43, layout=wq.WQ_LAYOUT_B200_V1)
    y = c.run()
    label = wq.last_kernel()
    assert f".t{T}." in label, label
    check(y, c.W(), c.x, f"v1tc T={T} ta={ta}")


@gpu
def test_gemm_v1tc_forced_split_follows_the_rule(monkeypatch):
    """A forced split must leave every CTA an even number of 128-k steps."""
    monkeypatch.setenv("WQ_V1TC_S", "4")
    monkeypatch.setenv("WQ_FORCE_KERNEL", "v1tc")
    c = Int4Case(16, 300, 768, 128, True, workload=41, layout=wq.WQ_LAYOUT_B200_V1)
    with pytest.raises(wq.WQError) as e:
        c.run()
    assert e.value.code == wq.WQ_ERR_ARG


@gpu
@pytest.mark.parametrize("ta", V1TC_A)
@pytest.mark.parametrize("S", [1, 4])
def test_gemm_v1tc_weights_beyond_fp16_range(S, ta, monkeypatch):
    """Half the rows with scales up to 9000 (|w| up to 135000): formed as
    w·2^-e and rescaled in fp32, every output finite and within tolerance."""
    monkeypatch.setenv("WQ_V1TC_TA", ta)
    monkeypatch.setenv("WQ_V1TC_S", str(S))
    monkeypatch.setenv("WQ_FORCE_KERNEL", "v1tc")
    M, N, K = 16, 300, 2048
    rng = np.random.default_rng(42)
    big = rng.random(N) < 0.5
    t = synth.int4_weights(N, K, 128, scale_lo=0.002, scale_hi=0.01, with_zeros=True, workload=42)
    s = t["scales"].copy()
    s[big] = rng.uniform(5000, 9000, (int(big.sum()), K // 128)).astype(np.float16)
    g = Guarded((wq.wq_int4_packed_bytes(N, K, 128),), torch.uint8)
    wq.wq_repack_int4(dev(t["w_packed"]), dev(s), dev(t["zeros"]), g.t, N, K, 128)
    x = (synth.activations_f16(M, K, workload=42).astype(np.float32) * 1e-4).astype(np.float16)
    gy = Guarded((M, N), torch.float16)
    wq.gemv_int4_blockwise(dev(x), g.t, None, None, gy.t, M, N, K, 128, layout=wq.WQ_LAYOUT_B200_V1)
    torch.cuda.synchronize()
    gy.check("v1tc large-scale y")
    label = wq.last_kernel()
    assert ".gemm.v1tc." in label and label.endswith(f".s{S}"), label
    y = gy.t.cpu().numpy().astype(np.float64)
    assert np.isfinite(y).all()
    check(y, oracle.dequant_int4(t["w_packed"], s, t["zeros"], N, K, 128), x, f"v1tc beyond fp16 range S={S}")


@gpu
@pytest.mark.parametrize("N,K", FULL_BATCHED)
def test_full_batched_v1tc_sampled(N, K):
    """The batched int4 workload in the B200_V1 layout at its full sizes
    (M = 16, 32, 64, 128) in the default launch configuration; sampled rows
    vs the oracle, guard bands around every output."""
    t = synth.int4_weights(N, K, 128, scale_lo=0.002, scale_hi=0.01, with_zeros=True, workload=5)
    g = Guarded((wq.wq_int4_packed_bytes(N, K, 128),), torch.uint8)
    wq.wq_repack_int4(dev(t["w_packed"]), dev(t["scales"]), dev(t["zeros"]), g.t, N, K, 128)
    torch.cuda.synchronize()
    rows = sample_rows(N)
    Wr = oracle.dequant_int4(t["w_packed"][rows], t["scales"][rows], t["zeros"][rows], len(rows), K, 128)
    for M in (16, 32, 64, 128):
        x = synth.activations_f16(M, K, workload=5)
        gy = Guarded((M, N), torch.float16)
        wq.gemv_int4_blockwise(dev(x), g.t, None, None, gy.t, M, N, K, 128, layout=wq.WQ_LAYOUT_B200_V1)
        torch.cuda.synchronize()
        label = wq.last_kernel()
        # the tcgen05 kernel from 25 rows, and from 9 when its 128-row tiles fill
        # the GPU without a K split (2·ceil(N/128) > SMs); else the warp-MMA GEMM
        fills = 2 * -(-N // 128) > torch.cuda.get_device_properties(0).multi_processor_count
        assert (".gemm.v1tc." in label) if (M > 24 or fills) else (".gemm.v1w." in label), label
        gy.check(f"v1tc full {N}x{K} M={M}")
        y = gy.t.cpu().numpy().astype(np.float64)
        check(y[:, rows], Wr, x, f"v1tc full {N}x{K} M={M} [{label}]")


# ----------------------------------------------------- warp-MMA GEMM over the B200_V1 stream

@gpu
@pytest.mark.parametrize("M", [9, 16, 17, 24, 25, 33, 40, 57, 64])
@pytest.mark.parametrize("N,K,bs", [(300, 1024, 128), (37, 4096, 256), (1000, 384, 128), (16, 128, 128), (129, 896, 256)])
def test_gemm_v1w_batched(M, N, K, bs, monkeypatch):
    """The warp-MMA GEMM over the B200_V1 stream (M = 9..64, every column-group
    count 2..8 and both warp arrangements): ragged row tiles, an odd number of
    128-k steps, a single step, a ragged last block (896 = 3·256 + 128).  Guard
    bands around every output; two calls agree bit for bit."""
    monkeypatch.setenv("WQ_FORCE_KERNEL", "v1w")
    c = Int4Case(M, N, K, bs, True, workload=44, layout=wq.WQ_LAYOUT_B200_V1)
    y = c.run()
    assert ".gemm.v1w." in wq.last_kernel(), wq.last_kernel()
    check(y, c.W(), c.x, f"v1w M={M} N={N} K={K} bs={bs}")
    assert np.array_equal(y, c.run())


@gpu
@pytest.mark.parametrize("S", [1, 2, 4, 8])
@pytest.mark.parametrize("M", [16, 48])
@pytest.mark.parametrize("K", [4096, 1408])
def test_gemm_v1w_cluster_split_k(S, M, K, monkeypatch):
    """K split over a cluster of S CTAs (K = 1408: eleven steps, uneven runs
    per rank), partials added through distributed shared memory in rank order."""
    monkeypatch.setenv("WQ_FORCE_KERNEL", "v1w")
    monkeypatch.setenv("WQ_V1W_S", str(S))
    c = Int4Case(M, 300, K, 128, True, workload=45, layout=wq.WQ_LAYOUT_B200_V1)
    y = c.run()
    label = wq.last_kernel()
    assert ".gemm.v1w." in label and label.endswith(f".s{S}"), label
    check(y, c.W(), c.x, f"v1w M={M} K={K} S={S}")
    assert np.array_equal(y, c.run())


@gpu
@pytest.mark.parametrize("T", [1, 2, 5])
def test_gemm_v1w_raw_slot_sizes(T, monkeypatch):
    monkeypatch.setenv("WQ_FORCE_KERNEL", "v1w")
    monkeypatch.setenv("WQ_V1W_T", str(T))
    monkeypatch.setenv("WQ_V1W_S", "1")  # all 16 steps in one CTA, so T is not capped by the slice
    c = Int4Case(33, 200, 2048, 128, True, workload=46, layout=wq.WQ_LAYOUT_B200_V1)
    y = c.run()
    assert f".t{T}." in wq.last_kernel(), wq.last_kernel()
    check(y, c.W(), c.x, f"v1w T={T}")


@gpu
@pytest.mark.parametrize("N,K", FULL_BATCHED)
def test_full_batched_v1w_sampled(N, K, monkeypatch):
    monkeypatch.setenv("WQ_FORCE_KERNEL", "v1w")
    t = synth.int4_weights(N, K, 128, scale_lo=0.002, scale_hi=0.01, with_zeros=True, workload=5)
    g = Guarded((wq.wq_int4_packed_bytes(N, K, 128),), torch.uint8)
    wq.wq_repack_int4(dev(t["w_packed"]), dev(t["scales"]), dev(t["zeros"]), g.t, N, K, 128)
    torch.cuda.synchronize()
    rows = sample_rows(N)
    Wr = oracle.dequant_int4(t["w_packed"][rows], t["scales"][rows], t["zeros"][rows], len(rows), K, 128)
    for M in (16, 32, 64):
        x = synth.activations_f16(M, K, workload=5)
        gy = Guarded((M, N), torch.float16)
        wq.gemv_int4_blockwise(dev(x), g.t, None, None, gy.t, M, N, K, 128, layout=wq.WQ_LAYOUT_B200_V1)
        torch.cuda.synchronize()
        assert ".gemm.v1w." in wq.last_kernel(), wq.last_kernel()
        gy.check(f"v1w full {N}x{K} M={M}")
        y = gy.t.cpu().numpy().astype(np.float64)
        check(y[:, rows], Wr, x, f"v1w full {N}x{K} M={M}")
