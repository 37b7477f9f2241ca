"""C ABI checks that need no GPU: the library loads, exports every entry point
declared in include/wq.h, rejects bad arguments with the documented codes
before touching a device, answers size queries, and its host W_dsc plane
builder matches the oracle bit for bit."""
import os
import re

import numpy as np
import pytest

import oracle
import weight_only_quantized_q4_b200 as wq
from weight_only_quantized_q4_b200 import _lib, synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built():
    from weight_only_quantized_q4_b200.build import build

    build()


def header_functions():
    with open(os.path.join(ROOT, "include", "wq.h")) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[a-z_]+\s*\*?\s*([a-z0-9_]+)\s*\(", text, flags=re.M)))


def test_every_header_symbol_is_exported():
    names = header_functions()
    assert "gemv_int4_blockwise" in names and "wq_device_status" in names
    lib = _lib.lib()
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(_lib.SIGNATURES), "binding signatures and header disagree"


A16 = 0x10000  # a 16-byte aligned fake device address (never dereferenced)


def rc_int4(**kw):
    a = dict(x=A16, w=A16, s=A16, z=None, y=A16, M=1, N=16, K=256, bs=32, layout=0)
    a.update(kw)
    return _lib.lib().gemv_int4_blockwise(a["x"], a["w"], a["s"], a["z"], a["y"], a["M"], a["N"], a["K"], a["bs"],
                                         a["layout"], None)


def test_int4_argument_errors():
    assert rc_int4(M=0) == _lib.WQ_ERR_ARG
    assert rc_int4(N=-1) == _lib.WQ_ERR_ARG
    assert rc_int4(bs=24) == _lib.WQ_ERR_ARG
    assert rc_int4(bs=8) == _lib.WQ_ERR_ARG
    assert rc_int4(bs=512) == _lib.WQ_ERR_ARG
    assert rc_int4(K=250) == _lib.WQ_ERR_ARG
    assert rc_int4(layout=3) == _lib.WQ_ERR_LAYOUT
    assert rc_int4(x=None) == _lib.WQ_ERR_ARG
    assert rc_int4(w=A16 + 8) == _lib.WQ_ERR_ALIGN
    assert rc_int4(z=A16 + 4) == _lib.WQ_ERR_ALIGN
    assert "16-byte" in wq.last_error()


def test_q4k_and_bf16_argument_errors():
    L = _lib.lib()
    assert L.gemv_q4k(A16, A16, A16, 1, 8, 300, 0, None) == _lib.WQ_ERR_ARG
    assert L.gemv_q4k(A16, A16 + 2, A16, 1, 8, 256, 0, None) == _lib.WQ_ERR_ALIGN
    assert L.gemv_q4k(A16, A16, A16, 1, 8, 256, 3, None) == _lib.WQ_ERR_LAYOUT
    assert L.gemv_q4k_dsc(A16, A16, None, A16, 1, 8, 256, 0, None) == _lib.WQ_ERR_ARG
    assert L.gemv_bf16(A16 + 1, A16, A16, 1, 8, 7, None) == _lib.WQ_ERR_ARG
    assert L.gemv_bf16(A16, A16, A16, 1, 0, 7, None) == _lib.WQ_ERR_ARG
    assert L.dequant_q4k(A16, None, A16, 4, 100, 0, None) == _lib.WQ_ERR_ARG
    assert L.wq_build_q4k_dsc(None, 4, 256, None) == _lib.WQ_ERR_ARG
    assert L.wq_repack_q4k(A16, A16, 16, 300, 1, None) == _lib.WQ_ERR_ARG
    assert L.wq_repack_q4k(A16, A16, 16, 256, 0, None) == _lib.WQ_ERR_LAYOUT
    assert L.wq_repack_q4k(A16 + 4, A16, 16, 256, 1, None) == _lib.WQ_ERR_ALIGN
    assert L.dequant_q4k(A16, A16, A16, 4, 256, 1, None) == _lib.WQ_ERR_LAYOUT
    assert L.wq_test_expire_wait(10, None) == _lib.WQ_ERR_ARG
    assert L.wq_test_expire_wait(2 * 10**9, None) == _lib.WQ_ERR_ARG


def test_v1_layout_argument_errors():
    assert rc_int4(layout=1, K=192, bs=64) == _lib.WQ_ERR_ARG   # K % 128 != 0
    assert rc_int4(layout=2) == _lib.WQ_ERR_LAYOUT
    assert rc_int4(layout=1, K=256, bs=16) == _lib.WQ_ERR_ARG   # B200_V1 needs block >= 32
    L = _lib.lib()
    assert L.wq_repack_int4(A16, A16, None, A16, 16, 192, 64, 1, None) == _lib.WQ_ERR_ARG
    assert L.wq_repack_int4(A16, A16, None, A16, 16, 256, 16, 1, None) == _lib.WQ_ERR_ARG
    assert L.wq_repack_int4(A16, A16, None, A16, 16, 256, 128, 0, None) == _lib.WQ_ERR_LAYOUT
    assert L.wq_repack_int4(A16 + 4, A16, None, A16, 16, 256, 128, 1, None) == _lib.WQ_ERR_ALIGN
    assert L.wq_repack_int4(A16, None, None, A16, 16, 256, 128, 1, None) == _lib.WQ_ERR_ARG


def test_size_queries():
    assert wq.wq_int4_codes_bytes(21, 256, 0) == 21 * 128
    assert wq.wq_int4_codes_bytes(21, 256, 1) == 0
    assert wq.wq_int4_packed_bytes(21, 256, 128) == 2 * 2 * 1072
    assert wq.wq_int4_packed_bytes(21, 256, 64) == 2 * 2 * 1104
    assert wq.wq_int4_packed_bytes(21, 256, 32) == 2 * 2 * 1184
    assert wq.wq_int4_packed_bytes(21, 192, 64) == 0
    assert wq.wq_int4_packed_bytes(21, 256, 16) == 0
    assert wq.wq_int4_bytes(4096, 14336, 128, 1) == 256 * 112 * 1072
    assert wq.wq_int4_bytes(256, 1024, 32) == 256 * 512 + 256 * 32 * 2 + 256 * 16
    assert wq.wq_int4_bytes(4, 96, 32) == 4 * 48 + 4 * 3 * 2 + 4 * 2  # odd block count: zero-point bytes round up
    assert wq.wq_int4_bytes(4, 100, 32) == 0  # K % 16 != 0
    # a ragged last block: 80 = 32 + 32 + 16 (three blocks), 896 = 3 x 256 + 128
    assert wq.wq_int4_bytes(4, 80, 32) == 4 * 40 + 4 * 3 * 2 + 4 * 2
    assert wq.wq_int4_bytes(2, 896, 256) == 2 * 448 + 2 * 4 * 2 + 2 * 2
    assert wq.wq_int4_packed_bytes(21, 896, 256) == 2 * 7 * 1072
    assert wq.wq_q4k_bytes(4096, 4096) == 4096 * 16 * 144
    assert wq.wq_q4k_dsc_bytes(4096, 11008) == 4096 * 11008 // 4
    assert wq.wq_q4k_dsc_bytes(4, 100) == 0
    assert wq.wq_q4k_packed_bytes(21, 512) == 2 * 2 * 2304
    assert wq.wq_q4k_packed_bytes(21, 512, 0) == 0
    assert wq.wq_q4k_packed_bytes(4096, 11008) == 256 * 43 * 2304 == wq.wq_q4k_bytes(4096, 11008)
    assert wq.wq_layout_version() == wq.WQ_LAYOUT_B200_V1 == 1


@pytest.mark.parametrize("N,K", [(1, 256), (5, 768), (64, 4096)])
def test_host_plane_matches_oracle(N, K):
    raw = synth.q4k_weights(N, K, workload=31)
    got = wq.wq_build_q4k_dsc(raw, N, K)
    ref = oracle.q4k_plane(raw, N, K)
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))


def test_host_plane_special_values():
    """fp16 subnormal and large d/dmin values go through the host fp16 decoder exactly."""
    raw = synth.q4k_weights(3, 256, workload=32).copy()
    raw[0, 0, 0:2] = np.array([0x0001], dtype=np.uint16).view(np.uint8)   # smallest subnormal d
    raw[1, 0, 2:4] = np.array([0x7BFF], dtype=np.uint16).view(np.uint8)   # 65504 dmin
    raw[2, 0, 0:2] = np.array([0x8400], dtype=np.uint16).view(np.uint8)   # negative normal d
    got = wq.wq_build_q4k_dsc(raw, 3, 256)
    ref = oracle.q4k_plane(raw, 3, 256)
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))


def test_product_path_does_not_import_oracle():
    pkg = os.path.join(ROOT, "weight_only_quantized_q4_b200")
    for name in os.listdir(pkg):
        if name.endswith(".py"):
            with open(os.path.join(pkg, name)) as f:
                src = f.read()
            assert "import oracle" not in src and "from oracle" not in src, name
