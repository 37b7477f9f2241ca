"""bench.py's contract on CPU: the algorithmic byte counts it reports agree
with the library's own size queries, and the reference arm (the CPU oracle)
prints one JSON line with the required keys."""
from __future__ import annotations

import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import weight_only_quantized_q4_b200 as wq  # noqa: E402


@pytest.mark.parametrize("name", sorted(bench.WORKLOADS))
def test_weight_bytes_match_library_size_queries(name):
    w = bench.WORKLOADS[name]
    N, K = w["N"], w["K"]
    got = bench.weight_bytes(w)
    if w["fmt"] == "int4":
        if w["zeros"]:
            assert got == wq.wq_int4_bytes(N, K, w["bs"], wq.WQ_LAYOUT_CANONICAL)
        else:
            assert got == wq.wq_int4_codes_bytes(N, K, wq.WQ_LAYOUT_CANONICAL) + 2 * N * (K // w["bs"])
        if w.get("layout", 0) == wq.WQ_LAYOUT_B200_V1:
            # the repacked stream holds the same bytes plus per-tile padding (< 1%)
            packed = wq.wq_int4_packed_bytes(N, K, w["bs"], wq.WQ_LAYOUT_B200_V1)
            assert got <= packed <= got * 1.01
    elif w["fmt"] == "q4k":
        if w["dsc"]:
            assert got == wq.wq_int4_codes_bytes(N, K, wq.WQ_LAYOUT_CANONICAL) + wq.wq_q4k_dsc_bytes(N, K)
        else:
            assert got == wq.wq_q4k_bytes(N, K)
    elif w["fmt"] == "swiglu":
        assert got == 2 * wq.wq_int4_bytes(N, K, w["bs"], wq.WQ_LAYOUT_CANONICAL)
        assert got <= wq.wq_int4_gate_up_packed_bytes(N, K, w["bs"]) <= got * 1.01
    elif w["fmt"] == "mmq":  # the q4_K weights (the int8 activations are like x, excluded)
        assert got == wq.wq_q4k_bytes(N, K)
    elif w["fmt"] == "mxfp4":
        # codes (two per byte) plus one E8M0 byte per 32-element block
        assert got == wq.wq_int4_codes_bytes(N, K, wq.WQ_LAYOUT_CANONICAL) + N * (K // 32)
    else:
        assert got == 2 * N * K


def test_default_workload_is_the_int4_target_shape():
    w = bench.WORKLOADS[bench.DEFAULT_WORKLOAD]
    assert (w["fmt"], w["M"], w["N"], w["K"], w["bs"], w["zeros"]) == ("int4", 1, 4096, 14336, 128, True)


def test_reference_arm_json_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                          "int4_b32_m1_256x1024", "--steps", "1", "--warmup", "0", "--cpu-budget", "0.2"],
                         capture_output=True, text=True, timeout=300, env=dict(os.environ, RANK="0", WORLD_SIZE="1"))
    assert out.returncode == 0, out.stderr
    lines = [ln for ln in out.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["metric"] == bench.METRIC  # the same metric as the product arm
    assert d["impl"] == "reference" and d["unit"] == "GB/s" and d["value"] > 0
    assert d["higher_is_better"] is True and d["config"]["workload"] == "int4_b32_m1_256x1024"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
