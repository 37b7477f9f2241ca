"""Host-side checks of the TMEM row map of the tcgen05 B200_V1 GEMM (no GPU).

With the fp16 A rows in tensor memory, a warp can only reach its own quarter
of the 128 TMEM lanes, and each thread forms one weight row.  v1ta_row(L)
names the tile row (16·band + 8·half + g) that TMEM lane L holds.  The kernel
relies on two properties of that map, checked here on the function itself
(compiled for the host from the kernel header):

* it is a bijection of the 128 rows, so every accumulator row is some weight
  row exactly once and the epilogue can map it back;
* for every quarter (warp) and code chunk t, the 16-byte chunks the 32 lanes
  read at once (chunk 4g + t of their band's tile, bands an odd number of
  16-byte units apart in the raw slot) fall into all eight 16-byte bank
  groups, so one 128-bit shared load costs the minimum two wavefronts.
"""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "weight_only_quantized_q4_b200", "csrc")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

PROGRAM = r"""
#include <cstdio>
#include "gemm_v1tc.cuh"
int main() {
  for (int L = 0; L < 128; ++L) std::printf("%d\n", wq::v1ta_row(L));
  return 0;
}
"""


@pytest.fixture(scope="module")
def row_map(tmp_path_factory):
    if not (os.path.exists(NVCC) or shutil.which("nvcc")):
        pytest.skip("nvcc not available")
    d = tmp_path_factory.mktemp("v1ta")
    src, exe = d / "rows.cu", d / "rows"
    src.write_text(PROGRAM)
    cmd = [NVCC, "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-I", CSRC,
           "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)]
    subprocess.run(cmd, check=True, capture_output=True, timeout=600)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True, timeout=60).stdout
    return [int(v) for v in out.split()]


def test_row_map_is_a_bijection(row_map):
    assert sorted(row_map) == list(range(128))


def test_each_quarter_holds_four_bands_and_four_row_indices(row_map):
    for q in range(4):
        rows = row_map[32 * q:32 * q + 32]
        bands = {r >> 4 for r in rows}
        gs = {r & 7 for r in rows}
        assert len(bands) == 4 and len(gs) == 4, (q, sorted(bands), sorted(gs))
        assert all(sum(1 for r in rows if (r >> 4, r & 7) == (b, g)) == 2 for b in bands for g in gs)


@pytest.mark.parametrize("T", [1, 2, 3, 4, 5, 6, 7, 8])
def test_code_chunk_reads_cover_all_bank_groups(row_map, T):
    tb = 1072
    band_stride = T * tb + (16 if (T * tb // 16) % 2 == 0 else 0)  # the planner's rule
    assert (band_stride // 16) % 2 == 1
    for q in range(4):
        rows = row_map[32 * q:32 * q + 32]
        for step in range(T):
            for gp in range(2):
                for t in range(4):
                    addrs = {(r >> 4) * band_stride + step * tb + gp * 512 + (4 * (r & 7) + t) * 16 for r in rows}
                    assert len(addrs) == 16  # two lanes (the row pair g, g + 8) share each chunk
                    groups = [(a // 16) % 8 for a in addrs]
                    assert sorted(set(groups)) == list(range(8)), (q, T, step, gp, t, groups)
                    assert max(groups.count(g) for g in range(8)) == 2
