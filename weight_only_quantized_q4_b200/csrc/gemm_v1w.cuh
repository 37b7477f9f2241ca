// gemm_v1w.cuh — batched GEMM (M = 9..64) over the int4 B200_V1 band stream
// with warp-level MMA (mma.sync m16n8k16, fp16 × fp16 -> fp32) and the A
// operand straight from the unpacking registers.
//
// y[m, n] = Σ_k W[n, k]·x[m, k], W = (q - z)·s (onnx-genai PR #1000, "What it
// does": int4 blockwise weights, fp16 scales, uint4 zero-points; blocks of at
// least 128 k, so every 16 × 128 tile has one scale and one zero-point per row).
//
// Why next to the tcgen05 kernel: at these batch sizes a 128-row tile gives
// each tcgen05.mma little work, and one thread issuing eight of them per 128-k
// step plus the fp16 A tile written to and read back from shared memory set
// the pace (about 1 µs per step whatever M is).  Here every weight code is
// unpacked once into registers — q - z exactly, through magic-number fp16
// codes — and multiplied against all M batch rows by the warp that unpacked
// it (M/8 MMA column groups), so there is no A tile and no issuing thread.
//
// Layout of the work.  A CTA owns R = 8 bands (128 rows) and a run of 128-k
// steps of K (the S CTAs of a cluster split K and add their partials through
// distributed shared memory in rank order):
//   * producer warp: one bulk copy per band for T consecutive steps (the
//     band's tiles are contiguous in the stream) into a raw slot, and one TMA
//     copy per step of the x slice [8·MG rows][128 k] (two 64-k boxes,
//     128-byte swizzle: the fragment reads of eight rows hit eight different
//     16-byte bank groups; rows past M read as zero);
//   * P·R consumer warps: warp w takes band w mod R on the steps ≡ w / R
//     (mod P), keeps its 16 rows × 8·MG outputs in registers over all its
//     steps, and applies each tile's fp32 scale to the tile's exact integer
//     sums (P = 2 for up to 24 batch rows, so that two warps per band hide the
//     MMA latency; P = 1 from 25 rows, where the MG independent MMA chains of
//     a warp do, and the register budget of a 9-warp CTA holds the accumulators);
//   * epilogue: the two parities and (cluster) the K slices are added in a
//     fixed order, y rounded once to fp16.
// Every mbarrier wait is bounded (wq_device.cuh); after a timeout the kernel
// records it, waits (bounded) for its copies in flight and returns.
#pragma once

#include "gemm_tc5.cuh"
#include "gemv_tc.cuh"

namespace wq {

struct V1WParams {
  CUtensorMap tmap_x;  // x [M][K] fp16, box 64 k × 8·MG rows, 128-byte swizzle
  const uint8_t* w;    // B200_V1 int4 stream
  void* y;             // [M][N] fp16
  int M, N, K;
  int n_bands, tpb, tb;  // bands, 128-k tiles per band, bytes per tile
  int S;                 // CTAs of a cluster (K slices); rank r takes steps [r·tpb/S, (r+1)·tpb/S)
  int T, NR, NX;         // steps per raw slot, raw slots, x slots
  int off_x, off_bar;    // shared-memory offsets (raw slots start at 0)
};

constexpr int kV1WBands = 8;  // bands per CTA (128 rows)

// consumer warps per band: two (step parities) for MG <= 3, one above
__host__ __device__ constexpr int v1w_par(int mg) { return mg <= 3 ? 2 : 1; }
__host__ __device__ constexpr int v1w_warps(int mg) { return kV1WBands * v1w_par(mg) + 1; }

template <int MG>
__global__ void __launch_bounds__(v1w_warps(MG) * 32, 1) gemm_v1w_kernel(const __grid_constant__ V1WParams p) {
  constexpr int R = kV1WBands;
  constexpr int P = v1w_par(MG);
  constexpr int XR = 8 * MG;          // batch rows of an x slice
  constexpr int XSLOT = XR * 256;     // two 64-k boxes of XR rows × 128 B
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* raw_full = reinterpret_cast<uint64_t*>(smem + p.off_bar);
  uint64_t* raw_empty = raw_full + p.NR;
  uint64_t* x_full = raw_empty + p.NR;
  uint64_t* x_empty = x_full + p.NX;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(x_empty + p.NX);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = p.S > 1 ? tc5_cluster_rank() : 0u;
  const int tile = blockIdx.x / p.S;
  const int n0 = tile * 16 * R, b0 = tile * R;
  const int nbt = min(R, p.n_bands - b0);  // bands present in this row tile
  const int s_begin = static_cast<int>((static_cast<long long>(rank) * p.tpb) / p.S);
  const int nks = static_cast<int>((static_cast<long long>(rank + 1) * p.tpb) / p.S) - s_begin;

  if (tid == 0) {
    for (int i = 0; i < p.NR; ++i) {
      mbar_init(&raw_full[i], 1);
      mbar_init(&raw_empty[i], P * R);  // every consumer warp, once per slot
    }
    for (int i = 0; i < p.NX; ++i) {
      mbar_init(&x_full[i], 1);
      mbar_init(&x_empty[i], R);  // the R warps that take the step
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();

  float yacc[MG][4];
#pragma unroll
  for (int j = 0; j < MG; ++j) yacc[j][0] = yacc[j][1] = yacc[j][2] = yacc[j][3] = 0.f;
  const int g = lane >> 2, t = lane & 3;
  const int band = warp % R, par = warp / R;

  if (warp == P * R) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const long long band_bytes = static_cast<long long>(p.tpb) * p.tb;
      const int nslots = (nks + p.T - 1) / p.T;
      int issued = 0, x_issued = 0;
      auto issue_raw = [&](int r) {
        const int rs = r % p.NR, ru = r / p.NR;
        if (ru > 0 && !mbar_wait_bounded(&raw_empty[rs], static_cast<uint32_t>((ru - 1) & 1))) return false;
        const int nt = min(p.T, nks - r * p.T);
        mbar_arrive_expect_tx(&raw_full[rs], static_cast<uint32_t>(nbt * nt * p.tb));
        uint8_t* dst = smem + rs * R * p.T * p.tb;
        for (int i = 0; i < nbt; ++i)
          bulk_g2s(dst + i * p.T * p.tb, p.w + (b0 + i) * band_bytes + static_cast<long long>(s_begin + r * p.T) * p.tb,
                   static_cast<uint32_t>(nt * p.tb), &raw_full[rs]);
        return true;
      };
      for (int ls = 0; ls < nks && !*abort_flag; ++ls) {
        const int xs = ls % p.NX, xu = ls / p.NX;
        if (xu > 0 && !mbar_wait_bounded(&x_empty[xs], static_cast<uint32_t>((xu - 1) & 1))) {
          *abort_flag = 1;
          break;
        }
        mbar_arrive_expect_tx(&x_full[xs], static_cast<uint32_t>(XSLOT));
        uint8_t* xd = smem + p.off_x + xs * XSLOT;
        tma_load_2d(xd, &p.tmap_x, (s_begin + ls) * 128, 0, &x_full[xs]);
        tma_load_2d(xd + XSLOT / 2, &p.tmap_x, (s_begin + ls) * 128 + 64, 0, &x_full[xs]);
        ++x_issued;
        bool okr = true;
        while (okr && issued < nslots && issued <= ls / p.T + p.NR - 1) okr = issue_raw(issued++);
        if (!okr) {
          *abort_flag = 1;
          break;
        }
      }
      // the latest copies into each slot have landed before the CTA may exit
      for (int r = issued > p.NR ? issued - p.NR : 0; r < issued; ++r)
        mbar_wait_bounded(&raw_full[r % p.NR], static_cast<uint32_t>((r / p.NR) & 1));
      for (int l = x_issued > p.NX ? x_issued - p.NX : 0; l < x_issued; ++l)
        mbar_wait_bounded(&x_full[l % p.NX], static_cast<uint32_t>((l / p.NX) & 1));
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ consumer warps
    const bool have = band < nbt;
    for (int r = 0; r * p.T < nks && !*abort_flag; ++r) {
      const int rs = r % p.NR;
      if (!mbar_wait_bounded(&raw_full[rs], static_cast<uint32_t>((r / p.NR) & 1))) {
        *abort_flag = 1;
        break;
      }
      const int l_end = min(nks, (r + 1) * p.T);
      int ls0 = r * p.T;
      while (ls0 % P != par) ++ls0;
      for (int ls = ls0; ls < l_end; ls += P) {
        const int xs = ls % p.NX;
        if (!mbar_wait_bounded(&x_full[xs], static_cast<uint32_t>((ls / p.NX) & 1))) {
          *abort_flag = 1;
          break;
        }
        if (have) {
          const uint8_t* tp = smem + (rs * R + band) * p.T * p.tb + (ls - r * p.T) * p.tb;
          const uint8_t* xsl = smem + p.off_x + xs * XSLOT;
          const uint4 qa = *reinterpret_cast<const uint4*>(tp + lane * 16);
          const uint4 qb = *reinterpret_cast<const uint4*>(tp + 512 + lane * 16);
          const uint16_t* sc = reinterpret_cast<const uint16_t*>(tp + 1024);
          const uint32_t sb0 = sc[g], sb1 = sc[g + 8];
          const uint32_t zb0 = tp[1056 + (g >> 1)], zb1 = tp[1056 + ((g + 8) >> 1)];
          const uint32_t z0 = (zb0 >> ((g & 1) * 4)) & 15u, z1 = (zb1 >> ((g & 1) * 4)) & 15u;
          const uint32_t zl0 = (0x6400u | z0) * 0x00010001u, zl1 = (0x6400u | z1) * 0x00010001u;
          const uint32_t zh0 = (0x5400u | (z0 << 4)) * 0x00010001u, zh1 = (0x5400u | (z1 << 4)) * 0x00010001u;
          const uint32_t v0[4] = {qa.x, qa.z, qb.x, qb.z}, v1[4] = {qa.y, qa.w, qb.y, qb.w};
          float d[MG][4];
#pragma unroll
          for (int j = 0; j < MG; ++j) d[j][0] = d[j][1] = d[j][2] = d[j][3] = 0.f;
#pragma unroll
          for (int gi = 0; gi < 4; ++gi) {
            const uint32_t a0 = v0[gi], a1 = v1[gi], a08 = a0 >> 8, a18 = a1 >> 8;
            // the exact integers q - z of rows g, g + 8 as fp16 pairs (codes
            // ordered k0 k2 k4 k6 k1 k3 k5 k7 in a word: natural x pairs)
            const uint32_t al[4] = {hsub2(lop3_and_or(a0, 0x000F000Fu, 0x64006400u), zl0),
                                    hsub2(lop3_and_or(a1, 0x000F000Fu, 0x64006400u), zl1),
                                    hsub2(lop3_and_or(a08, 0x000F000Fu, 0x64006400u), zl0),
                                    hsub2(lop3_and_or(a18, 0x000F000Fu, 0x64006400u), zl1)};
            const uint32_t ah[4] = {hsub2(lop3_and_or(a0, 0x00F000F0u, 0x54005400u), zh0),
                                    hsub2(lop3_and_or(a1, 0x00F000F0u, 0x54005400u), zh1),
                                    hsub2(lop3_and_or(a08, 0x00F000F0u, 0x54005400u), zh0),
                                    hsub2(lop3_and_or(a18, 0x00F000F0u, 0x54005400u), zh1)};
            // x row 8j + g at k = 32·gi + 8t .. + 7: 16-byte chunk 4(gi & 1) + t of
            // the 64-k box gi / 2, swizzled by the row
            const int c = 4 * (gi & 1) + t;
            const uint8_t* xb = xsl + (gi >> 1) * (XSLOT / 2);
#pragma unroll
            for (int j = 0; j < MG; ++j) {
              const int xr = 8 * j + g;
              const uint4 xv = *reinterpret_cast<const uint4*>(xb + xr * 128 + ((c ^ (xr & 7)) << 4));
              mma_f16(d[j], al, xv.x, xv.z);
              mma_f16(d[j], ah, xv.y, xv.w);
            }
          }
          const float s0 = h16_to_f32(sb0), s1 = h16_to_f32(sb1);
#pragma unroll
          for (int j = 0; j < MG; ++j) {
            yacc[j][0] = fmaf(s0, d[j][0], yacc[j][0]);
            yacc[j][1] = fmaf(s0, d[j][1], yacc[j][1]);
            yacc[j][2] = fmaf(s1, d[j][2], yacc[j][2]);
            yacc[j][3] = fmaf(s1, d[j][3], yacc[j][3]);
          }
        }
        __syncwarp();
        if (lane == 0) tc5_arrive(&x_empty[xs]);
      }
      __syncwarp();
      if (lane == 0) tc5_arrive(&raw_empty[rs]);
    }
  }

  // ---- epilogue: partials [parity][128 rows][XR] in the (drained) rings
  __syncthreads();
  float* red = reinterpret_cast<float*>(smem);
  if (warp < P * R) {
#pragma unroll
    for (int j = 0; j < MG; ++j) {
      const int r0 = (par * 16 * R + 16 * band + g) * XR + 8 * j + 2 * t;
      red[r0] = yacc[j][0];
      red[r0 + 1] = yacc[j][1];
      red[r0 + 8 * XR] = yacc[j][2];
      red[r0 + 8 * XR + 1] = yacc[j][3];
    }
  }
  __syncthreads();
  const bool ok = !*abort_flag;
  __half* y = reinterpret_cast<__half*>(p.y);
  const int nthr = v1w_warps(MG) * 32;
  if constexpr (P == 2) {  // the two parities, parity 0 first, into parity 0's slot
    for (int i = tid; i < 16 * R * XR; i += nthr) red[i] = red[i] + red[16 * R * XR + i];
  }
  if (p.S == 1) {
    __syncthreads();
    for (int i = tid; i < 16 * R * p.M; i += nthr) {
      const int row = i / p.M, m = i - row * p.M;
      if (n0 + row < p.N && ok) y[static_cast<long long>(m) * p.N + n0 + row] = __float2half_rn(red[row * XR + m]);
    }
  } else {
    // K split over the cluster: each rank adds 128/S rows over all ranks in rank order
    tc5_cluster_sync();
    const int rows_per = 16 * R / p.S;
    for (int i = tid; i < rows_per * p.M; i += nthr) {
      const int rr = static_cast<int>(rank) * rows_per + i / p.M, m = i % p.M;
      float sum = 0.f;
      for (int q = 0; q < p.S; ++q) sum += tc5_dsmem_ld(red + rr * XR + m, static_cast<uint32_t>(q));
      if (n0 + rr < p.N && ok) y[static_cast<long long>(m) * p.N + n0 + rr] = __float2half_rn(sum);
    }
    tc5_cluster_sync();
  }
}

}  // namespace wq
