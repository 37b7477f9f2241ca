// gemv_tc.cuh — tensor-pipe decode GEMV for M = 1..8 (sm_100a), register operands.
//
// Why this exists next to the CUDA-core family: with 4-bit weights at HBM
// speed a B200 SM must retire ~43 weights per clock.  The CUDA-core path
// spends one (half-rate) mixed-precision FMA per weight per batch row, so
// from M = 2 on the FP32 pipe, not HBM, sets the pace.  Here the
// multiply-accumulate runs on the tensor pipe with warp-level
// mma.m16n8k16 (fp16 × fp16 -> fp32) whose A operand comes straight from the
// unpacking registers: no shared-memory or TMEM round trip for the
// dequantized operand, and the fp32 accumulators stay in registers so the
// per-block / per-chunk scales are applied exactly in fp32.
//
// Exact codes: a nibble placed in bits 0-3 of an fp16 whose other bits are
// 0x6400 is 1024 + q; a nibble in bits 4-7 under 0x5400 is 64 + q.  One LOP3
// builds such a pair, one HSUB2 removes 1024 + z (or 64 + z): the MMA sees the
// exact small integers (q - z) (int4) or q (q4_K).  For q4_K the last row of
// every 16-row tile is a row of ones, so the same MMA also returns Σx per
// chunk, needed for the -dmin·m term (w = d·sc·q - dmin·m, minfer doc 62
// "r59 — q4_K W_dsc plane", §2.1).
//
// Work split: a CTA owns whole bands of 16 rows (15 for q4_K).  A producer
// warp streams each band in K-chunks (one bulk copy per row, padded row
// pitch so the fragment loads are bank-conflict free, plus the matching
// activation chunk and, for the W_dsc plane, the band's plane entries) into a
// ring of shared-memory stages.  W consumer warps split each stage's
// K-units (int4: one quantization block; q4_K: one 64-element run; bf16: 32
// k) and accumulate the band's 16×8 outputs in registers; at the end of the
// band a shared-memory pass adds the W partial tiles and writes y.
#pragma once

#include "gemv_cc.cuh"
#include "wq_device.cuh"

namespace wq {

struct TCParams {
  const void* x;
  const uint8_t* w;
  const uint8_t* scales;
  const uint8_t* zeros;
  const uint8_t* plane;
  void* y;
  int M, N, K;
  int nb, zb, block_shift;  // int4
  long long row_bytes;      // bytes per weight row in global memory
  int rpb;                  // rows per band: 16, or 15 for q4_K (row 15 is the ones row)
  int n_bands;
  int Kc;                   // k per stage (int4: multiple of the block; q4_K: of 256; bf16: of 32)
  int pitch;                // bytes per row inside a stage
  int n_kst;                // stages per band
  int NS;                   // ring depth
  int stage_bytes;
  int off_x;                // activation chunk [M][Kc] fp16/bf16 inside a stage
  int off_plane;            // q4_K plane slice [Kc/32][pstride] inside a stage
  int plane_stride;
  int off_meta;             // int4: band scales [16][nb] fp16 then zeros [16][zb]; after the ring
  int meta_zoff;
  int off_red;              // 2 × W × 16 × 8 floats
  int W;                    // consumer warps
  int x_res;                // 1: the whole x [M][K] sits in shared memory at off_xres (one copy per CTA)
  int off_xres;
  // B200_V1 int4 stream: tile bytes, tiles per band, tiles per stage
  int v1_tb, v1_tpb, v1_tps;
};

__device__ __forceinline__ void mma_f16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t lop3_and_or(uint32_t v, uint32_t mask, uint32_t magic) {
  uint32_t r;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(v), "r"(mask), "r"(magic));  // (v & mask) | magic
  return r;
}

__device__ __forceinline__ uint32_t hsub2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

__device__ __forceinline__ void named_bar(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// BIGB: int4 blocks of at least 128 k (one block per 128-k iteration); the
// band's zero-point magics and fp32 scales are then precomputed in shared
// memory as one 16-byte entry {1024+z pair, 64+z pair, scale, 0} per
// (block, row).
template <Fmt F, bool V1, bool BIGB>
__global__ void __launch_bounds__(544, 1) gemv_tc_kernel(const TCParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int W = p.W;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + p.off_red + 2 * W * 16 * 8 * 4);
  uint64_t* empty = full + p.NS;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + p.NS);

  const int k_rot = static_cast<int>(blockIdx.x % static_cast<unsigned>(p.n_kst));
  const int b_begin = static_cast<int>(static_cast<long long>(blockIdx.x) * p.n_bands / gridDim.x);
  const int b_end = static_cast<int>(static_cast<long long>(blockIdx.x + 1) * p.n_bands / gridDim.x);
  const int total = (b_end - b_begin) * p.n_kst;

  if (tid == 0) {
    for (int i = 0; i < p.NS; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], W);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  // The next kernel in the stream may start streaming its weights now; this one
  // waits for the previous kernel only where it reads x (producer) or writes y.
  grid_launch_dependents();

  // ------------------------------------------------------------ producer warp
  // All 32 lanes issue copies: lane 0 arms the stage's barrier, then lane j
  // issues row copies j, j+32, ..., activation rows and plane chunks likewise
  // (a single issuing thread caps the copy rate of small row segments).
  if (warp == W && V1) {
    // B200_V1: the CTA's bands are one contiguous byte range; stream it linearly.
    if (lane != 0) return;
    const uint64_t policy = policy_evict_first();
    const uint32_t sbytes = static_cast<uint32_t>(p.v1_tps * p.v1_tb);
    const uint8_t* src = p.w + static_cast<long long>(b_begin) * p.v1_tpb * p.v1_tb;
    // Until the previous kernel has completed only L2 may be filled (it is the
    // point of coherence, so a prefetch cannot return data older than a write
    // of that kernel): prefetch the first ring's worth of this CTA's stream,
    // then wait, then copy into shared memory.
    for (int S = 0; S < min(total, p.NS); ++S) prefetch_l2(src + static_cast<long long>(S) * sbytes, sbytes);
    grid_wait_prior();
    int ks = 0, slot = 0;
    uint32_t phase = 0;
    for (int S = 0; S < total; ++S) {
      if (S >= p.NS && (*abort_flag || !mbar_wait_bounded(&empty[slot], phase ^ 1u))) {
        *abort_flag = 1;
        return;
      }
      uint8_t* st = smem + slot * p.stage_bytes;
      const uint32_t kc = static_cast<uint32_t>(p.v1_tps * 128);
      const uint32_t xb = p.x_res ? (S == 0 ? p.M * 2u * p.K : 0u) : p.M * 2u * kc;
      mbar_arrive_expect_tx(&full[slot], sbytes + xb);
      bulk_g2s_stream(st, src + static_cast<long long>(S) * sbytes, sbytes, &full[slot], policy);
      if (p.x_res) {
        if (S == 0) bulk_g2s(smem + p.off_xres, p.x, p.M * 2u * p.K, &full[slot]);
      } else {
        const long long k0 = static_cast<long long>(ks) * kc;
        for (int m = 0; m < p.M; ++m)
          bulk_g2s(st + p.off_x + m * 2 * kc, reinterpret_cast<const uint8_t*>(p.x) + (m * 1ll * p.K + k0) * 2,
                   2u * kc, &full[slot]);
      }
      if (++ks == p.n_kst) ks = 0;
      if (++slot == p.NS) {
        slot = 0;
        phase ^= 1u;
      }
    }
    return;
  }
  if (warp == W) {
    const uint64_t policy = policy_evict_first();
    {
      // L2 prefetch of the rows of this CTA's first band (first ring's worth of
      // stages), the only weight traffic issued before the previous kernel
      // has completed (see the B200_V1 producer above)
      const int r0 = b_begin * p.rpb, nr = min(p.rpb, p.N - r0);
      const int ns = min(p.n_kst, p.NS);
      long long seg = 0;
      if constexpr (F == Fmt::Int4) seg = static_cast<long long>(min(p.K, ns * p.Kc)) / 2;
      else if constexpr (F == Fmt::BF16) seg = 2ll * min(p.K, ns * p.Kc);
      else seg = static_cast<long long>(min(p.K, ns * p.Kc) / 256) * 144;
      if (b_begin < b_end)
        for (int j = lane; j < nr; j += 32) {
          const uint8_t* rowp = p.w + static_cast<long long>(r0 + j) * p.row_bytes;
          // whole 16-byte units inside the segment only (never past the tensor)
          const uint64_t a = (reinterpret_cast<uint64_t>(rowp) + 15) & ~15ull;
          const uint64_t e = (reinterpret_cast<uint64_t>(rowp) + seg) & ~15ull;
          for (uint64_t o = a; o < e; o += 32768)
            prefetch_l2(reinterpret_cast<const void*>(o), static_cast<uint32_t>(e - o < 32768ull ? e - o : 32768ull));
        }
    }
    grid_wait_prior();
    int band = b_begin, ks = 0, slot = 0;  // stage bookkeeping kept incremental (no divisions)
    uint32_t phase = 0;
    for (int S = 0; S < total; ++S) {
      if (S >= p.NS) {
        bool ok = true;
        if (lane == 0) ok = !*abort_flag && mbar_wait_bounded(&empty[slot], phase ^ 1u);
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) {
          if (lane == 0) *abort_flag = 1;
          return;
        }
      }
      const int r0 = band * p.rpb;
      const int nr = min(p.rpb, p.N - r0);
      // CTAs walk K from different starting chunks so that, at any moment,
      // they fetch different activation chunks (no L2 hot spot)
      int kr = ks + (V1 ? 0 : k_rot);
      if (kr >= p.n_kst) kr -= p.n_kst;
      const int k0 = kr * p.Kc;
      const int kc = min(p.Kc, p.K - k0);
      uint32_t seg, kofs;  // bytes per row in this stage, byte offset of k0 in a row
      if constexpr (F == Fmt::Int4) {
        seg = kc / 2;
        kofs = k0 / 2;
      } else if constexpr (F == Fmt::BF16) {
        seg = 2 * kc;
        kofs = 2 * k0;
      } else {
        seg = (kc / 256) * 144;
        kofs = (k0 / 256) * 144;
      }
      if constexpr (V1) seg = 0;  // B200_V1: the band's tiles arrive as one contiguous range below
      const uint32_t vbytes = V1 ? (kc / 128) * 1024u : 0u;
      uint32_t bytes = nr * seg + vbytes + (p.x_res ? (S == 0 ? p.M * 2u * p.K : 0u) : p.M * 2u * kc);
      uint32_t n_chunks = 0, pl_len0 = 0, pl_len8 = 0;
      if constexpr (F == Fmt::Q4KDsc) {
        n_chunks = kc / 32;
        pl_len0 = (nr * 8u + 15u) & ~15u;
        pl_len8 = (nr * 8u + 8u + 15u) & ~15u;
        // chunk c's slice starts 8 bytes past a 16-byte boundary iff (c·N + r0) is odd
        uint32_t n8 = 0;
        if (p.N & 1) {
          const uint32_t c_first = k0 / 32;
          for (uint32_t c = 0; c < n_chunks; ++c) n8 += ((c_first + c) * 1u * p.N + r0) & 1u;
        }
        bytes += (n_chunks - n8) * pl_len0 + n8 * pl_len8;
      }
      uint8_t* st = smem + slot * p.stage_bytes;
      // The slot was released by the consumers' mbarrier arrivals (release) and
      // acquired by the wait above: their shared-memory reads are ordered
      // before these async-proxy writes, no proxy fence is needed.
      if (lane == 0) mbar_arrive_expect_tx(&full[slot], bytes);
      __syncwarp();
      if constexpr (V1) {
        if (lane == 0)
          bulk_g2s_stream(st, p.w + static_cast<long long>(band) * 8ll * p.K + (k0 / 128) * 1024ll, vbytes,
                          &full[slot], policy);
      } else {
        for (int j = lane; j < nr; j += 32)
          bulk_g2s_stream(st + j * p.pitch, p.w + static_cast<long long>(r0 + j) * p.row_bytes + kofs, seg,
                          &full[slot], policy);
      }
      if (p.x_res) {
        // activations for the whole kernel ride on the first stage's barrier
        if (S == 0 && lane == 0) bulk_g2s(smem + p.off_xres, p.x, p.M * 2u * p.K, &full[slot]);
      } else {
        for (int m = lane; m < p.M; m += 32)
          bulk_g2s(st + p.off_x + m * 2 * p.Kc,
                   reinterpret_cast<const uint8_t*>(p.x) + (static_cast<long long>(m) * p.K + k0) * 2, 2u * kc,
                   &full[slot]);
      }
      if constexpr (F == Fmt::Q4KDsc) {
        for (uint32_t c = lane; c < n_chunks; c += 32) {
          const uint64_t a = reinterpret_cast<uint64_t>(p.plane) + ((k0 / 32 + c) * 1ull * p.N + r0) * 8ull;
          bulk_g2s_stream(st + p.off_plane + c * p.plane_stride, reinterpret_cast<const void*>(a & ~15ull),
                          (a & 15u) ? pl_len8 : pl_len0, &full[slot], policy);
        }
      }
      if (++ks == p.n_kst) {
        ks = 0;
        ++band;
      }
      if (++slot == p.NS) {
        slot = 0;
        phase ^= 1u;
      }
    }
    return;
  }

  // ------------------------------------------------------------ consumer warps
  grid_wait_prior();  // y may still be read or written by the previous kernel
  const int g = lane >> 2;  // fragment row (and batch column of B)
  const int t = lane & 3;   // fragment k-pair / output column pair
  const int nthr = W * 32;
  float* red = reinterpret_cast<float*>(smem + p.off_red);
  const uint8_t* meta = smem + p.off_meta;
  int S = 0;

  for (int band = b_begin; band < b_end; ++band) {
    const int r0 = band * p.rpb;
    const int nr = min(p.rpb, p.N - r0);
    if constexpr (F == Fmt::Int4 && V1) {
      // tiles carry their own scales and zero-points: nothing to stage per band
    } else if constexpr (F == Fmt::Int4 && BIGB) {
      uint4* meta4 = reinterpret_cast<uint4*>(smem + p.off_meta);
      const int ne = 16 * p.nb;
      const uint16_t* gs = reinterpret_cast<const uint16_t*>(p.scales);
      for (int e0 = tid; e0 < ne; e0 += 8 * nthr) {
        uint32_t sv[8], zv[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {  // eight independent loads in flight per thread
          const int e = e0 + u * nthr;
          sv[u] = 0u;
          zv[u] = 8u;
          if (e < ne) {
            const int r = e / p.nb, b = e - r * p.nb;
            if (r < nr) {
              sv[u] = gs[static_cast<long long>(r0 + r) * p.nb + b];
              if (p.zeros) zv[u] = (p.zeros[static_cast<long long>(r0 + r) * p.zb + (b >> 1)] >> ((b & 1) * 4)) & 15u;
            }
          }
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int e = e0 + u * nthr;
          if (e < ne) {
            const int r = e / p.nb, b = e - r * p.nb;
            const float sc = r < nr ? h16_to_f32(sv[u]) : 0.f;
            meta4[b * 16 + r] = make_uint4((0x6400u | zv[u]) * 0x00010001u, (0x5400u | (zv[u] << 4)) * 0x00010001u,
                                           __float_as_uint(sc), 0u);
          }
        }
      }
      named_bar(1, nthr);
    } else if constexpr (F == Fmt::Int4) {
      // band scales (fp16, [16][nb]) and zero-points ([16][zb]) into shared memory
      uint16_t* ms = reinterpret_cast<uint16_t*>(smem + p.off_meta);
      uint8_t* mz = smem + p.off_meta + p.meta_zoff;
      const uint16_t* gs = reinterpret_cast<const uint16_t*>(p.scales) + static_cast<long long>(r0) * p.nb;
      for (int i = tid; i < nr * p.nb; i += nthr) ms[i] = gs[i];
      if (p.zeros) {
        const uint8_t* gz = p.zeros + static_cast<long long>(r0) * p.zb;
        for (int i = tid; i < nr * p.zb; i += nthr) mz[i] = gz[i];
      }
      named_bar(1, nthr);
    }
    float yacc[4] = {0.f, 0.f, 0.f, 0.f};  // rows g, g+8 × columns 2t, 2t+1

    for (int ks = 0; ks < p.n_kst; ++ks, ++S) {
      const int slot = S % p.NS;
      const uint8_t* st = smem + slot * p.stage_bytes;
      bool ok = !*abort_flag;
      if (ok && !mbar_wait_bounded(&full[slot], static_cast<uint32_t>((S / p.NS) & 1))) {
        *abort_flag = 1;
        ok = false;
      }
      int kr = ks + (V1 ? 0 : k_rot);
      if (kr >= p.n_kst) kr -= p.n_kst;
      const int k0 = kr * p.Kc;
      const int kc = min(p.Kc, p.K - k0);
      const uint8_t* rg = st + g * p.pitch;        // row g of the tile
      const uint8_t* rg8 = st + (g + 8) * p.pitch; // row g + 8
      // activation row g at the stage's k0 (valid when g < M)
      const uint8_t* xs = p.x_res ? smem + p.off_xres + (static_cast<long long>(g) * p.K + k0) * 2
                                  : st + p.off_x + g * 2 * p.Kc;
      const bool xrow = g < p.M;

      if constexpr (F == Fmt::Int4) {
        // Iterations of 128 k (4 groups of 32); every group has its own
        // accumulator so four MMA chains are in flight per warp (the warp-level
        // MMA has a long latency on sm_100).  Groups of one quantization block
        // are summed before the block's fp32 scale is applied.
        const int iters = kc >> 7;
        const uint16_t* ms = reinterpret_cast<const uint16_t*>(meta);
        const uint8_t* mz = meta + p.meta_zoff;
        if constexpr (V1 && BIGB) {
          // One block covers the whole 128-k tile: its two scales and zero-points
          // (rows g and g+8) are read and turned into fp16 magics once per tile.
          for (int u = warp; ok && u < p.v1_tps; u += W) {
            const uint8_t* tp = st + u * p.v1_tb;
            const uint16_t* sc = reinterpret_cast<const uint16_t*>(tp + 1024);
            const uint32_t sb0 = sc[g], sb1 = sc[g + 8];
            const uint32_t zb0 = tp[1024 + 32 + (g >> 1)], zb1 = tp[1024 + 32 + ((g + 8) >> 1)];
            const uint4 qa = *reinterpret_cast<const uint4*>(tp + lane * 16);
            const uint4 qb = *reinterpret_cast<const uint4*>(tp + 512 + lane * 16);
            const uint8_t* xt = xs + 2 * 128 * u;
            uint4 xv[4];
#pragma unroll
            for (int gi = 0; gi < 4; ++gi) {
              xv[gi] = make_uint4(0u, 0u, 0u, 0u);
              if (xrow) xv[gi] = *reinterpret_cast<const uint4*>(xt + 2 * (32 * gi + 8 * t));
            }
            const uint32_t z0 = (zb0 >> ((g & 1) * 4)) & 15u, z1 = (zb1 >> ((g & 1) * 4)) & 15u;
            const uint32_t zl0 = (0x6400u | z0) * 0x00010001u, zl1 = (0x6400u | z1) * 0x00010001u;
            const uint32_t zh0 = (0x5400u | (z0 << 4)) * 0x00010001u, zh1 = (0x5400u | (z1 << 4)) * 0x00010001u;
            const uint32_t v0[4] = {qa.x, qa.z, qb.x, qb.z}, v1[4] = {qa.y, qa.w, qb.y, qb.w};
            float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int gi = 0; gi < 4; ++gi) {
              const uint32_t a0 = v0[gi], a1 = v1[gi], a08 = a0 >> 8, a18 = a1 >> 8;
              const uint32_t al[4] = {hsub2(lop3_and_or(a0, 0x000F000Fu, 0x64006400u), zl0),
                                      hsub2(lop3_and_or(a1, 0x000F000Fu, 0x64006400u), zl1),
                                      hsub2(lop3_and_or(a08, 0x000F000Fu, 0x64006400u), zl0),
                                      hsub2(lop3_and_or(a18, 0x000F000Fu, 0x64006400u), zl1)};
              const uint32_t ah[4] = {hsub2(lop3_and_or(a0, 0x00F000F0u, 0x54005400u), zh0),
                                      hsub2(lop3_and_or(a1, 0x00F000F0u, 0x54005400u), zh1),
                                      hsub2(lop3_and_or(a08, 0x00F000F0u, 0x54005400u), zh0),
                                      hsub2(lop3_and_or(a18, 0x00F000F0u, 0x54005400u), zh1)};
              // codes ordered k0 k2 k4 k6 k1 k3 k5 k7: natural activation pairs
              mma_f16(d, al, xv[gi].x, xv[gi].z);
              mma_f16(d, ah, xv[gi].y, xv[gi].w);
            }
            const float s0 = h16_to_f32(sb0), s1 = h16_to_f32(sb1);
            yacc[0] = fmaf(s0, d[0], yacc[0]);
            yacc[1] = fmaf(s0, d[1], yacc[1]);
            yacc[2] = fmaf(s1, d[2], yacc[2]);
            yacc[3] = fmaf(s1, d[3], yacc[3]);
          }
        } else if constexpr (V1) {
          // tile u of the stage: 1024 code bytes in fragment order, then the
          // tile's scales [bpt][16] fp16 and zero-point bytes [bpt][8]
          const int bpt = p.block_shift >= 7 ? 1 : (128 >> p.block_shift);
          for (int u = warp; ok && u < p.v1_tps; u += W) {
            const uint8_t* tp = st + u * p.v1_tb;
            const uint4 qa = *reinterpret_cast<const uint4*>(tp + lane * 16);
            const uint4 qb = *reinterpret_cast<const uint4*>(tp + 512 + lane * 16);
            const uint32_t v0[4] = {qa.x, qa.z, qb.x, qb.z}, v1[4] = {qa.y, qa.w, qb.y, qb.w};
            const uint8_t* xt = xs + 2 * 128 * u;  // activations of this tile's 128 k
            float d[4] = {0.f, 0.f, 0.f, 0.f};
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int gi = 0; gi < 4; ++gi) {
              const int bt = bpt == 1 ? 0 : (gi * 32) >> p.block_shift;
              const uint32_t zb0 = tp[1024 + 32 * bpt + bt * 8 + (g >> 1)];
              const uint32_t zb1 = tp[1024 + 32 * bpt + bt * 8 + ((g + 8) >> 1)];
              const uint32_t z0 = (zb0 >> ((g & 1) * 4)) & 15u, z1 = (zb1 >> ((g & 1) * 4)) & 15u;
              const uint32_t zl0 = (0x6400u | z0) * 0x00010001u, zl1 = (0x6400u | z1) * 0x00010001u;
              const uint32_t zh0 = (0x5400u | (z0 << 4)) * 0x00010001u, zh1 = (0x5400u | (z1 << 4)) * 0x00010001u;
              uint32_t bl0 = 0, bl1 = 0, bh0 = 0, bh1 = 0;
              if (xrow) {
                const uint4 xv = *reinterpret_cast<const uint4*>(xt + 2 * (32 * gi + 8 * t));
                bl0 = xv.x; bh0 = xv.y; bl1 = xv.z; bh1 = xv.w;  // codes ordered k0 k2 k4 k6 k1 k3 k5 k7
              }
              const uint32_t a0 = v0[gi], a1 = v1[gi], a08 = a0 >> 8, a18 = a1 >> 8;
              const uint32_t al[4] = {hsub2(lop3_and_or(a0, 0x000F000Fu, 0x64006400u), zl0),
                                      hsub2(lop3_and_or(a1, 0x000F000Fu, 0x64006400u), zl1),
                                      hsub2(lop3_and_or(a08, 0x000F000Fu, 0x64006400u), zl0),
                                      hsub2(lop3_and_or(a18, 0x000F000Fu, 0x64006400u), zl1)};
              const uint32_t ah[4] = {hsub2(lop3_and_or(a0, 0x00F000F0u, 0x54005400u), zh0),
                                      hsub2(lop3_and_or(a1, 0x00F000F0u, 0x54005400u), zh1),
                                      hsub2(lop3_and_or(a08, 0x00F000F0u, 0x54005400u), zh0),
                                      hsub2(lop3_and_or(a18, 0x00F000F0u, 0x54005400u), zh1)};
              mma_f16(d, al, bl0, bl1);
              mma_f16(d, ah, bh0, bh1);
              const bool last = bpt == 1 ? gi == 3 : ((gi + 1) * 32) % (1 << p.block_shift) == 0;
              if (last) {
                const uint16_t* sc = reinterpret_cast<const uint16_t*>(tp + 1024) + bt * 16;
                const float s0 = h16_to_f32(sc[g]), s1 = h16_to_f32(sc[g + 8]);
                acc[0] = fmaf(s0, d[0], acc[0]);
                acc[1] = fmaf(s0, d[1], acc[1]);
                acc[2] = fmaf(s1, d[2], acc[2]);
                acc[3] = fmaf(s1, d[3], acc[3]);
                d[0] = d[1] = d[2] = d[3] = 0.f;
              }
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) yacc[e] += acc[e];
          }
        } else if constexpr (BIGB) {
          const uint4* meta4 = reinterpret_cast<const uint4*>(meta);
          for (int it = warp; ok && it < iters; it += W) {
            const int kb = it * 128;
            const int blk = (k0 + kb) >> p.block_shift;
            const uint4 m0 = meta4[blk * 16 + g], m1 = meta4[blk * 16 + g + 8];
            uint32_t v0[4], v1[4];
            if constexpr (V1) {
              const uint4 qa = *reinterpret_cast<const uint4*>(st + it * 1024 + lane * 16);
              const uint4 qb = *reinterpret_cast<const uint4*>(st + it * 1024 + 512 + lane * 16);
              v0[0] = qa.x; v1[0] = qa.y; v0[1] = qa.z; v1[1] = qa.w;
              v0[2] = qb.x; v1[2] = qb.y; v0[3] = qb.z; v1[3] = qb.w;
            } else {
#pragma unroll
              for (int gi = 0; gi < 4; ++gi) {
                const int kk = kb + 32 * gi + 8 * t;
                v0[gi] = *reinterpret_cast<const uint32_t*>(rg + kk / 2);
                v1[gi] = *reinterpret_cast<const uint32_t*>(rg8 + kk / 2);
              }
            }
            float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int gi = 0; gi < 4; ++gi) {
              const int kk = kb + 32 * gi + 8 * t;
              uint32_t bl0 = 0, bl1 = 0, bh0 = 0, bh1 = 0;
              if (xrow) {
                const uint4 xv = *reinterpret_cast<const uint4*>(xs + 2 * kk);
                if constexpr (V1) {  // codes ordered k0 k2 k4 k6 k1 k3 k5 k7: natural activation pairs
                  bl0 = xv.x; bh0 = xv.y; bl1 = xv.z; bh1 = xv.w;
                } else {
                  bl0 = __byte_perm(xv.x, xv.z, 0x5410);  // (x0, x4)
                  bh0 = __byte_perm(xv.x, xv.z, 0x7632);  // (x1, x5)
                  bl1 = __byte_perm(xv.y, xv.w, 0x5410);  // (x2, x6)
                  bh1 = __byte_perm(xv.y, xv.w, 0x7632);  // (x3, x7)
                }
              }
              const uint32_t a0 = v0[gi], a1 = v1[gi], a08 = a0 >> 8, a18 = a1 >> 8;
              const uint32_t al[4] = {hsub2(lop3_and_or(a0, 0x000F000Fu, 0x64006400u), m0.x),
                                      hsub2(lop3_and_or(a1, 0x000F000Fu, 0x64006400u), m1.x),
                                      hsub2(lop3_and_or(a08, 0x000F000Fu, 0x64006400u), m0.x),
                                      hsub2(lop3_and_or(a18, 0x000F000Fu, 0x64006400u), m1.x)};
              const uint32_t ah[4] = {hsub2(lop3_and_or(a0, 0x00F000F0u, 0x54005400u), m0.y),
                                      hsub2(lop3_and_or(a1, 0x00F000F0u, 0x54005400u), m1.y),
                                      hsub2(lop3_and_or(a08, 0x00F000F0u, 0x54005400u), m0.y),
                                      hsub2(lop3_and_or(a18, 0x00F000F0u, 0x54005400u), m1.y)};
              mma_f16(d, al, bl0, bl1);
              mma_f16(d, ah, bh0, bh1);
            }
            const float s0 = __uint_as_float(m0.z), s1 = __uint_as_float(m1.z);
            yacc[0] = fmaf(s0, d[0], yacc[0]);
            yacc[1] = fmaf(s0, d[1], yacc[1]);
            yacc[2] = fmaf(s1, d[2], yacc[2]);
            yacc[3] = fmaf(s1, d[3], yacc[3]);
          }
        } else
        for (int it = warp; ok && it < iters; it += W) {
          const int kb = it * 128;
          uint32_t v0[4], v1[4], bl0[4], bl1[4], bh0[4], bh1[4];
          if constexpr (V1) {
            const uint4 qa = *reinterpret_cast<const uint4*>(st + it * 1024 + lane * 16);
            const uint4 qb = *reinterpret_cast<const uint4*>(st + it * 1024 + 512 + lane * 16);
            v0[0] = qa.x; v1[0] = qa.y; v0[1] = qa.z; v1[1] = qa.w;
            v0[2] = qb.x; v1[2] = qb.y; v0[3] = qb.z; v1[3] = qb.w;
          }
#pragma unroll
          for (int gi = 0; gi < 4; ++gi) {
            const int kk = kb + 32 * gi + 8 * t;
            if constexpr (!V1) {
              v0[gi] = *reinterpret_cast<const uint32_t*>(rg + kk / 2);
              v1[gi] = *reinterpret_cast<const uint32_t*>(rg8 + kk / 2);
            }
            bl0[gi] = bl1[gi] = bh0[gi] = bh1[gi] = 0u;
            if (xrow) {
              const uint4 xv = *reinterpret_cast<const uint4*>(xs + 2 * kk);
              if constexpr (V1) {
                bl0[gi] = xv.x; bh0[gi] = xv.y; bl1[gi] = xv.z; bh1[gi] = xv.w;
              } else {
                bl0[gi] = __byte_perm(xv.x, xv.z, 0x5410);  // (x0, x4)
                bh0[gi] = __byte_perm(xv.x, xv.z, 0x7632);  // (x1, x5)
                bl1[gi] = __byte_perm(xv.y, xv.w, 0x5410);  // (x2, x6)
                bh1[gi] = __byte_perm(xv.y, xv.w, 0x7632);  // (x3, x7)
              }
            }
          }
          float d[4][4];
#pragma unroll
          for (int gi = 0; gi < 4; ++gi) {
            const int blk = (k0 + kb + 32 * gi) >> p.block_shift;
            uint32_t z0 = 8u, z1 = 8u;
            if (p.zeros) {
              if (g < nr) z0 = (mz[g * p.zb + (blk >> 1)] >> ((blk & 1) * 4)) & 15u;
              if (g + 8 < nr) z1 = (mz[(g + 8) * p.zb + (blk >> 1)] >> ((blk & 1) * 4)) & 15u;
            }
            const uint32_t zl0 = (0x6400u | z0) * 0x00010001u, zl1 = (0x6400u | z1) * 0x00010001u;
            const uint32_t zh0 = (0x5400u | (z0 << 4)) * 0x00010001u, zh1 = (0x5400u | (z1 << 4)) * 0x00010001u;
            const uint32_t a0 = v0[gi], a1 = v1[gi], a08 = a0 >> 8, a18 = a1 >> 8;
            const uint32_t al[4] = {hsub2(lop3_and_or(a0, 0x000F000Fu, 0x64006400u), zl0),
                                    hsub2(lop3_and_or(a1, 0x000F000Fu, 0x64006400u), zl1),
                                    hsub2(lop3_and_or(a08, 0x000F000Fu, 0x64006400u), zl0),
                                    hsub2(lop3_and_or(a18, 0x000F000Fu, 0x64006400u), zl1)};
            const uint32_t ah[4] = {hsub2(lop3_and_or(a0, 0x00F000F0u, 0x54005400u), zh0),
                                    hsub2(lop3_and_or(a1, 0x00F000F0u, 0x54005400u), zh1),
                                    hsub2(lop3_and_or(a08, 0x00F000F0u, 0x54005400u), zh0),
                                    hsub2(lop3_and_or(a18, 0x00F000F0u, 0x54005400u), zh1)};
            d[gi][0] = d[gi][1] = d[gi][2] = d[gi][3] = 0.f;
            mma_f16(d[gi], al, bl0[gi], bl1[gi]);
            mma_f16(d[gi], ah, bh0[gi], bh1[gi]);
          }
          // fold: consecutive groups of the same block share one scale
          float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int gi = 0; gi < 4; ++gi) {
            const int blk = (k0 + kb + 32 * gi) >> p.block_shift;
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[e] += d[gi][e];
            const bool last = (gi == 3) || (((k0 + kb + 32 * (gi + 1)) >> p.block_shift) != blk);
            if (last) {
              const float s0 = g < nr ? h16_to_f32(ms[g * p.nb + blk]) : 0.f;
              const float s1 = g + 8 < nr ? h16_to_f32(ms[(g + 8) * p.nb + blk]) : 0.f;
              yacc[0] = fmaf(s0, acc[0], yacc[0]);
              yacc[1] = fmaf(s0, acc[1], yacc[1]);
              yacc[2] = fmaf(s1, acc[2], yacc[2]);
              yacc[3] = fmaf(s1, acc[3], yacc[3]);
#pragma unroll
              for (int e = 0; e < 4; ++e) acc[e] = 0.f;
            }
          }
        }
      } else if constexpr (F == Fmt::Q4K || F == Fmt::Q4KDsc) {
        const int units = (kc / 256) * 4;  // runs of 64 elements
        const bool ones_row = (g == 7);    // fragment row g+8 == 15 carries ones
        for (int u = warp; ok && u < units; u += W) {
          const int sb = u >> 2, pp = u & 3;          // block in the stage, run
          const int qoff = sb * 144 + 16 + 32 * pp;   // code bytes of the run inside a row
          const int kx = sb * 256 + 64 * pp;          // k of chunk 2p inside the stage
          float d0h[2][4], d1h[2][4];  // one accumulator per half-run: four MMA chains in flight
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int i = 16 * h + 4 * t;             // element inside the chunks
            const uint32_t v0 = *reinterpret_cast<const uint32_t*>(rg + qoff + i);
            const uint32_t v1 = ones_row ? 0u : *reinterpret_cast<const uint32_t*>(rg8 + qoff + i);
            uint32_t b0 = 0, b1 = 0, c0 = 0, c1 = 0;
            if (xrow) {
              const uint2 xa = *reinterpret_cast<const uint2*>(xs + 2 * (kx + i));
              const uint2 xb = *reinterpret_cast<const uint2*>(xs + 2 * (kx + 32 + i));
              b0 = __byte_perm(xa.x, xa.y, 0x5410);  // (c0[i], c0[i+2])
              b1 = __byte_perm(xa.x, xa.y, 0x7632);  // (c0[i+1], c0[i+3])
              c0 = __byte_perm(xb.x, xb.y, 0x5410);
              c1 = __byte_perm(xb.x, xb.y, 0x7632);
            }
            const uint32_t v08 = v0 >> 8, v18 = v1 >> 8;
            const uint32_t k1024 = 0x64006400u, k64 = 0x54005400u, one = 0x3C003C00u;
            const uint32_t al[4] = {hsub2(lop3_and_or(v0, 0x000F000Fu, k1024), k1024),
                                    ones_row ? one : hsub2(lop3_and_or(v1, 0x000F000Fu, k1024), k1024),
                                    hsub2(lop3_and_or(v08, 0x000F000Fu, k1024), k1024),
                                    ones_row ? one : hsub2(lop3_and_or(v18, 0x000F000Fu, k1024), k1024)};
            const uint32_t ah[4] = {hsub2(lop3_and_or(v0, 0x00F000F0u, k64), k64),
                                    ones_row ? one : hsub2(lop3_and_or(v1, 0x00F000F0u, k64), k64),
                                    hsub2(lop3_and_or(v08, 0x00F000F0u, k64), k64),
                                    ones_row ? one : hsub2(lop3_and_or(v18, 0x00F000F0u, k64), k64)};
            d0h[h][0] = d0h[h][1] = d0h[h][2] = d0h[h][3] = 0.f;
            d1h[h][0] = d1h[h][1] = d1h[h][2] = d1h[h][3] = 0.f;
            mma_f16(d0h[h], al, b0, b1);
            mma_f16(d1h[h], ah, c0, c1);
          }
          float d0[4], d1[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            d0[e] = d0h[0][e] + d0h[1][e];
            d1[e] = d1h[0][e] + d1h[1][e];
          }
          // Σx of chunks 2p and 2p+1 for columns 2t, 2t+1 sit in lane (7, t), fragment row 15
          const float X00 = __shfl_sync(0xffffffffu, d0[2], 28 + t);
          const float X01 = __shfl_sync(0xffffffffu, d0[3], 28 + t);
          const float X10 = __shfl_sync(0xffffffffu, d1[2], 28 + t);
          const float X11 = __shfl_sync(0xffffffffu, d1[3], 28 + t);
          // coefficients (A, B) of chunks 2p, 2p+1 for rows g and g+8
          float A0[2], A1[2], B0[2], B1[2];
#pragma unroll
          for (int rr = 0; rr < 2; ++rr) {
            const int row = g + 8 * rr;
            A0[rr] = A1[rr] = B0[rr] = B1[rr] = 0.f;
            if (row < nr && row < 15) {
              if constexpr (F == Fmt::Q4KDsc) {
                const int cl = sb * 8 + 2 * pp;  // chunk inside the stage
                const uint64_t a0 =
                    reinterpret_cast<uint64_t>(p.plane) + ((k0 / 32 + cl) * 1ull * p.N + r0) * 8ull;
                const uint64_t a1 = a0 + static_cast<uint64_t>(p.N) * 8ull;
                const float2 P0 = *reinterpret_cast<const float2*>(st + p.off_plane + cl * p.plane_stride +
                                                                    (a0 & 15u) + row * 8);
                const float2 P1 = *reinterpret_cast<const float2*>(st + p.off_plane + (cl + 1) * p.plane_stride +
                                                                    (a1 & 15u) + row * 8);
                A0[rr] = P0.x;
                B0[rr] = P0.y;
                A1[rr] = P1.x;
                B1[rr] = P1.y;
              } else {
                const uint4 hd = *reinterpret_cast<const uint4*>(st + row * p.pitch + sb * 144);
                uint32_t sc2, mn2;
                q4k_scale_min_pair(hd.y, hd.z, hd.w, static_cast<uint32_t>(pp & 1), static_cast<uint32_t>(pp >> 1),
                                   sc2, mn2);
                const float dd = h16_to_f32(hd.x), dm = h16_to_f32(hd.x >> 16);
                A0[rr] = dd * static_cast<float>(sc2 & 0xFFu);
                A1[rr] = dd * static_cast<float>(sc2 >> 8);
                B0[rr] = -(dm * static_cast<float>(mn2 & 0xFFu));
                B1[rr] = -(dm * static_cast<float>(mn2 >> 8));
              }
            }
          }
          yacc[0] = fmaf(A0[0], d0[0], fmaf(A1[0], d1[0], fmaf(B0[0], X00, fmaf(B1[0], X10, yacc[0]))));
          yacc[1] = fmaf(A0[0], d0[1], fmaf(A1[0], d1[1], fmaf(B0[0], X01, fmaf(B1[0], X11, yacc[1]))));
          yacc[2] = fmaf(A0[1], d0[2], fmaf(A1[1], d1[2], fmaf(B0[1], X00, fmaf(B1[1], X10, yacc[2]))));
          yacc[3] = fmaf(A0[1], d0[3], fmaf(A1[1], d1[3], fmaf(B0[1], X01, fmaf(B1[1], X11, yacc[3]))));
        }
      } else {  // BF16: A is the weight itself, 16 k per MMA; four rotating accumulators
        const int units = kc / 64;
        float d[4][4];
#pragma unroll
        for (int q = 0; q < 4; ++q) d[q][0] = d[q][1] = d[q][2] = d[q][3] = 0.f;
        for (int u = warp; ok && u < units; u += W) {
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            const int kk = u * 64 + 16 * h + 2 * t;
            const uint32_t a[4] = {*reinterpret_cast<const uint32_t*>(rg + 2 * kk),
                                   *reinterpret_cast<const uint32_t*>(rg8 + 2 * kk),
                                   *reinterpret_cast<const uint32_t*>(rg + 2 * (kk + 8)),
                                   *reinterpret_cast<const uint32_t*>(rg8 + 2 * (kk + 8))};
            uint32_t b0 = 0, b1 = 0;
            if (xrow) {
              b0 = *reinterpret_cast<const uint32_t*>(xs + 2 * kk);
              b1 = *reinterpret_cast<const uint32_t*>(xs + 2 * (kk + 8));
            }
            mma_bf16(d[h], a, b0, b1);
          }
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) yacc[e] += (d[0][e] + d[1][e]) + (d[2][e] + d[3][e]);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot]);
    }

    // ---- band end: add the W partial tiles, write y
    float* rb = red + (band & 1) * (W * 16 * 8);
    rb[(warp * 16 + g) * 8 + 2 * t] = yacc[0];
    rb[(warp * 16 + g) * 8 + 2 * t + 1] = yacc[1];
    rb[(warp * 16 + g + 8) * 8 + 2 * t] = yacc[2];
    rb[(warp * 16 + g + 8) * 8 + 2 * t + 1] = yacc[3];
    named_bar(1, nthr);
    if (!*abort_flag) {
      for (int o = tid; o < nr * p.M; o += nthr) {
        const int row = o / p.M, n = o - row * p.M;
        float sum = 0.f;
        for (int w2 = 0; w2 < W; ++w2) sum += rb[(w2 * 16 + row) * 8 + n];
        const long long yo = static_cast<long long>(n) * p.N + r0 + row;
        if constexpr (F == Fmt::BF16)
          reinterpret_cast<__nv_bfloat16*>(p.y)[yo] = __float2bfloat16_rn(sum);
        else
          reinterpret_cast<__half*>(p.y)[yo] = __float2half_rn(sum);
      }
    }
  }
}

}  // namespace wq
