// gemv_v1.cuh — decode GEMV (M = 1..8) for int4 weights in the B200_V1 stream
// layout with quantization blocks of at least 128 k (one block per tile).
//
// What it computes (onnx-genai PR #1000, "What it does": int4 blockwise
// weights with fp16 scales and uint4 zero-points): y[m][n] = Σ_k x[m][k]·w[n][k]
// with w = (q − z)·s, accumulated in fp32 and rounded once to fp16.
//
// How, per 128-k tile of a 16-row band (one quantization block per row):
//   Σ_k (q − z)·s·x = s·(Σ_k q·x − z·Σ_k x)
// The code words are masked into fp16 subnormals, q·2^-24 (low nibbles) and
// q·2^-20 (high nibbles), exact, with no subtraction; two warp-level MMAs per
// 32 k (one per nibble half, each with its own fp32 accumulator) form
// 2^-24·Σ q·x.  Σ_k x per tile and batch column (×2^-24) is precomputed once
// per CTA from the resident activations, so the zero-point costs one FMA per
// output per tile.  The fp32 result is rescaled by 2^24 (exact) at the end.
//
// Work split.  A cluster of C CTAs (C = 1, 2 or 4) owns a contiguous range of
// bands; CTA rank r of the cluster streams k-tiles [r·tpb/C, (r+1)·tpb/C) of
// each band.  A CTA's tiles form one linear sequence (band-major); the
// producer warp copies it in stages of `tps` tiles with bulk copies (one per
// contiguous run) into a ring of NS shared-memory stages.  Consumer warp w
// takes tiles w, w+W, w+2W, ... of the sequence, so warps never wait for one
// another at band boundaries: each warp hands its partial sums for a band to
// a reducer warp through a two-slot shared buffer guarded by named barriers,
// and the reducer adds the W partials in fixed warp order (deterministic).
// With C > 1 the per-CTA band partials are added across the cluster through
// distributed shared memory, again in fixed rank order.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

#include "wq_device.cuh"

namespace wq {

constexpr int kV1MaxDst = 8;

struct V1Params {
  const void* x;     // [M][K] fp16
  const uint8_t* w;  // B200_V1 stream
  void* y;           // [M][N] fp16
  // Where y goes: n_dst buffers of [M][y_ld] fp16 (this GPU's output and, for
  // a row-split layer, the other GPUs' copies mapped into this process), the
  // N rows of this call landing at columns y_off .. y_off + N - 1 of each.
  // A plain call has one destination, y itself (y_ld = N, y_off = 0).
  void* ydst[kV1MaxDst];
  int n_dst, y_ld, y_off;
  int M, N, K;
  int n_bands;       // ceil(N / 16)
  int tpb;           // tiles per band (K / 128)
  int tpc;           // tiles per band handled by one CTA (tpb / C)
  int tps;           // tiles per stage (a multiple of W)
  int tps0;          // tiles of the first stage (a multiple of W, <= tps): a small first
                     // stage lands sooner after the wait for the previous kernel
  int tb;            // bytes per tile
  int NS;            // ring depth
  int stage_bytes;   // tps · tb
  int C;             // CTAs per cluster (along K)
  int W;             // consumer warps
  int hint;          // 1: weight copies carry the L2 evict-first policy
  int pre;           // stages copied to shared memory before waiting for the previous kernel
  int pf_bytes;      // bytes of the CTA's stream prefetched into L2 before that wait (pre == 0)
  int pfd;           // after the wait: stage S + pfd is prefetched into L2 as stage S is copied (0: off)
  int Mp;            // M rounded up to even (stride of a partial row)
  int off_x;         // activations [M][tpc·128] fp16
  int off_zero;      // 256 zero bytes
  int off_xs;        // Σx table [tpc][8] fp32 (×2^-24)
  int off_red;       // [2][W][16][Mp] fp32 warp partials
  int off_part;      // [bands per cluster][16][M] fp32 CTA partials (C > 1)
  int off_bar;       // full[NS], empty[NS], abort word
};

namespace v1d {

// y[n][r] (fp16, RN) into every destination of the call
__device__ __forceinline__ void store_y(const V1Params& p, int n, int r, float v) {
  const __half h = __float2half_rn(v);
  for (int d = 0; d < p.n_dst; ++d)
    reinterpret_cast<__half*>(p.ydst[d])[static_cast<long long>(n) * p.y_ld + p.y_off + r] = h;
}

constexpr int kBarFull0 = 1;  // named barriers 1, 2: partial slot s is full
constexpr int kBarFree0 = 3;  // named barriers 3, 4: partial slot s is free again
constexpr int kBarCons = 5;   // consumers only (prologue)

__device__ __forceinline__ void bar_sync(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory"); }
__device__ __forceinline__ void bar_arrive(int id, int n) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(n) : "memory");
}
__device__ __forceinline__ void mbar_arrive1(uint64_t* bar) {
  asm volatile("{\n .reg .b64 st;\n mbarrier.arrive.shared::cta.b64 st, [%0];\n}\n" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// One 128-k tile of a 16-row band (rows g, g + 8 of the lane) against batch
// row g (or a zero buffer for lanes past M):
//   y += s_r·(2^-24·Σ q·x − z_r·(2^-24·Σ x))   for columns 2t, 2t + 1.
// xt: this lane's activations of the tile; xsp: Σx (×2^-24) of columns 2t, 2t+1.
__device__ __forceinline__ void tile_fma(const uint8_t* tp, const uint8_t* xt, const float* xsp, int lane, int g,
                                         float (&y)[4]) {
  const uint4 qa = *reinterpret_cast<const uint4*>(tp + lane * 16);
  const uint4 qb = *reinterpret_cast<const uint4*>(tp + 512 + lane * 16);
  uint4 xv[4];
#pragma unroll
  for (int gi = 0; gi < 4; ++gi) xv[gi] = *reinterpret_cast<const uint4*>(xt + 64 * gi);
  const uint16_t* sc = reinterpret_cast<const uint16_t*>(tp + 1024);
  const uint32_t sb0 = sc[g], sb1 = sc[g + 8];
  const uint2 zz = *reinterpret_cast<const uint2*>(tp + 1056);
  const float2 X = *reinterpret_cast<const float2*>(xsp);
  const uint32_t v0[4] = {qa.x, qa.z, qb.x, qb.z}, v1[4] = {qa.y, qa.w, qb.y, qb.w};
  float dl[4] = {0.f, 0.f, 0.f, 0.f}, dh[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int gi = 0; gi < 4; ++gi) {
    const uint32_t a0 = v0[gi], a1 = v1[gi], a08 = a0 >> 8, a18 = a1 >> 8;
    // code pairs (k, k+1), (k+4, k+5) in the low nibbles, (k+2, k+3), (k+6, k+7) in the high
    mma16816(dl, a0 & 0x000F000Fu, a1 & 0x000F000Fu, a08 & 0x000F000Fu, a18 & 0x000F000Fu, xv[gi].x, xv[gi].z);
    mma16816(dh, a0 & 0x00F000F0u, a1 & 0x00F000F0u, a08 & 0x00F000F0u, a18 & 0x00F000F0u, xv[gi].y, xv[gi].w);
  }
  const float s0 = h16_to_f32(sb0), s1 = h16_to_f32(sb1);
  // zero-points as floats: 2^23 + z has z in its low mantissa bits
  const float z0 = __uint_as_float(((zz.x >> (4 * g)) & 15u) | 0x4B000000u) - 8388608.f;
  const float z1 = __uint_as_float(((zz.y >> (4 * g)) & 15u) | 0x4B000000u) - 8388608.f;
  y[0] = fmaf(s0, fmaf(-z0, X.x, fmaf(dh[0], 0.0625f, dl[0])), y[0]);
  y[1] = fmaf(s0, fmaf(-z0, X.y, fmaf(dh[1], 0.0625f, dl[1])), y[1]);
  y[2] = fmaf(s1, fmaf(-z1, X.x, fmaf(dh[2], 0.0625f, dl[2])), y[2]);
  y[3] = fmaf(s1, fmaf(-z1, X.y, fmaf(dh[3], 0.0625f, dl[3])), y[3]);
}

// int4 B200_V1 tile with the zero-point taken out of the MMA operand: a nibble
// masked under the fp16 pattern of 1024 (low nibbles) or 64 (high nibbles) is
// 1024 + q or 64 + q exactly; subtracting 1024 + z or 64 + z (one HSUB2 per
// pair) leaves the exact integer q − z.  The MMA then forms Σ (q − z)·x
// directly: no Σx table, no prologue, one fp32 FMA by the scale per output.
__device__ __forceinline__ uint32_t v1k_lop3_or(uint32_t v, uint32_t mask, uint32_t magic) {
  uint32_t r;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(v), "r"(mask), "r"(magic));  // (v & mask) | magic
  return r;
}
__device__ __forceinline__ uint32_t v1k_hsub2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

__device__ __forceinline__ void tile_fma_zq(const uint8_t* tp, const uint8_t* xt, int lane, int g, float (&y)[4]) {
  const uint4 qa = *reinterpret_cast<const uint4*>(tp + lane * 16);
  const uint4 qb = *reinterpret_cast<const uint4*>(tp + 512 + lane * 16);
  uint4 xv[4];
#pragma unroll
  for (int gi = 0; gi < 4; ++gi) xv[gi] = *reinterpret_cast<const uint4*>(xt + 64 * gi);
  const uint16_t* sc = reinterpret_cast<const uint16_t*>(tp + 1024);
  const uint32_t sb0 = sc[g], sb1 = sc[g + 8];
  const uint2 zz = *reinterpret_cast<const uint2*>(tp + 1056);
  const uint32_t z0 = (zz.x >> (4 * g)) & 15u, z1 = (zz.y >> (4 * g)) & 15u;
  const uint32_t zl0 = (0x6400u | z0) * 0x00010001u, zl1 = (0x6400u | z1) * 0x00010001u;
  const uint32_t zh0 = (0x5400u | (z0 << 4)) * 0x00010001u, zh1 = (0x5400u | (z1 << 4)) * 0x00010001u;
  const uint32_t v0[4] = {qa.x, qa.z, qb.x, qb.z}, v1[4] = {qa.y, qa.w, qb.y, qb.w};
  float da[4] = {0.f, 0.f, 0.f, 0.f}, db[4] = {0.f, 0.f, 0.f, 0.f};  // two chains: even / odd 32-k groups
#pragma unroll
  for (int gi = 0; gi < 4; ++gi) {
    const uint32_t a0 = v0[gi], a1 = v1[gi], a08 = a0 >> 8, a18 = a1 >> 8;
    float(&d)[4] = (gi & 1) ? db : da;
    mma16816(d, v1k_hsub2(v1k_lop3_or(a0, 0x000F000Fu, 0x64006400u), zl0),
                  v1k_hsub2(v1k_lop3_or(a1, 0x000F000Fu, 0x64006400u), zl1),
                  v1k_hsub2(v1k_lop3_or(a08, 0x000F000Fu, 0x64006400u), zl0),
                  v1k_hsub2(v1k_lop3_or(a18, 0x000F000Fu, 0x64006400u), zl1), xv[gi].x, xv[gi].z);
    mma16816(d, v1k_hsub2(v1k_lop3_or(a0, 0x00F000F0u, 0x54005400u), zh0),
                  v1k_hsub2(v1k_lop3_or(a1, 0x00F000F0u, 0x54005400u), zh1),
                  v1k_hsub2(v1k_lop3_or(a08, 0x00F000F0u, 0x54005400u), zh0),
                  v1k_hsub2(v1k_lop3_or(a18, 0x00F000F0u, 0x54005400u), zh1), xv[gi].y, xv[gi].w);
  }
  const float s0 = h16_to_f32(sb0), s1 = h16_to_f32(sb1);
  y[0] = fmaf(s0, da[0] + db[0], y[0]);
  y[1] = fmaf(s0, da[1] + db[1], y[1]);
  y[2] = fmaf(s1, da[2] + db[2], y[2]);
  y[3] = fmaf(s1, da[3] + db[3], y[3]);
}

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ float dsmem_ld(const float* local, uint32_t rank) {
  uint32_t a;
  float v;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(smem_u32(local)), "r"(rank));
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(a) : "memory");
  return v;
}

}  // namespace v1d

constexpr int kV1MaxWarps = 26;  // consumer warps + producer + reducer

// ZQ: tiles through v1d::tile_fma_zq (exact q − z in the MMA operand, no Σx
// table or prologue); otherwise subnormal codes with the per-tile Σx term.
template <bool ZQ = false>
__global__ void __launch_bounds__(kV1MaxWarps * 32, 1) gemv_v1_kernel(const V1Params p) {
  constexpr float kYScale = ZQ ? 1.f : 16777216.f;  // subnormal-code partials are in units of 2^-24
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int W = p.W;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + p.off_bar);
  uint64_t* empty = full + p.NS;
  uint64_t* xbar = empty + p.NS;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(xbar + 1);

  const uint32_t rank = p.C > 1 ? v1d::cluster_rank() : 0u;
  const int cid = blockIdx.x / p.C, n_cl = gridDim.x / p.C;
  const int b_begin = static_cast<int>(static_cast<long long>(cid) * p.n_bands / n_cl);
  const int b_end = static_cast<int>(static_cast<long long>(cid + 1) * p.n_bands / n_cl);
  const int n_bl = b_end - b_begin;
  const int n_tiles = n_bl * p.tpc;                   // this CTA's linear tile sequence
  // stage S covers tiles [stage_first(S), stage_first(S) + stage_tiles(S)) of the sequence
  const int n_stages = n_tiles <= p.tps0 ? 1 : 1 + (n_tiles - p.tps0 + p.tps - 1) / p.tps;
  auto stage_first = [&](int S) { return S == 0 ? 0 : p.tps0 + (S - 1) * p.tps; };
  auto stage_tiles = [&](int S) { return min(S == 0 ? p.tps0 : p.tps, n_tiles - stage_first(S)); };
  const int Kc = p.tpc * 128;                         // this CTA's k extent

  if (tid == 0) {
    for (int i = 0; i < p.NS; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], W);
    }
    mbar_init(xbar, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  // The next kernel in the stream may start its own weight stream now; this
  // one only waits for the previous kernel where it reads x or writes y.
  grid_launch_dependents();

  // ---------------------------------------------------------------- producer
  if (warp == W) {
    if (lane == 0) {
      const uint64_t policy = policy_evict_first();
      const long long band_bytes = static_cast<long long>(p.tpb) * p.tb;
      const uint8_t* base = p.w + static_cast<long long>(b_begin) * band_bytes + static_cast<long long>(rank) * p.tpc * p.tb;
      int slot = 0, bl = 0, ti = 0;  // next tile: band bl (local), k-tile ti (local)
      uint32_t phase = 0;
      const int pre = min(p.pre, n_stages);
      // Before the wait for the previous kernel, the head of this CTA's weight
      // stream is either prefetched into L2 (pf_bytes; L2 is the point of
      // coherence, so a prefetch can never return data older than a write of
      // the previous kernel) or, when the caller has declared that no kernel
      // right before a GEMV writes its weights, copied straight into the ring
      // (`pre` stages).  The activations may be the previous kernel's output;
      // they are copied right after the wait, ahead of the rest of the weight
      // stream (a load queued behind a deep weight stream waits for all of it).
      if (p.pf_bytes > 0) {
        long long left = p.pf_bytes;
        for (int b = 0; b < n_bl && left > 0; ++b) {
          const uint8_t* run = base + b * band_bytes;
          const long long rb = min(left, static_cast<long long>(p.tpc) * p.tb);
          for (long long o = 0; o < rb; o += 32768)
            prefetch_l2(run + o, static_cast<uint32_t>(min(rb - o, 32768ll)));
          left -= rb;
        }
      }
      auto copy_x = [&]() {
        grid_wait_prior();
        mbar_arrive_expect_tx(xbar, static_cast<uint32_t>(p.M) * 2u * Kc);
        for (int m = 0; m < p.M; ++m)
          bulk_g2s(smem + p.off_x + m * 2 * Kc,
                   reinterpret_cast<const uint8_t*>(p.x) + (static_cast<long long>(m) * p.K + rank * Kc) * 2, 2u * Kc,
                   xbar);
      };
      for (int S = 0; S < n_stages; ++S) {
        if (S == pre) copy_x();
        if (S >= p.NS && (*abort_flag || !mbar_wait_bounded(&empty[slot], phase ^ 1u))) {
          *abort_flag = 1;
          break;
        }
        const int nt = stage_tiles(S);
        mbar_arrive_expect_tx(&full[slot], static_cast<uint32_t>(nt) * p.tb);
        uint8_t* dst = smem + slot * p.stage_bytes;
        for (int left = nt; left > 0;) {  // one copy per run of tiles inside one band
          const int run = min(left, p.tpc - ti);
          const uint8_t* src = base + bl * band_bytes + static_cast<long long>(ti) * p.tb;
          if (p.hint)
            bulk_g2s_stream(dst, src, static_cast<uint32_t>(run) * p.tb, &full[slot], policy);
          else
            bulk_g2s(dst, src, static_cast<uint32_t>(run) * p.tb, &full[slot]);
          dst += run * p.tb;
          left -= run;
          ti += run;
          if (ti == p.tpc) {
            ti = 0;
            ++bl;
          }
        }
        // keep more of the stream in flight than the ring holds: move the
        // tiles of stage S + pfd from HBM to L2 now (C = 1: the CTA's tiles
        // are one contiguous range), so their copy into the ring later is an
        // L2 read
        if (p.pfd > 0 && p.C == 1 && S + p.pfd < n_stages) {
          const uint8_t* src = base + static_cast<long long>(stage_first(S + p.pfd)) * p.tb;
          const long long nb = static_cast<long long>(stage_tiles(S + p.pfd)) * p.tb;
          for (long long o = 0; o < nb; o += 32768) prefetch_l2(src + o, static_cast<uint32_t>(min(nb - o, 32768ll)));
        }
        if (++slot == p.NS) {
          slot = 0;
          phase ^= 1u;
        }
      }
      if (pre == n_stages) copy_x();
    }
    return;
  }

  const int nthr_all = (W + 1) * 32;  // consumers + reducer on the partial-slot barriers
  float* red = reinterpret_cast<float*>(smem + p.off_red);
  const int red_slot = W * 16 * p.Mp;
  float* part = reinterpret_cast<float*>(smem + p.off_part);

  // ---------------------------------------------------------------- reducer
  if (warp == W + 1) {
    grid_wait_prior();  // y may still be read or written by the previous kernel
    for (int bl = 0; bl < n_bl; ++bl) {
      const int s = bl & 1;
      v1d::bar_sync(v1d::kBarFull0 + s, nthr_all);
      const float* rs = red + s * red_slot;
      const int r0 = (b_begin + bl) * 16;
      for (int o = lane; o < 16 * p.M; o += 32) {
        const int row = o / p.M, n = o - row * p.M;
        float sum = 0.f;
        for (int w2 = 0; w2 < W; ++w2) sum += rs[(w2 * 16 + row) * p.Mp + n];
        if (p.C > 1) {
          part[(bl * 16 + row) * p.M + n] = sum;
        } else if (r0 + row < p.N && !*abort_flag) {
          v1d::store_y(p, n, r0 + row, sum * kYScale);
        }
      }
      if (bl + 2 < n_bl) v1d::bar_arrive(v1d::kBarFree0 + s, nthr_all);
    }
  } else {
    // -------------------------------------------------------------- consumers
    const int g = lane >> 2, t = lane & 3;
    const int nthr = W * 32;
    float* xs = reinterpret_cast<float*>(smem + p.off_xs);
    uint8_t* xsm = smem + p.off_x;
    uint8_t* zbuf = smem + p.off_zero;  // 256 zero bytes: the activations of lanes past M
    // Σx per (tile, batch column) of this CTA's k-range: sixteen threads per
    // tile and column, each adding 8 consecutive activations (consecutive
    // threads read consecutive 16-byte chunks: no bank conflicts), then four
    // shuffles within the 16
    bool ok = mbar_wait_bounded(xbar, 0u);
    if (!ok) *abort_flag = 1;
    {
      const int items = ZQ ? 0 : p.tpc * p.M * 16;
      for (int b0 = 0; b0 < items; b0 += nthr) {
        const int i = b0 + tid;
        float sum = 0.f;
        const int tm = i >> 4, m = tm % p.M, ti = tm / p.M;
        if (i < items && ok) {
          const uint4 v = *reinterpret_cast<const uint4*>(xsm + (static_cast<long long>(m) * Kc + ti * 128 + (i & 15) * 8) * 2);
          const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&u[e]));
            sum += f.x + f.y;
          }
        }
#pragma unroll
        for (int o = 1; o < 16; o <<= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        if (i < items && (i & 15) == 0) xs[ti * 8 + m] = sum * 5.9604644775390625e-08f;  // ×2^-24, exact
      }
      for (int i = tid; i < p.tpc * 8; i += nthr)
        if ((i & 7) >= p.M) xs[i] = 0.f;
      for (int i = tid; i < 64; i += nthr) reinterpret_cast<uint32_t*>(zbuf)[i] = 0u;
    }
    v1d::bar_sync(v1d::kBarCons, nthr);

    const bool xrow = g < p.M;
    const uint8_t* xbase = xrow ? xsm + static_cast<long long>(g) * Kc * 2 + 16 * t : zbuf + 16 * t;
    const int xstep = xrow ? 256 : 0;
    const float* xsl = xs + 2 * t;
    float yacc[4] = {0.f, 0.f, 0.f, 0.f};
    int cur_bl = 0;  // band the accumulator belongs to
    int bl = 0, ti = warp;  // this warp's next tile (band-local index, k-tile)
    while (ti >= p.tpc) {
      ti -= p.tpc;
      ++bl;
    }
    // hand the partials of band `b` to the reducer
    auto flush = [&](int b) {
      const int s = b & 1;
      if (b >= 2) v1d::bar_sync(v1d::kBarFree0 + s, nthr_all);
      float* rs = red + s * red_slot + warp * 16 * p.Mp;
      if (2 * t < p.M) {
        rs[g * p.Mp + 2 * t] = yacc[0];
        rs[(g + 8) * p.Mp + 2 * t] = yacc[2];
      }
      if (2 * t + 1 < p.M) {
        rs[g * p.Mp + 2 * t + 1] = yacc[1];
        rs[(g + 8) * p.Mp + 2 * t + 1] = yacc[3];
      }
      v1d::bar_arrive(v1d::kBarFull0 + s, nthr_all);
      yacc[0] = yacc[1] = yacc[2] = yacc[3] = 0.f;
    };

    int slot = 0;
    uint32_t phase = 0;
    for (int S = 0; S < n_stages; ++S) {
      if (ok && !*abort_flag) {
        if (!mbar_wait_bounded(&full[slot], phase)) {
          *abort_flag = 1;
          ok = false;
        }
      } else {
        ok = false;
      }
      const int nt = stage_tiles(S);
      const uint8_t* st = smem + slot * p.stage_bytes;
      for (int u = warp; u < nt; u += W) {
        while (cur_bl < bl) {  // this warp's tiles moved on to a later band
          flush(cur_bl);
          ++cur_bl;
        }
        if (ok) {
          if constexpr (ZQ)
            v1d::tile_fma_zq(st + u * p.tb, xbase + ti * xstep, lane, g, yacc);
          else
            v1d::tile_fma(st + u * p.tb, xbase + ti * xstep, xsl + ti * 8, lane, g, yacc);
        }
        ti += W;
        while (ti >= p.tpc) {
          ti -= p.tpc;
          ++bl;
        }
      }
      __syncwarp();
      if (lane == 0) v1d::mbar_arrive1(&empty[slot]);
      if (++slot == p.NS) {
        slot = 0;
        phase ^= 1u;
      }
    }
    while (cur_bl < n_bl) {
      flush(cur_bl);
      ++cur_bl;
    }
  }

  if (p.C > 1) {
    // partials of every band are in `part` of each CTA of the cluster: add them
    // in rank order, the CTAs splitting the outputs between them
    v1d::cluster_sync();
    // The producer warp (warp W) has exited: number the W consumer warps and
    // the reducer warp (W + 1) contiguously so every item has a thread.
    const int nthr_red = (W + 1) * 32;
    const int rt = warp == W + 1 ? W * 32 + lane : tid;
    const int items = n_bl * 16 * p.M;
    for (int i = static_cast<int>(rank) * nthr_red + rt; i < items; i += p.C * nthr_red) {
      const int n = i % p.M, br = i / p.M, row = br & 15, b = br >> 4;
      const int r = (b_begin + b) * 16 + row;
      float sum = 0.f;
      for (int c = 0; c < p.C; ++c) sum += v1d::dsmem_ld(part + i, static_cast<uint32_t>(c));
      if (r < p.N && !*abort_flag)
        v1d::store_y(p, n, r, sum * kYScale);
    }
    v1d::cluster_sync();
  }
}

// ---------------------------------------------------------------------------
// Register-streaming variant: no shared-memory ring.  Each consumer warp loads
// its own tiles (two 16-byte code loads and the tile's scales / zero-points
// per lane, coalesced) straight into registers, P tiles ahead of the one it
// computes; the first P tiles are requested before the wait for the previous
// kernel.  Shared memory holds only the activations, the Σx table and the
// partial-sum slots.
// ---------------------------------------------------------------------------
struct V1RParams {
  const void* x;     // [M][K] fp16
  const uint8_t* w;  // B200_V1 stream
  void* y;           // [M][N] fp16
  int M, N, K;
  int n_bands, tpb, tb, W, Mp;
  int off_x, off_zero, off_xs, off_red;
};

struct TileRegs {
  uint4 qa, qb;
  uint2 zz;
  uint32_t s0, s1;
};

__device__ __forceinline__ void tile_ldg(const uint8_t* tp, int lane, int g, TileRegs& r) {
  r.qa = __ldcs(reinterpret_cast<const uint4*>(tp + lane * 16));
  r.qb = __ldcs(reinterpret_cast<const uint4*>(tp + 512 + lane * 16));
  r.s0 = __ldcs(reinterpret_cast<const unsigned short*>(tp + 1024) + g);
  r.s1 = __ldcs(reinterpret_cast<const unsigned short*>(tp + 1024) + g + 8);
  r.zz = __ldcs(reinterpret_cast<const uint2*>(tp + 1056));
}

__device__ __forceinline__ void tile_fma_regs(const TileRegs& r, const uint8_t* xt, const float* xsp, int g,
                                              float (&y)[4]) {
  uint4 xv[4];
#pragma unroll
  for (int gi = 0; gi < 4; ++gi) xv[gi] = *reinterpret_cast<const uint4*>(xt + 64 * gi);
  const float2 X = *reinterpret_cast<const float2*>(xsp);
  const uint32_t v0[4] = {r.qa.x, r.qa.z, r.qb.x, r.qb.z}, v1[4] = {r.qa.y, r.qa.w, r.qb.y, r.qb.w};
  float dl[4] = {0.f, 0.f, 0.f, 0.f}, dh[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int gi = 0; gi < 4; ++gi) {
    const uint32_t a0 = v0[gi], a1 = v1[gi], a08 = a0 >> 8, a18 = a1 >> 8;
    v1d::mma16816(dl, a0 & 0x000F000Fu, a1 & 0x000F000Fu, a08 & 0x000F000Fu, a18 & 0x000F000Fu, xv[gi].x, xv[gi].z);
    v1d::mma16816(dh, a0 & 0x00F000F0u, a1 & 0x00F000F0u, a08 & 0x00F000F0u, a18 & 0x00F000F0u, xv[gi].y, xv[gi].w);
  }
  const float s0 = h16_to_f32(r.s0), s1 = h16_to_f32(r.s1);
  const float z0 = __uint_as_float(((r.zz.x >> (4 * g)) & 15u) | 0x4B000000u) - 8388608.f;
  const float z1 = __uint_as_float(((r.zz.y >> (4 * g)) & 15u) | 0x4B000000u) - 8388608.f;
  y[0] = fmaf(s0, fmaf(-z0, X.x, fmaf(dh[0], 0.0625f, dl[0])), y[0]);
  y[1] = fmaf(s0, fmaf(-z0, X.y, fmaf(dh[1], 0.0625f, dl[1])), y[1]);
  y[2] = fmaf(s1, fmaf(-z1, X.x, fmaf(dh[2], 0.0625f, dl[2])), y[2]);
  y[3] = fmaf(s1, fmaf(-z1, X.y, fmaf(dh[3], 0.0625f, dl[3])), y[3]);
}

constexpr int kV1RMaxWarps = 17;  // consumer warps + reducer

template <int P>
__global__ void __launch_bounds__(kV1RMaxWarps * 32, 1) gemv_v1r_kernel(const V1RParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int W = p.W;
  const int b_begin = static_cast<int>(static_cast<long long>(blockIdx.x) * p.n_bands / gridDim.x);
  const int b_end = static_cast<int>(static_cast<long long>(blockIdx.x + 1) * p.n_bands / gridDim.x);
  const int n_bl = b_end - b_begin;
  const int n_tiles = n_bl * p.tpb;  // the CTA's tiles are one contiguous range of the stream
  const uint8_t* base = p.w + static_cast<long long>(b_begin) * p.tpb * p.tb;
  grid_launch_dependents();

  const int nthr_all = (W + 1) * 32;
  float* red = reinterpret_cast<float*>(smem + p.off_red);
  const int red_slot = W * 16 * p.Mp;

  if (warp == W) {
    // ---------------------------------------------------------------- reducer
    grid_wait_prior();  // y may still be read or written by the previous kernel
    for (int bl = 0; bl < n_bl; ++bl) {
      const int s = bl & 1;
      v1d::bar_sync(v1d::kBarFull0 + s, nthr_all);
      const float* rs = red + s * red_slot;
      const int r0 = (b_begin + bl) * 16;
      for (int o = lane; o < 16 * p.M; o += 32) {
        const int row = o / p.M, n = o - row * p.M;
        float sum = 0.f;
        for (int w2 = 0; w2 < W; ++w2) sum += rs[(w2 * 16 + row) * p.Mp + n];
        if (r0 + row < p.N)
          reinterpret_cast<__half*>(p.y)[static_cast<long long>(n) * p.N + r0 + row] = __float2half_rn(sum * 16777216.f);
      }
      if (bl + 2 < n_bl) v1d::bar_arrive(v1d::kBarFree0 + s, nthr_all);
    }
    return;
  }

  // ------------------------------------------------------------------ consumers
  const int g = lane >> 2, t = lane & 3;
  const int nthr = W * 32;
  const int cnt = warp < n_tiles ? (n_tiles - warp + W - 1) / W : 0;  // this warp's tiles: warp + W·i
  TileRegs q[P];
  // Before the previous kernel has completed only L2 is warmed (a register
  // load could return weights older than a write of that kernel): lane 0
  // prefetches this warp's first P tiles, the loads follow the wait.
  if (lane == 0)
    for (int j = 0; j < P && j < cnt; ++j) prefetch_l2(base + static_cast<long long>(warp + W * j) * p.tb, p.tb);
  grid_wait_prior();  // x, and possibly the weights, may be the previous kernel's output
#pragma unroll
  for (int j = 0; j < P; ++j)
    if (j < cnt) tile_ldg(base + static_cast<long long>(warp + W * j) * p.tb, lane, g, q[j]);

  float* xs = reinterpret_cast<float*>(smem + p.off_xs);
  uint8_t* xsm = smem + p.off_x;
  uint8_t* zbuf = smem + p.off_zero;
  {
    // x -> shared memory, and Σx (×2^-24) per (tile, batch column): four
    // threads per tile and column, 32 k each
    const int items = p.tpb * p.M * 4;
    const uint8_t* xg = reinterpret_cast<const uint8_t*>(p.x);
    for (int b0 = 0; b0 < items; b0 += nthr) {
      const int i = b0 + tid;
      float sum = 0.f;
      if (i < items) {
        const int qq = i & 3, tm = i >> 2, m = tm % p.M, ti = tm / p.M;
        const long long off = (static_cast<long long>(m) * p.K + ti * 128 + qq * 32) * 2;
        const uint4* src = reinterpret_cast<const uint4*>(xg + off);
        uint4* dst = reinterpret_cast<uint4*>(xsm + off);
        uint4 v[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) v[c] = __ldcg(src + c);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          dst[c] = v[c];
          const uint32_t u[4] = {v[c].x, v[c].y, v[c].z, v[c].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&u[e]));
            sum += f.x + f.y;
          }
        }
      }
      sum += __shfl_xor_sync(0xffffffffu, sum, 1);
      sum += __shfl_xor_sync(0xffffffffu, sum, 2);
      if (i < items && (i & 3) == 0) {
        const int tm = i >> 2, m = tm % p.M, ti = tm / p.M;
        xs[ti * 8 + m] = sum * 5.9604644775390625e-08f;  // ×2^-24, exact
      }
    }
    for (int i = tid; i < p.tpb * 8; i += nthr)
      if ((i & 7) >= p.M) xs[i] = 0.f;
    for (int i = tid; i < 64; i += nthr) reinterpret_cast<uint32_t*>(zbuf)[i] = 0u;
  }
  v1d::bar_sync(v1d::kBarCons, nthr);

  const bool xrow = g < p.M;
  const uint8_t* xbase = xrow ? xsm + static_cast<long long>(g) * p.K * 2 + 16 * t : zbuf + 16 * t;
  const int xstep = xrow ? 256 : 0;
  const float* xsl = xs + 2 * t;
  float yacc[4] = {0.f, 0.f, 0.f, 0.f};
  int cur_bl = 0;
  int bl = 0, ti = warp;  // band and k-tile of this warp's next tile
  while (ti >= p.tpb) {
    ti -= p.tpb;
    ++bl;
  }
  auto flush = [&](int b) {
    const int s = b & 1;
    if (b >= 2) v1d::bar_sync(v1d::kBarFree0 + s, nthr_all);
    float* rs = red + s * red_slot + warp * 16 * p.Mp;
    if (2 * t < p.M) {
      rs[g * p.Mp + 2 * t] = yacc[0];
      rs[(g + 8) * p.Mp + 2 * t] = yacc[2];
    }
    if (2 * t + 1 < p.M) {
      rs[g * p.Mp + 2 * t + 1] = yacc[1];
      rs[(g + 8) * p.Mp + 2 * t + 1] = yacc[3];
    }
    v1d::bar_arrive(v1d::kBarFull0 + s, nthr_all);
    yacc[0] = yacc[1] = yacc[2] = yacc[3] = 0.f;
  };

  for (int i0 = 0; i0 < cnt; i0 += P) {
#pragma unroll
    for (int j = 0; j < P; ++j) {
      const int i = i0 + j;
      if (i < cnt) {
        while (cur_bl < bl) {
          flush(cur_bl);
          ++cur_bl;
        }
        tile_fma_regs(q[j], xbase + ti * xstep, xsl + ti * 8, g, yacc);
        if (i + P < cnt) tile_ldg(base + static_cast<long long>(warp + W * (i + P)) * p.tb, lane, g, q[j]);
        ti += W;
        while (ti >= p.tpb) {
          ti -= p.tpb;
          ++bl;
        }
      }
    }
  }
  while (cur_bl < n_bl) {
    flush(cur_bl);
    ++cur_bl;
  }
}

}  // namespace wq
