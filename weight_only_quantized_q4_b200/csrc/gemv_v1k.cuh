// gemv_v1k.cuh — decode GEMV (M = 1..8, activations resident in shared
// memory) for the B200_V1 band streams of int4 (blocks of at least 128 k) and
// q4_K, with the tile stream split evenly over the CTAs (stream-K).
//
// What it computes is what gemv_v1.cuh computes (onnx-genai PR #1000, "What it
// does": int4 blockwise weights, fp16 scales and uint4 zero-points, fp32
// accumulation, one rounding to fp16), with the same per-tile arithmetic
// (subnormal codes through warp-level MMA, the zero-point through a per-tile
// Σx term).  What changes is the work split and the pipeline:
//
//  * The B200_V1 stream is band-major, so the tiles [t0, t1) of a CTA are one
//    contiguous byte range.  CTA i takes tiles [i·T/G, (i+1)·T/G) of the T
//    tiles: every CTA streams the same number of bytes (±1 tile), instead of
//    whole 16-row bands (256 bands on 148 SMs leave some SMs with twice the
//    work of others).
//  * A band cut by a CTA boundary is finished in a fix-up: each CTA that holds
//    a piece of it stores its fp32 partial sums (16 rows × M) in a workspace
//    slot, fences, and counts itself in the band's counter; the CTA that
//    brings the count to the number of pieces adds the pieces in CTA order
//    (a fixed order: results are bitwise repeatable), writes y and resets the
//    counter to zero for the next call.
//  * Before waiting for the previous kernel only L2 is filled (a prefetch of
//    the head of the CTA's range); x, then the ring of weight stages, are
//    copied after the wait.  The Σx table is built by 16 threads per (tile,
//    batch row), each reading 16 consecutive bytes (no bank conflicts).
#pragma once

#include "gemv_v1.cuh"

namespace wq {

struct V1KParams {
  const void* x;     // [M][K] fp16
  const uint8_t* w;  // B200_V1 stream
  void* y;           // [M][N] fp16
  int M, N, K;
  int n_bands;       // ceil(N / 16)
  int tpb;           // tiles per band (K / 128 int4, K / 256 q4_K)
  long long T;       // tiles in the stream (n_bands · tpb)
  int tb;            // bytes per tile
  int tps;           // tiles per stage
  int NS;            // ring depth
  int stage_bytes;   // tps · tb
  int W;             // consumer warps
  int Mp;            // M rounded up to even
  int pf_bytes;      // bytes prefetched into L2 before the wait
  int* counters;     // [n_bands] pieces counted per split band (zero between calls)
  float* partials;   // [grid][2][kNS][16][8] fp32 partial sums of split bands
  int off_x;         // activations [M][K] fp16
  int off_zero;      // 256 zero bytes
  int off_xs;        // Σx table [k-units][8] fp32 (int4: per tile, ×2^-24; q4_K: per 32-k chunk)
  int off_red;       // [kRedSlots][kNS][W][16][Mp] fp32 warp partials
  int off_bar;       // full[NS], empty[NS], x barrier, abort word
};

// ---------------------------------------------------------------------------
// q4_K B200_V1 tile: 16 rows × one 256-k super-block (eight 32-k chunks with
// their own coefficients d·sc_c and −dmin·m_c, minfer doc 62 "r59 — q4_K
// W_dsc plane", §2.1).
//
// The codes are the subnormal fp16 codes of the int4 tile (q·2^-24 low
// nibbles, 16q·2^-24 high nibbles), so the per-chunk sums Σ q·x come out of
// the warp-level MMA exactly; the chunk coefficients are applied afterwards in
// fp32.  At M < 8 most of the MMA's 8 columns would carry no batch row, so
// the columns carry chunks instead: with MP2 = M rounded up to a power of two,
// column n = MP2·j + m holds batch row m of chunk slot j, and chunk c is
// accumulated in set c % MP2 at slot c / MP2.  A lane supplies the B operand
// of column g (its activations when the MMA's chunk sits in its slot, zeros
// otherwise) and receives columns 2t, 2t+1: the chunks it receives are few
// (2 at MP2 <= 2), so it decodes only their 6-bit scales and mins.
// ---------------------------------------------------------------------------

// 24-bit (scale, min) entry of (pair p, tile row r) from the tile's bytes 2112..
__device__ __forceinline__ uint32_t q4k_v1_entry_smem(const uint8_t* tp, int p, int r) {
  const int off = 2112 + 3 * (16 * p + r);
  const uint32_t* w = reinterpret_cast<const uint32_t*>(tp + (off & ~3));
  return __funnelshift_r(w[0], w[1], 8 * (off & 3)) & 0xFFFFFFu;
}

// xt: activations of this lane's batch row (g % MP2) at the tile's first k,
// + 16·t bytes; xrow: that row exists (< M); zt: 16 zero bytes; xc: Σx of the
// tile's chunks in real units, [8 chunks][8 batch rows].
template <int MP2>
__device__ __forceinline__ void q4k_tile_fma(const uint8_t* tp, const uint8_t* xt, bool xrow, const uint8_t* zt,
                                             const float* xc, int lane, int g, int t, float (&y)[4]) {
  const uint4 q0 = *reinterpret_cast<const uint4*>(tp + lane * 16);
  const uint4 q1 = *reinterpret_cast<const uint4*>(tp + 512 + lane * 16);
  const uint4 q2 = *reinterpret_cast<const uint4*>(tp + 1024 + lane * 16);
  const uint4 q3 = *reinterpret_cast<const uint4*>(tp + 1536 + lane * 16);
  const uint32_t v0[8] = {q0.x, q0.z, q1.x, q1.z, q2.x, q2.z, q3.x, q3.z};  // row g, chunk c
  const uint32_t v1[8] = {q0.y, q0.w, q1.y, q1.w, q2.y, q2.w, q3.y, q3.w};  // row g + 8
  const int jg = g / MP2;  // chunk slot of the B column this lane supplies
  float dl[MP2][4], dh[MP2][4];
#pragma unroll
  for (int S = 0; S < MP2; ++S)
#pragma unroll
    for (int e = 0; e < 4; ++e) dl[S][e] = dh[S][e] = 0.f;
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const uint4 xv = *reinterpret_cast<const uint4*>(xrow && jg == c / MP2 ? xt + 64 * c : zt);
    const uint32_t a0 = v0[c], a1 = v1[c], a08 = a0 >> 8, a18 = a1 >> 8;
    v1d::mma16816(dl[c % MP2], a0 & 0x000F000Fu, a1 & 0x000F000Fu, a08 & 0x000F000Fu, a18 & 0x000F000Fu, xv.x, xv.z);
    v1d::mma16816(dh[c % MP2], a0 & 0x00F000F0u, a1 & 0x00F000F0u, a08 & 0x00F000F0u, a18 & 0x00F000F0u, xv.y, xv.w);
  }
  // At MP2 = 1 the chunk sums come from the activations themselves: lane
  // (g, t) holds 8 of the 32 of chunk g; four lanes add up the chunk, and the
  // lane receiving chunk c reads the sum from lane 4c.
  float xown[2] = {0.f, 0.f};
  if constexpr (MP2 == 1) {
    float ps = 0.f;
    if (xrow) {
      const uint4 xo = *reinterpret_cast<const uint4*>(xt + 64 * g);
      const uint32_t u[4] = {xo.x, xo.y, xo.z, xo.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&u[e]));
        ps += f.x + f.y;
      }
    }
    ps += __shfl_xor_sync(0xffffffffu, ps, 1);
    ps += __shfl_xor_sync(0xffffffffu, ps, 2);
    xown[0] = __shfl_sync(0xffffffffu, ps, 8 * t);      // chunk 2t
    xown[1] = __shfl_sync(0xffffffffu, ps, 8 * t + 4);  // chunk 2t + 1
  }
  // coefficients of the chunks this lane receives, rows g and g + 8
  const uint32_t dd0 = *reinterpret_cast<const uint32_t*>(tp + 2048 + 4 * g);
  const uint32_t dd1 = *reinterpret_cast<const uint32_t*>(tp + 2048 + 4 * (g + 8));
  const float d0 = h16_to_f32(dd0) * 16777216.f, d1 = h16_to_f32(dd1) * 16777216.f;  // ×2^24: codes are q·2^-24
  const float m0 = h16_to_f32(dd0 >> 16), m1 = h16_to_f32(dd1 >> 16);
#pragma unroll
  for (int S = 0; S < MP2; ++S) {
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int n = 2 * t + e;
      const int c = S + MP2 * (n / MP2), m = n % MP2;
      const uint32_t en0 = q4k_v1_entry_smem(tp, c >> 1, g), en1 = q4k_v1_entry_smem(tp, c >> 1, g + 8);
      const int hi = c & 1;
      const float sc0 = static_cast<float>((en0 >> (6 * hi)) & 63u), sc1 = static_cast<float>((en1 >> (6 * hi)) & 63u);
      const float mn0 = static_cast<float>((en0 >> (12 + 6 * hi)) & 63u), mn1 = static_cast<float>((en1 >> (12 + 6 * hi)) & 63u);
      const float X = MP2 == 1 ? xown[e] : xc[c * 8 + m];
      // y += d·sc·Σqx − dmin·m·Σx  (codes ×2^-24 in the MMA, ×2^24 folded into d)
      y[e] = fmaf(d0 * sc0, fmaf(dh[S][e], 0.0625f, dl[S][e]), fmaf(-(m0 * mn0), X, y[e]));
      y[2 + e] = fmaf(d1 * sc1, fmaf(dh[S][2 + e], 0.0625f, dl[S][2 + e]), fmaf(-(m1 * mn1), X, y[2 + e]));
    }
  }
}

// Split-band counters: one atomic with acquire-release semantics both
// publishes this piece's partial sums (written by the warp before a
// __syncwarp) and, for the last piece, makes the other pieces visible.
__device__ __forceinline__ int atom_add_acq_rel(int* p, int v) {
  int old;
  asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

// Band partial slots between the consumer warps and the reducer: a ring of
// kRedSlots, so a slow fix-up of one band does not hold the consumers back.
constexpr int kRedSlots = 4;
constexpr int kBarRedFull = 1;   // named barriers 1..4: slot s holds a band's warp partials
constexpr int kBarRedFree = 5;   // named barriers 5..8: slot s is free again
constexpr int kBarPrologue = 9;  // consumers only

// CTA of tile t when CTA i owns [floor(i·T/G), floor((i+1)·T/G)).
__device__ __forceinline__ int v1k_cta_of(long long t, long long T, int G) {
  return static_cast<int>(((t + 1) * G - 1) / T);
}

constexpr int kV1KMaxWarps = 18;  // consumer warps + producer + reducer

// silu(a)·b in fp32 (the epilogue of the fused gate / up projection)
__device__ __forceinline__ float silu_mul(float a, float b) { return a / (1.f + __expf(-a)) * b; }

// F = Fmt::Int4 (128-k tiles of 1064 + 8 bytes) or Fmt::Q4K (256-k tiles of
// 2304 bytes); MP2 (q4_K only) = M rounded up to a power of two.  DUAL (int4):
// each tile of the stream is a gate tile followed by the up tile of the same
// 16 rows and 128 k (the fused gate-up stream); the CTA keeps both sums and
// writes y = silu(x·Wgᵀ)·(x·Wuᵀ).
template <Fmt F, int MP2, bool DUAL = false, bool ZQ = false>
__global__ void __launch_bounds__(kV1KMaxWarps * 32, 1) gemv_v1k_kernel(const V1KParams p) {
  constexpr bool kQ4K = F == Fmt::Q4K;
  // the Σx table is needed for the q4_K mins (MP2 > 1; at MP2 = 1 the tile forms its
  // chunk sums itself) and for the int4 Σx zero-point term (unless ZQ)
  constexpr bool kSumX = kQ4K ? MP2 > 1 : !ZQ;
  constexpr int kNS = DUAL ? 2 : 1;  // sums kept per output (gate and up for the fused stream)
  constexpr int kUnit = kQ4K ? 32 : 128;             // k per Σx entry (a q4_K chunk, an int4 tile)
  constexpr int kUnitsPerTile = kQ4K ? 8 : 1;
  constexpr float kYScale = !kQ4K && !ZQ ? 16777216.f : 1.f;  // subnormal-code int4 partials are ×2^-24
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int W = p.W, G = gridDim.x, cta = blockIdx.x;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + p.off_bar);
  uint64_t* empty = full + p.NS;
  uint64_t* xbar = empty + p.NS;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(xbar + 1);

  const long long t0 = static_cast<long long>(cta) * p.T / G, t1 = static_cast<long long>(cta + 1) * p.T / G;
  const int n_tiles = static_cast<int>(t1 - t0);
  const int b_first = static_cast<int>(t0 / p.tpb);
  const int b_last = n_tiles > 0 ? static_cast<int>((t1 - 1) / p.tpb) : b_first;
  const int n_bl = n_tiles > 0 ? b_last - b_first + 1 : 0;
  const int n_stages = (n_tiles + p.tps - 1) / p.tps;
  // Work order: the piece of the last band first (tiles max(t0, b_last·tpb)
  // .. t1), then the piece of the first band (t0 .. its end), then the whole
  // bands in between.  The pieces this CTA shares with its neighbours are
  // finished first, so their fix-ups overlap the rest of the work instead of
  // ending it.  Virtual tile v of the order maps to stream tile phys(v); band
  // position 0 is b_last, 1 is b_first, 2.. are b_first + 1 ...
  const long long tail0 = max(t0, static_cast<long long>(b_last) * p.tpb);
  const long long mid0 = static_cast<long long>(b_first + 1) * p.tpb;
  const int len_tail = static_cast<int>(t1 - tail0);
  const int len_head = b_last > b_first ? static_cast<int>(mid0 - t0) : 0;
  const int run_end[3] = {len_tail, len_tail + len_head, n_tiles};
  const long long run_start[3] = {tail0, t0, mid0};
  auto band_at = [&](int pos) { return pos == 0 ? b_last : pos == 1 ? b_first : b_first + pos - 1; };

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
  grid_launch_dependents();
  if (n_tiles == 0) return;

  // ---------------------------------------------------------------- producer
  if (warp == W) {
    if (lane == 0) {
      const uint64_t policy = policy_evict_first();
      {
        long long left = p.pf_bytes;  // the head of the work order, run by run
        for (int r = 0, vs = 0; r < 3 && left > 0; vs = run_end[r], ++r) {
          const long long bytes = min(left, static_cast<long long>(run_end[r] - vs) * p.tb);
          const uint8_t* src = p.w + run_start[r] * p.tb;
          for (long long o = 0; o < bytes; o += 32768)
            prefetch_l2(src + o, static_cast<uint32_t>(min(bytes - o, 32768ll)));
          left -= bytes;
        }
      }
      grid_wait_prior();  // x and the weights may be the previous kernel's output
      mbar_arrive_expect_tx(xbar, static_cast<uint32_t>(p.M) * 2u * p.K);
      for (int m = 0; m < p.M; ++m)
        bulk_g2s(smem + p.off_x + m * 2 * p.K, reinterpret_cast<const uint8_t*>(p.x) + static_cast<long long>(m) * p.K * 2,
                 2u * p.K, xbar);
      int slot = 0;
      uint32_t phase = 0;
      for (int S = 0; S < n_stages; ++S) {
        if (S >= p.NS && (*abort_flag || !mbar_wait_bounded(&empty[slot], phase ^ 1u))) {
          *abort_flag = 1;
          break;
        }
        const int v0 = S * p.tps, v1 = min(v0 + p.tps, n_tiles);
        mbar_arrive_expect_tx(&full[slot], static_cast<uint32_t>(v1 - v0) * p.tb);
        for (int r = 0, vs = 0; r < 3; vs = run_end[r], ++r) {  // one copy per run the stage overlaps
          const int a = max(v0, vs), b = min(v1, run_end[r]);
          if (a < b)
            bulk_g2s_stream(smem + slot * p.stage_bytes + (a - v0) * p.tb, p.w + (run_start[r] + (a - vs)) * p.tb,
                            static_cast<uint32_t>(b - a) * p.tb, &full[slot], policy);
        }
        if (++slot == p.NS) {
          slot = 0;
          phase ^= 1u;
        }
      }
    }
    return;
  }

  const int nthr_all = (W + 1) * 32;
  float* red = reinterpret_cast<float*>(smem + p.off_red);
  const int red_slot = kNS * W * 16 * p.Mp;  // [kNS][W][16][Mp] per slot

  // ---------------------------------------------------------------- reducer
  if (warp == W + 1) {
    grid_wait_prior();  // y, the counters and the partials may be in use by the previous kernel
    __half* y = reinterpret_cast<__half*>(p.y);
    for (int bl = 0; bl < n_bl; ++bl) {
      const int s = bl % kRedSlots;
      v1d::bar_sync(kBarRedFull + s, nthr_all);
      const float* rs = red + s * red_slot;
      const int b = band_at(bl);
      const long long bt0 = static_cast<long long>(b) * p.tpb, bt1 = bt0 + p.tpb;
      const bool whole = bt0 >= t0 && bt1 <= t1;
      const int r0 = b * 16;
      const int slot_here = b == b_first ? 0 : 1;
      float* mine = p.partials + (static_cast<long long>(cta) * 2 + slot_here) * 128 * kNS;
      for (int o = lane; o < 16 * p.M; o += 32) {
        const int row = o / p.M, n = o - row * p.M;
        float sum[kNS];
#pragma unroll
        for (int h = 0; h < kNS; ++h) {
          sum[h] = 0.f;
          for (int w2 = 0; w2 < W; ++w2) sum[h] += rs[((h * W + w2) * 16 + row) * p.Mp + n];
        }
        if (whole) {
          const float v = DUAL ? silu_mul(sum[0] * kYScale, sum[kNS - 1] * kYScale) : sum[0] * kYScale;
          if (r0 + row < p.N && !*abort_flag) y[static_cast<long long>(n) * p.N + r0 + row] = __float2half_rn(v);
        } else {
#pragma unroll
          for (int h = 0; h < kNS; ++h) mine[h * 128 + row * 8 + n] = sum[h];
        }
      }
      if (!whole) {
        // fix-up of a band cut by CTA boundaries: count this piece; the last
        // piece adds all pieces in CTA order and writes y
        __syncwarp();
        int seen = 0;
        if (lane == 0) seen = atom_add_acq_rel(&p.counters[b], 1);
        seen = __shfl_sync(0xffffffffu, seen, 0);
        const int c0 = v1k_cta_of(bt0, p.T, G), c1 = v1k_cta_of(bt1 - 1, p.T, G);
        if (seen == c1 - c0) {
          for (int o = lane; o < 16 * p.M; o += 32) {
            const int row = o / p.M, n = o - row * p.M;
            float sum[kNS];
#pragma unroll
            for (int h = 0; h < kNS; ++h) sum[h] = 0.f;
            for (int c = c0; c <= c1; ++c) {
              // the band is the first band of every piece holder but c0 (unless it is c0's first too)
              const long long ct0 = static_cast<long long>(c) * p.T / G;
              const int sl = (ct0 / p.tpb == b) ? 0 : 1;
              const float* src = p.partials + (static_cast<long long>(c) * 2 + sl) * 128 * kNS + row * 8 + n;
#pragma unroll
              for (int h = 0; h < kNS; ++h) sum[h] += __ldcg(src + h * 128);
            }
            const float v = DUAL ? silu_mul(sum[0] * kYScale, sum[kNS - 1] * kYScale) : sum[0] * kYScale;
            if (r0 + row < p.N && !*abort_flag) y[static_cast<long long>(n) * p.N + r0 + row] = __float2half_rn(v);
          }
          __syncwarp();
          if (lane == 0) p.counters[b] = 0;
        }
      }
      if (bl + kRedSlots < n_bl) v1d::bar_arrive(kBarRedFree + s, nthr_all);
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int g = lane >> 2, t = lane & 3;
  const int nthr = W * 32;
  float* xs = reinterpret_cast<float*>(smem + p.off_xs);
  uint8_t* xsm = smem + p.off_x;
  uint8_t* zbuf = smem + p.off_zero;
  bool ok = mbar_wait_bounded(xbar, 0u);
  if (!ok) *abort_flag = 1;
  {
    // Σx per (k-unit, batch row): kUnit / 8 threads per unit, each summing 8
    // consecutive activations (16 bytes, consecutive threads on consecutive
    // addresses), then a shuffle reduction over those threads.  int4 keeps
    // the sums in units of 2^-24 (the scale of its MMA results), q4_K in real
    // units.
    constexpr int kTpu = kUnit / 8;
    const int n_units = p.tpb * kUnitsPerTile;
    const int items = kSumX ? n_units * p.M * kTpu : 0;
    const int rounds = (items + nthr - 1) / nthr;
    for (int r = 0; r < rounds; ++r) {
      const int i = r * nthr + tid;
      const int j = i % kTpu, um = i / kTpu;
      const int un = um / p.M, m = um - un * p.M;
      float sum = 0.f;
      if (i < items && ok) {
        const uint4 v =
            *reinterpret_cast<const uint4*>(xsm + (static_cast<long long>(m) * p.K + un * kUnit + 8 * j) * 2);
        const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&u[e]));
          sum += f.x + f.y;
        }
      }
#pragma unroll
      for (int off = kTpu / 2; off >= 1; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
      if (i < items && j == 0) xs[un * 8 + m] = kQ4K ? sum : sum * 5.9604644775390625e-08f;  // ×2^-24, exact
    }
    for (int i = tid; i < n_units * 8; i += nthr)
      if ((i & 7) >= p.M) xs[i] = 0.f;
    for (int i = tid; i < 64; i += nthr) reinterpret_cast<uint32_t*>(zbuf)[i] = 0u;
  }
  v1d::bar_sync(kBarPrologue, nthr);

  // int4: the lane's B column is batch row g; q4_K: batch row g % MP2 (see q4k_tile_fma)
  const int mrow = kQ4K ? g % (MP2 > 0 ? MP2 : 1) : g;
  const bool xrow = mrow < p.M;
  const uint8_t* xbase = xrow ? xsm + static_cast<long long>(mrow) * p.K * 2 + 16 * t : zbuf + 16 * t;
  const int xstep = xrow ? (kQ4K ? 512 : 256) : 0;
  const float* xsl = xs + 2 * t;
  float yacc[4] = {0.f, 0.f, 0.f, 0.f};
  float yacc2[4] = {0.f, 0.f, 0.f, 0.f};  // up projection (DUAL)
  int cur_bl = 0;
  // band position and k-tile of virtual tile v
  auto locate = [&](int v, int& pos, int& k) {
    if (v < run_end[0]) {
      pos = 0;
      k = static_cast<int>(tail0 - static_cast<long long>(b_last) * p.tpb) + v;
    } else if (v < run_end[1]) {
      pos = 1;
      k = static_cast<int>(t0 - static_cast<long long>(b_first) * p.tpb) + (v - run_end[0]);
    } else {
      const int off = v - run_end[1];
      pos = 2 + off / p.tpb;
      k = off % p.tpb;
    }
  };
  auto run_of = [&](int v) { return v < run_end[0] ? 0 : v < run_end[1] ? 1 : 2; };
  int vw = warp;  // this warp's next virtual tile
  int bl = 0, ti = 0;
  locate(vw, bl, ti);
  auto flush = [&](int b) {
    const int s = b % kRedSlots;
    if (b >= kRedSlots) v1d::bar_sync(kBarRedFree + s, nthr_all);
    float* rs = red + s * red_slot + warp * 16 * p.Mp;
    if constexpr (kQ4K && MP2 < 8) {
      // columns 2t, 2t+1 of a lane hold batch rows (2t + e) % MP2 of different
      // chunks: add the lanes (and, at MP2 = 1, the two columns) that share a batch row
      if constexpr (MP2 == 1) {
        yacc[0] += yacc[1];
        yacc[2] += yacc[3];
        yacc[1] = yacc[3] = 0.f;
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if constexpr (MP2 <= 2) yacc[e] += __shfl_xor_sync(0xffffffffu, yacc[e], 1);
        yacc[e] += __shfl_xor_sync(0xffffffffu, yacc[e], 2);
      }
      const int writers = MP2 <= 2 ? 1 : 2;  // lanes t < writers hold distinct batch rows
      if (t < writers) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int m = (2 * t + e) % MP2;
          if (m < p.M && (MP2 > 1 || e == 0)) {
            rs[g * p.Mp + m] = yacc[e];
            rs[(g + 8) * p.Mp + m] = yacc[2 + e];
          }
        }
      }
    } else {
      auto put = [&](float* rh, float v0, float v1, float v2, float v3) {
        if (2 * t < p.M) {
          rh[g * p.Mp + 2 * t] = v0;
          rh[(g + 8) * p.Mp + 2 * t] = v2;
        }
        if (2 * t + 1 < p.M) {
          rh[g * p.Mp + 2 * t + 1] = v1;
          rh[(g + 8) * p.Mp + 2 * t + 1] = v3;
        }
      };
      put(rs, yacc[0], yacc[1], yacc[2], yacc[3]);
      if constexpr (DUAL) put(rs + W * 16 * p.Mp, yacc2[0], yacc2[1], yacc2[2], yacc2[3]);
    }
    v1d::bar_arrive(kBarRedFull + s, nthr_all);
    yacc[0] = yacc[1] = yacc[2] = yacc[3] = 0.f;
    yacc2[0] = yacc2[1] = yacc2[2] = yacc2[3] = 0.f;
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
    const int nt = min(p.tps, n_tiles - S * p.tps);
    const uint8_t* st = smem + slot * p.stage_bytes;
    for (int u = warp; u < nt; u += W) {
      while (cur_bl < bl) {
        flush(cur_bl);
        ++cur_bl;
      }
      if (ok) {
        if constexpr (kQ4K)
          q4k_tile_fma<MP2>(st + u * p.tb, xbase + ti * xstep, xrow, zbuf, xs + ti * 64, lane, g, t, yacc);
        else if constexpr (ZQ) {
          v1d::tile_fma_zq(st + u * p.tb, xbase + ti * xstep, lane, g, yacc);
          if constexpr (DUAL) v1d::tile_fma_zq(st + u * p.tb + p.tb / 2, xbase + ti * xstep, lane, g, yacc2);
        } else if constexpr (DUAL) {
          v1d::tile_fma(st + u * p.tb, xbase + ti * xstep, xsl + ti * 8, lane, g, yacc);
          v1d::tile_fma(st + u * p.tb + p.tb / 2, xbase + ti * xstep, xsl + ti * 8, lane, g, yacc2);
        } else
          v1d::tile_fma(st + u * p.tb, xbase + ti * xstep, xsl + ti * 8, lane, g, yacc);
      }
      const int vn = vw + W;
      if (vn < n_tiles && run_of(vn) != run_of(vw)) {
        locate(vn, bl, ti);
      } else {
        ti += W;
        while (ti >= p.tpb) {
          ti -= p.tpb;
          ++bl;
        }
      }
      vw = vn;
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

}  // namespace wq
