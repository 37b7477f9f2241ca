// gemm_v1tc.cuh — batched dequant-then-MMA on the tcgen05 tensor cores for
// int4 weights in the B200_V1 band stream (quantization blocks of at least
// 128 k, so every 16 × 128 tile carries one scale and one zero-point per row).
//
// y[m, n] = Σ_k W[n, k]·x[m, k] with W = (q - z)·s (onnx-genai PR #1000,
// "What it does": int4 blockwise weights, fp16 scales, uint4 zero-points),
// accumulated in fp32, one rounding to fp16.
//
// Layout of the work.  A CTA owns 128 weight rows (eight 16-row bands of the
// stream: the UMMA M side), BN batch rows (the UMMA N side) and one slice of
// K; the S CTAs of a cluster share the rows, split K and add their fp32
// accumulators through distributed shared memory in rank order.  The CTA's
// stream is consumed one 128-k step at a time (eight tiles, one per band):
//   * weight producer warp: one bulk copy per band and raw slot of T steps
//     (the tiles of a band are contiguous in the stream, so no tensor map is
//     needed for the weights);
//   * activation producer warp: two TMA copies of the BN × 128 activation
//     slice per step, 128-byte swizzled into the UMMA K-major layout (no
//     multicast).  A bulk copy can hold its issuing thread for about a
//     microsecond when many bytes are in flight, so the two streams do not
//     share a thread;
//   * sixteen dequant warps turn the tiles into fp16 A rows: (q - z) exactly
//     through magic-number codes, times s in one fp16 rounding (as the 64-k
//     kernel does);
//   * two MMA warps (even / odd steps): eight tcgen05.mma (K = 16) per step,
//     each warp into its own fp32 TMEM accumulators, alternating between two
//     per step where the columns allow.
// Rows whose weights could pass the fp16 range (15·max|s| > 65504 over the
// row's blocks) are formed as w·2^-e and their result multiplied by 2^e, as
// in the 64-k kernel.  Every mbarrier wait is bounded (wq_device.cuh).
//
// A in tensor memory (TA, the default).  The dequant warps store the fp16 A
// rows into TMEM (tcgen05.st, one row per TMEM lane) and the MMAs read A from
// there, so shared memory carries only the raw tiles and the activations.  A
// warp may only reach its own quarter of the TMEM lanes, so a thread holds one
// row and one 64-k half of a step: TMEM lane L carries tile row v1ta_row(L),
// chosen so that the 32 rows of a quarter come from four bands and four row
// indices g, and the 16-byte code chunks a warp reads at once fall into eight
// different bank groups (band stride in the raw slot an odd number of 16-byte
// units).  The epilogue maps the accumulator rows back.  One commit per step
// frees both the step's A slot and its activation slot (the activation ring is
// as deep as the A ring).
//
// A in shared memory (WQ_V1TC_TA=0).  Warp w turns the tile of band w mod 8 of
// every step of parity w / 8 into a 128-byte-swizzled fp16 A tile.  The
// tile's codes are in warp-MMA fragment order, so a lane holds 8 consecutive k
// of two rows per 32-bit word and writes them as one 16-byte chunk; lanes with
// odd row index take the two words of a pair in the opposite order, so the
// eight lanes of a quarter-warp always write eight different bank groups.
// Each weight then crosses shared memory twice as fp16 (about 89 KB of
// shared-memory traffic per 8.6 KB of weights per step), and the activation
// ring has a commit of its own.
#pragma once

#include "gemm_tc5.cuh"

namespace wq {

struct V1TCParams {
  CUtensorMap tmap_x;  // activations [M][K] fp16, box BN rows × 64, 128-byte swizzle
  const uint8_t* w;    // B200_V1 int4 stream
  void* y;             // [M, N] fp16
  int M, N, K;
  int n_bands;         // ceil(N / 16)
  int tpb;             // tiles (128-k steps) per band
  int tb;              // bytes per tile
  int BN;              // batch tile (UMMA N), multiple of 16, <= 128
  int tmem_cols;       // power of two >= max(32, 2·BN)
  int S;               // CTAs of a cluster (K slices)
  int nks;             // steps per CTA (tpb / S, even)
  int NA, NR, NX;      // A slots (32 KB), raw slots (8 bands × T tiles), activation slots (BN × 256 B)
  int NACC;            // accumulators per step parity (1 or 2: the MMAs of a step alternate between them)
  int T;               // 128-k steps per raw slot: one copy of T consecutive tiles per band
  int band_stride;     // bytes between the bands of a raw slot (T·tb, + 16 when that is an even number of 16 B units)
  int off_a;           // shared-memory A slots (shared-memory A form)
  int off_x, off_raw, off_rowe, off_bar;  // shared-memory offsets
};

constexpr int kV1TCWarps = 20;  // 16 dequant / epilogue warps, weight producer, activation producer, two MMA issuers
constexpr int kV1TCA = 32768;   // bytes of one A slot: 128 rows × 128 k fp16 (two 64-k atoms)
constexpr int kV1TANA = 4;      // TMEM A slots (A in tensor memory): 64 columns each, after 256 accumulator columns
constexpr int kV1TAColA = 256;  // first TMEM column of the A slots

// Tile row (16·band + 8·half + g) held in TMEM lane L when A lives in tensor
// memory: quarter Q = L / 32 takes bands 4·(Q / 2) .. + 3 and row indices
// g = 4·(Q mod 2) .. + 3 of both halves.
__host__ __device__ __forceinline__ int v1ta_row(int L) {
  const int Q = L >> 5, i = L & 31;
  const int band = 4 * (Q >> 1) + (i >> 3), g = 4 * (Q & 1) + ((i >> 1) & 3), half = i & 1;
  return 16 * band + 8 * half + g;
}

// One row's half of a B200_V1 tile (k = 64·gp .. + 63) as 32 fp16 pairs in k
// order, RN16((q − z)·s): the row's code words sit in the 16-byte chunks of
// lanes 4g + t (t = 0..3) of the fragment order, word 2·gl + half of chunk t
// holding k = 64·gp + 32·gl + 8·t .. + 7.
__device__ __forceinline__ void v1ta_row_half(const uint8_t* tp, int gp, int g, int half, uint32_t zl, uint32_t zh,
                                              uint32_t s2, uint32_t (&o)[32]) {
  const uint8_t* cp = tp + gp * 512 + g * 64;
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    const uint4 c = *reinterpret_cast<const uint4*>(cp + 16 * t);
#pragma unroll
    for (int gl = 0; gl < 2; ++gl) {
      const uint32_t a = gl == 0 ? (half ? c.y : c.x) : (half ? c.w : c.z), a8 = a >> 8;
      uint32_t* q = o + 16 * gl + 4 * t;
      q[0] = hmul2_f(hsub2_f(lop3_or(a, 0x000F000Fu, 0x64006400u), zl), s2);
      q[1] = hmul2_f(hsub2_f(lop3_or(a, 0x00F000F0u, 0x54005400u), zh), s2);
      q[2] = hmul2_f(hsub2_f(lop3_or(a8, 0x000F000Fu, 0x64006400u), zl), s2);
      q[3] = hmul2_f(hsub2_f(lop3_or(a8, 0x00F000F0u, 0x54005400u), zh), s2);
    }
  }
}

// One int4 B200_V1 tile (16 rows × 128 k) at tp into rows 16·band.. of the A
// slot at ab (two 128-byte-swizzled 64-k atoms).  s2: the two rows' scales as
// fp16 pairs (already multiplied by 2^-e where needed).
__device__ __forceinline__ void v1tc_tile_to_a(const uint8_t* tp, uint8_t* ab, int band, int lane, uint32_t s2g,
                                               uint32_t s2g8) {
  const int g = lane >> 2, t = lane & 3, odd = g & 1;
  // word pairs (row g, row g + 8) of gi = 0..3, gi ^ odd at position j
  const uint2 w0 = *reinterpret_cast<const uint2*>(tp + lane * 16 + 8 * odd);
  const uint2 w1 = *reinterpret_cast<const uint2*>(tp + lane * 16 + 8 * (1 - odd));
  const uint2 w2 = *reinterpret_cast<const uint2*>(tp + 512 + lane * 16 + 8 * odd);
  const uint2 w3 = *reinterpret_cast<const uint2*>(tp + 512 + lane * 16 + 8 * (1 - odd));
  const uint2 zz = *reinterpret_cast<const uint2*>(tp + 1056);
  const uint32_t z0 = (zz.x >> (4 * g)) & 15u, z1 = (zz.y >> (4 * g)) & 15u;
  const uint32_t zl0 = (0x6400u | z0) * 0x00010001u, zl1 = (0x6400u | z1) * 0x00010001u;
  const uint32_t zh0 = (0x5400u | (z0 << 4)) * 0x00010001u, zh1 = (0x5400u | (z1 << 4)) * 0x00010001u;
  const uint32_t wg[4] = {w0.x, w1.x, w2.x, w3.x}, wg8[4] = {w0.y, w1.y, w2.y, w3.y};
  const int r0 = 16 * band + g, r1 = r0 + 8;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int gi = j ^ odd;             // the word's 32-k group: k = 32·gi + 8·t .. + 7
    const int c = 4 * (gi & 1) + t;     // its 16-byte chunk inside the 64-k atom
    uint8_t* atom = ab + (j >> 1) * 16384;  // gi >> 1 == j >> 1
    {
      const uint32_t a = wg[j], a8 = a >> 8;
      const uint4 o = make_uint4(hmul2_f(hsub2_f(lop3_or(a, 0x000F000Fu, 0x64006400u), zl0), s2g),
                                 hmul2_f(hsub2_f(lop3_or(a, 0x00F000F0u, 0x54005400u), zh0), s2g),
                                 hmul2_f(hsub2_f(lop3_or(a8, 0x000F000Fu, 0x64006400u), zl0), s2g),
                                 hmul2_f(hsub2_f(lop3_or(a8, 0x00F000F0u, 0x54005400u), zh0), s2g));
      *reinterpret_cast<uint4*>(atom + sw128(r0, c)) = o;
    }
    {
      const uint32_t a = wg8[j], a8 = a >> 8;
      const uint4 o = make_uint4(hmul2_f(hsub2_f(lop3_or(a, 0x000F000Fu, 0x64006400u), zl1), s2g8),
                                 hmul2_f(hsub2_f(lop3_or(a, 0x00F000F0u, 0x54005400u), zh1), s2g8),
                                 hmul2_f(hsub2_f(lop3_or(a8, 0x000F000Fu, 0x64006400u), zl1), s2g8),
                                 hmul2_f(hsub2_f(lop3_or(a8, 0x00F000F0u, 0x54005400u), zh1), s2g8));
      *reinterpret_cast<uint4*>(atom + sw128(r1, c)) = o;
    }
  }
}

// 2^-e for the fp16 range of a row whose largest |scale| has bits smax (0x7FFF-masked, finite)
__device__ __forceinline__ int v1tc_row_exponent(uint32_t smax) {
  float bound = 15.f * h16_to_f32(smax);
  int e = 0;
  while (bound > 65504.f) {
    bound *= 0.5f;
    ++e;
  }
  return e;
}

template <bool TA>
__global__ void __launch_bounds__(kV1TCWarps * 32, 1) gemm_v1tc_kernel(const __grid_constant__ V1TCParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* raw_full = reinterpret_cast<uint64_t*>(smem + p.off_bar);
  uint64_t* raw_empty = raw_full + p.NR;
  uint64_t* x_full = raw_empty + p.NR;
  uint64_t* x_empty = x_full + p.NX;
  uint64_t* a_full = x_empty + p.NX;
  uint64_t* a_empty = a_full + p.NA;
  uint64_t* done = a_empty + p.NA;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* rowe = reinterpret_cast<int*>(smem + p.off_rowe);  // [128] exponent e of each tile row

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = p.S > 1 ? tc5_cluster_rank() : 0u;
  const int tile = blockIdx.x / p.S;
  const int n0 = tile * 128, b0 = tile * 8;
  const int nbt = min(8, p.n_bands - b0);  // bands present in this row tile
  const int m0 = blockIdx.y * p.BN;
  const int s_begin = static_cast<int>(rank) * p.nks;  // first 128-k step of this CTA
  const int nks = p.nks;
  const int x_slot = p.BN * 256;                        // two 64-k atoms of BN rows

  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(p.tmem_cols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (tid == 32) {
    for (int i = 0; i < p.NR; ++i) {
      mbar_init(&raw_full[i], 1);
      mbar_init(&raw_empty[i], 16);  // every dequant warp, once per slot
    }
    for (int i = 0; i < p.NX; ++i) {
      mbar_init(&x_full[i], 1);
      mbar_init(&x_empty[i], 1);  // tcgen05.commit
    }
    for (int i = 0; i < p.NA; ++i) {
      mbar_init(&a_full[i], 8);
      mbar_init(&a_empty[i], 1);
    }
    mbar_init(done, 2);  // one commit per MMA warp
    *abort_flag = 0;
    fence_barrier_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 16) {
    // ------------------------------------------------------------ weight producer
    // raw slot r (steps [r·T, r·T + T)): one bulk copy per band of its tiles,
    // which are contiguous in the band's stream.  A bulk copy can hold its
    // issuing thread for a while when many bytes are in flight, so the
    // activation copies have a warp of their own.
    if (lane == 0) {
      const long long band_bytes = static_cast<long long>(p.tpb) * p.tb;
      const int nslots = (nks + p.T - 1) / p.T;
      for (int r = 0; r < nslots && !*abort_flag; ++r) {
        const int rs = r % p.NR, ru = r / p.NR;
        if (ru > 0 && !mbar_wait_bounded(&raw_empty[rs], static_cast<uint32_t>((ru - 1) & 1))) {
          *abort_flag = 1;
          break;
        }
        const int nt = min(p.T, nks - r * p.T);
        mbar_arrive_expect_tx(&raw_full[rs], static_cast<uint32_t>(nbt * nt * p.tb));
        uint8_t* dst = smem + p.off_raw + rs * 8 * p.band_stride;
        for (int i = 0; i < nbt; ++i)
          bulk_g2s(dst + i * p.band_stride, p.w + (b0 + i) * band_bytes + static_cast<long long>(s_begin + r * p.T) * p.tb,
                   static_cast<uint32_t>(nt * p.tb), &raw_full[rs]);
      }
    }
  } else if (warp == 17) {
    // ------------------------------------------------------------ activation producer
    if (lane == 0) {
      for (int ls = 0; ls < nks && !*abort_flag; ++ls) {
        const int gs = s_begin + ls;
        const int xs = ls % p.NX, xu = ls / p.NX;
        // A in TMEM: the activation ring is as deep as the A ring (NX == NA), and
        // slot xs is free once the MMAs of step ls - NA have completed, which the
        // A slot's barrier already tracks (one commit per step instead of two)
        uint64_t* xfree = TA ? a_empty : x_empty;
        if (xu > 0 && !mbar_wait_bounded(&xfree[xs], static_cast<uint32_t>((xu - 1) & 1))) {
          *abort_flag = 1;
          break;
        }
        mbar_arrive_expect_tx(&x_full[xs], static_cast<uint32_t>(x_slot));
        uint8_t* xd = smem + p.off_x + xs * x_slot;
        tma_load_2d(xd, &p.tmap_x, gs * 128, m0, &x_full[xs]);
        tma_load_2d(xd + x_slot / 2, &p.tmap_x, gs * 128 + 64, m0, &x_full[xs]);
      }
    }
  } else if (warp >= 18) {
    // ------------------------------------------------------------ MMA issuers
    // Warp 18 takes the even steps, warp 19 the odd ones, each into its own
    // accumulators: on B200 one issuing thread is held about 100 cycles per
    // tcgen05.mma at these N (16 to 128), and a second issuing thread nearly
    // doubles the rate the tensor core receives them (107 -> 55-66 cycles per
    // MMA in a microbenchmark).  With NACC = 2 the MMAs of a step also
    // alternate between two accumulators (no measurable effect on B200).
    if (lane == 0) {
      const uint32_t idesc = umma_idesc_f16(p.BN);
      const int par = warp - 18;
      for (int ls = par; ls < nks && !*abort_flag; ls += 2) {
        const int a = ls % p.NA, au = ls / p.NA, xs = ls % p.NX, xu = ls / p.NX;
        if (!mbar_wait_bounded(&a_full[a], static_cast<uint32_t>(au & 1)) ||
            !mbar_wait_bounded(&x_full[xs], static_cast<uint32_t>(xu & 1))) {
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint32_t dacc = tmem + static_cast<uint32_t>((ls & 1) * p.NACC * p.BN);
        const uint32_t dsub = p.NACC > 1 ? static_cast<uint32_t>(p.BN) : 0u;  // second accumulator of the parity
#pragma unroll
        for (int h = 0; h < 2; ++h) {  // the two 64-k atoms of the step
          const uint64_t bd = umma_smem_desc_sw128(smem_u32(smem + p.off_x + xs * x_slot + h * (x_slot / 2)));
#pragma unroll
          for (int j = 0; j < 4; ++j) {  // K = 16 per MMA
            const int q = 4 * h + j;
            const uint32_t d = dacc + ((q & 1) ? dsub : 0u);
            // the first MMA into each accumulator (steps 0 and 1) overwrites it
            const uint32_t accum = (ls > 1 || q >= p.NACC) ? 1u : 0u;
            if constexpr (TA) {
              // A slot a: 64 TMEM columns, 16 k (8 columns) per MMA
              umma_f16_ta(d, tmem + static_cast<uint32_t>(kV1TAColA + 64 * a + 8 * q), bd + 2ull * j, idesc, accum);
            } else {
              // advance 32 bytes inside the swizzle atom per MMA
              const uint64_t ad = umma_smem_desc_sw128(smem_u32(smem + p.off_a + a * kV1TCA + h * 16384));
              umma_f16(d, ad + 2ull * j, bd + 2ull * j, idesc, accum);
            }
          }
        }
        umma_commit(&a_empty[a]);
        if constexpr (!TA) umma_commit(&x_empty[xs]);
      }
      umma_commit(done);  // arrives when every MMA this thread issued has completed
    }
  } else {
    // ------------------------------------------------------------ dequant warps
    const int band = warp & 7, par = warp >> 3;
    const int g = lane >> 2, t = lane & 3;
    const bool have = band < nbt;
    // fp16 range of every row: the largest finite |scale| over every tile of
    // the band (all of K, so that the CTAs of a cluster agree).  The two warps
    // of a band split its tiles; each lane loads the 32 scale bytes of its
    // tiles with two 16-byte loads, all issued before any is used; the warps
    // reduce per row and meet in shared memory.
    uint32_t* rmax = reinterpret_cast<uint32_t*>(rowe);  // [128] row maxima, then exponents in place
    if (tid < 128) rmax[tid] = 0u;
    asm volatile("bar.sync 1, 512;" ::: "memory");
    if (have) {
      const uint8_t* bb = p.w + static_cast<long long>(b0 + band) * p.tpb * p.tb + 1024;
      uint32_t mx[16];
#pragma unroll
      for (int r = 0; r < 16; ++r) mx[r] = 0u;
      constexpr int kPer = 4;  // tiles per lane per round (loads in flight)
      for (int j0 = 2 * lane + par; j0 < p.tpb; j0 += 64 * kPer) {
        uint4 v[kPer][2];
#pragma unroll
        for (int u = 0; u < kPer; ++u) {
          const int j = j0 + 64 * u;
          if (j < p.tpb) {
            v[u][0] = __ldg(reinterpret_cast<const uint4*>(bb + static_cast<long long>(j) * p.tb));
            v[u][1] = __ldg(reinterpret_cast<const uint4*>(bb + static_cast<long long>(j) * p.tb + 16));
          } else {
            v[u][0] = v[u][1] = make_uint4(0u, 0u, 0u, 0u);
          }
        }
#pragma unroll
        for (int u = 0; u < kPer; ++u)
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const uint32_t wv[4] = {v[u][hh].x, v[u][hh].y, v[u][hh].z, v[u][hh].w};
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const uint32_t m = (wv[q >> 1] >> (16 * (q & 1))) & 0x7FFFu;
              const int r = 8 * hh + q;
              if (m < 0x7C00u && m > mx[r]) mx[r] = m;
            }
          }
      }
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        const uint32_t m = __reduce_max_sync(0xffffffffu, mx[r]);
        if (lane == 0) atomicMax(&rmax[16 * band + r], m);
      }
    }
    asm volatile("bar.sync 1, 512;" ::: "memory");
    if (par == 0 && t == 0) {
      const int e_g = v1tc_row_exponent(rmax[16 * band + g]), e_g8 = v1tc_row_exponent(rmax[16 * band + g + 8]);
      __syncwarp(0x11111111u);
      rowe[16 * band + g] = e_g;
      rowe[16 * band + g + 8] = e_g8;
    }
    asm volatile("bar.sync 1, 512;" ::: "memory");  // the row exponents are in place
    const int e0 = rowe[16 * band + g], e1 = rowe[16 * band + g + 8];
    const float dn0 = __int_as_float((127 - e0) << 23), dn1 = __int_as_float((127 - e1) << 23);
    // A in tensor memory: this thread's row (TMEM lane 32·(warp mod 4) + lane)
    // and 64-k half gp of every step of parity par
    const int ta_q = warp & 3, ta_gp = (warp >> 2) & 1;
    const int ta_r = v1ta_row(32 * ta_q + lane);
    const int ta_band = ta_r >> 4, ta_g = ta_r & 7, ta_half = (ta_r >> 3) & 1;
    const bool ta_have = ta_band < nbt;
    const int ta_e = rowe[ta_r];
    const float ta_dn = __int_as_float((127 - ta_e) << 23);
    const uint32_t ta_col = tmem + (static_cast<uint32_t>(32 * ta_q) << 16) + static_cast<uint32_t>(kV1TAColA + 32 * ta_gp);
    // every dequant warp visits every raw slot (count 16 on its empty barrier)
    // and converts the slot's steps of its parity
    for (int r = 0; r * p.T < nks && !*abort_flag; ++r) {
      const int rs = r % p.NR, ru = r / p.NR;
      if (!mbar_wait_bounded(&raw_full[rs], static_cast<uint32_t>(ru & 1))) {
        *abort_flag = 1;
        break;
      }
      const int l_end = min(nks, (r + 1) * p.T);
      for (int ls = r * p.T + ((r * p.T + par) & 1); ls < l_end; ls += 2) {
        const int a = ls % p.NA, au = ls / p.NA;
        if (au > 0 && !mbar_wait_bounded(&a_empty[a], static_cast<uint32_t>((au - 1) & 1))) {
          *abort_flag = 1;
          break;
        }
        if constexpr (TA) {
          if (au > 0) tc_fence_after();  // the MMAs that read this slot have completed
          uint32_t o[32];
          if (ta_have) {
            const uint8_t* tp = smem + p.off_raw + (rs * 8 + ta_band) * p.band_stride + (ls - r * p.T) * p.tb;
            uint32_t sv = *reinterpret_cast<const unsigned short*>(tp + 1024 + 2 * (8 * ta_half + ta_g));
            if (ta_e) sv = __half_as_ushort(__float2half_rn(h16_to_f32(sv) * ta_dn));
            const uint32_t zw = *reinterpret_cast<const uint32_t*>(tp + 1056 + 4 * ta_half);
            const uint32_t z = (zw >> (4 * ta_g)) & 15u;
            v1ta_row_half(tp, ta_gp, ta_g, ta_half, (0x6400u | z) * 0x00010001u, (0x5400u | (z << 4)) * 0x00010001u,
                          sv * 0x00010001u, o);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) o[j] = 0u;
          }
          tmem_st32(ta_col + static_cast<uint32_t>(64 * a), o);
          tmem_wait_st();
          tc_fence_before();
        } else if (have) {
          const uint8_t* tp = smem + p.off_raw + (rs * 8 + band) * p.band_stride + (ls - r * p.T) * p.tb;
          uint32_t sg = *reinterpret_cast<const unsigned short*>(tp + 1024 + 2 * g);
          uint32_t sg8 = *reinterpret_cast<const unsigned short*>(tp + 1024 + 2 * (g + 8));
          if (e0) sg = __half_as_ushort(__float2half_rn(h16_to_f32(sg) * dn0));
          if (e1) sg8 = __half_as_ushort(__float2half_rn(h16_to_f32(sg8) * dn1));
          v1tc_tile_to_a(tp, smem + p.off_a + a * kV1TCA, band, lane, sg * 0x00010001u, sg8 * 0x00010001u);
          fence_proxy_async_smem();  // generic-proxy writes -> visible to the tensor core
        }
        __syncwarp();
        if (lane == 0) tc5_arrive(&a_full[a]);
      }
      __syncwarp();
      if (lane == 0) tc5_arrive(&raw_empty[rs]);
    }
  }

  // ---- epilogue: every thread waits for the last MMAs, warps 0..7 read TMEM
  // (warp w: lanes 32(w mod 4).., column half (w / 4) mod 2)
  bool ok = !*abort_flag && mbar_wait_bounded(done, 0u);
  tc_fence_after();
  const int lq = warp & 3, ch = (warp >> 2) & 1;
  const uint32_t lane_base = tmem + (static_cast<uint32_t>(lq * 32) << 16);
  const int tlane = lq * 32 + lane;                  // TMEM lane this thread reads back
  const int trow = TA ? v1ta_row(tlane) : tlane;     // its tile row
  const bool split_cols = p.BN % 32 == 0;
  const int cols_per = split_cols ? p.BN / 2 : p.BN;
  const int c_begin = split_cols ? ch * cols_per : 0;
  const bool reads = warp < 8 && (split_cols || ch == 0);
  const float row_up = __int_as_float((127 + rowe[trow & 127]) << 23);  // 2^e
  // the accumulators in a fixed order: even steps (NACC of them), then odd steps
  const int n_acc = (nks > 1 ? 2 : 1) * p.NACC;
  auto acc16 = [&](int c0, float (&v)[16]) {
    uint32_t r0[16];
    tmem_ld16(lane_base + c0, r0);
#pragma unroll
    for (int j = 0; j < 16; ++j) v[j] = __uint_as_float(r0[j]);
    for (int c = 1; c < n_acc; ++c) {
      tmem_ld16(lane_base + c * p.BN + c0, r0);
#pragma unroll
      for (int j = 0; j < 16; ++j) v[j] += __uint_as_float(r0[j]);
    }
#pragma unroll
    for (int j = 0; j < 16; ++j) v[j] *= row_up;
  };
  __half* y = reinterpret_cast<__half*>(p.y);
  if (p.S == 1) {
    if (ok && reads) {
      for (int c0 = c_begin; c0 < c_begin + cols_per; c0 += 16) {
        float v[16];
        acc16(c0, v);
        const int yrow = n0 + trow;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int m = m0 + c0 + j;
          if (m < p.M && yrow < p.N) y[static_cast<long long>(m) * p.N + yrow] = __float2half_rn(v[j]);
        }
      }
    }
  } else {
    // K split over the cluster: park the fp32 tile [128][BN] in this CTA's
    // shared memory (the rings are drained), then each rank adds 128/S rows
    // over all ranks in rank order
    float* acc = reinterpret_cast<float*>(smem);
    __syncthreads();
    if (reads) {
      for (int c0 = c_begin; c0 < c_begin + cols_per; c0 += 16) {
        float v[16];
        if (ok) acc16(c0, v);
#pragma unroll
        for (int j = 0; j < 16; ++j) acc[trow * p.BN + c0 + j] = ok ? v[j] : 0.f;
      }
    }
    tc5_cluster_sync();
    const int rows_per = 128 / p.S;
    const int items = rows_per * p.BN;
    for (int i = tid; i < items; i += kV1TCWarps * 32) {
      const int rr = static_cast<int>(rank) * rows_per + i / p.BN, c = i % p.BN;
      float sum = 0.f;
      for (int q = 0; q < p.S; ++q) sum += tc5_dsmem_ld(acc + rr * p.BN + c, static_cast<uint32_t>(q));
      const int m = m0 + c, yrow = n0 + rr;
      if (m < p.M && yrow < p.N && !*abort_flag) y[static_cast<long long>(m) * p.N + yrow] = __float2half_rn(sum);
    }
    tc5_cluster_sync();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(p.tmem_cols) : "memory");
}

}  // namespace wq
