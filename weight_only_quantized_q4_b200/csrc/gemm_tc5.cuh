// gemm_tc5.cuh — batched dequant-then-MMA on the 5th-generation tensor cores
// (tcgen05, sm_100a) for M >= 9 decode/prefill batches.
//
// y[m, n] = Σ_k W[n, k]·x[m, k].  A CTA owns 128 weight rows (the UMMA M side),
// BN batch rows (the UMMA N side, a multiple of 16, <= 256) and one K slice;
// the S CTAs of a thread-block cluster share the rows and split K, and add
// their fp32 accumulators through distributed shared memory (fixed rank
// order).  Warp-specialized pipeline over 64-k stages, with full / empty
// mbarrier rings and no block-wide synchronisation in the main loop:
//   * weight producer warp: 2-D TMA copies (tensor maps, no multicast) of the
//     raw weight bytes, 128 rows × 256 k per copy (int4: 128 B per row; q4_K:
//     one 144-byte super-block per row);
//   * activation producer warp: the BN × 64 activation slice per stage,
//     128-byte swizzled so it lands in the UMMA K-major layout;
//   * eight dequant warps (two threads per weight row, 32 k each) turn the raw
//     bytes into fp16 A rows in natural k order: int4 as RN16((q - z)·s)
//     (q - z exact via magic-number codes, one rounding of the exact product),
//     q4_K as RN16(d·sc·q - dmin·m) from the exact fp32 value.  With batch
//     tiles of at most 128 columns a thread stores its row's 32 k into tensor
//     memory (its row is its TMEM lane) and the MMAs read A from there;
//     otherwise the rows go to a 128-byte-swizzled shared-memory tile;
//   * two MMA warps (even / odd stages) issue four tcgen05.mma (K = 16 each)
//     per stage into fp32 TMEM accumulators of 128 lanes × BN columns and
//     commit them to the mbarriers that free the A and activation slots.
// The epilogue reads the accumulator with tcgen05.ld (warps w and w + 4 share
// TMEM lanes 32(w mod 4).. and split the columns) and stores fp16 y.  Weights
// are rounded to fp16 once before the MMA (error <= 2^-11 relative per weight,
// within the 2e-3·Σ|w·x| acceptance bound); the device dequant exports stay
// exact fp32.  Every mbarrier wait is bounded (wq_device.cuh).
#pragma once

#include <cuda.h>

#include "gemv_cc.cuh"
#include "wq_device.cuh"

namespace wq {

struct TC5Params {
  CUtensorMap tmap_w;  // raw weight bytes: [N][K/2] (int4) or [N][K/256·144] (q4_K), box 128 rows
  CUtensorMap tmap_x;  // activations [M][K] fp16, box BN rows × 64, 128-byte swizzle
  const void* x;       // [M, K] fp16
  const uint8_t* w;    // int4 codes [N][K/2] or q4_K blocks [N][K/256][144]
  const uint8_t* scales;
  const uint8_t* zeros;
  void* y;             // [M, N] fp16
  int M, N, K;
  int nb, zb, block_shift;
  int BN;              // batch tile (UMMA N), multiple of 16
  int tmem_cols;       // power of two >= max(32, 2·BN): two accumulator tiles
  int S;               // CTAs of a cluster (K slices)
  int nks;             // 64-k stages per CTA (K / S / 64, a multiple of 4)
  int NR, NX;          // raw-weight slots, activation slots (64 k each)
  int spr;             // 64-k stages per raw slot (a power of two)
  int raw_pitch;       // bytes per weight row in a raw slot
  int raw_bytes;       // bytes of one raw slot (128 rows)
  int off_x, off_raw, off_bar;  // shared-memory offsets (A slots start at 0)
};

__device__ __forceinline__ uint64_t umma_smem_desc_sw128(uint32_t saddr) {
  // K-major, 128-byte swizzle: rows of 128 B in 8-row (1024 B) atoms.
  // start >> 4 at [0,14), LBO (unused for this layout, 1) at [16,30),
  // SBO = 1024 B >> 4 at [32,46), version 1 at [46,48), layout 2 at [61,64).
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (1ull << 16) | (64ull << 32) | (1ull << 46) |
         (2ull << 61);
}

// kind::f16 instruction descriptor: D f32, A/B f16 (or both bf16), both K-major, N = bn, M = 128.
__host__ __device__ __forceinline__ uint32_t umma_idesc_f16(int bn, bool bf16 = false) {
  return (1u << 4) | (bf16 ? (1u << 7) | (1u << 10) : 0u) | (static_cast<uint32_t>(bn >> 3) << 17) |
         (static_cast<uint32_t>(128 >> 4) << 24);
}

__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// tcgen05.mma kind::f16 with A read from tensor memory (a_tmem) and B from a
// shared-memory descriptor
__device__ __forceinline__ void umma_f16_ta(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 32 consecutive TMEM columns of this thread's lane from registers
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
// 16 consecutive TMEM columns of this thread's lane from registers
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};\n" ::"r"(
          taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ uint32_t lop3_or(uint32_t v, uint32_t mask, uint32_t magic) {
  uint32_t r;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(v), "r"(mask), "r"(magic));  // (v & mask) | magic
  return r;
}
__device__ __forceinline__ uint32_t hsub2_f(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
__device__ __forceinline__ uint32_t hmul2_f(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// swizzled byte offset of 16-byte chunk c (0..7) of row r in a 128-B-row tile
__device__ __forceinline__ uint32_t sw128(int r, int c) { return r * 128 + ((c ^ (r & 7)) << 4); }

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Dequantize half h (32 k) of one stage of one weight row into 16 fp16x2
// words in natural k order.  raw: the stage's 32 code bytes of the row in
// shared memory; hdr (q4_K): the super-block's 16-byte header; sz (int4): fp16
// scale bits | zero-point << 16.
template <Fmt F>
__device__ __forceinline__ void dequant_stage(int s, int h, const uint8_t* raw, const uint8_t* hdr, uint32_t sz,
                                              float down, uint32_t (&o)[16]) {
  if constexpr (F == Fmt::Int4) {
    const uint4 c = *reinterpret_cast<const uint4*>(raw);  // this thread's 16 code bytes (32 k)
    const uint32_t sbits = sz & 0xFFFFu, z = sz >> 16;
    const uint32_t s2 = sbits | (sbits << 16);
    // (1024 + z, 64 + z): subtracted from (1024 + q_even, 64 + q_odd) gives (q - z) exactly
    const uint32_t zz = (0x6400u | z) | ((0x5400u | (z << 4)) << 16);
    const uint32_t words[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
    for (int wd = 0; wd < 4; ++wd) {
#pragma unroll
      for (int bt = 0; bt < 4; ++bt) {
        // byte bt (codes k = 2bt, 2bt+1) into both halves, then the low nibble
        // in the low half and the high nibble in the high half
        const uint32_t t = __byte_perm(words[wd], 0u, 0x1010u + 0x0101u * static_cast<uint32_t>(bt));
        o[wd * 4 + bt] = hmul2_f(hsub2_f(lop3_or(t, 0x00F0000Fu, 0x54006400u), zz), s2);
      }
    }
  } else {
    const uint4 c1 = *reinterpret_cast<const uint4*>(raw), c2 = *reinterpret_cast<const uint4*>(raw + 16);
    const uint4 hd = *reinterpret_cast<const uint4*>(hdr);
    const int pp = ((s * 64) & 255) >> 6;
    uint32_t sc2, mn2;
    q4k_scale_min_pair(hd.y, hd.z, hd.w, static_cast<uint32_t>(pp & 1), static_cast<uint32_t>(pp >> 1), sc2, mn2);
    const float d = h16_to_f32(hd.x) * down, dm = h16_to_f32(hd.x >> 16) * down;  // ×2^-e: exact
    // half 0: chunk 2pp (low nibbles), half 1: chunk 2pp+1 (high nibbles)
    const uint32_t scv = h ? (sc2 >> 8) : (sc2 & 0xFFu), mnv = h ? (mn2 >> 8) : (mn2 & 0xFFu);
    const float A = __fmul_rn(d, static_cast<float>(scv)), B = -__fmul_rn(dm, static_cast<float>(mnv));
    const uint32_t words[8] = {c1.x, c1.y, c1.z, c1.w, c2.x, c2.y, c2.z, c2.w};
    const int sh = 4 * h;
#pragma unroll
    for (int wd = 0; wd < 8; ++wd) {
      const uint32_t v = words[wd] >> sh;
      float f[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) f[e] = fmaf(A, __uint_as_float(0x4B000000u | ((v >> (8 * e)) & 15u)) - 8388608.0f, B);
      o[wd * 2 + 0] = pack_f16x2(f[0], f[1]);
      o[wd * 2 + 1] = pack_f16x2(f[2], f[3]);
    }
  }
}

// fp16 range of the weight tile.  A dequantized weight must be finite in fp16
// (|w| <= 65504) to enter the MMA; the bound of a row is 15·max|s| (int4) or
// max(|d|·63·15 + |dmin|·63) (q4_K).  A row whose bound is above 65504 is
// dequantized as w·2^-e, with the least e that brings the bound within range,
// and its fp32 result is multiplied by 2^e (both exact).  Rows within range
// (every row of ordinary weights) have e = 0 and are unchanged.  Non-finite
// scales are left out of the bound: they propagate as in IEEE arithmetic.
template <Fmt F>
__device__ __forceinline__ int row_exponent(const TC5Params& p, int row) {
  if constexpr (F == Fmt::BF16) {
    return 0;
  } else {
    if (row >= p.N) return 0;
    float bound = 0.f;
    if constexpr (F == Fmt::Int4) {
      const unsigned short* sr = reinterpret_cast<const unsigned short*>(p.scales) + static_cast<long long>(row) * p.nb;
      uint32_t mx = 0;
      auto take = [&](uint32_t bits) {
        const uint32_t m = bits & 0x7FFFu;
        if (m < 0x7C00u && m > mx) mx = m;
      };
      if ((p.nb & 7) == 0) {  // whole 16-byte groups (the scale array is 16-byte aligned)
        const uint4* s4 = reinterpret_cast<const uint4*>(sr);
#pragma unroll 4
        for (int b = 0; b < p.nb / 8; ++b) {
          const uint4 v = __ldg(s4 + b);
          take(v.x), take(v.x >> 16), take(v.y), take(v.y >> 16);
          take(v.z), take(v.z >> 16), take(v.w), take(v.w >> 16);
        }
      } else {
#pragma unroll 8
        for (int b = 0; b < p.nb; ++b) take(__ldg(sr + b));
      }
      bound = 15.f * h16_to_f32(mx);
    } else {
      const int nsb = p.K / 256;
      const uint8_t* wr = p.w + static_cast<long long>(row) * nsb * 144;
#pragma unroll 8
      for (int j = 0; j < nsb; ++j) {
        const uint32_t dd = __ldg(reinterpret_cast<const unsigned int*>(wr + 144ll * j));
        const float b = fabsf(h16_to_f32(dd)) * 945.f + fabsf(h16_to_f32(dd >> 16)) * 63.f;
        if (b <= 3.0e38f && b > bound) bound = b;  // finite d and dmin only
      }
    }
    int e = 0;
    while (bound > 65504.f) {
      bound *= 0.5f;
      ++e;
    }
    return e;
  }
}

// int4 scale and zero-point of stage s of weight row `row`, as the two loaded
// words (fp16 scale bits; the zero-point byte holding blocks 2j and 2j+1).
// Nothing here uses the loaded values, so the loads stay in flight until the
// stage that needs them (sz_of combines them there): an operation on a load's
// result at issue time would stall the thread for the whole load latency.
// Rows past N read row N-1 (their outputs are never stored).
__device__ __forceinline__ void fetch_sz(const TC5Params& p, int row, int s, uint32_t& sraw, uint32_t& zraw) {
  const long long r = row < p.N ? row : p.N - 1;
  const int b = (s * 64) >> p.block_shift;  // blocks of >= 64 k: one scale / zero-point per stage
  const uint8_t* zp = p.zeros ? p.zeros + r * p.zb + (b >> 1) : p.scales;  // any readable byte without zeros
  sraw = __ldg(reinterpret_cast<const unsigned short*>(p.scales) + r * p.nb + b);
  zraw = __ldg(zp);
}
// packed fp16 scale | z << 16 of stage s from its two loaded words
__device__ __forceinline__ uint32_t sz_of(const TC5Params& p, int s, uint32_t sraw, uint32_t zraw) {
  const int b = (s * 64) >> p.block_shift;
  const uint32_t z = p.zeros ? (zraw >> ((b & 1) * 4)) & 15u : 8u;
  return (sraw & 0xFFFFu) | (z << 16);
}

__device__ __forceinline__ void cp_async16(void* dst, const void* src, uint32_t bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// wait until at most n of this thread's commit groups are pending (n = 0..7)
__device__ __forceinline__ void cp_async_wait_n(int n) {
  switch (n) {
    case 0: asm volatile("cp.async.wait_group 0;" ::: "memory"); break;
    case 1: asm volatile("cp.async.wait_group 1;" ::: "memory"); break;
    case 2: asm volatile("cp.async.wait_group 2;" ::: "memory"); break;
    case 3: asm volatile("cp.async.wait_group 3;" ::: "memory"); break;
    case 4: asm volatile("cp.async.wait_group 4;" ::: "memory"); break;
    case 5: asm volatile("cp.async.wait_group 5;" ::: "memory"); break;
    case 6: asm volatile("cp.async.wait_group 6;" ::: "memory"); break;
    default: asm volatile("cp.async.wait_group 7;" ::: "memory"); break;
  }
}

__device__ __forceinline__ uint32_t tc5_cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void tc5_cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ float tc5_dsmem_ld(const float* local, uint32_t rank) {
  uint32_t a;
  float v;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(smem_u32(local)), "r"(rank));
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(a) : "memory");
  return v;
}

constexpr int kTc5SzAhead = 8;  // int4 scale / zero-point words fetched ahead in registers
constexpr int kTc5NA = 4;       // A slots (16 KB each)
constexpr int kTc5Warps = 12;   // 8 dequant / epilogue warps, weight producer, activation producer, two MMA issuers

__device__ __forceinline__ void tc5_arrive(uint64_t* bar) {
  asm volatile("{\n .reg .b64 st;\n mbarrier.arrive.shared::cta.b64 st, [%0];\n}\n" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int c0, int c1, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

// TA (int4, q4_K with BN <= 128): the dequant threads store their fp16 A rows
// into tensor memory (tcgen05.st; a thread's weight row is its TMEM lane) and
// the MMAs read A from there, instead of a 128-byte-swizzled shared-memory
// tile that the tensor core reads back.
constexpr int kTc5TAColA = 256;  // first TMEM column of the A slots (4 × 32 columns)

template <Fmt F, bool TA = false>
__global__ void __launch_bounds__(kTc5Warps * 32, 1) gemm_tc5_kernel(const __grid_constant__ TC5Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte alignment for the swizzle atoms
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* raw_full = reinterpret_cast<uint64_t*>(smem + p.off_bar);
  uint64_t* raw_empty = raw_full + p.NR;
  uint64_t* x_full = raw_empty + p.NR;
  uint64_t* x_empty = x_full + p.NX;
  uint64_t* a_full = x_empty + p.NX;
  uint64_t* a_empty = a_full + kTc5NA;
  uint64_t* done = a_empty + kTc5NA;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = p.S > 1 ? tc5_cluster_rank() : 0u;
  const int n0 = (blockIdx.x / p.S) * 128;
  const int m0 = blockIdx.y * p.BN;
  const int s_begin = static_cast<int>(rank) * p.nks;  // first global 64-k stage of this CTA
  const int nks = p.nks;
  const int x_bytes = p.BN * 128;

  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(p.tmem_cols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (tid == 32) {
    for (int i = 0; i < p.NR; ++i) {
      mbar_init(&raw_full[i], 1);
      mbar_init(&raw_empty[i], 8);  // one arrival per dequant warp
    }
    for (int i = 0; i < p.NX; ++i) {
      mbar_init(&x_full[i], 1);
      mbar_init(&x_empty[i], 1);  // tcgen05.commit
    }
    for (int i = 0; i < kTc5NA; ++i) {
      mbar_init(&a_full[i], F == Fmt::BF16 ? 1 : 8);  // bf16: the producer's TMA fills A directly
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
  // dequant / epilogue warps: thread tid handles weight row n0 + (tid & 127) in both roles
  const int row_e = warp < 8 ? row_exponent<F>(p, n0 + (tid & 127)) : 0;
  const float row_up = __int_as_float((127 + row_e) << 23);  // 2^e

  if (warp == 8) {
    // ------------------------------------------------------------ weight producer
    // (the activation copies have a warp of their own: a weight copy waits for
    // its ring slot, which the activation stream should not wait behind)
    if (lane == 0) {
      int rs = 0, ru = 0;  // slot index and use count of the raw ring
      for (int ls = 0; ls < nks && !*abort_flag; ++ls) {
        const int gs = s_begin + ls;
        if constexpr (F == Fmt::BF16) {
          // bf16 weights are the MMA operand as stored: 128 rows × 64 k straight into an A slot
          const int a = ls & (kTc5NA - 1), au = ls / kTc5NA;
          if (au > 0 && !mbar_wait_bounded(&a_empty[a], static_cast<uint32_t>((au - 1) & 1))) {
            *abort_flag = 1;
            break;
          }
          mbar_arrive_expect_tx(&a_full[a], 16384u);
          tma_load_2d(smem + a * 16384, &p.tmap_w, gs * 64, n0, &a_full[a]);
        } else if ((ls & (p.spr - 1)) == 0) {
          if (ru > 0 && !mbar_wait_bounded(&raw_empty[rs], static_cast<uint32_t>((ru - 1) & 1))) {
            *abort_flag = 1;
            break;
          }
          mbar_arrive_expect_tx(&raw_full[rs], static_cast<uint32_t>(p.raw_bytes));
          const int c0 = F == Fmt::Int4 ? gs * 32 : (gs >> 2) * 144;  // byte column of the slot's first k
          tma_load_2d(smem + p.off_raw + rs * p.raw_bytes, &p.tmap_w, c0, n0, &raw_full[rs]);
          if (++rs == p.NR) {
            rs = 0;
            ++ru;
          }
        }
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ activation producer
    if (lane == 0) {
      int xs = 0, xu = 0;  // slot index and use count of the activation ring
      for (int ls = 0; ls < nks && !*abort_flag; ++ls) {
        const int gs = s_begin + ls;
        if (xu > 0 && !mbar_wait_bounded(&x_empty[xs], static_cast<uint32_t>((xu - 1) & 1))) {
          *abort_flag = 1;
          break;
        }
        mbar_arrive_expect_tx(&x_full[xs], static_cast<uint32_t>(x_bytes));
        tma_load_2d(smem + p.off_x + xs * ((x_bytes + 1023) & ~1023), &p.tmap_x, gs * 64, m0, &x_full[xs]);
        if (++xs == p.NX) {
          xs = 0;
          ++xu;
        }
      }
    }
  } else if (warp >= 10) {
    // ------------------------------------------------------------ MMA issuers
    // warp 10 the even stages, warp 11 the odd ones (a second issuing thread
    // nearly doubles the rate tcgen05.mma instructions reach the tensor core)
    if (lane == 0) {
      const uint32_t idesc = umma_idesc_f16(p.BN, F == Fmt::BF16);
      for (int ls = warp - 10; ls < nks && !*abort_flag; ls += 2) {
        const int a = ls & (kTc5NA - 1), au = ls / kTc5NA;
        const int xs = ls % p.NX, xu = ls / p.NX;
        if (!mbar_wait_bounded(&a_full[a], static_cast<uint32_t>(au & 1)) ||
            !mbar_wait_bounded(&x_full[xs], static_cast<uint32_t>(xu & 1))) {
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint64_t bd = umma_smem_desc_sw128(smem_u32(smem + p.off_x + xs * ((x_bytes + 1023) & ~1023)));
        // even and odd stages accumulate into two TMEM tiles (columns [0, BN) and
        // [BN, 2BN)), so consecutive stages' MMAs do not wait for each other
        const uint32_t dacc = tmem + static_cast<uint32_t>((ls & 1) * p.BN);
        if constexpr (TA) {
          // A slot a: 32 TMEM columns (64 k), 8 columns per MMA
          const uint32_t at = tmem + static_cast<uint32_t>(kTc5TAColA + 32 * a);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            umma_f16_ta(dacc, at + 8u * j, bd + 2ull * j, idesc, (ls > 1 || j > 0) ? 1u : 0u);
        } else {
          const uint64_t ad = umma_smem_desc_sw128(smem_u32(smem + a * 16384));
#pragma unroll
          for (int j = 0; j < 4; ++j)  // K = 16 per MMA: advance 32 bytes inside the swizzle atom
            umma_f16(dacc, ad + 2ull * j, bd + 2ull * j, idesc, (ls > 1 || j > 0) ? 1u : 0u);
        }
        umma_commit(&a_empty[a]);
        umma_commit(&x_empty[xs]);
      }
      umma_commit(done);  // arrives when every MMA this thread issued has completed
    }
  } else {
    // ------------------------------------------------------------ dequant warps
    const int rl = tid & 127, h = tid >> 7;  // weight row (TMEM lane) and which 32 k of a stage
    const int row = n0 + rl;
    const float down = __int_as_float((127 - row_e) << 23);  // 2^-e of this row
    uint32_t sra[kTc5SzAhead], zra[kTc5SzAhead];
    if constexpr (F == Fmt::Int4) {
#pragma unroll
      for (int i = 0; i < kTc5SzAhead; ++i) {
        sra[i] = zra[i] = 0u;
        if (i < nks) fetch_sz(p, row, s_begin + i, sra[i], zra[i]);
      }
    }
    int rs = 0, ru = 0;
    for (int s0 = 0; s0 < (F == Fmt::BF16 ? 0 : nks); s0 += kTc5SzAhead) {
#pragma unroll
      for (int i = 0; i < kTc5SzAhead; ++i) {
        const int ls = s0 + i;
        if (ls >= nks || *abort_flag) break;
        if ((ls & (p.spr - 1)) == 0 && !mbar_wait_bounded(&raw_full[rs], static_cast<uint32_t>(ru & 1))) {
          *abort_flag = 1;
          break;
        }
        const int a = ls & (kTc5NA - 1), au = ls / kTc5NA;
        if (au > 0 && !mbar_wait_bounded(&a_empty[a], static_cast<uint32_t>((au - 1) & 1))) {
          *abort_flag = 1;
          break;
        }
        uint32_t sz = 0u;
        if constexpr (F == Fmt::Int4) {
          sz = sz_of(p, s_begin + ls, sra[i], zra[i]);
          if (ls + kTc5SzAhead < nks) fetch_sz(p, row, s_begin + ls + kTc5SzAhead, sra[i], zra[i]);
          if (row_e) {  // s·2^-e, rounded to fp16 (exact unless it falls below the normal range)
            const uint32_t sb = __half_as_ushort(__float2half_rn(h16_to_f32(sz) * down));
            sz = (sz & 0xFFFF0000u) | sb;
          }
        }
        const uint8_t* rrow = smem + p.off_raw + rs * p.raw_bytes + rl * p.raw_pitch;
        // int4 raw slots arrive 128-byte swizzled (16-byte chunk c of row r at
        // c ^ (r & 7)): the 8 rows a quarter-warp reads fall in 8 different banks
        const uint8_t* codes = F == Fmt::Int4 ? smem + p.off_raw + rs * p.raw_bytes + sw128(rl, 2 * (ls & 3) + h)
                                              : rrow + 16 + 32 * (ls & 3);
        uint32_t o[16];
        if constexpr (F != Fmt::BF16) dequant_stage<F>(s_begin + ls, h, codes, rrow, sz, down, o);
        if constexpr (TA) {
          // row rl is TMEM lane rl (warp w reaches lanes 32·(w mod 4) ..); k = 32·h .. + 31 of the stage
          if (au > 0) tc_fence_after();  // the MMAs that read this slot have completed
          tmem_st16(tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16) +
                        static_cast<uint32_t>(kTc5TAColA + 32 * a + 16 * h),
                    o);
          tmem_wait_st();
          tc_fence_before();
        } else {
          uint8_t* at = smem + a * 16384;
#pragma unroll
          for (int c = 0; c < 4; ++c)
            *reinterpret_cast<uint4*>(at + sw128(rl, 4 * h + c)) =
                make_uint4(o[4 * c], o[4 * c + 1], o[4 * c + 2], o[4 * c + 3]);
          fence_proxy_async_smem();  // generic-proxy writes -> visible to the tensor core
        }
        __syncwarp();
        if (lane == 0) tc5_arrive(&a_full[a]);
        if ((ls & (p.spr - 1)) == p.spr - 1) {  // every stage of the raw slot is dequantized
          if (lane == 0) tc5_arrive(&raw_empty[rs]);
          if (++rs == p.NR) {
            rs = 0;
            ++ru;
          }
        }
      }
    }
  }

  // ---- epilogue: every thread waits for the last MMAs, the dequant warps read TMEM
  bool ok = !*abort_flag && mbar_wait_bounded(done, 0u);
  tc_fence_after();
  const int lq = warp & 3, ch = (warp >> 2) & 1;  // TMEM lane quarter, column half
  const uint32_t lane_base = tmem + (static_cast<uint32_t>(lq * 32) << 16);
  const int trow = lq * 32 + lane;                // tile row this thread reads back
  const bool split_cols = p.BN % 32 == 0;        // both column halves are whole 16-column groups
  const int cols_per = split_cols ? p.BN / 2 : p.BN;
  const int c_begin = split_cols ? ch * cols_per : 0;
  const bool reads = warp < 8 && (split_cols || ch == 0);
  // fp16 y (int4, q4_K) or bf16 y (bf16 weights and activations)
  auto store_y = [&](long long o, float v) {
    if constexpr (F == Fmt::BF16)
      reinterpret_cast<__nv_bfloat16*>(p.y)[o] = __float2bfloat16_rn(v);
    else
      reinterpret_cast<__half*>(p.y)[o] = __float2half_rn(v);
  };
  // the two accumulator tiles of a 16-column group, added (fixed order); a CTA
  // with a single stage (bf16, K <= 64) never wrote the odd tile
  auto acc16 = [&](int c0, float (&v)[16]) {
    uint32_t r0[16], r1[16];
    tmem_ld16(lane_base + c0, r0);
    if (nks > 1) {
      tmem_ld16(lane_base + p.BN + c0, r1);
#pragma unroll
      for (int j = 0; j < 16; ++j) v[j] = __uint_as_float(r0[j]) + __uint_as_float(r1[j]);
    } else {
#pragma unroll
      for (int j = 0; j < 16; ++j) v[j] = __uint_as_float(r0[j]);
    }
  };
  if (p.S == 1) {
    if (ok && reads) {
      for (int c0 = c_begin; c0 < c_begin + cols_per; c0 += 16) {
        float v[16];
        acc16(c0, v);
        const int yrow = n0 + trow;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int m = m0 + c0 + j;
          if (m < p.M && yrow < p.N) store_y(static_cast<long long>(m) * p.N + yrow, v[j] * row_up);
        }
      }
    }
  } else {
    // K split over the cluster: park the fp32 tile [128][BN] in this CTA's shared
    // memory (the rings are drained), then each rank adds 128/S rows over all ranks
    float* acc = reinterpret_cast<float*>(smem);
    __syncthreads();
    if (reads) {
      for (int c0 = c_begin; c0 < c_begin + cols_per; c0 += 16) {
        float v[16];
        if (ok) acc16(c0, v);
#pragma unroll
        for (int j = 0; j < 16; ++j) acc[trow * p.BN + c0 + j] = ok ? v[j] * row_up : 0.f;
      }
    }
    tc5_cluster_sync();
    const int rows_per = 128 / p.S;
    const int items = rows_per * p.BN;
    for (int i = tid; i < items; i += kTc5Warps * 32) {
      const int rr = static_cast<int>(rank) * rows_per + i / p.BN, c = i % p.BN;
      float sum = 0.f;
      for (int q = 0; q < p.S; ++q) sum += tc5_dsmem_ld(acc + rr * p.BN + c, static_cast<uint32_t>(q));
      const int m = m0 + c, yrow = n0 + rr;
      if (m < p.M && yrow < p.N && !*abort_flag) store_y(static_cast<long long>(m) * p.N + yrow, sum);
    }
    tc5_cluster_sync();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(p.tmem_cols) : "memory");
}

}  // namespace wq
