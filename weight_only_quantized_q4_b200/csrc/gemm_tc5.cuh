// gemm_tc5.cuh — batched dequant-then-MMA on the 5th-generation tensor cores
// (tcgen05, sm_100a) for M >= 9 decode/prefill batches.
//
// y[m, n] = Σ_k W[n, k]·x[m, k].  A CTA owns 128 weight rows (the UMMA M side)
// and BN batch rows (the UMMA N side, a multiple of 16, <= 256).  For every
// 64-k stage:
//   * the 128 threads dequantize their row's 64 weights to fp16 and store them
//     into a 128-byte-swizzled K-major A tile (16 KB); int4 as
//     RN16((q - z)·s) (q - z exact in fp16, one rounding of the exact
//     product), q4_K as RN16(d·sc·q - dmin·m) from the exact fp32 value;
//   * they copy the BN × 64 activation slice into a B tile of the same layout;
//   * one thread issues four tcgen05.mma (K = 16 each) accumulating into an
//     fp32 TMEM accumulator of 128 lanes × BN columns, and commits them to an
//     mbarrier that frees the stage's A/B buffers (two buffers: dequantizing
//     stage s+1 overlaps the MMAs of stage s).
// The epilogue reads the accumulator with tcgen05.ld (warp w owns TMEM lanes
// 32w..32w+31 = weight rows) and stores fp16 y.  Weights are rounded to fp16
// once before the MMA (error <= 2^-11 relative per weight, within the
// 2e-3·Σ|w·x| acceptance bound); the device dequant exports stay exact fp32.
// Every mbarrier wait is bounded (wq_device.cuh).
#pragma once

#include "gemv_cc.cuh"
#include "wq_device.cuh"

namespace wq {

struct TC5Params {
  const void* x;       // [M, K] fp16
  const uint8_t* w;    // int4 codes [N][K/2] or q4_K blocks [N][K/256][144]
  const uint8_t* scales;
  const uint8_t* zeros;
  void* y;             // [M, N] fp16
  int M, N, K;
  int nb, zb, block_shift;
  int BN;              // batch tile (UMMA N), multiple of 16
  int tmem_cols;       // power of two >= max(32, BN)
};

__device__ __forceinline__ uint64_t umma_smem_desc_sw128(uint32_t saddr) {
  // K-major, 128-byte swizzle: rows of 128 B in 8-row (1024 B) atoms.
  // start >> 4 at [0,14), LBO (unused for this layout, 1) at [16,30),
  // SBO = 1024 B >> 4 at [32,46), version 1 at [46,48), layout 2 at [61,64).
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (1ull << 16) | (64ull << 32) | (1ull << 46) |
         (2ull << 61);
}

// kind::f16 instruction descriptor: D f32, A/B f16, both K-major, N = bn, M = 128.
__host__ __device__ __forceinline__ uint32_t umma_idesc_f16(int bn) {
  return (1u << 4) | (static_cast<uint32_t>(bn >> 3) << 17) | (static_cast<uint32_t>(128 >> 4) << 24);
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

// Raw data of one 64-k stage of one weight row, fetched ahead into registers.
struct RawStage {
  uint4 c0, c1, c2;  // int4: codes in c0, c1; q4_K: header in c0, codes in c1, c2
  uint32_t sz;       // int4: fp16 scale bits | zero-point << 16
};

template <Fmt F>
__device__ __forceinline__ void fetch_stage(const TC5Params& p, int row, int s, RawStage& r) {
  const int k0 = s * 64;
  if (row >= p.N) {
    r.c0 = r.c1 = r.c2 = make_uint4(0u, 0u, 0u, 0u);
    r.sz = 8u << 16;
    return;
  }
  if constexpr (F == Fmt::Int4) {
    const uint4* src = reinterpret_cast<const uint4*>(p.w + static_cast<long long>(row) * (p.K / 2) + k0 / 2);
    r.c0 = __ldcs(src);
    r.c1 = __ldcs(src + 1);
    const int b = k0 >> p.block_shift;  // blocks of >= 64 k: one scale / zero-point per stage
    uint32_t z = 8u;
    if (p.zeros) z = (p.zeros[static_cast<long long>(row) * p.zb + (b >> 1)] >> ((b & 1) * 4)) & 15u;
    r.sz = reinterpret_cast<const uint16_t*>(p.scales)[static_cast<long long>(row) * p.nb + b] | (z << 16);
  } else {
    const int sb = k0 >> 8, pp = (k0 & 255) >> 6;
    const uint8_t* blk = p.w + (static_cast<long long>(row) * (p.K / 256) + sb) * 144;
    r.c0 = __ldcs(reinterpret_cast<const uint4*>(blk));
    r.c1 = __ldcs(reinterpret_cast<const uint4*>(blk + 16 + 32 * pp));
    r.c2 = __ldcs(reinterpret_cast<const uint4*>(blk + 32 + 32 * pp));
  }
}

// Dequantize one stage of one row into 32 fp16x2 words (8 chunks of 8).
// int4 chunk c holds codes of k = 8c + {0,4,1,5,2,6,3,7} (the activation tile
// is permuted the same way); q4_K chunks are in natural k order.
template <Fmt F>
__device__ __forceinline__ void dequant_stage(const TC5Params& p, int s, const RawStage& r, uint32_t (&h)[32]) {
  if constexpr (F == Fmt::Int4) {
    const uint32_t sbits = r.sz & 0xFFFFu, z = r.sz >> 16;
    const uint32_t s2 = sbits | (sbits << 16);
    const uint32_t zl = (0x6400u | z) * 0x00010001u, zh = (0x5400u | (z << 4)) * 0x00010001u;
    const uint32_t words[8] = {r.c0.x, r.c0.y, r.c0.z, r.c0.w, r.c1.x, r.c1.y, r.c1.z, r.c1.w};
#pragma unroll
    for (int wd = 0; wd < 8; ++wd) {
      const uint32_t v = words[wd], v8 = v >> 8;
      uint32_t q[4];
      q[0] = hsub2_f(lop3_or(v, 0x000F000Fu, 0x64006400u), zl);   // (n0, n4) - z, exact
      q[1] = hsub2_f(lop3_or(v, 0x00F000F0u, 0x54005400u), zh);   // (n1, n5) - z
      q[2] = hsub2_f(lop3_or(v8, 0x000F000Fu, 0x64006400u), zl);  // (n2, n6) - z
      q[3] = hsub2_f(lop3_or(v8, 0x00F000F0u, 0x54005400u), zh);  // (n3, n7) - z
#pragma unroll
      for (int e = 0; e < 4; ++e) h[wd * 4 + e] = hmul2_f(q[e], s2);  // RN16((q - z)·s): one rounding
    }
  } else {
    const int pp = ((s * 64) & 255) >> 6;
    uint32_t sc2, mn2;
    q4k_scale_min_pair(r.c0.y, r.c0.z, r.c0.w, static_cast<uint32_t>(pp & 1), static_cast<uint32_t>(pp >> 1), sc2, mn2);
    const float d = h16_to_f32(r.c0.x), dm = h16_to_f32(r.c0.x >> 16);
    const float A0 = __fmul_rn(d, static_cast<float>(sc2 & 0xFFu)), A1 = __fmul_rn(d, static_cast<float>(sc2 >> 8));
    const float B0 = -__fmul_rn(dm, static_cast<float>(mn2 & 0xFFu)), B1 = -__fmul_rn(dm, static_cast<float>(mn2 >> 8));
    const uint32_t words[8] = {r.c1.x, r.c1.y, r.c1.z, r.c1.w, r.c2.x, r.c2.y, r.c2.z, r.c2.w};
#pragma unroll
    for (int wd = 0; wd < 8; ++wd) {
      const uint32_t v = words[wd];
      float lo[4], hi[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        lo[e] = fmaf(A0, __uint_as_float(0x4B000000u | ((v >> (8 * e)) & 15u)) - 8388608.0f, B0);
        hi[e] = fmaf(A1, __uint_as_float(0x4B000000u | ((v >> (8 * e + 4)) & 15u)) - 8388608.0f, B1);
      }
      h[wd * 2 + 0] = pack_f16x2(lo[0], lo[1]);
      h[wd * 2 + 1] = pack_f16x2(lo[2], lo[3]);
      h[16 + wd * 2 + 0] = pack_f16x2(hi[0], hi[1]);
      h[16 + wd * 2 + 1] = pack_f16x2(hi[2], hi[3]);
    }
  }
}

constexpr int kTc5Prefetch = 4;  // stages of raw weights in flight per thread

template <Fmt F>
__global__ void __launch_bounds__(128, 2) gemm_tc5_kernel(const TC5Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte alignment for the swizzle atoms
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* A[2] = {smem, smem + 16384};
  const int bsz = ((p.BN * 128) + 1023) & ~1023;
  uint8_t* B[2] = {smem + 32768, smem + 32768 + bsz};
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + 32768 + 2 * bsz);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 4);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5;
  const int n0 = blockIdx.x * 128;
  const int m0 = blockIdx.y * p.BN;
  const int row = n0 + tid;  // weight row this thread dequantizes (TMEM lane tid)

  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(p.tmem_cols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (tid == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t idesc = umma_idesc_f16(p.BN);
  const int nks = p.K / 64;
  const uint16_t* xg = reinterpret_cast<const uint16_t*>(p.x);

  RawStage raw[kTc5Prefetch];
#pragma unroll
  for (int i = 0; i < kTc5Prefetch; ++i)
    if (i < nks) fetch_stage<F>(p, row, i, raw[i]);

  for (int s0 = 0; s0 < nks; s0 += kTc5Prefetch) {
#pragma unroll
    for (int i = 0; i < kTc5Prefetch; ++i) {
      const int s = s0 + i;
      if (s >= nks) break;
      const int slot = s & 1;
      if (s >= 2 && !*abort_flag) {
        if (!mbar_wait_bounded(&bars[slot], static_cast<uint32_t>(((s - 2) >> 1) & 1))) *abort_flag = 1;
      }
      __syncthreads();
      if (*abort_flag) break;
      const int k0 = s * 64;
      uint32_t h[32];
      dequant_stage<F>(p, s, raw[i], h);
      if (s + kTc5Prefetch < nks) fetch_stage<F>(p, row, s + kTc5Prefetch, raw[i]);
      uint8_t* a = A[slot];
#pragma unroll
      for (int c = 0; c < 8; ++c)
        *reinterpret_cast<uint4*>(a + sw128(tid, c)) = make_uint4(h[4 * c], h[4 * c + 1], h[4 * c + 2], h[4 * c + 3]);
      // ---- B: activation rows m0 .. m0+BN-1, k0 .. k0+63 (zero past M)
      uint8_t* bt = B[slot];
      for (int c = tid; c < p.BN * 8; c += 128) {
        const int n = c >> 3, kc = c & 7;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (m0 + n < p.M) v = *reinterpret_cast<const uint4*>(xg + static_cast<long long>(m0 + n) * p.K + k0 + 8 * kc);
        if constexpr (F == Fmt::Int4)  // same k order as the A chunks: x0 x4 x1 x5 x2 x6 x3 x7
          v = make_uint4(__byte_perm(v.x, v.z, 0x5410), __byte_perm(v.x, v.z, 0x7632), __byte_perm(v.y, v.w, 0x5410),
                         __byte_perm(v.y, v.w, 0x7632));
        *reinterpret_cast<uint4*>(bt + sw128(n, kc)) = v;
      }
      fence_proxy_async_smem();  // generic-proxy writes -> visible to the tensor core
      tc_fence_before();
      __syncthreads();
      if (tid == 0) {
        tc_fence_after();
        const uint64_t ad = umma_smem_desc_sw128(smem_u32(a));
        const uint64_t bd = umma_smem_desc_sw128(smem_u32(bt));
#pragma unroll
        for (int j = 0; j < 4; ++j)  // K = 16 per MMA: advance 32 bytes inside the swizzle atom
          umma_f16(tmem, ad + 2ull * j, bd + 2ull * j, idesc, (s > 0 || j > 0) ? 1u : 0u);
        umma_commit(&bars[slot]);
      }
    }
    if (*abort_flag) break;
  }
  // ---- wait for the last stage's MMAs, then read the accumulator
  const int last = nks - 1;
  bool ok = !*abort_flag;
  if (ok && !mbar_wait_bounded(&bars[last & 1], static_cast<uint32_t>((last >> 1) & 1))) ok = false;
  if (ok && nks >= 2 && !mbar_wait_bounded(&bars[(last - 1) & 1], static_cast<uint32_t>(((last - 1) >> 1) & 1)))
    ok = false;
  tc_fence_after();
  if (ok) {
    __half* y = reinterpret_cast<__half*>(p.y);
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    for (int c0 = 0; c0 < p.BN; c0 += 16) {
      uint32_t r[16];
      tmem_ld16(lane_base + c0, r);
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int m = m0 + c0 + j;
        if (m < p.M && row < p.N) y[static_cast<long long>(m) * p.N + row] = __float2half_rn(__uint_as_float(r[j]));
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(p.tmem_cols) : "memory");
}

}  // namespace wq
