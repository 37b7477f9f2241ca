// gemm_mmq.cuh — int8-activation batched q4_K on the tcgen05 tensor cores
// (minfer doc 62 "r59 — q4_K W_dsc plane": §3.2 the MMQ dispatch arm, an
// int8 prepass over the activations feeding an integer GEMM; §2.1 the
// rank-1 rescale of every (chunk, row) pair by (d·sc, −dmin·m)).
//
// Prepass (quantize_q8_kernel), per token m and 32-element chunk c, binary32
// with one rounding per operation: amax = max|x|, d = amax / 127,
// q = rint(x / d) (ties to even; 0 when d = 0), s = d·Σq.  q is stored
// token-major int8 [M][K]; (d, s) chunk-major float2 [K/32][Mp], Mp = M
// rounded up to 16 (the padding entries are zero).
//
// GEMM (gemm_mmq_kernel):
//   y[m, n] = Σ_c (d·sc)[n, c]·d[m, c]·I[m, n, c] + (−dmin·m)[n, c]·s[m, c],
//   I[m, n, c] = Σ_{k in chunk c} q4[n, k]·q8[m, k]   (exact, int32)
// A CTA owns 128 weight rows (the UMMA M side), BN tokens (the UMMA N side)
// and a slice of K; the S CTAs of a cluster split K and add their fp32
// partials through distributed shared memory in rank order.  Per q4_K
// super-block (256 k):
//   * producer warp: one TMA copy of the 128 rows' 144-byte blocks, two of
//     the BN × 128 int8 activation slices (128-byte swizzle, the UMMA K-major
//     layout; no multicast) and one of the 8 × BN (d, s) pairs;
//   * four unpack warps (a thread per weight row) spread the row's 4-bit
//     codes into bytes of a 128-byte-swizzled A tile (two 128-k atoms) and
//     form the row's eight (d·sc, −dmin·m) pairs (each one fp32 multiply, the
//     W_dsc plane entries of §2.2 — or read them from the plane when given);
//   * one MMA warp issues one tcgen05.mma kind::i8 (K = 32, s32 accumulate)
//     per chunk into its own TMEM accumulator: a chunk's integer sums must
//     stay apart because its rescale differs;
//   * sixteen rescale warps read each chunk's 128 × BN int32 sums with
//     tcgen05.ld and add dv·(d·I) + mv·s into fp32 registers (the four warps
//     w ≡ q mod 4 share TMEM lanes 32q.. and split the columns); the int32
//     sum becomes fp32 exactly by the magic-number route (|I| < 2^22), which
//     keeps the conversion off the slow conversion pipe.
// TMEM holds two buffers of U = 256 / BN chunk accumulators, so the MMAs of
// one buffer overlap the rescale of the other.  Every mbarrier wait is
// bounded (wq_device.cuh); on a timeout the kernel stops, waits (bounded) for
// its copies and MMAs in flight, frees TMEM and returns.
#pragma once

#include "gemm_tc5.cuh"

namespace wq {

struct MMQParams {
  CUtensorMap tmap_w;  // raw q4_K bytes [N][K/256·144], box 144 B × 128 rows
  CUtensorMap tmap_a;  // int8 activations [M][K], box 128 B × BN rows, 128-byte swizzle
  CUtensorMap tmap_s;  // (d, s) as floats [K/32][2·Mp], box 2·BN × 8 chunks
  const float* plane;  // W_dsc plane [K/32][N] float2, or null (coefficients formed in the kernel)
  void* y;             // [M, N] fp16
  int M, N, K;
  int S;               // CTAs of a cluster (K slices)
  int nsb_total;       // super-blocks of K; rank r of a cluster takes [r·nsb_total/S, (r+1)·nsb_total/S)
  int NS, NA;          // stages (TMA ring), A slots
  int stage_bytes, a_bytes;
  int off_a, off_bar;  // shared-memory offsets (stages start at 0)
};

constexpr int kMMQWarps = 22;  // producer, MMA issuer, 4 unpack warps, 16 rescale warps
constexpr int kMMQRescale = 16;
constexpr int kMMQRaw = 128 * 144;  // raw bytes of one stage

template <int BN>
struct MMQShape {
  static constexpr int U = (256 / BN) < 8 ? (256 / BN) : 8;  // chunk accumulators per TMEM buffer
  static constexpr int TMEM_COLS = 2 * U * BN;
  static constexpr int STAGE = kMMQRaw + 256 * BN + 64 * BN;     // raw, int8 x (2 atoms), (d, s)
  static constexpr int A_SLOT = 32768 + 8192 + 64 * BN;          // A tile, (dv, mv)[8][128], d[8][BN] | s[8][BN]
  static constexpr int CP = BN >= 64 ? BN / 4 : 16;              // columns per rescale warp
  static constexpr int GROUPS = BN / CP;                          // column groups in use (of four)
};

// kind::i8 instruction descriptor: D s32, A and B signed 8-bit, both K-major, N = bn, M = 128.
__host__ __device__ __forceinline__ uint32_t umma_idesc_i8(int bn) {
  return (2u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(bn >> 3) << 17) |
         (static_cast<uint32_t>(128 >> 4) << 24);
}

// One MMA that overwrites its accumulator (enable-input-d false): every chunk
// starts a fresh integer sum.
__device__ __forceinline__ void umma_i8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, 0, 0;\n"
      " tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc)
      : "memory");
}

// 16 consecutive TMEM columns of this warp's 32 lanes, without waiting (the
// caller issues several, then tcgen05.wait::ld once).
__device__ __forceinline__ void tmem_ld16_nowait(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// acc[tokens] += dv·(d·I) + mv·s over 16 columns of one chunk: v the int32
// sums, d4 / s4 the tokens' d and s (four per float4), two tokens per
// instruction.  The int32 sum becomes fp32 exactly (|I| < 2^22).
template <int NP>
__device__ __forceinline__ void mmq_rescale16(float2 (&acc)[NP], int a0, const uint32_t (&v)[16], const float4* d4,
                                              const float4* s4, float2 dv2, float2 mv2) {
#pragma unroll
  for (int t = 0; t < 16; t += 4) {
    const float4 dq = d4[t >> 2], sq = s4[t >> 2];
    float2 i01 = __fadd2_rn(make_float2(__int_as_float(static_cast<int>(v[t]) + 0x4B400000),
                                        __int_as_float(static_cast<int>(v[t + 1]) + 0x4B400000)),
                            make_float2(-12582912.0f, -12582912.0f));
    float2 i23 = __fadd2_rn(make_float2(__int_as_float(static_cast<int>(v[t + 2]) + 0x4B400000),
                                        __int_as_float(static_cast<int>(v[t + 3]) + 0x4B400000)),
                            make_float2(-12582912.0f, -12582912.0f));
    i01 = __fmul2_rn(make_float2(dq.x, dq.y), i01);
    i23 = __fmul2_rn(make_float2(dq.z, dq.w), i23);
    float2& x01 = acc[a0 + (t >> 1)];
    float2& x23 = acc[a0 + (t >> 1) + 1];
    x01 = __ffma2_rn(dv2, i01, x01);
    x23 = __ffma2_rn(dv2, i23, x23);
    x01 = __ffma2_rn(mv2, make_float2(sq.x, sq.y), x01);
    x23 = __ffma2_rn(mv2, make_float2(sq.z, sq.w), x23);
  }
}

// int32 |v| < 2^22 -> fp32, exactly: 1.5·2^23 + v has v in its mantissa field.
__device__ __forceinline__ float mmq_i2f(uint32_t v) {
  return __int_as_float(static_cast<int>(v) + 0x4B400000) - 12582912.0f;
}

// ---------------------------------------------------------------- prepass

// Thread per (chunk c, token m), m fastest: reads the chunk's 32 fp16 values
// (four 16-byte loads), writes 32 int8 codes and the (d, s) pair.  Tokens
// M..Mp-1 only write zero pairs.
__global__ void quantize_q8_kernel(const __half* x, int8_t* qa, float2* sda, int M, int Mp, int K) {
  const int C = K / 32;
  const long long items = static_cast<long long>(C) * Mp;
  for (long long it = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; it < items;
       it += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int c = static_cast<int>(it / Mp), m = static_cast<int>(it - static_cast<long long>(c) * Mp);
    if (m >= M) {
      sda[it] = make_float2(0.f, 0.f);
      continue;
    }
    const uint4* src = reinterpret_cast<const uint4*>(x + static_cast<long long>(m) * K + 32 * c);
    uint32_t h[16];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint4 v = src[i];
      h[4 * i] = v.x;
      h[4 * i + 1] = v.y;
      h[4 * i + 2] = v.z;
      h[4 * i + 3] = v.w;
    }
    float f[32];
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      f[2 * i] = h16_to_f32(h[i]);
      f[2 * i + 1] = h16_to_f32(h[i] >> 16);
      amax = fmaxf(amax, fmaxf(fabsf(f[2 * i]), fabsf(f[2 * i + 1])));
    }
    const float d = __fdiv_rn(amax, 127.0f);
    int sum = 0;
    uint32_t packed[8];
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      uint32_t word = 0;
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const int q = d > 0.f ? __float2int_rn(__fdiv_rn(f[4 * w + b], d)) : 0;
        sum += q;
        word |= (static_cast<uint32_t>(q) & 0xFFu) << (8 * b);
      }
      packed[w] = word;
    }
    uint4* dst = reinterpret_cast<uint4*>(qa + static_cast<long long>(m) * K + 32 * c);
    dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
    sda[it] = make_float2(d, __fmul_rn(d, static_cast<float>(sum)));
  }
}

// ---------------------------------------------------------------- GEMM

// (scale, min) of chunk j (0..7) from the 12 packed bytes (§2.1 / §3.2: chunks
// 0..3 take the low 6 bits of bytes j and j + 4; chunks 4..7 a nibble of byte
// j + 4 and the top two bits of byte j − 4 (scale) or byte j (min)).
__device__ __forceinline__ void mmq_scale_min(const uint8_t* sc, int j, uint32_t& s, uint32_t& m) {
  if (j < 4) {
    s = sc[j] & 63u;
    m = sc[j + 4] & 63u;
  } else {
    s = (sc[j + 4] & 15u) | ((sc[j - 4] >> 6) << 4);
    m = (sc[j + 4] >> 4) | ((sc[j] >> 6) << 4);
  }
}

template <int BN>
__global__ void __launch_bounds__(kMMQWarps * 32, 1) gemm_mmq_kernel(const __grid_constant__ MMQParams p) {
  using SH = MMQShape<BN>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + p.off_bar);
  uint64_t* stage_empty = full + p.NS;
  uint64_t* a_full = stage_empty + p.NS;
  uint64_t* a_empty = a_full + p.NA;
  uint64_t* acc_full = a_empty + p.NA;  // [2]
  uint64_t* acc_empty = acc_full + 2;   // [2]
  uint64_t* done = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = p.S > 1 ? tc5_cluster_rank() : 0u;
  const int tile = blockIdx.x / p.S;
  const int n0 = tile * 128;
  const int m0 = blockIdx.y * BN;
  const int sb0 = static_cast<int>((static_cast<long long>(rank) * p.nsb_total) / p.S);  // this CTA's K slice
  const int nsb = static_cast<int>((static_cast<long long>(rank + 1) * p.nsb_total) / p.S) - sb0;

  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(SH::TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (tid == 32) {
    for (int i = 0; i < p.NS; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&stage_empty[i], 2);  // the unpack warps (raw, (d, s)) and the MMA commit (int8 x)
    }
    for (int i = 0; i < p.NA; ++i) {
      mbar_init(&a_full[i], 1);
      mbar_init(&a_empty[i], 1 + kMMQRescale);  // MMA commit (A tile) and every rescale warp (coefficients)
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], kMMQRescale);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int issued = 0;
      for (int j = 0; j < nsb && !*abort_flag; ++j) {
        const int s = j % p.NS, su = j / p.NS;
        if (su > 0 && !mbar_wait_bounded(&stage_empty[s], static_cast<uint32_t>((su - 1) & 1))) {
          *abort_flag = 1;
          break;
        }
        uint8_t* st = smem + s * p.stage_bytes;
        mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(SH::STAGE));
        const int sb = sb0 + j;
        tma_load_2d(st, &p.tmap_w, sb * 144, n0, &full[s]);
        tma_load_2d(st + kMMQRaw, &p.tmap_a, sb * 256, m0, &full[s]);
        tma_load_2d(st + kMMQRaw + 128 * BN, &p.tmap_a, sb * 256 + 128, m0, &full[s]);
        tma_load_2d(st + kMMQRaw + 256 * BN, &p.tmap_s, 2 * m0, 8 * sb, &full[s]);
        ++issued;
      }
      // the latest copy issued into each stage has landed before the CTA may exit
      for (int j = issued > p.NS ? issued - p.NS : 0; j < issued; ++j)
        mbar_wait_bounded(&full[j % p.NS], static_cast<uint32_t>((j / p.NS) & 1));
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // The eight MMAs of a super-block are unrolled (compile-time chunk,
    // accumulator and descriptor offsets): a rolled chunk loop around the
    // bounded accumulator waits ran about ten times slower per MMA.
    if (lane == 0) {
      const uint32_t idesc = umma_idesc_i8(BN);
      constexpr int kUnits = 8 / SH::U;  // TMEM buffers a super-block fills
      for (int j = 0; j < nsb && !*abort_flag; ++j) {
        const int s = j % p.NS, a = j % p.NA;
        if (!mbar_wait_bounded(&full[s], static_cast<uint32_t>((j / p.NS) & 1)) ||
            !mbar_wait_bounded(&a_full[a], static_cast<uint32_t>((j / p.NA) & 1))) {
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint64_t ad0 = umma_smem_desc_sw128(smem_u32(smem + p.off_a + a * p.a_bytes));
        const uint64_t bd0 = umma_smem_desc_sw128(smem_u32(smem + s * p.stage_bytes + kMMQRaw));
        bool ok = true;
#pragma unroll
        for (int q = 0; q < kUnits; ++q) {
          const int u = j * kUnits + q, slot = u & 1;
          if (u >= 2) {
            if (!mbar_wait_bounded(&acc_empty[slot], static_cast<uint32_t>(((u >> 1) - 1) & 1))) {
              ok = false;
              break;
            }
            tc_fence_after();
          }
#pragma unroll
          for (int e = 0; e < SH::U; ++e) {
            const int c = q * SH::U + e;  // chunk of the super-block: atom c / 4, 32 bytes (c % 4) into it
            umma_i8(tmem + static_cast<uint32_t>(slot * SH::U * BN + e * BN),
                    ad0 + static_cast<uint64_t>((c >> 2) * (16384 >> 4) + 2 * (c & 3)),
                    bd0 + static_cast<uint64_t>((c >> 2) * ((128 * BN) >> 4) + 2 * (c & 3)), idesc);
          }
          umma_commit(&acc_full[slot]);
        }
        if (!ok) {
          *abort_flag = 1;
          break;
        }
        umma_commit(&stage_empty[s]);
        umma_commit(&a_empty[a]);
      }
      umma_commit(done);  // arrives when every MMA issued above has completed
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------ unpack warps
    const int r = tid - 64;  // weight row of the tile
    const int n = n0 + r;
    for (int j = 0; j < nsb && !*abort_flag; ++j) {
      const int s = j % p.NS, a = j % p.NA, au = j / p.NA;
      if (!mbar_wait_bounded(&full[s], static_cast<uint32_t>((j / p.NS) & 1)) ||
          (au > 0 && !mbar_wait_bounded(&a_empty[a], static_cast<uint32_t>((au - 1) & 1)))) {
        *abort_flag = 1;
        break;
      }
      const uint8_t* st = smem + s * p.stage_bytes;
      uint8_t* ab = smem + p.off_a + a * p.a_bytes;
      const uint8_t* rb = st + r * 144;
      // codes: run p (32 bytes) holds chunk 2p in its low nibbles and chunk
      // 2p + 1 in its high nibbles; 16 bytes give 16 consecutive k of each
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int run = q >> 1, half = q & 1;
        const uint4 v = *reinterpret_cast<const uint4*>(rb + 16 + 32 * run + 16 * half);
        const int klo = 4 * run + half, khi = klo + 2;  // 16-byte chunk index over the 256 k
        const uint4 lo = make_uint4(v.x & 0x0F0F0F0Fu, v.y & 0x0F0F0F0Fu, v.z & 0x0F0F0F0Fu, v.w & 0x0F0F0F0Fu);
        const uint4 hi = make_uint4((v.x >> 4) & 0x0F0F0F0Fu, (v.y >> 4) & 0x0F0F0F0Fu, (v.z >> 4) & 0x0F0F0F0Fu,
                                    (v.w >> 4) & 0x0F0F0F0Fu);
        *reinterpret_cast<uint4*>(ab + (klo >> 3) * 16384 + sw128(r, klo & 7)) = lo;
        *reinterpret_cast<uint4*>(ab + (khi >> 3) * 16384 + sw128(r, khi & 7)) = hi;
      }
      // the row's eight (d·sc, −dmin·m) pairs
      float2* coef = reinterpret_cast<float2*>(ab + 32768);
      const int sb = sb0 + j;
      if (p.plane) {
#pragma unroll
        for (int c = 0; c < 8; ++c)
          coef[c * 128 + r] = n < p.N ? reinterpret_cast<const float2*>(p.plane)[static_cast<long long>(8 * sb + c) * p.N + n]
                                      : make_float2(0.f, 0.f);
      } else {
        const float d = h16_to_f32(*reinterpret_cast<const unsigned short*>(rb));
        const float dmin = h16_to_f32(*reinterpret_cast<const unsigned short*>(rb + 2));
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint32_t sc, mn;
          mmq_scale_min(rb + 4, c, sc, mn);
          coef[c * 128 + r] = make_float2(__fmul_rn(d, static_cast<float>(sc)), -__fmul_rn(dmin, static_cast<float>(mn)));
        }
      }
      // the (d, s) pairs of the BN tokens, chunk by chunk: [8][BN] pairs ->
      // per chunk BN values of d, then BN values of s (two-token operands)
      const float2* sd_src = reinterpret_cast<const float2*>(st + kMMQRaw + 256 * BN);
      float* sd_dst = reinterpret_cast<float*>(ab + 32768 + 8192);
      for (int i = r; i < 8 * BN; i += 128) {
        const int c = i / BN, t = i - c * BN;
        const float2 v = sd_src[i];
        sd_dst[c * 2 * BN + t] = v.x;
        sd_dst[c * 2 * BN + BN + t] = v.y;
      }
      fence_proxy_async_smem();  // generic-proxy writes of the A tile -> visible to the tensor core
      asm volatile("bar.sync 1, 128;" ::: "memory");
      if (r == 0) {
        tc5_arrive(&stage_empty[s]);
        tc5_arrive(&a_full[a]);
      }
    }
  } else {
    // ------------------------------------------------------------ rescale warps
    const int lq = warp & 3, cg = (warp - 6) >> 2;
    const int trow = lq * 32 + lane;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(lq * 32) << 16);
    const bool active = cg < SH::GROUPS;
    const int c_begin = active ? cg * SH::CP : 0;
    float2 acc[SH::CP / 2];  // tokens (2i, 2i + 1) of the warp's columns
#pragma unroll
    for (int i = 0; i < SH::CP / 2; ++i) acc[i] = make_float2(0.f, 0.f);
    constexpr int kUnits = 8 / SH::U;
    for (int j = 0; j < nsb && !*abort_flag; ++j) {
      const int a = j % p.NA;
      if (!mbar_wait_bounded(&a_full[a], static_cast<uint32_t>((j / p.NA) & 1))) {
        *abort_flag = 1;
        break;
      }
      const uint8_t* ab = smem + p.off_a + a * p.a_bytes;
      const float2* coef = reinterpret_cast<const float2*>(ab + 32768);
      const float* sd = reinterpret_cast<const float*>(ab + 32768 + 8192);
      bool ok = true;
#pragma unroll
      for (int q = 0; q < kUnits; ++q) {
        const int u = j * kUnits + q, slot = u & 1;
        if (!mbar_wait_bounded(&acc_full[slot], static_cast<uint32_t>((u >> 1) & 1))) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (active && SH::CP > 16) {
#pragma unroll
          for (int e = 0; e < SH::U; ++e) {
#pragma unroll
            for (int cc = 0; cc < SH::CP; cc += 16) {
              const int c = q * SH::U + e;
              const float2 cf = coef[c * 128 + trow];
              uint32_t v[16];
              tmem_ld16_nowait(lane_base + static_cast<uint32_t>(slot * SH::U * BN + e * BN + c_begin + cc), v);
              tmem_wait_ld();
              mmq_rescale16(acc, cc >> 1, v, reinterpret_cast<const float4*>(sd + c * 2 * BN + c_begin + cc),
                            reinterpret_cast<const float4*>(sd + c * 2 * BN + BN + c_begin + cc),
                            make_float2(cf.x, cf.x), make_float2(cf.y, cf.y));
            }
          }
        } else if (active) {
          // two chunks per round: both TMEM loads in flight before one wait
#pragma unroll
          for (int e = 0; e < SH::U; e += 2) {
#pragma unroll
            for (int cc = 0; cc < SH::CP; cc += 16) {  // 16 columns per load (register budget)
              const int c0 = q * SH::U + e, c1 = c0 + 1;
              const uint32_t col = static_cast<uint32_t>(slot * SH::U * BN + e * BN + c_begin + cc);
              uint32_t va[16], vb[16];
              tmem_ld16_nowait(lane_base + col, va);
              tmem_ld16_nowait(lane_base + col + BN, vb);
              const float2 cf0 = coef[c0 * 128 + trow], cf1 = coef[c1 * 128 + trow];
              tmem_wait_ld();
              mmq_rescale16(acc, cc >> 1, va, reinterpret_cast<const float4*>(sd + c0 * 2 * BN + c_begin + cc),
                            reinterpret_cast<const float4*>(sd + c0 * 2 * BN + BN + c_begin + cc),
                            make_float2(cf0.x, cf0.x), make_float2(cf0.y, cf0.y));
              mmq_rescale16(acc, cc >> 1, vb, reinterpret_cast<const float4*>(sd + c1 * 2 * BN + c_begin + cc),
                            reinterpret_cast<const float4*>(sd + c1 * 2 * BN + BN + c_begin + cc),
                            make_float2(cf1.x, cf1.x), make_float2(cf1.y, cf1.y));
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) tc5_arrive(&acc_empty[slot]);
      }
      if (!ok) {
        *abort_flag = 1;
        break;
      }
      __syncwarp();
      if (lane == 0) tc5_arrive(&a_empty[a]);
    }

    // ---- epilogue (rescale warps hold the CTA's fp32 partial tile)
    __half* y = reinterpret_cast<__half*>(p.y);
    if (p.S == 1) {
      if (active && !*abort_flag) {
        const int yrow = n0 + trow;
#pragma unroll
        for (int i = 0; i < SH::CP; ++i) {
          const int m = m0 + c_begin + i;
          const float v = (i & 1) ? acc[i >> 1].y : acc[i >> 1].x;
          if (m < p.M && yrow < p.N) y[static_cast<long long>(m) * p.N + yrow] = __float2half_rn(v);
        }
      }
    }
    if (p.S > 1) {
      // park the partial tile [128][BN] in the stage memory once every warp
      // of the CTA is past the main loop (named barrier 2 over the rescale
      // warps only after the block-wide sync below)
      float* part = reinterpret_cast<float*>(smem);
      asm volatile("bar.sync 2, 512;" ::: "memory");
      if (active)
#pragma unroll
        for (int i = 0; i < SH::CP; ++i) part[trow * BN + c_begin + i] = (i & 1) ? acc[i >> 1].y : acc[i >> 1].x;
    }
  }

  // every thread: the MMAs have completed before TMEM is released or reused
  const bool mma_done = mbar_wait_bounded(done, 0u);
  if (p.S > 1) {
    __syncthreads();
    tc5_cluster_sync();
    const int rows_per = 128 / p.S;
    const int items = rows_per * BN;
    __half* y = reinterpret_cast<__half*>(p.y);
    for (int i = tid; i < items; i += kMMQWarps * 32) {
      const int rr = static_cast<int>(rank) * rows_per + i / BN, c = i % BN;
      float sum = 0.f;
      for (int q = 0; q < p.S; ++q)
        sum += tc5_dsmem_ld(reinterpret_cast<const float*>(smem) + rr * BN + c, static_cast<uint32_t>(q));
      const int m = m0 + c, yrow = n0 + rr;
      if (m < p.M && yrow < p.N && !*abort_flag && mma_done) y[static_cast<long long>(m) * p.N + yrow] = __float2half_rn(sum);
    }
    tc5_cluster_sync();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(SH::TMEM_COLS)
                 : "memory");
}

}  // namespace wq
