// gemv_cc.cuh — CUDA-core decode GEMV family (M = 1..8) for sm_100a.
//
// y[m, n] = Σ_k W[n, k]·x[m, k], W dequantized on the fly, fp32 accumulation.
//
// Design (B200-first; the pages' multicol / cp.async designs are prior art):
//  * Weight rows are contiguous, so the rows a CTA owns form one contiguous
//    byte range.  One thread streams it into a ring of shared-memory stages
//    with 1-D bulk copies (cp.async.bulk, completion on an mbarrier).  The
//    prefetch depth therefore costs no registers and no occupancy, which is
//    what the int4 decode GEMV was found to be bound by (onnx-genai PR #1000,
//    "ncu — cp.async worked, but is occupancy-negative").
//  * Activations are stationary: a thread owns one K-segment of KS elements
//    for the whole kernel and keeps x[m, segment] in registers, arranged to
//    match the code pairs the unpacking produces.  Each warp covers 32
//    consecutive segments; WK warps cover a full row ("row group"); G row
//    groups work on different rows of the same stage.
//  * 4-bit codes are unpacked by masking only (see wq_device.cuh) into fp16
//    subnormals q·2^-24 and multiplied by fp16 x with the mixed-precision
//    fma.rn.f32.f16 (exact product, fp32 accumulate, full FMA rate on B200).
//    Zero-points and q4_K mins never touch the per-weight loop: per segment
//    y += s·(Σ q·x − z·Σ x) (int4) and y += A·Σ q·x + B·Σ x (q4_K, with
//    A = d·sc, B = −dmin·m: the rank-1 form of minfer doc 62 §2.1).
//  * Per stage each thread holds RG rows × M partial sums; a reduce-scatter
//    butterfly over the warp leaves one sum per lane, a shared-memory pass
//    adds the WK warps of a row group and writes y.
#pragma once

#include "wq_device.cuh"

namespace wq {

enum class Fmt : int { Int4 = 0, Q4K = 1, Q4KDsc = 2, BF16 = 3 };

struct CCParams {
  const void* x;          // [M, K] fp16 (int4, q4_K) or bf16
  const uint8_t* w;       // codes / q4_K blocks / bf16 rows, row stride row_bytes
  const uint8_t* scales;  // int4: fp16 [N][nb]
  const uint8_t* zeros;   // int4: uint4 pairs [N][zb], or null (z = 8)
  const uint8_t* plane;   // q4_K W_dsc plane: float2 [K/32][N]
  void* y;                // [M, N] fp16 or bf16
  int N, K;
  int nb, zb;             // int4: blocks per row, zero-point bytes per row
  int block_shift;        // int4: log2(block_size)
  long long row_bytes;    // bytes per weight row
  int S;                  // segments per row (K / KS)
  int WK;                 // warps per row group
  int G;                  // row groups per CTA
  int RG;                 // rows per row group per stage (<= the kernel's RGMAX)
  int RS;                 // rows per stage (= G · RG)
  int NS;                 // stages in the ring
  int n_granules;         // ceil(N / 2): rows are split across CTAs in pairs
  int stage_bytes;        // bytes of one stage
  int off_scales, off_zeros, off_plane;  // offsets inside a stage
  int plane_stride;       // bytes per chunk inside a stage's plane area
  int red_offset;         // offset of the reduction buffers after the ring
};

template <Fmt F>
struct FmtTraits;
template <>
struct FmtTraits<Fmt::Int4> {
  static constexpr int kBitsPerWeight = 4;
};
template <>
struct FmtTraits<Fmt::Q4K> {
  static constexpr int kBitsPerWeight = 4;
};
template <>
struct FmtTraits<Fmt::Q4KDsc> {
  static constexpr int kBitsPerWeight = 4;
};
template <>
struct FmtTraits<Fmt::BF16> {
  static constexpr int kBitsPerWeight = 16;
};

__host__ __device__ constexpr int pow2_ceil(int v) { return v <= 1 ? 1 : 2 * pow2_ceil((v + 1) / 2); }
__host__ __device__ constexpr int ilog2(int v) { return v <= 1 ? 0 : 1 + ilog2(v / 2); }

// Reduce-scatter of V (power of two, <= 32) values over the 32 lanes of a
// warp.  On return lanes whose low (5 - log2 V) bits are zero hold, in v[0],
// the warp-wide sum of value index lane >> (5 - log2 V).
template <int V>
__device__ __forceinline__ void warp_reduce_scatter(float (&v)[V], int lane) {
  int n = V;
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    if (n > 1) {
      const bool upper = (lane & off) != 0;
#pragma unroll
      for (int i = 0; i < V / 2; ++i) {
        if (i < n / 2) {
          const float send = upper ? v[i] : v[i + n / 2];
          const float keep = upper ? v[i + n / 2] : v[i];
          v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
      }
      n >>= 1;
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], off);
    }
  }
}

__device__ __forceinline__ uint32_t aligned_down16(uint64_t a) { return static_cast<uint32_t>(a & 15u); }

// Issue the bulk copies of stage `s` into `dst` (run by every lane of warp 0;
// lane 0 arms the barrier with the exact byte total first).
template <Fmt F>
__device__ __forceinline__ void issue_stage(const CCParams& p, uint8_t* dst, uint64_t* bar, int r0, int nr,
                                            int lane, uint64_t policy) {
  // Weight rows: one contiguous, 16-byte aligned range (row_bytes % 16 == 0).
  const uint32_t wbytes = static_cast<uint32_t>(nr * p.row_bytes);
  uint32_t total = wbytes;
  uint32_t sc_len = 0, z_len = 0, pl_len0 = 0, pl_len8 = 0, n_pl8 = 0, n_chunks = 0;
  const uint8_t* sc_lo = nullptr;
  const uint8_t* z_lo = nullptr;
  if constexpr (F == Fmt::Int4) {
    const uint64_t a = reinterpret_cast<uint64_t>(p.scales) + 2ull * p.nb * r0;
    const uint64_t b = a + 2ull * p.nb * nr;
    sc_lo = reinterpret_cast<const uint8_t*>(a & ~15ull);
    sc_len = static_cast<uint32_t>(((b + 15) & ~15ull) - (a & ~15ull));
    total += sc_len;
    if (p.zeros) {
      const uint64_t za = reinterpret_cast<uint64_t>(p.zeros) + 1ull * p.zb * r0;
      const uint64_t zb = za + 1ull * p.zb * nr;
      z_lo = reinterpret_cast<const uint8_t*>(za & ~15ull);
      z_len = static_cast<uint32_t>(((zb + 15) & ~15ull) - (za & ~15ull));
      total += z_len;
    }
  }
  if constexpr (F == Fmt::Q4KDsc) {
    n_chunks = static_cast<uint32_t>(p.K / 32);
    pl_len0 = (nr * 8u + 15u) & ~15u;
    pl_len8 = (nr * 8u + 8u + 15u) & ~15u;
    n_pl8 = (p.N & 1) ? n_chunks / 2 : 0u;  // r0 even: chunk c is 8 mod 16 iff c·N is odd
    total += (n_chunks - n_pl8) * pl_len0 + n_pl8 * pl_len8;
  }
  if (lane == 0) {
    // slot reuse is ordered by the __syncthreads that ended its last use
    mbar_arrive_expect_tx(bar, total);
    bulk_g2s_stream(dst, p.w + static_cast<long long>(r0) * p.row_bytes, wbytes, bar, policy);
    if constexpr (F == Fmt::Int4) {
      bulk_g2s(dst + p.off_scales, sc_lo, sc_len, bar);
      if (p.zeros) bulk_g2s(dst + p.off_zeros, z_lo, z_len, bar);
    }
  }
  if constexpr (F == Fmt::Q4KDsc) {
    __syncwarp();
    for (uint32_t c = lane; c < n_chunks; c += 32) {
      const uint64_t a = reinterpret_cast<uint64_t>(p.plane) + (static_cast<uint64_t>(c) * p.N + r0) * 8ull;
      const uint32_t len = (a & 15u) ? pl_len8 : pl_len0;
      bulk_g2s_stream(dst + p.off_plane + c * p.plane_stride, reinterpret_cast<const void*>(a & ~15ull), len, bar,
                      policy);
    }
  }
}

// Largest rows-per-group a kernel instance can hold (RGMAX·M partial sums).
__host__ __device__ constexpr int rg_max(int M) { return M == 1 ? 8 : (M == 2 ? 4 : (M <= 4 ? 2 : 1)); }

template <Fmt F, int M, int KS>
__global__ void __launch_bounds__(512, 1) gemv_cc_kernel(const CCParams p) {
  constexpr int RG = rg_max(M);
  constexpr bool kFour = FmtTraits<F>::kBitsPerWeight == 4;
  constexpr int V = pow2_ceil(RG * M);        // values per lane in the reduction
  constexpr int XW = KS / 2;                  // 32-bit x registers per m (fp16/bf16 pairs)
  constexpr int SEG_BYTES = kFour ? KS / 2 : KS * 2;
  static_assert(SEG_BYTES % 4 == 0, "segment must hold whole 32-bit words");
  constexpr int WORDS = SEG_BYTES / 4;

  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + p.red_offset + 2 * p.RS * p.WK * M * 4);
  int* abort_flag = reinterpret_cast<int*>(bars + p.NS);
  float* red = reinterpret_cast<float*>(smem + p.red_offset);

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int g = warp / p.WK;
  const int kw = warp - g * p.WK;
  const int seg = kw * 32 + lane;
  const bool active = seg < p.S;

  // Balanced split of row pairs over the grid.
  const long long gb = static_cast<long long>(blockIdx.x) * p.n_granules / gridDim.x;
  const long long ge = static_cast<long long>(blockIdx.x + 1) * p.n_granules / gridDim.x;
  const int row_begin = static_cast<int>(2 * gb);
  const int row_end = min(static_cast<int>(2 * ge), p.N);
  const int n_rows = max(row_end - row_begin, 0);
  const int n_stages = (n_rows + p.RS - 1) / p.RS;

  if (tid == 0) {
    for (int i = 0; i < p.NS; ++i) mbar_init(&bars[i], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();

  const uint64_t policy = policy_evict_first();
  if (warp == 0) {
    for (int s = 0; s < p.NS - 1 && s < n_stages; ++s) {
      const int r0 = row_begin + s * p.RS;
      issue_stage<F>(p, smem + s * p.stage_bytes, &bars[s], r0, min(p.RS, row_end - r0), lane, policy);
    }
  }

  // ---- stationary activations: x[m][seg·KS .. +KS) in the pairing the unpack uses
  uint32_t xr[M][XW];
  float xs[M][2];  // Σx over the segment (int4: [0]; q4_K: chunk 2p in [0], 2p+1 in [1])
  int q_sb = 0, q_p = 0;  // q4_K: super-block and run of this segment
  {
    const uint16_t* xg = reinterpret_cast<const uint16_t*>(p.x);
    int kbase = seg * KS;  // first k of this segment (int4, bf16)
    int kc0 = 0;           // q4_K: first k of this segment's slice of chunk 2p
    if constexpr (F == Fmt::Q4K || F == Fmt::Q4KDsc) {
      constexpr int SEGS_PER_SB = 256 / KS;
      q_sb = seg / SEGS_PER_SB;
      const int byte0 = (seg % SEGS_PER_SB) * (KS / 2);  // offset inside the 128 code bytes
      q_p = byte0 / 32;
      kc0 = q_sb * 256 + 64 * q_p + (byte0 % 32);
    }
#pragma unroll
    for (int m = 0; m < M; ++m) {
      xs[m][0] = 0.f;
      xs[m][1] = 0.f;
#pragma unroll
      for (int i = 0; i < XW; ++i) xr[m][i] = 0u;
      if (!active) continue;
      const uint16_t* xm = xg + static_cast<long long>(m) * p.K;
      if constexpr (F == Fmt::Int4) {
        // word wd covers k = kbase + 8wd .. +7; pairs (x0,x4) (x1,x5) (x2,x6) (x3,x7)
#pragma unroll
        for (int wd = 0; wd < WORDS; ++wd) {
          const uint4 v = *reinterpret_cast<const uint4*>(xm + kbase + 8 * wd);
          xr[m][4 * wd + 0] = __byte_perm(v.x, v.z, 0x5410);
          xr[m][4 * wd + 1] = __byte_perm(v.x, v.z, 0x7632);
          xr[m][4 * wd + 2] = __byte_perm(v.y, v.w, 0x5410);
          xr[m][4 * wd + 3] = __byte_perm(v.y, v.w, 0x7632);
          const __half* h = reinterpret_cast<const __half*>(&v);
#pragma unroll
          for (int e = 0; e < 8; ++e) xs[m][0] += __half2float(h[e]);
        }
      } else if constexpr (F == Fmt::Q4K || F == Fmt::Q4KDsc) {
        // word wd covers code bytes i..i+3 (i = 4wd): elements i..i+3 of both chunks;
        // pairs (c0[i], c0[i+2]) (c1[i], c1[i+2]) (c0[i+1], c0[i+3]) (c1[i+1], c1[i+3])
#pragma unroll
        for (int wd = 0; wd < WORDS; ++wd) {
          const uint2 a = *reinterpret_cast<const uint2*>(xm + kc0 + 4 * wd);
          const uint2 b = *reinterpret_cast<const uint2*>(xm + kc0 + 32 + 4 * wd);
          xr[m][4 * wd + 0] = __byte_perm(a.x, a.y, 0x5410);
          xr[m][4 * wd + 1] = __byte_perm(b.x, b.y, 0x5410);
          xr[m][4 * wd + 2] = __byte_perm(a.x, a.y, 0x7632);
          xr[m][4 * wd + 3] = __byte_perm(b.x, b.y, 0x7632);
          const __half* ha = reinterpret_cast<const __half*>(&a);
          const __half* hb = reinterpret_cast<const __half*>(&b);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            xs[m][0] += __half2float(ha[e]);
            xs[m][1] += __half2float(hb[e]);
          }
        }
      } else {  // BF16: natural pairs
#pragma unroll
        for (int i = 0; i < XW / 4; ++i) {
          const uint4 v = *reinterpret_cast<const uint4*>(xm + kbase + 8 * i);
          xr[m][4 * i + 0] = v.x;
          xr[m][4 * i + 1] = v.y;
          xr[m][4 * i + 2] = v.z;
          xr[m][4 * i + 3] = v.w;
        }
      }
    }
    if constexpr (F == Fmt::Int4) {
#pragma unroll
      for (int m = 0; m < M; ++m) xs[m][0] *= 5.9604644775390625e-08f;  // ·2^-24, matches the code scale
    }
  }

  const int int4_block = (F == Fmt::Int4) ? ((seg * KS) >> p.block_shift) : 0;
  // q4_K raw decode selectors for the chunk pair (2p, 2p+1)
  const uint32_t q_hp = static_cast<uint32_t>(q_p & 1);
  const uint32_t q_up = static_cast<uint32_t>(q_p >> 1);

  for (int s = 0; s < n_stages; ++s) {
    const int slot = s % p.NS;
    if (warp == 0 && s + p.NS - 1 < n_stages) {
      const int sn = s + p.NS - 1;
      const int r0n = row_begin + sn * p.RS;
      issue_stage<F>(p, smem + (sn % p.NS) * p.stage_bytes, &bars[sn % p.NS], r0n, min(p.RS, row_end - r0n),
                     lane, policy);
    }
    const int r0 = row_begin + s * p.RS;
    const int nr = min(p.RS, row_end - r0);
    const uint8_t* st = smem + slot * p.stage_bytes;

    if (!mbar_wait_bounded(&bars[slot], static_cast<uint32_t>((s / p.NS) & 1))) *abort_flag = 1;

    float acc_out[V];
#pragma unroll
    for (int i = 0; i < V; ++i) acc_out[i] = 0.f;

#pragma unroll
    for (int rr = 0; rr < RG; ++rr) {
      const int j = g + rr * p.G;  // row inside the stage
      if (active && rr < p.RG && j < nr) {
        const uint8_t* wrow = st + static_cast<long long>(j) * p.row_bytes;
        uint32_t wv[WORDS];
        if constexpr (F == Fmt::Int4) {
#pragma unroll
          for (int q = 0; q < WORDS; q += 4) {
            if constexpr (WORDS >= 4) {
              const uint4 t = *reinterpret_cast<const uint4*>(wrow + seg * SEG_BYTES + 4 * q);
              wv[q] = t.x; wv[q + 1] = t.y; wv[q + 2] = t.z; wv[q + 3] = t.w;
            }
          }
          if constexpr (WORDS == 2) {
            const uint2 t = *reinterpret_cast<const uint2*>(wrow + seg * SEG_BYTES);
            wv[0] = t.x; wv[1] = t.y;
          }
          if constexpr (WORDS == 1) wv[0] = *reinterpret_cast<const uint32_t*>(wrow + seg * SEG_BYTES);
        } else if constexpr (F == Fmt::Q4K || F == Fmt::Q4KDsc) {
          const uint8_t* qs = wrow + q_sb * 144 + 16 + (seg % (256 / KS)) * SEG_BYTES;
          // blocks are 144 B and the codes start at +16, so a segment of
          // SEG_BYTES is SEG_BYTES-aligned (up to 16)
          if constexpr (WORDS >= 4) {
#pragma unroll
            for (int q = 0; q < WORDS; q += 4) {
              const uint4 t = *reinterpret_cast<const uint4*>(qs + 4 * q);
              wv[q] = t.x; wv[q + 1] = t.y; wv[q + 2] = t.z; wv[q + 3] = t.w;
            }
          } else if constexpr (WORDS == 2) {
            const uint2 t = *reinterpret_cast<const uint2*>(qs);
            wv[0] = t.x; wv[1] = t.y;
          } else {
            wv[0] = *reinterpret_cast<const uint32_t*>(qs);
          }
        } else {
#pragma unroll
          for (int q = 0; q < WORDS; q += 4) {
            const uint4 t = *reinterpret_cast<const uint4*>(wrow + seg * SEG_BYTES + 4 * q);
            wv[q] = t.x; wv[q + 1] = t.y; wv[q + 2] = t.z; wv[q + 3] = t.w;
          }
        }

        float a[M][4];
#pragma unroll
        for (int m = 0; m < M; ++m) a[m][0] = a[m][1] = a[m][2] = a[m][3] = 0.f;

        if constexpr (kFour) {
#pragma unroll
          for (int q = 0; q < WORDS; ++q) {
            const uint32_t v = wv[q];
            const uint32_t v8 = v >> 8;
            const uint32_t p0 = lo4(v), p1 = hi4(v), p2 = lo4(v8), p3 = hi4(v8);
#pragma unroll
            for (int m = 0; m < M; ++m) {
              // ×1 positions into a[m][0..1], ×16 positions into a[m][2..3];
              // from M = 4 on the batch gives enough independent chains and
              // one accumulator per class keeps the register count down
              if constexpr (M >= 4) {
                mfma2_f16_1(a[m][0], p0, xr[m][4 * q + 0]);
                mfma2_f16_1(a[m][2], p1, xr[m][4 * q + 1]);
                mfma2_f16_1(a[m][0], p2, xr[m][4 * q + 2]);
                mfma2_f16_1(a[m][2], p3, xr[m][4 * q + 3]);
              } else {
                mfma2_f16(a[m][0], a[m][1], p0, xr[m][4 * q + 0]);
                mfma2_f16(a[m][2], a[m][3], p1, xr[m][4 * q + 1]);
                mfma2_f16(a[m][0], a[m][1], p2, xr[m][4 * q + 2]);
                mfma2_f16(a[m][2], a[m][3], p3, xr[m][4 * q + 3]);
              }
            }
          }
        } else {
#pragma unroll
          for (int q = 0; q < WORDS; ++q) {
#pragma unroll
            for (int m = 0; m < M; ++m) {
              if constexpr (M >= 4) {
                mfma2_bf16_1(a[m][(q & 1) * 2], wv[q], xr[m][q]);
              } else {
                if (q & 1)
                  mfma2_bf16(a[m][2], a[m][3], wv[q], xr[m][q]);
                else
                  mfma2_bf16(a[m][0], a[m][1], wv[q], xr[m][q]);
              }
            }
          }
        }

        // ---- per-segment coefficients and fold into the row's partial sums
        if constexpr (F == Fmt::Int4) {
          const int jrow = j;
          const uint8_t* sc_base = st + p.off_scales + aligned_down16(reinterpret_cast<uint64_t>(p.scales) +
                                                                      2ull * p.nb * r0);
          const uint16_t sbits = reinterpret_cast<const uint16_t*>(sc_base)[jrow * p.nb + int4_block];
          const float s24 = h16_to_f32(sbits) * 16777216.0f;  // ·2^24 undoes the code scale
          float z = 8.0f;
          if (p.zeros) {
            const uint8_t* z_base =
                st + p.off_zeros + aligned_down16(reinterpret_cast<uint64_t>(p.zeros) + 1ull * p.zb * r0);
            const uint32_t zbyte = z_base[jrow * p.zb + (int4_block >> 1)];
            z = static_cast<float>((zbyte >> ((int4_block & 1) * 4)) & 15u);
          }
#pragma unroll
          for (int m = 0; m < M; ++m) {
            const float lo = a[m][0] + a[m][1];
            const float hi = a[m][2] + a[m][3];
            const float t = fmaf(hi, 0.0625f, lo);      // Σ q·x · 2^-24
            const float u = fmaf(-z, xs[m][0], t);     // Σ (q − z)·x · 2^-24
            acc_out[rr * M + m] = fmaf(s24, u, acc_out[rr * M + m]);
          }
        } else if constexpr (F == Fmt::Q4K || F == Fmt::Q4KDsc) {
          float A0, A1, B0, B1;  // A·2^24 / A·2^20 for the two code scales, B plain
          if constexpr (F == Fmt::Q4K) {
            const uint4 h = *reinterpret_cast<const uint4*>(wrow + q_sb * 144);
            uint32_t sc2, mn2;
            q4k_scale_min_pair(h.y, h.z, h.w, q_hp, q_up, sc2, mn2);
            const float d = h16_to_f32(h.x);
            const float dmin = h16_to_f32(h.x >> 16);
            const float sc0 = __uint_as_float(0x4B000000u | (sc2 & 0xFFu)) - 8388608.0f;
            const float sc1 = __uint_as_float(0x4B000000u | (sc2 >> 8)) - 8388608.0f;
            const float mn0 = __uint_as_float(0x4B000000u | (mn2 & 0xFFu)) - 8388608.0f;
            const float mn1 = __uint_as_float(0x4B000000u | (mn2 >> 8)) - 8388608.0f;
            A0 = (d * sc0) * 16777216.0f;
            A1 = (d * sc1) * 1048576.0f;
            B0 = -(dmin * mn0);
            B1 = -(dmin * mn1);
          } else {
            const int c0 = q_sb * 8 + 2 * q_p;
            const uint8_t* pl = st + p.off_plane;
            const uint64_t a0 = reinterpret_cast<uint64_t>(p.plane) + (static_cast<uint64_t>(c0) * p.N + r0) * 8ull;
            const uint64_t a1 = a0 + static_cast<uint64_t>(p.N) * 8ull;
            const float2 P0 = *reinterpret_cast<const float2*>(pl + c0 * p.plane_stride + (a0 & 15u) + j * 8);
            const float2 P1 = *reinterpret_cast<const float2*>(pl + (c0 + 1) * p.plane_stride + (a1 & 15u) + j * 8);
            A0 = P0.x * 16777216.0f;
            A1 = P1.x * 1048576.0f;
            B0 = P0.y;
            B1 = P1.y;
          }
#pragma unroll
          for (int m = 0; m < M; ++m) {
            float o = acc_out[rr * M + m];
            o = fmaf(A0, a[m][0] + a[m][1], o);
            o = fmaf(A1, a[m][2] + a[m][3], o);
            o = fmaf(B0, xs[m][0], o);
            o = fmaf(B1, xs[m][1], o);
            acc_out[rr * M + m] = o;
          }
        } else {
#pragma unroll
          for (int m = 0; m < M; ++m) acc_out[rr * M + m] += (a[m][0] + a[m][1]) + (a[m][2] + a[m][3]);
        }
      }
    }

    // ---- reduce over the warp, then over the WK warps of the row group
    warp_reduce_scatter<V>(acc_out, lane);
    float* redb = red + (s & 1) * (p.RS * p.WK * M);
    constexpr int SH = 5 - ilog2(V);
    if ((lane & ((1 << SH) - 1)) == 0) {
      const int idx = lane >> SH;
      if (idx < RG * M) {
        const int rr = idx / M, m = idx - rr * M;
        const int j = g + rr * p.G;
        if (j < p.RS) redb[(j * p.WK + kw) * M + m] = acc_out[0];
      }
    }
    __syncthreads();
    if (*abort_flag) break;
    for (int t = tid; t < nr * M; t += blockDim.x) {
      const int j = t / M, m = t - j * M;
      float sum = 0.f;
      for (int w2 = 0; w2 < p.WK; ++w2) sum += redb[(j * p.WK + w2) * M + m];
      const long long o = static_cast<long long>(m) * p.N + (r0 + j);
      if constexpr (F == Fmt::BF16)
        reinterpret_cast<__nv_bfloat16*>(p.y)[o] = __float2bfloat16_rn(sum);
      else
        reinterpret_cast<__half*>(p.y)[o] = __float2half_rn(sum);
    }
  }
  if (*abort_flag && tid == 0) {
    // A wait gave up: before the CTA exits, give every stage that was issued
    // and not yet consumed a bounded chance to land in shared memory.
    for (int t = 0; t < n_stages; ++t) {
      if (!mbar_try_wait(&bars[t % p.NS], static_cast<uint32_t>((t / p.NS) & 1))) {
        if (t < n_stages && t >= 0) (void)mbar_wait_bounded(&bars[t % p.NS], static_cast<uint32_t>((t / p.NS) & 1));
        break;
      }
    }
  }
}

}  // namespace wq
