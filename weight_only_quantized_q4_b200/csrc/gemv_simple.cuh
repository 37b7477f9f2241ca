// gemv_simple.cuh — general-shape kernels: the fallback GEMV (any alignment,
// any K, any M in chunks of 8), the dequantization exports and the device
// W_dsc plane builder.
//
// The exports walk the codes exactly the way the streaming GEMV does (one
// 32-bit word -> four fp16x2 subnormal code pairs via lo4/hi4, q4_K chunk
// pairs via q4k_scale_min_pair), then widen each code exactly to fp32, so a
// bit-exact comparison of the export against the oracle checks the unpacking
// and coefficient decoding the fast kernels rely on.
#pragma once

#include "wq_device.cuh"
#include "gemv_cc.cuh"

namespace wq {

// B200_V1 stores the eight codes of a word in the order k0 k2 k4 k6 k1 k3 k5 k7
// (nibble positions 0..7), so that the pair extractions lo4 / hi4 / lo4(>>8) /
// hi4(>>8) yield (k0,k1) (k2,k3) (k4,k5) (k6,k7): consecutive activation
// pairs.  Nibble position of code k (0..7) inside such a word:
__host__ __device__ __forceinline__ int int4_v1_nibble_pos(int k) { return (k >> 1) | ((k & 1) << 2); }

// B200_V1 int4 stream geometry (see include/wq.h): bands of 16 rows, K/128
// tiles per band, each tile = 1024 code bytes + bpt·16 fp16 scales + bpt·8
// zero-point bytes, padded to 16 bytes.
__host__ __device__ __forceinline__ int int4_v1_bpt(int bs) { return bs >= 128 ? 1 : 128 / bs; }
__host__ __device__ __forceinline__ int int4_v1_tile_bytes(int bs) {
  return (1024 + int4_v1_bpt(bs) * 40 + 15) / 16 * 16;
}
__host__ __device__ __forceinline__ long long int4_v1_tile_offset(long long row, int k, int K, int bs) {
  return ((row >> 4) * (K / 128) + (k >> 7)) * static_cast<long long>(int4_v1_tile_bytes(bs));
}
// Byte offset of the 32-bit code word covering k = k8 .. k8+7 (k8 % 8 == 0) of `row`.
__host__ __device__ __forceinline__ long long int4_v1_word_offset(long long row, int k8, int K, int bs) {
  const int r = static_cast<int>(row & 15);
  const int g = r & 7, r8 = r >> 3;
  const int kk = k8 & 127;
  const int gi = kk >> 5, t = (kk & 31) >> 3;
  return int4_v1_tile_offset(row, k8, K, bs) + (gi >> 1) * 512 + (4 * g + t) * 16 + 4 * (2 * (gi & 1) + r8);
}
// Block slot inside a tile for k (0 when blocks span >= 128 k).
__host__ __device__ __forceinline__ int int4_v1_block_in_tile(int k, int bs) { return bs >= 128 ? 0 : (k & 127) / bs; }
__host__ __device__ __forceinline__ long long int4_v1_scale_offset(long long row, int k, int K, int bs) {
  return int4_v1_tile_offset(row, k, K, bs) + 1024 + (int4_v1_block_in_tile(k, bs) * 16 + (row & 15)) * 2;
}
__host__ __device__ __forceinline__ long long int4_v1_zero_offset(long long row, int k, int K, int bs) {
  return int4_v1_tile_offset(row, k, K, bs) + 1024 + 32 * int4_v1_bpt(bs) + int4_v1_block_in_tile(k, bs) * 8 +
         ((row & 15) >> 1);
}

// B200_V1 q4_K stream geometry (see include/wq.h): bands of 16 rows, K/256
// tiles per band, one super-block of the band's rows per tile, 2304 bytes:
// 2048 code bytes in warp-MMA fragment order (the int4 B200_V1 code order over
// eight 32-k groups, group = chunk), 16 (d, dmin) fp16 pairs, then 64 24-bit
// scale entries: entry (pair p, row r) at 2112 + 3·(16p + r) holds
// sc_{2p} | sc_{2p+1} << 6 | m_{2p} << 12 | m_{2p+1} << 18.
constexpr int kQ4KV1TileBytes = 2304;
__host__ __device__ __forceinline__ long long q4k_v1_tile_offset(long long row, int k, int K) {
  return ((row >> 4) * (K / 256) + (k >> 8)) * static_cast<long long>(kQ4KV1TileBytes);
}
__host__ __device__ __forceinline__ long long q4k_v1_word_offset(long long row, int k8, int K) {
  const int r = static_cast<int>(row & 15);
  const int g = r & 7, r8 = r >> 3;
  const int kk = k8 & 255;
  const int gi = kk >> 5, t = (kk & 31) >> 3;
  return q4k_v1_tile_offset(row, k8, K) + (gi >> 1) * 512 + (4 * g + t) * 16 + 4 * (2 * (gi & 1) + r8);
}
__host__ __device__ __forceinline__ long long q4k_v1_dd_offset(long long row, int k, int K) {
  return q4k_v1_tile_offset(row, k, K) + 2048 + 4 * (row & 15);
}
__host__ __device__ __forceinline__ long long q4k_v1_entry_offset(long long row, int k, int K) {
  const int c = (k & 255) >> 5;
  return q4k_v1_tile_offset(row, k, K) + 2112 + 3 * (16 * (c >> 1) + (row & 15));
}
// The 24-bit entry of (pair, row) from three bytes.
__device__ __forceinline__ uint32_t q4k_v1_entry(const uint8_t* e) {
  return static_cast<uint32_t>(e[0]) | (static_cast<uint32_t>(e[1]) << 8) | (static_cast<uint32_t>(e[2]) << 16);
}

struct SimpleParams {
  const void* x;
  const uint8_t* w;
  const uint8_t* scales;
  const uint8_t* zeros;
  const uint8_t* plane;
  void* y;
  int M, N, K;
  int nb, zb, block_shift;
  int layout;  // int4: 0 canonical, 1 B200_V1 (codes, scales and zero-points all in w)
};

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b16) { return __uint_as_float((b16 & 0xFFFFu) << 16); }

// Exact fp32 weight W[row, k] for the scalar fallback (plain byte reads).
template <Fmt F>
__device__ __forceinline__ float weight_scalar(const SimpleParams& p, int row, int k) {
  if constexpr (F == Fmt::Int4) {
    uint32_t q, sb, z = 8u;
    if (p.layout == 1) {
      const int bs = 1 << p.block_shift;
      const int pos = int4_v1_nibble_pos(k & 7);
      const uint32_t byte = p.w[int4_v1_word_offset(row, k & ~7, p.K, bs) + (pos >> 1)];
      q = (pos & 1) ? (byte >> 4) : (byte & 15u);
      sb = *reinterpret_cast<const uint16_t*>(p.w + int4_v1_scale_offset(row, k, p.K, bs));
      const uint32_t zbyte = p.w[int4_v1_zero_offset(row, k, p.K, bs)];
      z = (row & 1) ? (zbyte >> 4) : (zbyte & 15u);
    } else {
      const uint32_t byte = p.w[static_cast<long long>(row) * (p.K / 2) + (k >> 1)];
      q = (k & 1) ? (byte >> 4) : (byte & 15u);
      const int b = k >> p.block_shift;
      sb = reinterpret_cast<const uint16_t*>(p.scales)[static_cast<long long>(row) * p.nb + b];
      if (p.zeros) {
        const uint32_t zb = p.zeros[static_cast<long long>(row) * p.zb + (b >> 1)];
        z = (b & 1) ? (zb >> 4) : (zb & 15u);
      }
    }
    return static_cast<float>(static_cast<int>(q) - static_cast<int>(z)) * h16_to_f32(sb);
  } else if constexpr (F == Fmt::Q4K || F == Fmt::Q4KDsc) {
    if (F == Fmt::Q4K && p.layout == 1) {
      const int pos = int4_v1_nibble_pos(k & 7);
      const uint32_t byte = p.w[q4k_v1_word_offset(row, k & ~7, p.K) + (pos >> 1)];
      const uint32_t q = (pos & 1) ? (byte >> 4) : (byte & 15u);
      const uint32_t dd = *reinterpret_cast<const uint32_t*>(p.w + q4k_v1_dd_offset(row, k, p.K));
      const uint32_t ent = q4k_v1_entry(p.w + q4k_v1_entry_offset(row, k, p.K));
      const int hi = ((k & 255) >> 5) & 1;
      const uint32_t sc = (ent >> (6 * hi)) & 63u, mn = (ent >> (12 + 6 * hi)) & 63u;
      const float A = __fmul_rn(h16_to_f32(dd), static_cast<float>(sc));
      const float B = -__fmul_rn(h16_to_f32(dd >> 16), static_cast<float>(mn));
      return fmaf(A, static_cast<float>(q), B);
    }
    const uint8_t* blk = p.w + (static_cast<long long>(row) * (p.K / 256) + (k >> 8)) * 144;
    const int e = k & 255;
    const int c = e >> 5;
    const uint32_t byte = blk[16 + 32 * (e >> 6) + (e & 31)];
    const uint32_t q = (e & 32) ? (byte >> 4) : (byte & 15u);
    float A, B;
    if constexpr (F == Fmt::Q4K) {
      const uint32_t* hw = reinterpret_cast<const uint32_t*>(blk);
      uint32_t sc, mn;
      q4k_scale_min(hw[1], hw[2], hw[3], c, sc, mn);
      A = __fmul_rn(h16_to_f32(hw[0]), static_cast<float>(sc));
      B = -__fmul_rn(h16_to_f32(hw[0] >> 16), static_cast<float>(mn));
    } else {
      const float2 P = reinterpret_cast<const float2*>(p.plane)[static_cast<long long>((k >> 5)) * p.N + row];
      A = P.x;
      B = P.y;
    }
    return fmaf(A, static_cast<float>(q), B);
  } else {
    return bf16_bits_to_f32(reinterpret_cast<const uint16_t*>(p.w)[static_cast<long long>(row) * p.K + k]);
  }
}

template <Fmt F>
__device__ __forceinline__ float act_scalar(const SimpleParams& p, int m, int k) {
  const uint16_t b = reinterpret_cast<const uint16_t*>(p.x)[static_cast<long long>(m) * p.K + k];
  if constexpr (F == Fmt::BF16)
    return bf16_bits_to_f32(b);
  else
    return h16_to_f32(b);
}

// One warp per row (grid-stride), lanes stride over K, fp32 products and sums.
template <Fmt F, int M>
__global__ void __launch_bounds__(256) gemv_simple_kernel(const SimpleParams p) {
  const int lane = threadIdx.x & 31;
  const long long warp = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const long long n_warps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
  for (long long row = warp; row < p.N; row += n_warps) {
    float acc[M];
#pragma unroll
    for (int m = 0; m < M; ++m) acc[m] = 0.f;
    for (int k = lane; k < p.K; k += 32) {
      const float wv = weight_scalar<F>(p, static_cast<int>(row), k);
#pragma unroll
      for (int m = 0; m < M; ++m) acc[m] = fmaf(wv, act_scalar<F>(p, m, k), acc[m]);
    }
#pragma unroll
    for (int m = 0; m < M; ++m) {
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) acc[m] += __shfl_xor_sync(0xffffffffu, acc[m], off);
    }
    if (lane == 0) {
#pragma unroll
      for (int m = 0; m < M; ++m) {
        const long long o = static_cast<long long>(m) * p.N + row;
        if constexpr (F == Fmt::BF16)
          reinterpret_cast<__nv_bfloat16*>(p.y)[o] = __float2bfloat16_rn(acc[m]);
        else
          reinterpret_cast<__half*>(p.y)[o] = __float2half_rn(acc[m]);
      }
    }
  }
}

// ---------------------------------------------------------------------------
// dequantization exports (fp32 [N, K]); one thread per 32-bit word of codes
// ---------------------------------------------------------------------------

// Exact value of a code held as a subnormal in half `h` of a pair produced by
// lo4 (scale 2^-24) or hi4 (scale 2^-20).
__device__ __forceinline__ float code_of(uint32_t pair, int h, bool high_class) {
  const float v = h16_to_f32(pair >> (16 * h));
  return high_class ? v * 1048576.0f : v * 16777216.0f;
}

__global__ void dequant_int4_kernel(const uint8_t* w, const uint8_t* scales, const uint8_t* zeros, float* out,
                                    int N, int K, int nb, int zb, int block_shift, int layout) {
  const long long words_per_row = K / 8;
  const long long total = static_cast<long long>(N) * words_per_row;
  for (long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; t < total;
       t += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long row = t / words_per_row;
    const int wd = static_cast<int>(t - row * words_per_row);
    const int bs = 1 << block_shift;
    const uint32_t v = layout == 1 ? *reinterpret_cast<const uint32_t*>(w + int4_v1_word_offset(row, 8 * wd, K, bs))
                                   : reinterpret_cast<const uint32_t*>(w + row * (K / 2))[wd];
    // pairs by nibble position: (p0,p4) (p1,p5) (p2,p6) (p3,p7)
    const uint32_t pr[4] = {lo4(v), hi4(v), lo4(v >> 8), hi4(v >> 8)};
    const int k0 = 8 * wd;
    const int b = k0 >> block_shift;  // a word never straddles a block (block >= 16)
    float s, z = 8.f;
    if (layout == 1) {
      s = h16_to_f32(*reinterpret_cast<const uint16_t*>(w + int4_v1_scale_offset(row, k0, K, bs)));
      const uint32_t zbyte = w[int4_v1_zero_offset(row, k0, K, bs)];
      z = static_cast<float>((row & 1) ? (zbyte >> 4) : (zbyte & 15u));
    } else {
      s = h16_to_f32(reinterpret_cast<const uint16_t*>(scales)[row * nb + b]);
      if (zeros) {
        const uint32_t zbyte = zeros[row * zb + (b >> 1)];
        z = static_cast<float>((b & 1) ? (zbyte >> 4) : (zbyte & 15u));
      }
    }
    float* o = out + row * K + k0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const bool high = (i & 1) != 0;
      const int p0 = (i >> 1) * 2 + (high ? 1 : 0);  // nibble position of the pair's low half
      // canonical: position == k; B200_V1: position p holds k = 2·(p & 3) + (p >> 2)
      const int e0 = layout == 1 ? 2 * (p0 & 3) + (p0 >> 2) : p0;
      const int e1 = layout == 1 ? 2 * ((p0 + 4) & 3) + ((p0 + 4) >> 2) : p0 + 4;
      o[e0] = (code_of(pr[i], 0, high) - z) * s;
      o[e1] = (code_of(pr[i], 1, high) - z) * s;
    }
  }
}

// q4_K: thread per 32-bit word of codes; word t of block covers code bytes
// 4t'..4t'+3 of run p, i.e. elements i..i+3 of chunks 2p and 2p+1.
__global__ void dequant_q4k_kernel(const uint8_t* w, const uint8_t* plane, float* out, int N, int K) {
  const long long words_per_row = (K / 256) * 32;
  const long long total = static_cast<long long>(N) * words_per_row;
  for (long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; t < total;
       t += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long row = t / words_per_row;
    const int wr = static_cast<int>(t - row * words_per_row);
    const int sb = wr >> 5;
    const int wq = wr & 31;            // word inside the 128 code bytes
    const int pp = wq >> 3;            // run
    const int i = (wq & 7) * 4;        // first element inside the chunk
    const uint8_t* blk = w + (row * (K / 256) + sb) * 144;
    const uint32_t v = reinterpret_cast<const uint32_t*>(blk + 16)[wq];
    float A0, A1, B0, B1;
    if (plane) {
      const int c0 = sb * 8 + 2 * pp;
      const float2 P0 = reinterpret_cast<const float2*>(plane)[static_cast<long long>(c0) * N + row];
      const float2 P1 = reinterpret_cast<const float2*>(plane)[static_cast<long long>(c0 + 1) * N + row];
      A0 = P0.x; B0 = P0.y; A1 = P1.x; B1 = P1.y;
    } else {
      const uint32_t* hw = reinterpret_cast<const uint32_t*>(blk);
      uint32_t sc2, mn2;
      q4k_scale_min_pair(hw[1], hw[2], hw[3], static_cast<uint32_t>(pp & 1), static_cast<uint32_t>(pp >> 1), sc2,
                         mn2);
      const float d = h16_to_f32(hw[0]);
      const float dmin = h16_to_f32(hw[0] >> 16);
      A0 = __fmul_rn(d, static_cast<float>(sc2 & 0xFFu));
      A1 = __fmul_rn(d, static_cast<float>(sc2 >> 8));
      B0 = -__fmul_rn(dmin, static_cast<float>(mn2 & 0xFFu));
      B1 = -__fmul_rn(dmin, static_cast<float>(mn2 >> 8));
    }
    // pairs: lo4(v) = (c0[i], c0[i+2]); hi4(v) = (c1[i], c1[i+2]);
    //        lo4(v>>8) = (c0[i+1], c0[i+3]); hi4(v>>8) = (c1[i+1], c1[i+3])
    const uint32_t p0 = lo4(v), p1 = hi4(v), p2 = lo4(v >> 8), p3 = hi4(v >> 8);
    float* o0 = out + row * K + sb * 256 + 64 * pp + i;  // chunk 2p
    float* o1 = o0 + 32;                                 // chunk 2p+1
    o0[0] = fmaf(A0, code_of(p0, 0, false), B0);
    o0[2] = fmaf(A0, code_of(p0, 1, false), B0);
    o0[1] = fmaf(A0, code_of(p2, 0, false), B0);
    o0[3] = fmaf(A0, code_of(p2, 1, false), B0);
    o1[0] = fmaf(A1, code_of(p1, 0, true), B1);
    o1[2] = fmaf(A1, code_of(p1, 1, true), B1);
    o1[1] = fmaf(A1, code_of(p3, 0, true), B1);
    o1[3] = fmaf(A1, code_of(p3, 1, true), B1);
  }
}

// Canonical int4 -> B200_V1, codes: thread per 16-byte code chunk of a tile
// (rows past N get zero codes).  Tile i of the stream is written at tile slot
// i·tile_mul + tile_add of `out` (1, 0 for a plain stream; 2, 0 / 2, 1 for the
// gate / up halves of the fused gate-up stream).
__global__ void repack_int4_v1_codes_kernel(const uint8_t* w, uint8_t* out, int N, int K, int bs, int tile_mul = 1,
                                            int tile_add = 0) {
  const long long n_bands = (N + 15) / 16;
  const int tpb = K / 128;
  const int tb = int4_v1_tile_bytes(bs);
  const long long chunks = n_bands * tpb * 64;
  for (long long c = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; c < chunks;
       c += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long tile = c >> 6;  // band * tpb + s
    const int q = static_cast<int>(c & 63);
    const long long band = tile / tpb;
    const int s = static_cast<int>(tile - band * tpb);
    const int h = q >> 5, lane = q & 31;
    const int g = lane >> 2, t = lane & 3;
    uint32_t v[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int gi = 2 * h + (j >> 1), r8 = j & 1;
      const long long row = 16 * band + g + 8 * r8;
      const int k = 128 * s + 32 * gi + 8 * t;
      const uint32_t cw = row < N ? *reinterpret_cast<const uint32_t*>(w + row * (K / 2) + k / 2) : 0u;
      uint32_t o = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) o |= ((cw >> (4 * e)) & 15u) << (4 * int4_v1_nibble_pos(e));
      v[j] = o;
    }
    *reinterpret_cast<uint4*>(out + (tile * tile_mul + tile_add) * tb + q * 16) = make_uint4(v[0], v[1], v[2], v[3]);
  }
}

// Canonical int4 -> B200_V1, metadata: thread per (tile, block slot, row pair):
// the two rows' fp16 scales and their shared zero-point byte (pads: scale 0,
// zero-point 8); the 16-byte tail padding of a tile is zeroed by slot 0.
__global__ void repack_int4_v1_meta_kernel(const uint8_t* scales, const uint8_t* zeros, uint8_t* out, int N, int K,
                                           int bs, int tile_mul = 1, int tile_add = 0) {
  const long long n_bands = (N + 15) / 16;
  const int tpb = K / 128;
  const int bpt = int4_v1_bpt(bs);
  const int tb = int4_v1_tile_bytes(bs);
  const int nb = (K + bs - 1) / bs, zb = (nb + 1) / 2;  // a shorter last block is allowed
  const long long items = n_bands * tpb * bpt * 8;
  for (long long it = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; it < items;
       it += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int rp = static_cast<int>(it & 7);
    const long long rest = it >> 3;
    const int bt = static_cast<int>(rest % bpt);
    const long long tile = rest / bpt;
    const long long band = tile / tpb;
    const int s = static_cast<int>(tile - band * tpb);
    const int blk = (128 * s + bt * (bs < 128 ? bs : 0)) / bs;
    uint8_t* tp = out + (tile * tile_mul + tile_add) * tb;
    uint32_t zbyte = 0;
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int r = 2 * rp + e;
      const long long row = 16 * band + r;
      uint16_t sv = 0;
      uint32_t z = 8u;
      if (row < N) {
        sv = reinterpret_cast<const uint16_t*>(scales)[row * nb + blk];
        if (zeros) z = (zeros[row * zb + (blk >> 1)] >> ((blk & 1) * 4)) & 15u;
      }
      reinterpret_cast<uint16_t*>(tp + 1024)[bt * 16 + r] = sv;
      zbyte |= z << (4 * e);
    }
    tp[1024 + 32 * bpt + bt * 8 + rp] = static_cast<uint8_t>(zbyte);
    if (bt == 0 && rp == 0)
      for (int o = 1024 + 40 * bpt; o < tb; ++o) tp[o] = 0;
  }
}

// q4_K B200_V1 export: thread per 32-bit code word (8 codes of one chunk of
// one row), coefficients from the tile's (d, dmin) pair and 24-bit entry.
__global__ void dequant_q4k_v1_kernel(const uint8_t* w, float* out, int N, int K) {
  const long long words_per_row = K / 8;
  const long long total = static_cast<long long>(N) * words_per_row;
  for (long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; t < total;
       t += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long row = t / words_per_row;
    const int k0 = 8 * static_cast<int>(t - row * words_per_row);
    const uint32_t v = *reinterpret_cast<const uint32_t*>(w + q4k_v1_word_offset(row, k0, K));
    const uint32_t dd = *reinterpret_cast<const uint32_t*>(w + q4k_v1_dd_offset(row, k0, K));
    const uint32_t ent = q4k_v1_entry(w + q4k_v1_entry_offset(row, k0, K));
    const int hi = ((k0 & 255) >> 5) & 1;
    const float A = __fmul_rn(h16_to_f32(dd), static_cast<float>((ent >> (6 * hi)) & 63u));
    const float B = -__fmul_rn(h16_to_f32(dd >> 16), static_cast<float>((ent >> (12 + 6 * hi)) & 63u));
    // pairs by nibble position (p0,p4) (p1,p5) (p2,p6) (p3,p7); position p holds code e = 2·(p & 3) + (p >> 2)
    const uint32_t pr[4] = {lo4(v), hi4(v), lo4(v >> 8), hi4(v >> 8)};
    float* o = out + row * K + k0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const bool high = (i & 1) != 0;
      const int p0 = (i >> 1) * 2 + (high ? 1 : 0);
      const int e0 = 2 * (p0 & 3) + (p0 >> 2), e1 = 2 * ((p0 + 4) & 3) + ((p0 + 4) >> 2);
      o[e0] = fmaf(A, code_of(pr[i], 0, high), B);
      o[e1] = fmaf(A, code_of(pr[i], 1, high), B);
    }
  }
}

// Canonical q4_K -> B200_V1, codes: thread per 16-byte code chunk of a tile
// (128 per tile; rows past N get zero codes).
__global__ void repack_q4k_v1_codes_kernel(const uint8_t* w, uint8_t* out, int N, int K) {
  const long long n_bands = (N + 15) / 16;
  const int tpb = K / 256;
  const long long chunks = n_bands * tpb * 128;
  for (long long c = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; c < chunks;
       c += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long tile = c >> 7;  // band * tpb + sb
    const int q = static_cast<int>(c & 127);
    const long long band = tile / tpb;
    const int sb = static_cast<int>(tile - band * tpb);
    const int h = q >> 5, lane = q & 31;
    const int g = lane >> 2, t = lane & 3;
    uint32_t v[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int gi = 2 * h + (j >> 1), r8 = j & 1;  // gi = chunk of the super-block
      const long long row = 16 * band + g + 8 * r8;
      uint32_t o = 0;
      if (row < N) {
        const uint8_t* qs = w + (row * tpb + sb) * 144 + 16 + 32 * (gi >> 1) + 8 * t;
        const int sh = 4 * (gi & 1);  // even chunk: low nibbles of its run, odd: high
#pragma unroll
        for (int e = 0; e < 8; ++e) o |= ((static_cast<uint32_t>(qs[e]) >> sh) & 15u) << (4 * int4_v1_nibble_pos(e));
      }
      v[j] = o;
    }
    *reinterpret_cast<uint4*>(out + tile * kQ4KV1TileBytes + q * 16) = make_uint4(v[0], v[1], v[2], v[3]);
  }
}

// Canonical q4_K -> B200_V1, coefficients: thread per (tile, row): the row's
// (d, dmin) word and its four 24-bit (scale, min) pair entries (zeros for pad rows).
__global__ void repack_q4k_v1_meta_kernel(const uint8_t* w, uint8_t* out, int N, int K) {
  const long long n_bands = (N + 15) / 16;
  const int tpb = K / 256;
  const long long items = n_bands * tpb * 16;
  for (long long it = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; it < items;
       it += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int r = static_cast<int>(it & 15);
    const long long tile = it >> 4;
    const long long band = tile / tpb;
    const int sb = static_cast<int>(tile - band * tpb);
    const long long row = 16 * band + r;
    uint8_t* tp = out + tile * kQ4KV1TileBytes;
    uint32_t dd = 0, e[4] = {0u, 0u, 0u, 0u};
    if (row < N) {
      const uint32_t* hw = reinterpret_cast<const uint32_t*>(w + (row * tpb + sb) * 144);
      dd = hw[0];
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        uint32_t s0, m0, s1, m1;
        q4k_scale_min(hw[1], hw[2], hw[3], 2 * p, s0, m0);
        q4k_scale_min(hw[1], hw[2], hw[3], 2 * p + 1, s1, m1);
        e[p] = s0 | (s1 << 6) | (m0 << 12) | (m1 << 18);
      }
    }
    *reinterpret_cast<uint32_t*>(tp + 2048 + 4 * r) = dd;
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      uint8_t* ep = tp + 2112 + 3 * (16 * p + r);
      ep[0] = static_cast<uint8_t>(e[p]);
      ep[1] = static_cast<uint8_t>(e[p] >> 8);
      ep[2] = static_cast<uint8_t>(e[p] >> 16);
    }
  }
}

// W_dsc plane on the device (minfer doc 62, §2.2-§2.3): thread per (chunk, row).
__global__ void build_q4k_dsc_kernel(const uint8_t* w, float2* plane, int N, int K) {
  const long long n_chunks = K / 32;
  const long long total = n_chunks * N;
  for (long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; t < total;
       t += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long c = t / N;
    const long long row = t - c * N;
    const uint32_t* hw = reinterpret_cast<const uint32_t*>(w + (row * (K / 256) + c / 8) * 144);
    uint32_t sc, mn;
    q4k_scale_min(hw[1], hw[2], hw[3], static_cast<int>(c & 7), sc, mn);
    const float px = __fmul_rn(h16_to_f32(hw[0]), static_cast<float>(sc));
    const float py = -__fmul_rn(h16_to_f32(hw[0] >> 16), static_cast<float>(mn));
    plane[t] = make_float2(px, py);
  }
}

// Test hook for the failure path of bounded waits: one thread waits on an
// mbarrier that nothing arrives at (no copy in flight), gives up after
// limit_ns and records the timeout in the device error word, as a real wait
// that gives up does; the kernel then returns normally.
__global__ void expire_wait_kernel(unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait_bounded_ns(&bar, 0u, limit_ns);
  __syncthreads();
}

}  // namespace wq
