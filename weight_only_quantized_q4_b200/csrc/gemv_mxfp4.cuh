// gemv_mxfp4.cuh — decode GEMV (M = 1..8) for mxfp4 blockwise weights.
//
// Format (onnx-genai PR #1000, CPU criterion bench block: the mxfp4
// block-quantized matmul rows; the page does not print the format, the
// reading is the OCP microscaling FP4 definition): blocks of 32 elements
// along K share one E8M0 scale byte E (value 2^(E - 127), 255 = NaN); each
// element is a 4-bit E2M1 code (sign, 2-bit exponent with bias 1, 1-bit
// mantissa).  Codes [N][K/2], two per byte, low nibble = even k (the int4
// layout); scales [N][K/32] bytes.
//
// y[m][n] = Σ_b 2^(E[n][b] - 127) · Σ_{k in b} e2m1(q[n][k]) · x[m][k]
//
// How.  One warp-level MMA (m16n8k16, fp16 × fp16 -> fp32) per 16 k of a
// 16-row band: every code byte (two consecutive k of one row) becomes an fp16
// pair with one cvt.rn.f16x2.e2m1x2 — exact, E2M1 values are fp16 values —
// and the activations are the fp16 x as stored.  Each 32-k block gets its own
// fp32 accumulator fragment (two MMAs), multiplied by the block's power-of-two
// scale and added to the running sum: the products are exact in fp32 and the
// scale is applied in fp32 (fp16 could not hold 2^-127 .. 2^127).
//
// The k order inside an MMA is a permutation of the block's 32 k, the same
// for the A and B operands: lane (g, t) holds the code bytes 4t .. 4t+3 of
// rows g and g+8 (k = 8t .. 8t+7) and the activations x[g][8t .. 8t+7], so
// every load is one 32-bit word of codes per row and one 16-byte word of x.
//
// Work split: a CTA of W warps owns one band; warp w takes blocks w, w + W,
// ... and the W partial fragments are added in fixed warp order through
// shared memory (deterministic).  Loads are plain cached global loads; the
// warps of all resident CTAs keep the weight stream in flight.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

#include "wq_device.cuh"

namespace wq {

struct MXParams {
  const void* x;          // [M][K] fp16
  const uint8_t* w;       // codes [N][K/2]
  const uint8_t* scales;  // E8M0 [N][K/32]
  void* y;                // [M][N] fp16
  int M, N, K;
};

constexpr int kMXWarps = 8;

// Two E2M1 codes (one byte: low nibble first) -> fp16 pair (low half = low nibble).
__device__ __forceinline__ uint32_t e2m1x2_to_f16x2(uint32_t byte) {
  uint32_t r;
  asm("{\n .reg .b8 b;\n cvt.u8.u32 b, %1;\n cvt.rn.f16x2.e2m1x2 %0, b;\n}" : "=r"(r) : "r"(byte));
  return r;
}

// 2^(E - 127) as fp32 (E = 0 is the subnormal 2^-127; E = 255 is NaN).
__device__ __forceinline__ float e8m0_to_f32(uint32_t e) {
  e &= 0xFFu;
  return e == 255u ? __uint_as_float(0x7FC00000u) : (e == 0u ? __uint_as_float(0x00400000u) : __uint_as_float(e << 23));
}

__device__ __forceinline__ void mx_mma(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                       uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__global__ void __launch_bounds__(kMXWarps * 32) gemv_mxfp4_kernel(const MXParams p) {
  __shared__ float red[kMXWarps][16][8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int band = blockIdx.x;
  const int r0 = band * 16 + g, r1 = r0 + 8;
  const bool ok0 = r0 < p.N, ok1 = r1 < p.N;
  const int nb = p.K / 32;
  const long long rb = p.K / 2;  // code bytes per row
  const uint8_t* w0 = p.w + static_cast<long long>(ok0 ? r0 : 0) * rb + 4 * t;
  const uint8_t* w1 = p.w + static_cast<long long>(ok1 ? r1 : 0) * rb + 4 * t;
  const uint8_t* s0 = p.scales + static_cast<long long>(ok0 ? r0 : 0) * nb;
  const uint8_t* s1 = p.scales + static_cast<long long>(ok1 ? r1 : 0) * nb;
  const bool xrow = g < p.M;
  const __half* xr = reinterpret_cast<const __half*>(p.x) + static_cast<long long>(xrow ? g : 0) * p.K + 8 * t;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  constexpr int kU = 8;  // blocks in flight per warp
  for (int b0 = warp; b0 < nb; b0 += kMXWarps * kU) {
    uint32_t c0[kU], c1[kU], e0[kU], e1[kU];
    uint4 xv[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int b = b0 + u * kMXWarps;
      const bool in = b < nb;
      c0[u] = in && ok0 ? __ldg(reinterpret_cast<const unsigned int*>(w0 + 16ll * b)) : 0u;
      c1[u] = in && ok1 ? __ldg(reinterpret_cast<const unsigned int*>(w1 + 16ll * b)) : 0u;
      e0[u] = in && ok0 ? __ldg(s0 + b) : 127u;
      e1[u] = in && ok1 ? __ldg(s1 + b) : 127u;
      xv[u] = in && xrow ? __ldg(reinterpret_cast<const uint4*>(xr + 32ll * b)) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      float d[4] = {0.f, 0.f, 0.f, 0.f};
      // k = 8t + {0,1 | 2,3} in the first MMA, 8t + {4,5 | 6,7} in the second
      mx_mma(d, e2m1x2_to_f16x2(c0[u]), e2m1x2_to_f16x2(c1[u]), e2m1x2_to_f16x2(c0[u] >> 8),
             e2m1x2_to_f16x2(c1[u] >> 8), xv[u].x, xv[u].y);
      mx_mma(d, e2m1x2_to_f16x2(c0[u] >> 16), e2m1x2_to_f16x2(c1[u] >> 16), e2m1x2_to_f16x2(c0[u] >> 24),
             e2m1x2_to_f16x2(c1[u] >> 24), xv[u].z, xv[u].w);
      const float sg = e8m0_to_f32(e0[u]), sg8 = e8m0_to_f32(e1[u]);
      acc[0] = fmaf(sg, d[0], acc[0]);
      acc[1] = fmaf(sg, d[1], acc[1]);
      acc[2] = fmaf(sg8, d[2], acc[2]);
      acc[3] = fmaf(sg8, d[3], acc[3]);
    }
  }
  red[warp][g][2 * t] = acc[0];
  red[warp][g][2 * t + 1] = acc[1];
  red[warp][g + 8][2 * t] = acc[2];
  red[warp][g + 8][2 * t + 1] = acc[3];
  __syncthreads();
  for (int o = threadIdx.x; o < 16 * p.M; o += blockDim.x) {
    const int row = o / p.M, m = o - row * p.M;
    float sum = 0.f;
#pragma unroll
    for (int w2 = 0; w2 < kMXWarps; ++w2) sum += red[w2][row][m];
    const int n = band * 16 + row;
    if (n < p.N) reinterpret_cast<__half*>(p.y)[static_cast<long long>(m) * p.N + n] = __float2half_rn(sum);
  }
}

// Exact fp32 export W[n][k] = 2^(E - 127)·e2m1(q) (values past the fp32 range
// are ±inf, E = 255 gives NaN); one thread per code byte.
__global__ void dequant_mxfp4_kernel(const uint8_t* w, const uint8_t* scales, float* out, int N, int K) {
  const long long bytes = static_cast<long long>(N) * (K / 2);
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < bytes;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long row = i / (K / 2);
    const int k = static_cast<int>(i - row * (K / 2)) * 2;
    const float s = e8m0_to_f32(scales[row * (K / 32) + k / 32]);
    const uint32_t h2 = e2m1x2_to_f16x2(w[i]);
    out[row * K + k] = h16_to_f32(h2) * s;
    out[row * K + k + 1] = h16_to_f32(h2 >> 16) * s;
  }
}

}  // namespace wq
