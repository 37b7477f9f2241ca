// pack.cpp — load-time host packing for libwq (compiled with -ffp-contract=off).
//
// The W_dsc plane (minfer doc 62 "r59 — q4_K W_dsc plane", §2.2-§2.3): for
// every 32-element chunk c of every row n, the pair (d·sc_c, -(dmin·m_c)) is
// computed with exactly one IEEE binary32 multiply each and an exact
// negation, and stored chunk-major at float2 index c·N + n.  fp16 -> fp32 and
// 6-bit integer -> fp32 are exact, and this file is built with FMA
// contraction disabled, so the host plane is bit-identical to the device one.
#include <cstdint>
#include <cstring>

#include "../../include/wq.h"
#include "wq_host.h"

namespace {

// IEEE binary16 -> binary32, exact (normal, subnormal, inf, nan).
float half_bits_to_float(uint16_t h) {
  const uint32_t sign = static_cast<uint32_t>(h & 0x8000u) << 16;
  uint32_t exp = (h >> 10) & 0x1Fu;
  uint32_t man = h & 0x3FFu;
  uint32_t bits;
  if (exp == 0) {
    if (man == 0) {
      bits = sign;
    } else {  // subnormal: renormalize
      int e = -1;
      do {
        man <<= 1;
        ++e;
      } while ((man & 0x400u) == 0);
      man &= 0x3FFu;
      bits = sign | (static_cast<uint32_t>(127 - 15 - e) << 23) | (man << 13);
    }
  } else if (exp == 0x1Fu) {
    bits = sign | 0x7F800000u | (man << 13);
  } else {
    bits = sign | ((exp + 127 - 15) << 23) | (man << 13);
  }
  float f;
  std::memcpy(&f, &bits, 4);
  return f;
}

// 6-bit (scale, min) of chunk j from the 12 packed bytes (§2.1).
void scale_min(const uint8_t* b, int j, uint32_t* sc, uint32_t* mn) {
  if (j < 4) {
    *sc = b[j] & 63u;
    *mn = b[j + 4] & 63u;
  } else {
    *sc = (b[j + 4] & 0x0Fu) | ((b[j - 4] >> 6) << 4);
    *mn = (b[j + 4] >> 4) | ((b[j] >> 6) << 4);
  }
}

}  // namespace

extern "C" size_t wq_q4k_bytes(int N, int K) {
  if (N <= 0 || K <= 0 || K % 256) return 0;
  return static_cast<size_t>(N) * (K / 256) * 144;
}

extern "C" size_t wq_q4k_dsc_bytes(int N, int K) {
  if (N <= 0 || K <= 0 || K % 256) return 0;
  return static_cast<size_t>(N) * (K / 32) * 8;
}

extern "C" size_t wq_int4_codes_bytes(int N, int K, int layout) {
  if (N <= 0 || K <= 0 || K % 2 || layout != WQ_LAYOUT_CANONICAL) return 0;
  return static_cast<size_t>(N) * (K / 2);
}

extern "C" size_t wq_int4_packed_bytes(int N, int K, int block_size, int layout) {
  if (N <= 0 || K <= 0 || layout != WQ_LAYOUT_B200_V1) return 0;
  if (block_size < 32 || block_size > 256 || (block_size & (block_size - 1)) || K % 128) return 0;
  return static_cast<size_t>((N + 15) / 16) * (K / 128) * WQ_INT4_V1_TILE_BYTES(block_size);
}

extern "C" size_t wq_int4_gate_up_packed_bytes(int N, int K, int block_size, int layout) {
  if (block_size < 128) return 0;
  return 2 * wq_int4_packed_bytes(N, K, block_size, layout);
}

extern "C" size_t wq_q4k_packed_bytes(int N, int K, int layout) {
  if (N <= 0 || K <= 0 || K % 256 || layout != WQ_LAYOUT_B200_V1) return 0;
  return static_cast<size_t>((N + 15) / 16) * (K / 256) * WQ_Q4K_V1_TILE_BYTES;
}

extern "C" size_t wq_int4_bytes(int N, int K, int block_size, int layout) {
  if (N <= 0 || K <= 0) return 0;
  if (block_size < 16 || block_size > 256 || (block_size & (block_size - 1)) || K % 16) return 0;
  if (layout == WQ_LAYOUT_B200_V1) return wq_int4_packed_bytes(N, K, block_size, layout);
  if (layout != WQ_LAYOUT_CANONICAL) return 0;
  const size_t nb = (K + block_size - 1) / block_size;  // the last block may be shorter
  return static_cast<size_t>(N) * (K / 2) + static_cast<size_t>(N) * nb * 2 + static_cast<size_t>(N) * ((nb + 1) / 2);
}

extern "C" int wq_build_q4k_dsc(const void* w_q4k_host, int N, int K, void* out_host) {
  if (!w_q4k_host || !out_host) return wq::fail(WQ_ERR_ARG, "wq_build_q4k_dsc: null pointer");
  if (N <= 0 || K <= 0 || K % 256) return wq::fail(WQ_ERR_ARG, "wq_build_q4k_dsc: need N > 0 and K % 256 == 0");
  const uint8_t* w = static_cast<const uint8_t*>(w_q4k_host);
  float* out = static_cast<float*>(out_host);
  const int nsb = K / 256;
  for (int n = 0; n < N; ++n) {
    for (int sb = 0; sb < nsb; ++sb) {
      const uint8_t* blk = w + (static_cast<size_t>(n) * nsb + sb) * 144;
      const float d = half_bits_to_float(static_cast<uint16_t>(blk[0] | (blk[1] << 8)));
      const float dmin = half_bits_to_float(static_cast<uint16_t>(blk[2] | (blk[3] << 8)));
      for (int j = 0; j < 8; ++j) {
        uint32_t sc, mn;
        scale_min(blk + 4, j, &sc, &mn);
        const size_t c = static_cast<size_t>(sb) * 8 + j;
        const float px = d * static_cast<float>(sc);     // one binary32 multiply
        const float pm = dmin * static_cast<float>(mn);  // one binary32 multiply
        out[(c * N + n) * 2 + 0] = px;
        out[(c * N + n) * 2 + 1] = -pm;                   // exact negation
      }
    }
  }
  return wq::ok();
}
