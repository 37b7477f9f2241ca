// wq_device.cuh — device helpers shared by every libwq kernel (sm_100a).
//
// * bounded mbarrier waits (give up after ~1 s of %globaltimer, set the
//   device error word, let the caller drain and return),
// * 1-D bulk copies global -> shared (cp.async.bulk) completing on an mbarrier,
// * the 4-bit unpacking used by the GEMV kernels and the dequant exports:
//   a 32-bit word of codes is split into four fp16x2 registers by masking
//   only.  A nibble sitting in bits 0-3 of a 16-bit half, read as IEEE
//   binary16, is the subnormal q·2^-24 (exact); a nibble in bits 4-7 is
//   16·q·2^-24 (exact).  The mixed-precision fma.rn.f32.f16 multiplies such a
//   code by an fp16 activation exactly and accumulates in fp32, so the
//   integer code never needs a conversion instruction.
#pragma once

#include <cstdint>
#include <cuda_fp16.h>
#include <cuda_bf16.h>

namespace wq {

// Device-side error word: bounded waits OR a code in here instead of hanging.
__device__ unsigned int g_device_error;
constexpr unsigned int kDevErrTimeout = 1u;

constexpr unsigned long long kWaitLimitNs = 1000000000ull;  // 1 s

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

// Programmatic dependent launch: let the next kernel in the stream start its
// independent prologue now / wait until the previous kernel has completed and
// its writes are visible (both are no-ops when the launch carries no
// programmatic-serialization attribute).
__device__ __forceinline__ void grid_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void grid_wait_prior() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Same test, but a thread whose phase is still open is suspended (up to
// `hint_ns`, or until the phase completes) instead of spinning, so waiting
// warps leave their issue slots to the warps that have work.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

// Wait for phase `parity` of `bar` to complete, for at most `limit_ns`.
// Returns false (and records kDevErrTimeout) when the limit is reached.
__device__ __forceinline__ bool mbar_wait_bounded_ns(uint64_t* bar, uint32_t parity, unsigned long long limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  while (true) {
    if (mbar_try_wait_sleep(bar, parity, 20000u)) return true;
    if (global_ns() - t0 > limit_ns) {
      atomicOr(&g_device_error, kDevErrTimeout);
      return false;
    }
  }
}

__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity) {
  return mbar_wait_bounded_ns(bar, parity, kWaitLimitNs);
}

// 1-D bulk copy of `bytes` (multiple of 16, both addresses 16-byte aligned)
// from global to this CTA's shared memory, completing tx-bytes on `bar`.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Same, with an L2 evict-first hint (weights are read exactly once).
__device__ __forceinline__ void bulk_g2s_stream(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                                uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], "
      "%4;" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// Bulk prefetch of `bytes` (multiple of 16, 16-byte aligned) from global
// memory into L2; no data reaches the SM, so it is safe ahead of a
// griddepcontrol.wait (L2 is the point of coherence).
__device__ __forceinline__ void prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// ---------------------------------------------------------------------------
// mixed-precision FMAs: fp32 accumulator, fp16 / bf16 operands (exact products)
// ---------------------------------------------------------------------------

// acc0 += w.lo·x.lo ; acc1 += w.hi·x.hi
__device__ __forceinline__ void mfma2_f16(float& acc0, float& acc1, uint32_t w, uint32_t x) {
  asm("{\n .reg .b16 wl, wh, xl, xh;\n mov.b32 {wl, wh}, %2;\n mov.b32 {xl, xh}, %3;\n"
      " fma.rn.f32.f16 %0, wl, xl, %0;\n fma.rn.f32.f16 %1, wh, xh, %1;\n}\n"
      : "+f"(acc0), "+f"(acc1)
      : "r"(w), "r"(x));
}

// acc += w.lo·x.lo + w.hi·x.hi (one accumulator, two chained FMAs)
__device__ __forceinline__ void mfma2_f16_1(float& acc, uint32_t w, uint32_t x) {
  asm("{\n .reg .b16 wl, wh, xl, xh;\n mov.b32 {wl, wh}, %1;\n mov.b32 {xl, xh}, %2;\n"
      " fma.rn.f32.f16 %0, wl, xl, %0;\n fma.rn.f32.f16 %0, wh, xh, %0;\n}\n"
      : "+f"(acc)
      : "r"(w), "r"(x));
}

__device__ __forceinline__ void mfma2_bf16_1(float& acc, uint32_t w, uint32_t x) {
  asm("{\n .reg .b16 wl, wh, xl, xh;\n mov.b32 {wl, wh}, %1;\n mov.b32 {xl, xh}, %2;\n"
      " fma.rn.f32.bf16 %0, wl, xl, %0;\n fma.rn.f32.bf16 %0, wh, xh, %0;\n}\n"
      : "+f"(acc)
      : "r"(w), "r"(x));
}

__device__ __forceinline__ void mfma2_bf16(float& acc0, float& acc1, uint32_t w, uint32_t x) {
  asm("{\n .reg .b16 wl, wh, xl, xh;\n mov.b32 {wl, wh}, %2;\n mov.b32 {xl, xh}, %3;\n"
      " fma.rn.f32.bf16 %0, wl, xl, %0;\n fma.rn.f32.bf16 %1, wh, xh, %1;\n}\n"
      : "+f"(acc0), "+f"(acc1)
      : "r"(w), "r"(x));
}

// ---------------------------------------------------------------------------
// 4-bit unpacking into fp16x2 subnormal codes (no conversion instructions)
// ---------------------------------------------------------------------------
//
// For a 32-bit word v holding nibbles n0..n7 in bits 4i..4i+3:
//   lo4(v)      = v & 0x000F000F  -> halves (n0, n4) as q·2^-24
//   hi4(v)      = v & 0x00F000F0  -> halves (n1, n5) as 16·q·2^-24
//   lo4(v >> 8) -> (n2, n6) ; hi4(v >> 8) -> (n3, n7)
__device__ __forceinline__ uint32_t lo4(uint32_t v) { return v & 0x000F000Fu; }
__device__ __forceinline__ uint32_t hi4(uint32_t v) { return v & 0x00F000F0u; }

// Exact float of a code held as a subnormal fp16 (used by the dequant exports
// and the coefficient builders; the GEMV kernels never convert codes).
__device__ __forceinline__ float code_lo_to_f32(uint32_t pair, int half) {
  return (float)((pair >> (16 * half)) & 0xFu);
}

// ---------------------------------------------------------------------------
// q4_K 6-bit scale / min decode (minfer doc 62 "r59 — q4_K W_dsc plane", §2.1)
// ---------------------------------------------------------------------------
// The 12 packed bytes b[0..11] arrive as three little-endian words
// s0 = b0..b3, s1 = b4..b7, s2 = b8..b11.  Chunks j < 4 keep their scale in
// the low 6 bits of b[j] and their min in the low 6 bits of b[j+4]; chunks
// j >= 4 take the low (scale) or high (min) nibble of b[j+4] and the top two
// bits of b[j-4] (scale) or b[j] (min) as bits 4-5.  Returned as integers.
__device__ __forceinline__ void q4k_scale_min(uint32_t s0, uint32_t s1, uint32_t s2, int j, uint32_t& sc,
                                              uint32_t& mn) {
  if (j < 4) {
    sc = (s0 >> (8 * j)) & 63u;
    mn = (s1 >> (8 * j)) & 63u;
  } else {
    const int jj = j - 4;
    const uint32_t b8 = (s2 >> (8 * jj)) & 0xFFu;   // byte j+4
    const uint32_t blo = (s0 >> (8 * jj)) & 0xFFu;  // byte j-4
    const uint32_t bhi = (s1 >> (8 * jj)) & 0xFFu;  // byte j
    sc = (b8 & 0x0Fu) | ((blo >> 6) << 4);
    mn = (b8 >> 4) | ((bhi >> 6) << 4);
  }
}

// Branch-free decode of a consecutive chunk pair (2p, 2p+1), p in 0..3, as two
// packed byte lanes: sc2 = sc_{2p} | sc_{2p+1} << 8, mn2 likewise.  `hp` = p & 1
// selects the byte pair inside a word, `upper` = p >= 2 selects the rule.
__device__ __forceinline__ void q4k_scale_min_pair(uint32_t s0, uint32_t s1, uint32_t s2, uint32_t hp,
                                                   uint32_t upper, uint32_t& sc2, uint32_t& mn2) {
  const uint32_t sh = 16u * hp;
  const uint32_t a = (s0 >> sh) & 0xFFFFu;  // bytes 2hp, 2hp+1      (b[j] or b[j-4])
  const uint32_t b = (s1 >> sh) & 0xFFFFu;  // bytes 4+2hp, 5+2hp    (b[j+4] or b[j])
  const uint32_t c = (s2 >> sh) & 0xFFFFu;  // bytes 8+2hp, 9+2hp    (b[j+4] for j >= 4)
  if (upper) {
    sc2 = (c & 0x0F0Fu) | ((a >> 2) & 0x3030u);
    mn2 = ((c >> 4) & 0x0F0Fu) | ((b >> 2) & 0x3030u);
  } else {
    sc2 = a & 0x3F3Fu;
    mn2 = b & 0x3F3Fu;
  }
}

__device__ __forceinline__ float h16_to_f32(uint32_t bits16) {
  return __half2float(__ushort_as_half(static_cast<unsigned short>(bits16 & 0xFFFFu)));
}

}  // namespace wq
