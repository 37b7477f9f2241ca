// api.cu — the extern "C" entry points of libwq.so (declared in include/wq.h):
// argument validation, kernel choice, launch, status and liveness labels.
//
// Nothing here computes on the host: every entry point either rejects its
// arguments or enqueues kernels on the caller's stream.  There is no CPU
// fallback and no silent kernel fallback: wq_last_kernel() names the kernel
// each call launched.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <utility>

#include "../../include/wq.h"
#include "gemv_cc.cuh"
#include "gemv_simple.cuh"
#include "gemv_tc.cuh"
#include "gemv_v1.cuh"
#include "gemv_v1k.cuh"
#include "gemm_tc5.cuh"
#include "gemm_v1tc.cuh"
#include "gemv_mxfp4.cuh"
#include "gemm_mmq.cuh"
#include "gemm_v1w.cuh"
#include "wq_host.h"

namespace wq {

namespace {
thread_local std::string t_last_error;
thread_local std::string t_last_kernel = "none";

struct DeviceInfo {
  int sms = 0;
  bool is_sm100 = false;
  bool valid = false;
};
DeviceInfo g_dev[64];
std::mutex g_dev_mu;

int device_info(DeviceInfo* out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(WQ_ERR_CUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
  if (dev < 0 || dev >= 64) return fail(WQ_ERR_DEVICE, "device ordinal out of range");
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.valid) {
    int major = 0, minor = 0, sms = 0;
    if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
      return fail(WQ_ERR_CUDA, std::string("cudaDeviceGetAttribute: ") + cudaGetErrorString(e));
    d.sms = sms;
    d.is_sm100 = (major == 10 && minor == 0);
    d.valid = true;
  }
  *out = d;
  if (!d.is_sm100) return fail(WQ_ERR_DEVICE, "libwq is built for sm_100a (B200); the current device is not sm_100");
  return WQ_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned2(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 1u) == 0; }
int ilog2_int(int v) {
  int r = 0;
  while ((1 << r) < v) ++r;
  return r;
}

// WQ_PDL=0 turns programmatic dependent launch off (A/B runs).
bool pdl_enabled() {
  const char* v = std::getenv("WQ_PDL");
  return !(v && std::atoi(v) == 0);
}

int launch_check(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(WQ_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
  return WQ_OK;
}

// ---------------------------------------------------------------------------
// streaming CUDA-core GEMV: kernel table and planner
// ---------------------------------------------------------------------------
using CCKernel = void (*)(const CCParams);

template <Fmt F, int M, int KS>
CCKernel cc_ptr() {
  return &gemv_cc_kernel<F, M, KS>;
}

// Instantiated segment sizes per format and batch (activation registers stay
// at or below 32 per thread for the preferred choice, 64 for the fallback).
template <Fmt F, int M>
CCKernel cc_lookup(int KS) {
  constexpr bool four = F != Fmt::BF16;
  if constexpr (four) {
    switch (KS) {
      case 64:
        if constexpr (M <= 1) return cc_ptr<F, M, 64>();
        break;
      case 32:
        if constexpr (M <= 4) return cc_ptr<F, M, 32>();
        break;
      case 16:
        if constexpr (M <= 8) return cc_ptr<F, M, 16>();
        break;
      case 8:
        if constexpr (M >= 5) return cc_ptr<F, M, 8>();
        break;
      default:
        break;
    }
  } else {
    switch (KS) {
      case 32:
        if constexpr (M <= 2) return cc_ptr<F, M, 32>();
        break;
      case 16:
        if constexpr (M <= 8) return cc_ptr<F, M, 16>();
        break;
      case 8:
        if constexpr (M >= 2) return cc_ptr<F, M, 8>();
        break;
      default:
        break;
    }
  }
  return nullptr;
}

template <Fmt F>
CCKernel cc_kernel_for(int M, int KS) {
  switch (M) {
    case 1: return cc_lookup<F, 1>(KS);
    case 2: return cc_lookup<F, 2>(KS);
    case 3: return cc_lookup<F, 3>(KS);
    case 4: return cc_lookup<F, 4>(KS);
    case 5: return cc_lookup<F, 5>(KS);
    case 6: return cc_lookup<F, 6>(KS);
    case 7: return cc_lookup<F, 7>(KS);
    case 8: return cc_lookup<F, 8>(KS);
    default: return nullptr;
  }
}

CCKernel cc_kernel(Fmt f, int M, int KS) {
  switch (f) {
    case Fmt::Int4: return cc_kernel_for<Fmt::Int4>(M, KS);
    case Fmt::Q4K: return cc_kernel_for<Fmt::Q4K>(M, KS);
    case Fmt::Q4KDsc: return cc_kernel_for<Fmt::Q4KDsc>(M, KS);
    case Fmt::BF16: return cc_kernel_for<Fmt::BF16>(M, KS);
  }
  return nullptr;
}

// Segment-size preference per format and batch.
int ks_candidates(Fmt f, int M, int* out) {
  if (f != Fmt::BF16) {
    if (M == 1) { out[0] = 64; out[1] = 32; out[2] = 16; return 3; }
    if (M == 2) { out[0] = 32; out[1] = 16; return 2; }
    if (M <= 4) { out[0] = 16; out[1] = 32; return 2; }
    out[0] = 8; out[1] = 16; return 2;
  }
  if (M == 1) { out[0] = 32; out[1] = 16; return 2; }
  if (M == 2) { out[0] = 32; out[1] = 16; out[2] = 8; return 3; }
  if (M <= 4) { out[0] = 16; out[1] = 8; return 2; }
  out[0] = 8; out[1] = 16; return 2;
}

constexpr int kStageCap = 32 * 1024;
constexpr int kSmemPerSm = 220 * 1024;

struct CCPlan {
  CCKernel fn = nullptr;
  CCParams p{};
  int threads = 0, grid = 0, smem = 0, KS = 0;
};

int round16(long long v) { return static_cast<int>((v + 15) & ~15ll); }

bool plan_cc(Fmt f, int M, int N, int K, long long row_bytes, int nb, int zb, int block_size, bool has_zeros,
             int sms, CCPlan* plan) {
  int cands[4];
  const int nc = ks_candidates(f, M, cands);
  // Prefer a candidate without idle lanes in the last warp of a row group.
  int best = -1;
  double best_idle = 2.0;
  for (int i = 0; i < nc; ++i) {
    const int KS = cands[i];
    if (K % KS) continue;
    if (f == Fmt::Int4 && KS > block_size) continue;
    const int S = K / KS;
    const int WK = (S + 31) / 32;
    if (WK * 32 > 512) continue;
    if (!cc_kernel(f, M, KS)) continue;
    const double idle = double(WK * 32 - S) / double(WK * 32);
    if (idle < best_idle - 0.05) {  // earlier candidates win unless clearly less idle
      best_idle = idle;
      best = KS;
    }
  }
  if (best < 0) return false;
  const int KS = best;
  const int S = K / KS;
  const int WK = (S + 31) / 32;
  const int RGMAX = rg_max(M);

  auto stage_bytes_for = [&](int RS, int* o_sc, int* o_z, int* o_pl, int* pstride) {
    long long off = round16(RS * row_bytes);
    *o_sc = *o_z = *o_pl = 0;
    *pstride = 0;
    if (f == Fmt::Int4) {
      *o_sc = static_cast<int>(off);
      off += round16(2ll * RS * nb + 32);
      if (has_zeros) {
        *o_z = static_cast<int>(off);
        off += round16(1ll * RS * zb + 32);
      }
    }
    if (f == Fmt::Q4KDsc) {
      *o_pl = static_cast<int>(off);
      *pstride = round16(8ll * RS + 16);
      off += static_cast<long long>(*pstride) * (K / 32);
    }
    return off;
  };

  const int Gmax = std::max(1, 512 / (WK * 32));
  int G = std::min(Gmax, std::max(1, (256 + WK * 32 - 1) / (WK * 32)));
  int RG = RGMAX;
  int o_sc, o_z, o_pl, pstride;
  long long sb = 0;
  while (true) {
    sb = stage_bytes_for(G * RG, &o_sc, &o_z, &o_pl, &pstride);
    if (sb <= kStageCap) break;
    if (RG > 1) {
      --RG;
    } else if (G > 1) {
      --G;
    } else {
      break;  // one row per stage is over the cap: accept a bigger stage
    }
  }
  const int RS = G * RG;
  const long long red = 2ll * RS * WK * M * 4;
  const long long tail = red + 8ll * 8 + 16;
  int NS = 4, ctas_per_sm = 2;
  if (NS * sb + tail > kSmemPerSm / 2) {
    ctas_per_sm = 1;
    NS = static_cast<int>(std::min<long long>(6, (kSmemPerSm - tail) / sb));
  }
  if (NS < 2) return false;
  const int n_granules = (N + 1) / 2;
  const int grid = std::max(1, std::min(ctas_per_sm * sms, n_granules));

  CCParams& p = plan->p;
  p.N = N;
  p.K = K;
  p.nb = nb;
  p.zb = zb;
  p.block_shift = block_size > 0 ? ilog2_int(block_size) : 0;
  p.row_bytes = row_bytes;
  p.S = S;
  p.WK = WK;
  p.G = G;
  p.RG = RG;
  p.RS = RS;
  p.NS = NS;
  p.n_granules = n_granules;
  p.stage_bytes = static_cast<int>(sb);
  p.off_scales = o_sc;
  p.off_zeros = o_z;
  p.off_plane = o_pl;
  p.plane_stride = pstride;
  p.red_offset = static_cast<int>(NS * sb);
  plan->fn = cc_kernel(f, M, KS);
  plan->threads = G * WK * 32;
  plan->grid = grid;
  plan->smem = static_cast<int>(NS * sb + tail);
  plan->KS = KS;
  return plan->fn != nullptr;
}

int launch_cc(const CCPlan& plan, cudaStream_t st) {
  static std::mutex mu;
  static std::pair<CCKernel, int> configured[512];
  static int n_configured = 0;
  {
    std::lock_guard<std::mutex> lk(mu);
    int dev = 0;
    cudaGetDevice(&dev);
    bool found = false;
    for (int i = 0; i < n_configured; ++i)
      if (configured[i].first == plan.fn && configured[i].second == dev) found = true;
    if (!found) {
      cudaError_t e = cudaFuncSetAttribute(reinterpret_cast<const void*>(plan.fn),
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemPerSm + 4096);
      if (e != cudaSuccess) return fail(WQ_ERR_CUDA, std::string("cudaFuncSetAttribute: ") + cudaGetErrorString(e));
      if (n_configured < 512) configured[n_configured++] = {plan.fn, dev};
    }
  }
  plan.fn<<<plan.grid, plan.threads, plan.smem, st>>>(plan.p);
  return launch_check("gemv_cc launch");
}

std::string cc_label(const char* fmt, int M, int KS, const char* extra) {
  char buf[96];
  std::snprintf(buf, sizeof(buf), "%s.gemv.cc.m%d.ks%d%s", fmt, M, KS, extra);
  return buf;
}

// ---------------------------------------------------------------------------
// tensor-pipe GEMV (warp MMA, register operands): planner and launcher
// ---------------------------------------------------------------------------
struct TCPlan {
  TCParams p{};
  int threads = 0, grid = 0, smem = 0;
};

bool plan_tc(Fmt f, int M, int N, int K, long long row_bytes, int nb, int zb, int block_size, int layout,
             int sms, TCPlan* plan) {
  if (M < 1 || M > 8) return false;
  int Kc = 0;
  long long seg_full = 0;  // weight bytes per row of a full stage
  // WQ_TC_KC overrides the k-extent of a stage (tuning; rounded to the format's unit)
  const char* kc_env = std::getenv("WQ_TC_KC");
  const int kc_req = kc_env ? std::atoi(kc_env) : 0;
  int v1_tb = 0, v1_tpb = 0, v1_tps = 0;
  if (f == Fmt::Int4 && layout == WQ_LAYOUT_B200_V1) {
    if (block_size < 32 || K % 128) return false;
    v1_tb = int4_v1_tile_bytes(block_size);
    v1_tpb = K / 128;
    // tiles per stage: the largest divisor of the band's tile count within
    // the stage budget (WQ_TC_KC, in k, overrides the budget)
    const int cap_tiles = std::max(1, kc_req > 0 ? kc_req / 128 : (24 * 1024) / v1_tb);
    for (int d = 1; d <= v1_tpb; ++d)
      if (v1_tpb % d == 0 && d <= cap_tiles) v1_tps = d;
    Kc = 128 * v1_tps;
    seg_full = 0;
  } else if (f == Fmt::Int4) {
    if (block_size < 32 || K % 128) return false;
    Kc = std::max(std::max(block_size, 128), kc_req > 0 ? kc_req / 256 * 256 : 4096);
    Kc = std::min(Kc, K);
    seg_full = Kc / 2;
  } else if (f == Fmt::BF16) {
    if (K % 64) return false;
    Kc = std::min(kc_req > 0 ? std::max(64, kc_req / 64 * 64) : 2048, K);
    seg_full = 2ll * Kc;
  } else {
    if (K % 256) return false;
    Kc = std::min(kc_req > 0 ? std::max(256, kc_req / 256 * 256) : (f == Fmt::Q4K && M <= 2 ? 2048 : 1024), K);
    seg_full = (Kc / 256) * 144;
  }
  TCParams& p = plan->p;
  p.M = M;
  p.N = N;
  p.K = K;
  p.nb = nb;
  p.zb = zb;
  p.block_shift = block_size > 0 ? ilog2_int(block_size) : 0;
  p.row_bytes = row_bytes;
  p.rpb = (f == Fmt::Q4K || f == Fmt::Q4KDsc) ? 15 : 16;
  p.n_bands = (N + p.rpb - 1) / p.rpb;
  p.Kc = Kc;
  p.pitch = static_cast<int>(seg_full + 16);
  p.n_kst = (K + Kc - 1) / Kc;
  p.v1_tb = v1_tb;
  p.v1_tpb = v1_tpb;
  p.v1_tps = v1_tps;
  long long off = layout == WQ_LAYOUT_B200_V1 ? round16(1ll * v1_tps * v1_tb) : round16(16ll * p.pitch);
  p.off_x = static_cast<int>(off);
  // Activations resident for the whole kernel when small (one copy per CTA
  // instead of one per stage); WQ_TC_XRES=0/1 overrides (tuning).
  const char* xr_env = std::getenv("WQ_TC_XRES");
  const long long x_bytes = 2ll * M * K;
  p.x_res = xr_env ? (std::atoi(xr_env) != 0 && x_bytes <= 96 * 1024) : (x_bytes <= 64 * 1024);
  if (!p.x_res) off += round16(2ll * M * Kc);
  p.off_plane = static_cast<int>(off);
  p.plane_stride = round16(8ll * p.rpb + 16);
  if (f == Fmt::Q4KDsc) off += static_cast<long long>(p.plane_stride) * (Kc / 32);
  p.stage_bytes = static_cast<int>(round16(off));
  // WQ_TC_W overrides the number of consumer warps (tuning)
  // one CTA per SM for the B200_V1 stream needs 16 consumer warps (4 per
  // scheduler) to cover the load / MMA latency chains of the tile loop;
  // canonical int4 streams best with 12 warps over 4096-k stages, raw q4_K at
  // M <= 2 with 12 warps over 2048 k (B200, against 8 warps over 1024 k:
  // int4 M=1 4096x14336 22.8 -> 18.7 us, M=4 25.0 -> 20.4 us; q4_K M=1
  // 4096x11008 20.4 -> 18.0 us; q4_K M=4 stays faster at 8 warps / 1024 k)
  const char* w_env = std::getenv("WQ_TC_W");
  const int w_def = layout == WQ_LAYOUT_B200_V1 ? 16 : (f == Fmt::Int4 || (f == Fmt::Q4K && M <= 2)) ? 12 : 8;
  const int W = w_env ? std::max(1, std::min(16, std::atoi(w_env))) : w_def;
  p.W = W;
  long long meta = 0;
  if (f == Fmt::Int4 && layout == WQ_LAYOUT_B200_V1) {
    meta = 0;  // scales and zero-points travel inside the tiles
  } else if (f == Fmt::Int4 && block_size >= 128) {
    meta = 16ll * 16 * nb;  // one 16-byte entry per (block, row)
  } else if (f == Fmt::Int4) {
    p.meta_zoff = round16(2ll * 16 * nb);
    meta = p.meta_zoff + round16(16ll * zb);
  }
  const long long xres = p.x_res ? round16(x_bytes) : 0;
  const long long tail = meta + xres + 2ll * W * 16 * 8 * 4 + 2 * 16 * 8 + 16;
  // WQ_TC_NS overrides the ring depth (tuning); WQ_TC_CTAS the CTAs per SM (1 or 2)
  const char* ns_env = std::getenv("WQ_TC_NS");
  const char* cps_env = std::getenv("WQ_TC_CTAS");
  const int ns_cap = ns_env ? std::max(2, std::atoi(ns_env)) : 8;
  // B200_V1 streams want one CTA per SM with the deepest ring (the CTA's data is
  // one contiguous range, so almost all of it can be requested at once).
  int ctas_per_sm = cps_env ? std::max(1, std::min(2, std::atoi(cps_env))) : (layout == WQ_LAYOUT_B200_V1 ? 1 : 2);
  int NS = static_cast<int>(std::min<long long>(ns_cap, (kSmemPerSm / ctas_per_sm - tail) / p.stage_bytes));
  if (layout == WQ_LAYOUT_B200_V1 && ctas_per_sm == 1 && !ns_env)
    NS = static_cast<int>(std::min<long long>(16, (kSmemPerSm - tail) / p.stage_bytes));
  if (NS < 4 && ctas_per_sm == 2) {
    ctas_per_sm = 1;
    NS = static_cast<int>(std::min<long long>(std::max(ns_cap, 16), (kSmemPerSm - tail) / p.stage_bytes));
  }
  if (NS < 2) return false;
  p.NS = NS;
  p.off_meta = NS * p.stage_bytes;
  p.off_xres = static_cast<int>(p.off_meta + meta);
  p.off_red = static_cast<int>(p.off_xres + xres);
  plan->threads = (W + 1) * 32;
  plan->grid = std::max(1, std::min(p.n_bands, ctas_per_sm * sms));
  plan->smem = static_cast<int>(p.off_red + tail - meta - xres);
  return true;
}

using TCKernel = void (*)(const TCParams);

TCKernel tc_kernel(Fmt f, int layout, bool bigb) {
  const bool v1 = layout == WQ_LAYOUT_B200_V1;
  switch (f) {
    case Fmt::Int4:
      if (v1) return bigb ? &gemv_tc_kernel<Fmt::Int4, true, true> : &gemv_tc_kernel<Fmt::Int4, true, false>;
      return bigb ? &gemv_tc_kernel<Fmt::Int4, false, true> : &gemv_tc_kernel<Fmt::Int4, false, false>;
    case Fmt::Q4K: return &gemv_tc_kernel<Fmt::Q4K, false, false>;
    case Fmt::Q4KDsc: return &gemv_tc_kernel<Fmt::Q4KDsc, false, false>;
    case Fmt::BF16: return &gemv_tc_kernel<Fmt::BF16, false, false>;
  }
  return nullptr;
}

int launch_tc(Fmt f, int layout, const TCPlan& plan, cudaStream_t st) {
  static std::mutex mu;
  static bool configured[8][64] = {};
  const bool bigb = f == Fmt::Int4 && plan.p.block_shift >= 7;
  TCKernel fn = tc_kernel(f, layout, bigb);
  const int slot = f == Fmt::Int4 ? 4 + (layout == WQ_LAYOUT_B200_V1 ? 2 : 0) + (bigb ? 1 : 0) : static_cast<int>(f);
  {
    std::lock_guard<std::mutex> lk(mu);
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !configured[slot][dev]) {
      cudaError_t e = cudaFuncSetAttribute(reinterpret_cast<const void*>(fn),
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemPerSm + 4096);
      if (e != cudaSuccess) return fail(WQ_ERR_CUDA, std::string("cudaFuncSetAttribute: ") + cudaGetErrorString(e));
      configured[slot][dev] = true;
    }
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(plan.grid, 1, 1);
  cfg.blockDim = dim3(plan.threads, 1, 1);
  cfg.dynamicSmemBytes = plan.smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  cudaError_t e = cudaLaunchKernelEx(&cfg, fn, plan.p);
  if (e != cudaSuccess) return fail(WQ_ERR_CUDA, std::string("gemv_tc launch: ") + cudaGetErrorString(e));
  return launch_check("gemv_tc launch");
}

// ---------------------------------------------------------------------------
// B200_V1 int4 GEMV (blocks >= 128 k): planner and launcher
// ---------------------------------------------------------------------------
struct V1Plan {
  V1Params p;
  int grid = 0, threads = 0, smem = 0;
};

constexpr int kV1XBudget = 120 * 1024;   // resident activations per CTA
constexpr int kV1PartBudget = 16 * 1024;  // per-CTA band partials of a cluster split

// Clusters of C CTAs (one CTA per SM) that can be resident at once, per device.
int v1_max_clusters(int C, int smem, int threads, int sms) {
  if (C == 1) return sms;
  static std::mutex mu;
  static int cache[64][5] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lk(mu);
  if (dev >= 0 && dev < 64 && cache[dev][C] > 0) return cache[dev][C];
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(C * sms, 1, 1);
  cfg.blockDim = dim3(threads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, reinterpret_cast<const void*>(&gemv_v1_kernel<true>), &cfg) != cudaSuccess) {
    cudaGetLastError();
    n = 0;
  }
  if (dev >= 0 && dev < 64) cache[dev][C] = n > 0 ? n : -1;
  return n;
}

// WQ_V1_ZQ=0/1 picks the B200_V1 band kernel's tile arithmetic (A/B runs):
// 1 (default) forms the exact q − z in the MMA operand, 0 uses subnormal
// codes with a per-tile Σx zero-point term.
bool v1_zq() {
  const char* v = std::getenv("WQ_V1_ZQ");
  return !(v && std::atoi(v) == 0);
}

using V1Kernel = void (*)(const V1Params);
V1Kernel v1_kernel_fn() { return v1_zq() ? &gemv_v1_kernel<true> : &gemv_v1_kernel<false>; }

int v1_configure() {
  static std::mutex mu;
  static bool configured[2][64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lk(mu);
  const V1Kernel fns[2] = {&gemv_v1_kernel<false>, &gemv_v1_kernel<true>};
  for (int z = 0; z < 2; ++z)
    if (dev >= 0 && dev < 64 && !configured[z][dev]) {
      cudaError_t e = cudaFuncSetAttribute(reinterpret_cast<const void*>(fns[z]),
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemPerSm + 4096);
      if (e != cudaSuccess) return fail(WQ_ERR_CUDA, std::string("cudaFuncSetAttribute: ") + cudaGetErrorString(e));
      configured[z][dev] = true;
    }
  return WQ_OK;
}

// Geometry for cluster size C over n_clusters clusters; false if it does not fit.
bool plan_v1_geom(int M, int N, int K, int block_size, int C, int W, int n_clusters, V1Plan* plan, int stage_kb,
                  int cps) {
  const char* w_env = std::getenv("WQ_V1_W");  // consumer warps (tuning)
  if (w_env) W = std::max(4, std::min(kV1MaxWarps - 2, std::atoi(w_env)));
  const int tpb = K / 128;
  if (C < 1 || tpb % C || n_clusters < 1) return false;
  V1Params& p = plan->p;
  p.M = M;
  p.N = N;
  p.K = K;
  p.n_dst = 0;  // y only, unless the caller names destinations (row-split layers)
  p.y_ld = 0;
  p.y_off = 0;
  p.n_bands = (N + 15) / 16;
  p.tpb = tpb;
  p.tpc = tpb / C;
  p.tb = int4_v1_tile_bytes(block_size);
  p.W = W;
  // tiles per stage: a multiple of W, about stage_kb KB (larger bulk copies
  // stream faster on B200; WQ_V1_STAGE_KB overrides, for tuning)
  const char* sk_env = std::getenv("WQ_V1_STAGE_KB");
  const int stage_budget = (sk_env ? std::max(1, std::atoi(sk_env)) : stage_kb) * 1024;
  p.tps = W * std::max(1, stage_budget / (W * p.tb));
  // first stage: WQ_V1_FIRST tiles (tuning; rounded to whole multiples of W)
  const char* f_env = std::getenv("WQ_V1_FIRST");
  // (a first stage of one tile per warp lands sooner after the wait: B200, M=1
  // 4096x14336 12.08 -> 11.98 us, 4096x4096 5.21 -> 5.01 us)
  p.tps0 = f_env ? std::max(W, std::min(p.tps, std::atoi(f_env) / W * W)) : W;
  // Before waiting for the previous kernel: an L2 prefetch of the head of the
  // CTA's stream (safe whatever that kernel wrote; WQ_V1_PFKB, KB), or ring
  // stages copied to shared memory (WQ_V1_PRE, stages; only correct when the
  // kernel right before the GEMV does not write its weights).
  const char* pre_env = std::getenv("WQ_V1_PRE");
  p.pre = pre_env ? std::max(0, std::atoi(pre_env)) : 0;
  const char* pf_env = std::getenv("WQ_V1_PFKB");
  p.pf_bytes = p.pre > 0 ? 0 : (pf_env ? std::max(0, std::atoi(pf_env)) : 96) * 1024;
  const char* pfd_env = std::getenv("WQ_V1_PFD");  // L2 prefetch distance in stages (tuning)
  p.pfd = pfd_env ? std::max(0, std::atoi(pfd_env)) : 0;
  const char* h_env = std::getenv("WQ_V1_HINT");
  p.hint = h_env ? (std::atoi(h_env) != 0) : 1;
  p.stage_bytes = p.tps * p.tb;
  p.C = C;
  p.Mp = (M + 1) & ~1;
  const int bpc = (p.n_bands + n_clusters - 1) / n_clusters;  // bands per cluster, at most
  const long long x_bytes = 2ll * M * p.tpc * 128;
  const long long xs_bytes = 32ll * p.tpc;
  const long long red_bytes = 2ll * W * 16 * p.Mp * 4;
  const long long part_bytes = C > 1 ? 4ll * bpc * 16 * M : 0;
  if (x_bytes > kV1XBudget || part_bytes > kV1PartBudget) return false;
  const long long fixed = round16(x_bytes) + 256 + round16(xs_bytes) + round16(red_bytes) + round16(part_bytes);
  const long long room = kSmemPerSm / cps - 1024 - fixed - (2ll * 16 * 8 + 8 + 16);
  const char* ns_env = std::getenv("WQ_V1_NS");
  const int NS = static_cast<int>(
      std::min<long long>(ns_env ? std::max(2, std::atoi(ns_env)) : 16, room / p.stage_bytes));
  if (NS < 3) return false;
  p.NS = NS;
  p.pre = std::min(p.pre, NS);  // the x copy must not wait for a ring slot
  long long off = static_cast<long long>(NS) * p.stage_bytes;
  p.off_x = static_cast<int>(off);
  off += round16(x_bytes);
  p.off_zero = static_cast<int>(off);
  off += 256;
  p.off_xs = static_cast<int>(off);
  off += round16(xs_bytes);
  p.off_red = static_cast<int>(off);
  off += round16(red_bytes);
  p.off_part = static_cast<int>(off);
  off += round16(part_bytes);
  p.off_bar = static_cast<int>(off);
  off += 2ll * NS * 8 + 8 + 16;
  plan->smem = static_cast<int>(off);
  plan->threads = (W + 2) * 32;
  plan->grid = n_clusters * C;
  return true;
}

// Pick the cluster size that minimises the tiles of the busiest CTA
// (WQ_V1_C forces one, for tests and tuning).
bool plan_v1(int M, int N, int K, int block_size, int sms, V1Plan* out) {
  if (M < 1 || M > 8 || K % 128 || block_size < 128) return false;
  if (v1_configure() != WQ_OK) return false;
  const char* c_env = std::getenv("WQ_V1_C");
  const int c_force = c_env ? std::atoi(c_env) : 0;
  const char* cps_env = std::getenv("WQ_V1_CTAS");
  const int cps_force = cps_env ? std::max(1, std::min(4, std::atoi(cps_env))) : 0;
  const int n_bands = (N + 15) / 16;
  // Explicit geometry (tuning): WQ_V1_BPC bands per cluster, WQ_V1_CTAS CTAs
  // per SM (1..4), WQ_V1_C CTAs per cluster along K, WQ_V1_W consumer warps,
  // WQ_V1_STAGE_KB stage size.
  if (const char* bpc_env = std::getenv("WQ_V1_BPC")) {
    const int bpc = std::max(1, std::atoi(bpc_env));
    const int C = c_force > 1 ? c_force : 1;
    const int cps = cps_force > 0 ? cps_force : 1;
    const int ncl = (n_bands + bpc - 1) / bpc;
    for (int kb : {52, 36, 24, 18, 12, 8, 4})
      if (plan_v1_geom(M, N, K, block_size, C, 8, ncl, out, kb, cps)) return true;
    return false;
  }
  if (c_force > 1) {
    // cluster split along K (measured slower than whole bands per CTA on B200:
    // smaller copies per band and an extra cluster reduction), on request only
    const int W = 16;
    int ncl = v1_max_clusters(c_force, kSmemPerSm, (W + 2) * 32, sms);
    if (ncl <= 0) return false;
    ncl = std::min(ncl, n_bands);
    for (int kb : {52, 36, 24, 18})
      if (plan_v1_geom(M, N, K, block_size, c_force, W, ncl, out, kb, 1)) return true;
    return false;
  }
  // Two CTAs per SM (12 consumer warps each) when 36 KB stages still fit: the
  // next call's CTAs then start beside the current ones and fill their rings
  // while these finish.  Otherwise one CTA per SM with 16 consumer warps and the
  // largest stages that leave three in the ring.
  if (cps_force != 1 &&
      plan_v1_geom(M, N, K, block_size, 1, 12, std::min(n_bands, 2 * sms), out, 36, 2))
    return true;
  if (cps_force == 2) return false;
  for (int kb : {52, 36, 24, 18})
    if (plan_v1_geom(M, N, K, block_size, 1, 16, std::min(n_bands, sms), out, kb, 1)) return true;
  return false;
}


// ---------------------------------------------------------------------------
// B200_V1 int4 GEMV, register-streaming kernel: planner and launcher
// ---------------------------------------------------------------------------
struct V1RPlan {
  V1RParams p;
  int P = 4, grid = 0, threads = 0, smem = 0;
};

constexpr int kV1RXBudget = 200 * 1024;  // activations resident in shared memory

bool plan_v1r(int M, int N, int K, int block_size, int sms, V1RPlan* out) {
  if (M < 1 || M > 8 || K % 128 || block_size < 128) return false;
  V1RParams& p = out->p;
  const char* w_env = std::getenv("WQ_V1R_W");  // consumer warps (tuning)
  const char* p_env = std::getenv("WQ_V1R_P");  // tiles in flight per warp (tuning)
  p.W = w_env ? std::max(4, std::min(kV1RMaxWarps - 1, std::atoi(w_env))) : 16;
  out->P = p_env ? std::atoi(p_env) : 4;
  if (out->P != 2 && out->P != 3 && out->P != 4) out->P = 4;
  p.M = M;
  p.N = N;
  p.K = K;
  p.n_bands = (N + 15) / 16;
  p.tpb = K / 128;
  p.tb = int4_v1_tile_bytes(block_size);
  p.Mp = (M + 1) & ~1;
  const long long x_bytes = 2ll * M * K;
  if (x_bytes > kV1RXBudget) return false;
  long long off = 0;
  p.off_x = 0;
  off += round16(x_bytes);
  p.off_zero = static_cast<int>(off);
  off += 256;
  p.off_xs = static_cast<int>(off);
  off += round16(32ll * p.tpb);
  p.off_red = static_cast<int>(off);
  off += 2ll * p.W * 16 * p.Mp * 4;
  if (off > kSmemPerSm) return false;
  out->smem = static_cast<int>(off);
  out->threads = (p.W + 1) * 32;
  out->grid = std::max(1, std::min(p.n_bands, sms));
  return true;
}

template <int P>
int launch_v1r_p(const V1RPlan& plan, cudaStream_t st) {
  static std::mutex mu;
  static bool configured[64] = {};
  {
    int dev = 0;
    cudaGetDevice(&dev);
    std::lock_guard<std::mutex> lk(mu);
    if (dev >= 0 && dev < 64 && !configured[dev]) {
      cudaError_t e = cudaFuncSetAttribute(reinterpret_cast<const void*>(&gemv_v1r_kernel<P>),
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemPerSm + 4096);
      if (e != cudaSuccess) return fail(WQ_ERR_CUDA, std::string("cudaFuncSetAttribute: ") + cudaGetErrorString(e));
      configured[dev] = true;
    }
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(plan.grid, 1, 1);
  cfg.blockDim = dim3(plan.threads, 1, 1);
  cfg.dynamicSmemBytes = plan.smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  cudaError_t e = cudaLaunchKernelEx(&cfg, &gemv_v1r_kernel<P>, plan.p);
  if (e != cudaSuccess) return fail(WQ_ERR_CUDA, std::string("gemv_v1r launch: ") + cudaGetErrorString(e));
  return launch_check("gemv_v1r launch");
}

int launch_v1r(const V1RPlan& plan, cudaStream_t st) {
  switch (plan.P) {
    case 2: return launch_v1r_p<2>(plan, st);
    case 3: return launch_v1r_p<3>(plan, st);
    default: return launch_v1r_p<4>(plan, st);
  }
}


int launch_v1(const V1Plan& plan_in, cudaStream_t st) {
  int rc = v1_configure();
  if (rc) return rc;
  V1Plan plan = plan_in;
  if (plan.p.n_dst == 0) {  // a plain call: y is the only destination
    plan.p.ydst[0] = plan.p.y;
    plan.p.n_dst = 1;
    plan.p.y_ld = plan.p.N;
    plan.p.y_off = 0;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(plan.grid, 1, 1);
  cfg.blockDim = dim3(plan.threads, 1, 1);
  cfg.dynamicSmemBytes = plan.smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int na = 0;
  if (pdl_enabled()) {
    // programmatic dependent launch: the kernel requests its read-only weights
    // while the previous kernel in the stream finishes (it waits for that
    // kernel before it reads x or writes y)
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  if (plan.p.C > 1) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = plan.p.C;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  cudaError_t e = cudaLaunchKernelEx(&cfg, v1_kernel_fn(), plan.p);
  if (e != cudaSuccess) return fail(WQ_ERR_CUDA, std::string("gemv_v1 launch: ") + cudaGetErrorString(e));
  return launch_check("gemv_v1 launch");
}

// ---------------------------------------------------------------------------
// Split-band workspace: counters and partial sums of bands cut by CTA
// boundaries (stream-K kernels).  One per (device, stream), allocated and
// zeroed at the first such call on that stream; the kernels leave every
// counter at zero when they finish.  Calls on one stream are ordered (the
// kernels touch the workspace only after waiting for the previous kernel);
// separate streams have separate workspaces.
// ---------------------------------------------------------------------------
constexpr long long kWsMaxBands = 65536;   // rows up to 1,048,576
constexpr long long kWsMaxCtas = 1024;
// partials: [CTA][first / last band][gate, up][16 rows][8 batch rows] fp32
constexpr size_t kWsBytes = static_cast<size_t>(kWsMaxBands * 4 + kWsMaxCtas * 2 * 2 * 128 * 4);

std::mutex g_ws_mu;
std::map<std::pair<int, cudaStream_t>, void*> g_ws;

int split_workspace(cudaStream_t st, int** counters, float** partials) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(WQ_ERR_CUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
  std::lock_guard<std::mutex> lk(g_ws_mu);
  auto it = g_ws.find({dev, st});
  void* ptr = nullptr;
  if (it != g_ws.end()) {
    ptr = it->second;
  } else {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(st, &cs) == cudaSuccess && cs != cudaStreamCaptureStatusNone)
      return fail(WQ_ERR_CUDA,
                  "the first decode call on a stream sets up that stream's split-band workspace and cannot be "
                  "captured: make one call on this stream before capturing a CUDA graph");
    if ((e = cudaMalloc(&ptr, kWsBytes)) != cudaSuccess)
      return fail(WQ_ERR_CUDA, std::string("workspace cudaMalloc: ") + cudaGetErrorString(e));
    if ((e = cudaMemset(ptr, 0, kWsBytes)) != cudaSuccess)
      return fail(WQ_ERR_CUDA, std::string("workspace cudaMemset: ") + cudaGetErrorString(e));
    g_ws[{dev, st}] = ptr;
  }
  *counters = static_cast<int*>(ptr);
  *partials = reinterpret_cast<float*>(static_cast<uint8_t*>(ptr) + kWsMaxBands * 4);
  return WQ_OK;
}

// Zero every split-band workspace of the current device (after a kernel gave
// up, its counters may not have been reset).
int reset_workspaces() {
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lk(g_ws_mu);
  for (auto& kv : g_ws)
    if (kv.first.first == dev && cudaMemset(kv.second, 0, kWsBytes) != cudaSuccess)
      return fail(WQ_ERR_CUDA, "workspace reset failed");
  return WQ_OK;
}

// ---------------------------------------------------------------------------
// Allocation-free variant of the split-band workspace (gemv_q4k_noalloc): a
// fixed array in the library's own device memory, reserved when the library
// is loaded and kept until the process exits, so that a call never allocates.
// It serves at most kNaMaxBands bands (N <= 16 · kNaMaxBands rows) and
// kNaMaxCtas CTAs.  Every such call on every stream uses this one array.
// ---------------------------------------------------------------------------
constexpr int kNaMaxBands = 4096;  // rows up to 65,536
constexpr int kNaMaxCtas = 256;
constexpr size_t kNaBytes = static_cast<size_t>(kNaMaxBands) * 4 + static_cast<size_t>(kNaMaxCtas) * 2 * 128 * 4;
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNaBytes];

// The array's device address, looked up once per device with that device
// current (in host code the symbol is only a host-side handle).
int noalloc_scratch(uint8_t** out) {
  static std::mutex mu;
  static uint8_t* addr[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(WQ_ERR_CUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
  if (dev < 0 || dev >= 64) return fail(WQ_ERR_DEVICE, "device ordinal out of range");
  std::lock_guard<std::mutex> lk(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p)
      return fail(WQ_ERR_CUDA, std::string("cudaGetSymbolAddress(scratch): ") + cudaGetErrorString(e));
    addr[dev] = static_cast<uint8_t*>(p);
  }
  *out = addr[dev];
  return WQ_OK;
}

// ---------------------------------------------------------------------------
// B200_V1 int4 GEMV, stream-K: planner and launcher
// ---------------------------------------------------------------------------
struct V1KPlan {
  V1KParams p;
  int grid = 0, threads = 0, smem = 0;
  Fmt fmt = Fmt::Int4;
  int mp2 = 8;
  bool dual = false;
};

using V1KKernel = void (*)(const V1KParams);

// WQ_V1K_ZQ=1 selects the int4 tile with the zero-point inside the MMA operand (tuning)
bool v1k_zq() {
  const char* v = std::getenv("WQ_V1K_ZQ");
  return v && std::atoi(v) != 0;
}

V1KKernel v1k_kernel(Fmt f, int mp2, bool dual) {
  if (f == Fmt::Int4) {
    if (v1k_zq()) return dual ? &gemv_v1k_kernel<Fmt::Int4, 8, true, true> : &gemv_v1k_kernel<Fmt::Int4, 8, false, true>;
    return dual ? &gemv_v1k_kernel<Fmt::Int4, 8, true> : &gemv_v1k_kernel<Fmt::Int4, 8>;
  }
  switch (mp2) {
    case 1: return &gemv_v1k_kernel<Fmt::Q4K, 1>;
    case 2: return &gemv_v1k_kernel<Fmt::Q4K, 2>;
    case 4: return &gemv_v1k_kernel<Fmt::Q4K, 4>;
    default: return &gemv_v1k_kernel<Fmt::Q4K, 8>;
  }
}

constexpr int kV1KXBudget = 120 * 1024;  // resident activations per CTA

bool plan_v1k(Fmt f, int M, int N, int K, int block_size, int sms, V1KPlan* out, bool dual = false) {
  if (M < 1 || M > 8) return false;
  if (dual && f != Fmt::Int4) return false;
  if (f == Fmt::Int4 && (K % 128 || block_size < 128)) return false;
  if (f == Fmt::Q4K && K % 256) return false;
  if (f != Fmt::Int4 && f != Fmt::Q4K) return false;
  const bool q4k = f == Fmt::Q4K;
  const char* w_env = std::getenv("WQ_V1K_W");       // consumer warps (tuning)
  const char* c_env = std::getenv("WQ_V1K_CTAS");    // CTAs per SM (tuning)
  const char* st_env = std::getenv("WQ_V1K_STAGE");  // tiles per stage (tuning)
  const char* ns_env = std::getenv("WQ_V1K_NS");     // ring depth cap (tuning)
  const char* pf_env = std::getenv("WQ_V1K_PFKB");   // KB prefetched into L2 before the wait (tuning)
  const char* r_env = std::getenv("WQ_V1K_RES");     // CTAs each SM must be able to hold (tuning)
  V1KParams& p = out->p;
  const int W = w_env ? std::max(1, std::min(kV1KMaxWarps - 2, std::atoi(w_env))) : 16;
  const int cps = c_env ? std::max(1, std::min(4, std::atoi(c_env))) : 1;
  // shared memory is sized so that `res` CTAs fit on an SM: with res > cps the
  // next call's CTAs are resident while this call runs (and prefetch into L2)
  const int res = std::max(cps, r_env ? std::max(1, std::min(4, std::atoi(r_env))) : cps);
  const int stage_tiles = st_env ? std::max(1, std::atoi(st_env)) : 16;
  p.M = M;
  p.N = N;
  p.K = K;
  p.n_bands = (N + 15) / 16;
  if (p.n_bands > kWsMaxBands) return false;
  p.tpb = q4k ? K / 256 : K / 128;
  p.T = static_cast<long long>(p.n_bands) * p.tpb;
  p.tb = q4k ? kQ4KV1TileBytes : int4_v1_tile_bytes(block_size) * (dual ? 2 : 1);
  out->fmt = f;
  out->dual = dual;
  const int nsum = dual ? 2 : 1;
  int mp2 = 1;
  while (mp2 < M) mp2 *= 2;
  out->mp2 = mp2;
  p.W = W;
  p.tps = W * std::max(1, stage_tiles / W);  // a multiple of W: every warp's tile sequence runs on across stages
  p.stage_bytes = p.tps * p.tb;
  p.Mp = (M + 1) & ~1;
  p.pf_bytes = (pf_env ? std::max(0, std::atoi(pf_env)) : 96) * 1024;
  const long long x_bytes = 2ll * M * K;
  if (x_bytes > kV1KXBudget) return false;
  const long long xs_bytes = (q4k ? 256ll : 32ll) * p.tpb;  // Σx table: 8 floats per k-unit
  const long long fixed =
      round16(x_bytes) + 256 + round16(xs_bytes) + round16(1ll * kRedSlots * nsum * W * 16 * p.Mp * 4);
  const long long room = kSmemPerSm / res - 1024 - fixed - (2ll * 16 * 8 + 8 + 16);
  const int ns_cap = ns_env ? std::max(2, std::atoi(ns_env)) : 16;
  // smaller stages (still a multiple of W tiles) until at least two fit
  while (room / p.stage_bytes < 2 && p.tps > W) {
    p.tps = W * std::max(1, p.tps / W / 2);
    p.stage_bytes = p.tps * p.tb;
  }
  const int NS = static_cast<int>(std::min<long long>(ns_cap, room / p.stage_bytes));
  if (NS < 2) return false;
  p.NS = NS;
  long long off = static_cast<long long>(NS) * p.stage_bytes;
  p.off_x = static_cast<int>(off);
  off += round16(x_bytes);
  p.off_zero = static_cast<int>(off);
  off += 256;
  p.off_xs = static_cast<int>(off);
  off += round16(xs_bytes);
  p.off_red = static_cast<int>(off);
  off += round16(1ll * kRedSlots * nsum * W * 16 * p.Mp * 4);
  p.off_bar = static_cast<int>(off);
  off += 2ll * NS * 8 + 8 + 16;
  out->smem = static_cast<int>(off);
  out->threads = (W + 2) * 32;
  out->grid = static_cast<int>(std::min<long long>(std::min<long long>(sms * cps, p.T), kWsMaxCtas));
  return true;
}

int launch_v1k(V1KPlan& plan, cudaStream_t st, bool use_stream_workspace = true) {
  static std::mutex mu;
  static bool configured[8][64] = {};
  const V1KKernel fn = v1k_kernel(plan.fmt, plan.mp2, plan.dual);
  const int ki = plan.fmt == Fmt::Int4 ? 4 + (plan.dual ? 2 : 0) + (v1k_zq() ? 1 : 0)
                                       : (plan.mp2 == 1 ? 0 : plan.mp2 == 2 ? 1 : plan.mp2 == 4 ? 2 : 3);
  {
    int dev = 0;
    cudaGetDevice(&dev);
    std::lock_guard<std::mutex> lk(mu);
    if (dev >= 0 && dev < 64 && !configured[ki][dev]) {
      cudaError_t e = cudaFuncSetAttribute(reinterpret_cast<const void*>(fn),
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemPerSm + 4096);
      if (e != cudaSuccess) return fail(WQ_ERR_CUDA, std::string("cudaFuncSetAttribute: ") + cudaGetErrorString(e));
      configured[ki][dev] = true;
    }
  }
  if (use_stream_workspace) {
    int rc = split_workspace(st, &plan.p.counters, &plan.p.partials);
    if (rc) return rc;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(plan.grid, 1, 1);
  cfg.blockDim = dim3(plan.threads, 1, 1);
  cfg.dynamicSmemBytes = plan.smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  cudaError_t e = cudaLaunchKernelEx(&cfg, fn, plan.p);
  if (e != cudaSuccess) return fail(WQ_ERR_CUDA, std::string("gemv_v1k launch: ") + cudaGetErrorString(e));
  return launch_check("gemv_v1k launch");
}

// WQ_FORCE_KERNEL = "cc" | "tc" | "simple" pins the GEMV variant (A/B runs and
// per-variant parity tests); unset means the default choice below.
const char* forced_variant() {
  const char* v = std::getenv("WQ_FORCE_KERNEL");
  return (v && *v) ? v : nullptr;
}

template <Fmt F>
int launch_simple(const SimpleParams& sp, int M, int sms, cudaStream_t st) {
  const int threads = 256;
  const int rows_per_block = threads / 32;
  const int grid = std::max(1, std::min((sp.N + rows_per_block - 1) / rows_per_block, sms * 16));
  switch (M) {
    case 1: gemv_simple_kernel<F, 1><<<grid, threads, 0, st>>>(sp); break;
    case 2: gemv_simple_kernel<F, 2><<<grid, threads, 0, st>>>(sp); break;
    case 3: gemv_simple_kernel<F, 3><<<grid, threads, 0, st>>>(sp); break;
    case 4: gemv_simple_kernel<F, 4><<<grid, threads, 0, st>>>(sp); break;
    case 5: gemv_simple_kernel<F, 5><<<grid, threads, 0, st>>>(sp); break;
    case 6: gemv_simple_kernel<F, 6><<<grid, threads, 0, st>>>(sp); break;
    case 7: gemv_simple_kernel<F, 7><<<grid, threads, 0, st>>>(sp); break;
    case 8: gemv_simple_kernel<F, 8><<<grid, threads, 0, st>>>(sp); break;
    default: return fail(WQ_ERR_ARG, "simple kernel: M chunk out of range");
  }
  return launch_check("gemv_simple launch");
}

// ---------------------------------------------------------------------------
// tcgen05 batched path (M >= 9): planner and launcher
// ---------------------------------------------------------------------------
// cuTensorMapEncodeTiled from the driver, looked up once (no link-time
// dependency on libcuda).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, []() {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    else
      cudaGetLastError();
  });
  return fn;
}

int encode_2d(CUtensorMap* map, CUtensorMapDataType dt, const void* base, unsigned long long inner,
              unsigned long long outer, unsigned long long row_bytes, unsigned box_inner, unsigned box_outer,
              CUtensorMapSwizzle sw) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return fail(WQ_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(WQ_ERR_CUDA, "cuTensorMapEncodeTiled failed (" + std::to_string(static_cast<int>(r)) + ")");
  return WQ_OK;
}

template <Fmt F>
int launch_tc5(const void* x, const uint8_t* w, const uint8_t* scales, const uint8_t* zeros, void* y, int M, int N,
               int K, int nb, int zb, int block_size, int sms, cudaStream_t st, std::string* label) {
  TC5Params p{};
  p.x = x;
  p.w = w;
  p.scales = scales;
  p.zeros = zeros;
  p.y = y;
  p.M = M;
  p.N = N;
  p.K = K;
  p.nb = nb;
  p.zb = zb;
  p.block_shift = block_size > 0 ? ilog2_int(block_size) : 0;
  p.BN = std::min(256, (M + 15) / 16 * 16);
  // int4 and q4_K with BN <= 128: fp16 A rows in tensor memory (columns 256 ..
  // 383, after the two accumulator tiles); WQ_TC5_TA=0 keeps them in shared memory
  const char* ta_env = std::getenv("WQ_TC5_TA");
  const bool ta = F != Fmt::BF16 && p.BN <= 128 && !(ta_env && std::atoi(ta_env) == 0);
  int cols = 32;
  while (cols < 2 * p.BN) cols *= 2;  // two accumulator tiles (even / odd stages)
  p.tmem_cols = ta ? 512 : cols;
  // shared memory: 4 A slots (16 KB; none with A in TMEM), NX activation slots, NR raw slots, barriers
  const int x_slot = (p.BN * 128 + 1023) / 1024 * 1024;
  // raw slots of 256 k: int4 128 B per row, q4_K one 144-byte super-block per row
  // (256-byte int4 rows measured no faster on B200)
  p.spr = F == Fmt::BF16 ? 1 : 4;
  p.raw_pitch = F == Fmt::Int4 ? 128 : 144;
  p.raw_bytes = F == Fmt::BF16 ? 0 : 128 * p.raw_pitch;  // bf16 weights go straight into the A slots
  p.NR = F == Fmt::BF16 ? 0 : 3;
  const int budget = kSmemPerSm - 1024 - 1024;
  const int a_bytes = ta ? 0 : kTc5NA * 16384;
  p.NX = std::max(2, std::min(8, (budget - a_bytes - p.NR * p.raw_bytes) / x_slot));
  p.off_x = a_bytes;
  p.off_raw = p.off_x + p.NX * x_slot;
  p.off_bar = (p.off_raw + p.NR * p.raw_bytes + 127) / 128 * 128;
  const int smem = 1024 + p.off_bar + (2 * p.NR + 2 * p.NX + 2 * kTc5NA + 1) * 8 + 16;
  if (smem > kSmemPerSm + 4096) return fail(WQ_ERR_UNSUPPORTED, "gemm_tc5: shared memory plan too large");
  // Split K over a cluster of S CTAs (one CTA per SM) until the CTAs fill the
  // SMs; every CTA keeps a whole number of 256-k raw slots.
  const int n_tiles = (N + 127) / 128, m_tiles = (M + p.BN - 1) / p.BN;
  const int nst = (K + 63) / 64;  // bf16: a partial last stage reads zeros past K (TMA bounds fill)
  int S = 1;
  // the largest power-of-two split that still fits one wave, every CTA keeping an even number of raw slots
  while (S < 8 && n_tiles * m_tiles * S * 2 <= sms && nst % (2 * p.spr * S * 2) == 0) S *= 2;
  if (const char* s_env = std::getenv("WQ_TC5_S")) {  // tests and tuning
    const int sf = std::atoi(s_env);
    if (sf == 1 || sf == 2 || sf == 4 || sf == 8) {
      // the same rule as the automatic choice: every CTA gets an even number of
      // raw slots, so its even / odd accumulator tiles see the same stage count
      if (nst % (2 * p.spr * sf)) return fail(WQ_ERR_ARG, "WQ_TC5_S does not split K into an even number of raw slots per CTA");
      S = sf;
    }
  }
  if (S > 1 && 512 * p.BN > p.off_bar) return fail(WQ_ERR_UNSUPPORTED, "gemm_tc5: cluster partials do not fit");
  p.S = S;
  p.nks = nst / S;
  int rc;
  if constexpr (F == Fmt::Int4)
    rc = encode_2d(&p.tmap_w, CU_TENSOR_MAP_DATA_TYPE_UINT8, w, K / 2, N, K / 2, 128, 128, CU_TENSOR_MAP_SWIZZLE_128B);
  else if constexpr (F == Fmt::BF16)
    rc = encode_2d(&p.tmap_w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w, K, N, 2ull * K, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B);
  else
    rc = encode_2d(&p.tmap_w, CU_TENSOR_MAP_DATA_TYPE_UINT8, w, (K / 256) * 144ull, N, (K / 256) * 144ull, 144, 128,
                   CU_TENSOR_MAP_SWIZZLE_NONE);
  if (rc) return rc;
  rc = encode_2d(&p.tmap_x, F == Fmt::BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, x, K,
                 M, 2ull * K, 64, p.BN, CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc) return rc;
  static std::mutex mu;
  static bool configured[3][2][64] = {};
  const int fi = F == Fmt::Int4 ? 0 : F == Fmt::Q4K ? 1 : 2;
  constexpr bool kTA = F != Fmt::BF16;  // (bf16 weights are the A operand as stored: never TA)
  const void* fn = ta ? reinterpret_cast<const void*>(&gemm_tc5_kernel<F, kTA>)
                      : reinterpret_cast<const void*>(&gemm_tc5_kernel<F, false>);
  {
    std::lock_guard<std::mutex> lk(mu);
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !configured[fi][ta][dev]) {
      cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemPerSm + 4096);
      if (e != cudaSuccess) return fail(WQ_ERR_CUDA, std::string("cudaFuncSetAttribute: ") + cudaGetErrorString(e));
      configured[fi][ta][dev] = true;
    }
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(n_tiles * S, m_tiles, 1);
  cfg.blockDim = dim3(kTc5Warps * 32, 1, 1);
  // with A in TMEM a CTA holds all 512 TMEM columns: one CTA per SM (a second
  // one would wait in tcgen05.alloc, and with clusters two waits could cycle)
  cfg.dynamicSmemBytes = ta ? std::max(smem, kSmemPerSm / 2 + 8192) : smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = S;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = S > 1 ? 1 : 0;
  cudaError_t e = ta ? cudaLaunchKernelEx(&cfg, &gemm_tc5_kernel<F, kTA>, p)
                     : cudaLaunchKernelEx(&cfg, &gemm_tc5_kernel<F, false>, p);
  if (e != cudaSuccess) return fail(WQ_ERR_CUDA, std::string("gemm_tc5 launch: ") + cudaGetErrorString(e));
  rc = launch_check("gemm_tc5 launch");
  if (rc) return rc;
  char buf[64];
  std::snprintf(buf, sizeof(buf), "%s.gemm.tc5.%sbn%d.s%d", F == Fmt::Int4 ? "int4" : F == Fmt::Q4K ? "q4k" : "bf16",
                ta ? "ta." : "", p.BN, S);
  *label = buf;
  return WQ_OK;
}

// tcgen05 batched GEMM over the int4 B200_V1 stream (blocks >= 128): planner and launcher
int launch_v1tc(const void* x, const uint8_t* w, void* y, int M, int N, int K, int block_size, int sms,
                cudaStream_t st, std::string* label) {
  if (K % 128 || block_size < 128) return fail(WQ_ERR_UNSUPPORTED, "gemm_v1tc: needs K % 128 == 0 and blocks >= 128");
  V1TCParams p{};
  p.w = w;
  p.y = y;
  p.M = M;
  p.N = N;
  p.K = K;
  p.n_bands = (N + 15) / 16;
  p.tpb = K / 128;
  p.tb = int4_v1_tile_bytes(block_size);
  p.BN = std::min(128, (M + 15) / 16 * 16);
  // A operand in tensor memory (default) or in shared memory (WQ_V1TC_TA=0)
  const char* ta_env = std::getenv("WQ_V1TC_TA");
  const bool ta = !(ta_env && std::atoi(ta_env) == 0);
  // accumulators: even / odd steps, and NACC = 2 per parity (the MMAs of a
  // step alternate between them) where the columns allow; WQ_V1TC_NACC=1
  // keeps one per parity (tuning)
  const char* nacc_env = std::getenv("WQ_V1TC_NACC");
  p.NACC = (ta ? 4 * p.BN <= kV1TAColA : 4 * p.BN <= 512) ? 2 : 1;
  if (nacc_env && std::atoi(nacc_env) == 1) p.NACC = 1;
  int cols = 32;
  while (cols < 2 * p.NACC * p.BN) cols *= 2;
  p.tmem_cols = ta ? 512 : cols;      // A slots after the accumulators: 256 + 4 × 64 columns
  const int n_tiles = (p.n_bands + 7) / 8, m_tiles = (M + p.BN - 1) / p.BN;
  // Split K over a cluster of S CTAs (one CTA per SM) while the CTAs still fit
  // one wave; every CTA keeps an even number of 128-k steps.
  int S = 1;
  while (S < 8 && n_tiles * m_tiles * S * 2 <= sms && p.tpb % (4 * S) == 0) S *= 2;
  if (const char* s_env = std::getenv("WQ_V1TC_S")) {  // tests and tuning
    const int sf = std::atoi(s_env);
    if (sf == 1 || sf == 2 || sf == 4 || sf == 8) {
      if (sf > 1 && p.tpb % (2 * sf)) return fail(WQ_ERR_ARG, "WQ_V1TC_S does not split K into an even number of steps per CTA");
      S = sf;
    }
  }
  p.S = S;
  p.nks = p.tpb / S;
  // shared memory: NA A slots (32 KB), NX activation slots, NR raw slots of T
  // steps (one bulk copy of T tiles per band: few, large copies keep the
  // copy engine streaming), row exponents, barriers
  const int x_slot = p.BN * 256;
  p.NA = ta ? kV1TANA : 2;
  // activation slots: with A in TMEM as many as A slots (an activation slot is
  // freed by the same commit as its step's A slot: one commit per step, B200
  // M=32/64/128 14336x4096 25.2/25.9/27.9 us against 25.7/26.4/28.2 with six
  // activation slots and a commit each); with A in shared memory a ring of
  // its own (WQ_V1TC_NX overrides, tuning)
  p.NX = ta ? p.NA : (p.BN <= 32 ? 4 : p.BN <= 64 ? 3 : 2);
  if (const char* nx_env = std::getenv("WQ_V1TC_NX"); nx_env && !ta) p.NX = std::max(2, std::min(8, std::atoi(nx_env)));
  const int budget = kSmemPerSm + 4096 - 1024;
  p.off_a = 0;
  p.off_x = ta ? 0 : p.NA * 32768;
  p.off_raw = p.off_x + p.NX * x_slot;
  const int fixed = 512 + 16 + 8 * (2 * 4 + 2 * p.NX + 2 * p.NA + 1) + 16;
  const char* t_env = std::getenv("WQ_V1TC_T");  // steps per raw slot (tuning)
  p.NR = 3;
  // (+16: room for the band-stride pad below)
  p.T = std::min(16, (budget - p.off_raw - fixed) / (p.NR * 8 * p.tb + p.NR * 8 * 16));
  if (p.T < 2) {
    p.NR = 2;
    p.T = std::min(16, (budget - p.off_raw - fixed) / (p.NR * 8 * p.tb + p.NR * 8 * 16));
  }
  if (t_env) p.T = std::max(1, std::min(p.T, std::atoi(t_env)));
  p.T = std::max(1, std::min(p.T, p.nks));
  if (p.T < 1 || p.NR < 2) return fail(WQ_ERR_UNSUPPORTED, "gemm_v1tc: shared memory plan too large");
  // bands of a raw slot an odd number of 16-byte units apart (the TMEM-A
  // dequant reads chunks of four bands at once: eight bank groups)
  p.band_stride = p.T * p.tb + ((p.T * p.tb / 16) % 2 == 0 ? 16 : 0);
  p.off_rowe = static_cast<int>(round16(static_cast<long long>(p.off_raw) + static_cast<long long>(p.NR) * 8 * p.band_stride));
  p.off_bar = p.off_rowe + 512;
  const int smem = 1024 + p.off_bar + 8 * (2 * p.NR + 2 * p.NX + 2 * p.NA + 1) + 16;
  if (smem > kSmemPerSm + 4096) return fail(WQ_ERR_UNSUPPORTED, "gemm_v1tc: shared memory plan too large");
  if (S > 1 && 512 * p.BN > p.off_rowe) return fail(WQ_ERR_UNSUPPORTED, "gemm_v1tc: cluster partials do not fit");
  int rc = encode_2d(&p.tmap_x, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, x, K, M, 2ull * K, 64, p.BN, CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc) return rc;
  {
    static std::mutex mu;
    static bool configured[2][64] = {};
    std::lock_guard<std::mutex> lk(mu);
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !configured[ta][dev]) {
      cudaError_t e = cudaFuncSetAttribute(
          ta ? reinterpret_cast<const void*>(&gemm_v1tc_kernel<true>) : reinterpret_cast<const void*>(&gemm_v1tc_kernel<false>),
          cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemPerSm + 4096);
      if (e != cudaSuccess) return fail(WQ_ERR_CUDA, std::string("cudaFuncSetAttribute: ") + cudaGetErrorString(e));
      configured[ta][dev] = true;
    }
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(n_tiles * S, m_tiles, 1);
  cfg.blockDim = dim3(kV1TCWarps * 32, 1, 1);
  // one CTA per SM: a second CTA would wait in tcgen05.alloc for the first
  // one's 512 columns, and with clusters two such waits could close a cycle
  cfg.dynamicSmemBytes = ta ? std::max(smem, kSmemPerSm / 2 + 8192) : smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = S;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = S > 1 ? 1 : 0;
  cudaError_t e = ta ? cudaLaunchKernelEx(&cfg, &gemm_v1tc_kernel<true>, p)
                     : cudaLaunchKernelEx(&cfg, &gemm_v1tc_kernel<false>, p);
  if (e != cudaSuccess) return fail(WQ_ERR_CUDA, std::string("gemm_v1tc launch: ") + cudaGetErrorString(e));
  rc = launch_check("gemm_v1tc launch");
  if (rc) return rc;
  char buf[64];
  std::snprintf(buf, sizeof(buf), "int4.gemm.v1tc.%sbn%d.x%d.a%d.t%d.s%d", ta ? "ta." : "", p.BN, p.NX, p.NACC, p.T, S);
  *label = buf;
  return WQ_OK;
}

// int8-activation q4_K GEMM: BN = M rounded up to 16 (at most 128), clusters
// of S CTAs splitting the super-blocks while the CTAs fit one wave.
template <int BN>
int launch_mmq_bn(const void* qa8, const void* sda, const void* w, const void* plane, void* y, int M, int N, int K,
                  int sms, cudaStream_t st, std::string* label) {
  using SH = MMQShape<BN>;
  MMQParams p{};
  p.plane = static_cast<const float*>(plane);
  p.y = y;
  p.M = M;
  p.N = N;
  p.K = K;
  const int Mp = (M + 15) / 16 * 16;
  const int nsb_total = K / 256;
  const int n_tiles = (N + 127) / 128, m_tiles = (M + BN - 1) / BN;
  // the ranks of a cluster take consecutive, nearly equal runs of super-blocks
  int S = 1;
  while (S < 8 && n_tiles * m_tiles * S * 2 <= sms && nsb_total >= 2 * S) S *= 2;
  if (const char* s_env = std::getenv("WQ_MMQ_S")) {  // tests and tuning
    const int sf = std::atoi(s_env);
    if (sf == 1 || sf == 2 || sf == 4 || sf == 8) {
      if (nsb_total < sf) return fail(WQ_ERR_ARG, "WQ_MMQ_S exceeds the super-blocks of K");
      S = sf;
    }
  }
  p.S = S;
  p.nsb_total = nsb_total;
  p.stage_bytes = (SH::STAGE + 1023) / 1024 * 1024;
  p.a_bytes = (SH::A_SLOT + 1023) / 1024 * 1024;
  // three A slots (the unpack warps run a super-block ahead of the rescale)
  // when two stages still fit beside them, else two
  const int bars = 8 * (2 * 8 + 2 * 4 + 5) + 16;
  const int budget = kSmemPerSm + 4096 - 1024 - bars;
  p.NA = budget - 3 * p.a_bytes >= 2 * p.stage_bytes ? 3 : 2;
  if (const char* na_env = std::getenv("WQ_MMQ_NA")) p.NA = std::max(2, std::min(p.NA, std::atoi(na_env)));
  p.NS = std::min(4, (budget - p.NA * p.a_bytes) / p.stage_bytes);
  if (const char* ns_env = std::getenv("WQ_MMQ_NS")) p.NS = std::max(2, std::min(p.NS, std::atoi(ns_env)));
  if (p.NS < 2) return fail(WQ_ERR_UNSUPPORTED, "gemm_q4k_q8: shared memory plan too large");
  p.off_a = p.NS * p.stage_bytes;
  p.off_bar = p.off_a + p.NA * p.a_bytes;
  const int smem = 1024 + p.off_bar + 8 * (2 * p.NS + 2 * p.NA + 5) + 16;
  if (smem > kSmemPerSm + 4096) return fail(WQ_ERR_UNSUPPORTED, "gemm_q4k_q8: shared memory plan too large");
  if (S > 1 && 512 * BN > p.off_a) return fail(WQ_ERR_UNSUPPORTED, "gemm_q4k_q8: cluster partials do not fit");
  const unsigned long long row_bytes = 144ull * nsb_total;
  int rc = encode_2d(&p.tmap_w, CU_TENSOR_MAP_DATA_TYPE_UINT8, w, row_bytes, N, row_bytes, 144, 128,
                     CU_TENSOR_MAP_SWIZZLE_NONE);
  if (rc) return rc;
  if ((rc = encode_2d(&p.tmap_a, CU_TENSOR_MAP_DATA_TYPE_UINT8, qa8, K, M, K, 128, BN, CU_TENSOR_MAP_SWIZZLE_128B)))
    return rc;
  if ((rc = encode_2d(&p.tmap_s, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, sda, 2ull * Mp, K / 32, 8ull * Mp, 2 * BN, 8,
                      CU_TENSOR_MAP_SWIZZLE_NONE)))
    return rc;
  {
    static std::mutex mu;
    static bool configured[64] = {};
    std::lock_guard<std::mutex> lk(mu);
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !configured[dev]) {
      cudaError_t e = cudaFuncSetAttribute(reinterpret_cast<const void*>(&gemm_mmq_kernel<BN>),
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemPerSm + 4096);
      if (e != cudaSuccess) return fail(WQ_ERR_CUDA, std::string("cudaFuncSetAttribute: ") + cudaGetErrorString(e));
      configured[dev] = true;
    }
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(n_tiles * S, m_tiles, 1);
  cfg.blockDim = dim3(kMMQWarps * 32, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = S;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = S > 1 ? 1 : 0;
  cudaError_t e = cudaLaunchKernelEx(&cfg, &gemm_mmq_kernel<BN>, p);
  if (e != cudaSuccess) return fail(WQ_ERR_CUDA, std::string("gemm_q4k_q8 launch: ") + cudaGetErrorString(e));
  if ((rc = launch_check("gemm_q4k_q8 launch"))) return rc;
  char buf[64];
  std::snprintf(buf, sizeof(buf), "q4k.mmq.bn%d.ns%d.na%d.s%d%s", BN, p.NS, p.NA, S, plane ? ".dsc" : "");
  *label = buf;
  return WQ_OK;
}

// Warp-MMA GEMM over the int4 B200_V1 stream (M = 9..64): MG = ceil(M / 8)
// column groups of 8 batch rows, one CTA per 8 bands and K slice, clusters of
// S CTAs splitting K while the CTAs still fit one wave.
template <int MG>
int launch_v1w_mg(const void* x, const uint8_t* w, void* y, int M, int N, int K, int block_size, int sms,
                  cudaStream_t st, std::string* label) {
  V1WParams p{};
  p.w = w;
  p.y = y;
  p.M = M;
  p.N = N;
  p.K = K;
  p.n_bands = (N + 15) / 16;
  p.tpb = K / 128;
  p.tb = int4_v1_tile_bytes(block_size);
  const int n_tiles = (p.n_bands + kV1WBands - 1) / kV1WBands;
  int S = 1;
  while (S < 8 && n_tiles * S * 2 <= sms && p.tpb >= 4 * S) S *= 2;  // every rank keeps at least two steps
  if (const char* s_env = std::getenv("WQ_V1W_S")) {  // tests and tuning
    const int sf = std::atoi(s_env);
    if (sf == 1 || sf == 2 || sf == 4 || sf == 8) {
      if (p.tpb < sf) return fail(WQ_ERR_ARG, "WQ_V1W_S exceeds the 128-k steps of K");
      S = sf;
    }
  }
  p.S = S;
  const int xslot = 8 * MG * 256;
  p.NX = 4;
  p.NR = 3;
  const int bars = 8 * (2 * p.NR + 2 * p.NX) + 16;
  const int budget = kSmemPerSm + 4096 - 1024 - bars;
  const int min_steps = p.tpb / S;
  p.T = std::min(16, (budget - p.NX * xslot - 1024) / (p.NR * kV1WBands * p.tb));
  if (const char* t_env = std::getenv("WQ_V1W_T")) p.T = std::max(1, std::min(p.T, std::atoi(t_env)));
  p.T = std::max(1, std::min(p.T, std::max(1, min_steps)));
  p.off_x = (p.NR * kV1WBands * p.T * p.tb + 1023) / 1024 * 1024;
  p.off_bar = p.off_x + p.NX * xslot;
  const int smem = 1024 + p.off_bar + bars;
  if (smem > kSmemPerSm + 4096 || p.T < 1) return fail(WQ_ERR_UNSUPPORTED, "gemm_v1w: shared memory plan too large");
  if (v1w_par(MG) * 16 * kV1WBands * 8 * MG * 4 > p.off_bar) return fail(WQ_ERR_UNSUPPORTED, "gemm_v1w: partials do not fit");
  int rc = encode_2d(&p.tmap_x, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, x, K, M, 2ull * K, 64, 8 * MG,
                     CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc) return rc;
  {
    static std::mutex mu;
    static bool configured[64] = {};
    std::lock_guard<std::mutex> lk(mu);
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !configured[dev]) {
      cudaError_t e = cudaFuncSetAttribute(reinterpret_cast<const void*>(&gemm_v1w_kernel<MG>),
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemPerSm + 4096);
      if (e != cudaSuccess) return fail(WQ_ERR_CUDA, std::string("cudaFuncSetAttribute: ") + cudaGetErrorString(e));
      configured[dev] = true;
    }
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(n_tiles * S, 1, 1);
  cfg.blockDim = dim3(v1w_warps(MG) * 32, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = S;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = S > 1 ? 1 : 0;
  cudaError_t e = cudaLaunchKernelEx(&cfg, &gemm_v1w_kernel<MG>, p);
  if (e != cudaSuccess) return fail(WQ_ERR_CUDA, std::string("gemm_v1w launch: ") + cudaGetErrorString(e));
  if ((rc = launch_check("gemm_v1w launch"))) return rc;
  char buf[64];
  std::snprintf(buf, sizeof(buf), "int4.gemm.v1w.g%d.t%d.s%d", MG, p.T, S);
  *label = buf;
  return WQ_OK;
}

int launch_v1w(const void* x, const uint8_t* w, void* y, int M, int N, int K, int block_size, int sms,
               cudaStream_t st, std::string* label) {
  if (K % 128 || block_size < 128 || M < 1 || M > 64)
    return fail(WQ_ERR_UNSUPPORTED, "gemm_v1w: needs K % 128 == 0, blocks >= 128 and M <= 64");
  switch ((M + 7) / 8) {
    case 1: return launch_v1w_mg<1>(x, w, y, M, N, K, block_size, sms, st, label);
    case 2: return launch_v1w_mg<2>(x, w, y, M, N, K, block_size, sms, st, label);
    case 3: return launch_v1w_mg<3>(x, w, y, M, N, K, block_size, sms, st, label);
    case 4: return launch_v1w_mg<4>(x, w, y, M, N, K, block_size, sms, st, label);
    case 5: return launch_v1w_mg<5>(x, w, y, M, N, K, block_size, sms, st, label);
    case 6: return launch_v1w_mg<6>(x, w, y, M, N, K, block_size, sms, st, label);
    case 7: return launch_v1w_mg<7>(x, w, y, M, N, K, block_size, sms, st, label);
    default: return launch_v1w_mg<8>(x, w, y, M, N, K, block_size, sms, st, label);
  }
}

// Run one format over all M in chunks of at most 8 rows of x.
template <Fmt F>
int run_gemv(const char* fmt_name, const void* x, const uint8_t* w, const uint8_t* scales, const uint8_t* zeros,
             const uint8_t* plane, void* y, int M, int N, int K, long long row_bytes, int nb, int zb,
             int block_size, bool fast_ok, cudaStream_t st, int layout = WQ_LAYOUT_CANONICAL) {
  DeviceInfo di;
  int rc = device_info(&di);
  if (rc) return rc;
  std::string label;
  const int x_elt = 2;
  {
    // batches of 9 and more: one tcgen05 dequant-then-MMA launch (int4 canonical, q4_K)
    const char* force = forced_variant();
    const bool tc5_ok = (F == Fmt::Int4 && layout == WQ_LAYOUT_CANONICAL && K % 256 == 0 && block_size >= 64) ||
                        (F == Fmt::Q4K && layout == WQ_LAYOUT_CANONICAL && K % 256 == 0) ||
                        (F == Fmt::BF16 && K % 8 == 0 && aligned16(w));
    const bool want = force ? std::strcmp(force, "tc5") == 0 : M >= 9;
    if constexpr (F == Fmt::Int4) {
      // B200_V1 int4 with blocks of at least 128: the tcgen05 kernel reads the band stream itself
      const bool v1tc_ok = layout == WQ_LAYOUT_B200_V1 && K % 128 == 0 && block_size >= 128 && aligned16(x);
      // The tcgen05 kernel from 25 rows, and from 9 rows when its 128-row tiles
      // alone fill the GPU (no K split); otherwise the warp-MMA GEMM over the
      // stream up to 24 rows.  B200, M=16 / 24: 14336x4096 v1tc 25.7 / 25.6 us
      // against v1w 26.6 / 32.4, 32000x4096 50.4 / 50.3 against 53.1 / 64.5;
      // 4096x14336 (K split) v1w 25.1 / 27.5 against 26.9 / 29.4, 4096x4096
      // 11.6 / 13.1 against 13.9 / 16.4.  M=64 14336x4096: v1tc 25.9, v1w 64.5.
      const bool v1tc_fills = ((N + 127) / 128) * ((M + 127) / 128) * 2 > di.sms;
      const bool want_v1w = force ? std::strcmp(force, "v1w") == 0 : (M >= 9 && M <= 24 && !v1tc_fills);
      if (v1tc_ok && want_v1w) {
        rc = launch_v1w(x, w, y, M, N, K, block_size, di.sms, st, &label);
        if (rc) return rc;
        set_last_kernel(label);
        return WQ_OK;
      }
      const bool want_v1tc = force ? std::strcmp(force, "v1tc") == 0 : (M > 24 || (M >= 9 && v1tc_fills));
      if (v1tc_ok && want_v1tc) {
        rc = launch_v1tc(x, w, y, M, N, K, block_size, di.sms, st, &label);
        if (rc) return rc;
        set_last_kernel(label);
        return WQ_OK;
      }
    }
    if (tc5_ok && want && aligned16(x)) {
      if constexpr (F == Fmt::Int4 || F == Fmt::Q4K || F == Fmt::BF16) {
        rc = launch_tc5<F>(x, w, scales, zeros, y, M, N, K, nb, zb, block_size, di.sms, st, &label);
        if (rc) return rc;
        set_last_kernel(label);
        return WQ_OK;
      }
    }
  }
  for (int m0 = 0; m0 < M; m0 += 8) {
    const int mc = std::min(8, M - m0);
    const void* xc = static_cast<const uint8_t*>(x) + static_cast<long long>(m0) * K * x_elt;
    void* yc = static_cast<uint8_t*>(y) + static_cast<long long>(m0) * N * 2;
    const char* force = forced_variant();
    if constexpr (F == Fmt::Q4K) {
      if (layout == WQ_LAYOUT_B200_V1) {
        // B200_V1 q4_K: the stream-K band kernel, or the scalar kernel (which
        // reads every layout) when the activations do not fit or it is forced
        V1KPlan kplan;
        const bool want_v1k = force ? std::strcmp(force, "v1k") == 0 : true;
        if (want_v1k && aligned16(xc) && plan_v1k(Fmt::Q4K, mc, N, K, 0, di.sms, &kplan)) {
          kplan.p.x = xc;
          kplan.p.w = w;
          kplan.p.y = yc;
          rc = launch_v1k(kplan, st);
          if (rc) return rc;
          char buf[64];
          std::snprintf(buf, sizeof(buf), "%s.gemv.v1k.m%d.g%d%s", fmt_name, mc, kplan.grid, M > 8 ? ".chunked" : "");
          label = buf;
          continue;
        }
      }
    }
    if constexpr (F == Fmt::Int4) {
      V1RPlan rplan;
      // (the register-streaming kernel measured slower than the bulk-copy ring
      // on B200 for the 4096x14336-class shapes: it runs on request only)
      const bool want_v1r = force ? std::strcmp(force, "v1r") == 0 : false;
      if (want_v1r && layout == WQ_LAYOUT_B200_V1 && aligned16(xc) && plan_v1r(mc, N, K, block_size, di.sms, &rplan)) {
        rplan.p.x = xc;
        rplan.p.w = w;
        rplan.p.y = yc;
        rc = launch_v1r(rplan, st);
        if (rc) return rc;
        char buf[64];
        std::snprintf(buf, sizeof(buf), "%s.gemv.v1r.m%d.p%d%s", fmt_name, mc, rplan.P, M > 8 ? ".chunked" : "");
        label = buf;
        continue;
      }
      // (the stream-K kernel measured slower than the band kernel for int4 on
      // B200 at the 4096x14336 class shapes: it runs on request only)
      V1KPlan kplan;
      const bool want_v1k = force ? std::strcmp(force, "v1k") == 0 : false;
      if (want_v1k && layout == WQ_LAYOUT_B200_V1 && aligned16(xc) &&
          plan_v1k(Fmt::Int4, mc, N, K, block_size, di.sms, &kplan)) {
        kplan.p.x = xc;
        kplan.p.w = w;
        kplan.p.y = yc;
        rc = launch_v1k(kplan, st);
        if (rc) return rc;
        char buf[64];
        std::snprintf(buf, sizeof(buf), "%s.gemv.v1k.m%d.g%d%s", fmt_name, mc, kplan.grid, M > 8 ? ".chunked" : "");
        label = buf;
        continue;
      }
      V1Plan vplan;
      // the band-stream kernel for up to 3 rows of x per chunk; from 4 rows the
      // warp-MMA GEMV over the same stream is faster (B200, M=4 / 6 / 8:
      // 4096x4096 5.7 / 5.8 / 5.9 against 6.6 / 7.4 / 8.2 us; 11008x4096 12.0 /
      // 12.1 / 12.2 against 12.2 / 14.2 / 15.5; 4096x14336 M=4 13.2 against
      // 13.6; 14336x4096 M=4 15.8 against 15.3, M=6 15.9 against 18.2)
      const bool want_v1 = force ? std::strcmp(force, "v1s") == 0 : mc <= 3;
      if (want_v1 && layout == WQ_LAYOUT_B200_V1 && aligned16(xc) &&
          plan_v1(mc, N, K, block_size, di.sms, &vplan)) {
        vplan.p.x = xc;
        vplan.p.w = w;
        vplan.p.y = yc;
        rc = launch_v1(vplan, st);
        if (rc) return rc;
        char buf[64];
        std::snprintf(buf, sizeof(buf), "%s.gemv.v1s.m%d.c%d%s", fmt_name, mc, vplan.p.C, M > 8 ? ".chunked" : "");
        label = buf;
        continue;
      }
    }
    const bool want_tc = force ? std::strcmp(force, "tc") == 0 : true;
    const bool want_cc = force ? std::strcmp(force, "cc") == 0 : true;
    TCPlan tplan;
    const bool tc_layout_ok = layout == WQ_LAYOUT_CANONICAL || F == Fmt::Int4;  // q4_K B200_V1: v1k / scalar only
    if (want_tc && fast_ok && tc_layout_ok && aligned16(xc) &&
        plan_tc(F, mc, N, K, row_bytes, nb, zb, block_size, layout, di.sms, &tplan)) {
      tplan.p.x = xc;
      tplan.p.w = w;
      tplan.p.scales = scales;
      tplan.p.zeros = zeros;
      tplan.p.plane = plane;
      tplan.p.y = yc;
      rc = launch_tc(F, layout, tplan, st);
      if (rc) return rc;
      char buf[64];
      std::snprintf(buf, sizeof(buf), "%s.gemv.tc.m%d%s%s", fmt_name, mc, layout == WQ_LAYOUT_B200_V1 ? ".v1" : "",
                    M > 8 ? ".chunked" : "");
      label = buf;
      continue;
    }
    CCPlan plan;
    const bool use_cc = want_cc && fast_ok && layout == WQ_LAYOUT_CANONICAL && aligned16(xc) &&
                        plan_cc(F, mc, N, K, row_bytes, nb, zb, block_size, zeros != nullptr, di.sms, &plan);
    if (use_cc) {
      plan.p.x = xc;
      plan.p.w = w;
      plan.p.scales = scales;
      plan.p.zeros = zeros;
      plan.p.plane = plane;
      plan.p.y = yc;
      rc = launch_cc(plan, st);
      if (rc) return rc;
      label = cc_label(fmt_name, mc, plan.KS, M > 8 ? ".chunked" : "");
    } else {
      if (force && std::strcmp(force, "simple") != 0)
        return fail(WQ_ERR_UNSUPPORTED, std::string("WQ_FORCE_KERNEL=") + force +
                                            ": that kernel family cannot run this call (format, layout, shape or alignment)");
      SimpleParams sp{};
      sp.x = xc;
      sp.w = w;
      sp.scales = scales;
      sp.zeros = zeros;
      sp.plane = plane;
      sp.y = yc;
      sp.M = mc;
      sp.N = N;
      sp.K = K;
      sp.nb = nb;
      sp.zb = zb;
      sp.block_shift = block_size > 0 ? ilog2_int(block_size) : 0;
      sp.layout = layout;
      rc = launch_simple<F>(sp, mc, di.sms, st);
      if (rc) return rc;
      char buf[64];
      std::snprintf(buf, sizeof(buf), "%s.gemv.simple.m%d%s", fmt_name, mc, M > 8 ? ".chunked" : "");
      label = buf;
    }
  }
  set_last_kernel(label);
  return WQ_OK;
}

int check_dims(int M, int N, int K) {
  if (M <= 0 || N <= 0 || K <= 0) return fail(WQ_ERR_ARG, "M, N and K must be >= 1");
  return WQ_OK;
}

int check_int4(int K, int block_size, int layout) {
  if (layout != WQ_LAYOUT_CANONICAL && layout != WQ_LAYOUT_B200_V1)
    return fail(WQ_ERR_LAYOUT, "unknown int4 layout version");
  if (block_size < 16 || block_size > 256 || (block_size & (block_size - 1)))
    return fail(WQ_ERR_ARG, "block_size must be a power of two in [16, 256]");
  // the last block of a row may be shorter (K - (nb - 1)·block_size codes)
  if (K % 16) return fail(WQ_ERR_ARG, "int4 needs K % 16 == 0");
  if (layout == WQ_LAYOUT_B200_V1 && (K % 128 || block_size < 32))
    return fail(WQ_ERR_ARG, "the B200_V1 int4 layout needs K % 128 == 0 and block_size >= 32");
  return WQ_OK;
}

}  // namespace

int fail(int code, const std::string& msg) {
  t_last_error = msg;
  return code;
}
int ok() { return WQ_OK; }
void set_last_kernel(const std::string& label) { t_last_kernel = label; }

}  // namespace wq

using namespace wq;

extern "C" {

int gemv_int4_blockwise(const void* x_f16, const void* w_packed, const void* scales_f16, const void* zeros_u4,
                        void* y_f16, int M, int N, int K, int block_size, int layout, void* stream) {
  int rc = check_dims(M, N, K);
  if (rc) return rc;
  if ((rc = check_int4(K, block_size, layout))) return rc;
  const bool v1 = layout == WQ_LAYOUT_B200_V1;
  if (v1) {
    scales_f16 = nullptr;  // carried inside the repacked stream
    zeros_u4 = nullptr;
  }
  if (!x_f16 || !w_packed || (!v1 && !scales_f16) || !y_f16)
    return fail(WQ_ERR_ARG, "gemv_int4_blockwise: null pointer");
  if (!aligned16(x_f16) || !aligned16(w_packed) || (scales_f16 && !aligned16(scales_f16)) || !aligned16(y_f16) ||
      (zeros_u4 && !aligned16(zeros_u4)))
    return fail(WQ_ERR_ALIGN, "gemv_int4_blockwise: device pointers must be 16-byte aligned");
  const int nb = (K + block_size - 1) / block_size;
  const int zb = (nb + 1) / 2;
  const long long row_bytes = K / 2;
  const bool fast = (row_bytes % 16) == 0;
  return run_gemv<Fmt::Int4>("int4", x_f16, static_cast<const uint8_t*>(w_packed),
                             static_cast<const uint8_t*>(scales_f16), static_cast<const uint8_t*>(zeros_u4), nullptr,
                             y_f16, M, N, K, row_bytes, nb, zb, block_size, fast, static_cast<cudaStream_t>(stream),
                             layout);
}

int gemv_q4k(const void* x_f16, const void* w_q4k, void* y_f16, int M, int N, int K, int layout, void* stream) {
  int rc = check_dims(M, N, K);
  if (rc) return rc;
  if (layout != WQ_LAYOUT_CANONICAL && layout != WQ_LAYOUT_B200_V1)
    return fail(WQ_ERR_LAYOUT, "unknown q4_K layout version");
  if (K % 256) return fail(WQ_ERR_ARG, "gemv_q4k: K must be a multiple of 256");
  if (!x_f16 || !w_q4k || !y_f16) return fail(WQ_ERR_ARG, "gemv_q4k: null pointer");
  if (!aligned16(x_f16) || !aligned16(w_q4k) || !aligned16(y_f16))
    return fail(WQ_ERR_ALIGN, "gemv_q4k: device pointers must be 16-byte aligned");
  return run_gemv<Fmt::Q4K>("q4k", x_f16, static_cast<const uint8_t*>(w_q4k), nullptr, nullptr, nullptr, y_f16, M,
                            N, K, static_cast<long long>(K / 256) * 144, 0, 0, 0, true,
                            static_cast<cudaStream_t>(stream), layout);
}

int gemv_q4k_noalloc(const void* x_f16, const void* w_q4k, void* y_f16, int M, int N, int K, int layout,
                     void* stream) {
  int rc = check_dims(M, N, K);
  if (rc) return rc;
  if (layout != WQ_LAYOUT_B200_V1)
    return fail(WQ_ERR_LAYOUT, "gemv_q4k_noalloc: reads the B200_V1 q4_K stream (wq_repack_q4k) only");
  if (K % 256) return fail(WQ_ERR_ARG, "gemv_q4k_noalloc: K must be a multiple of 256");
  if ((N + 15) / 16 > kNaMaxBands)
    return fail(WQ_ERR_ARG, "gemv_q4k_noalloc: N above the fixed scratch maximum of 65536 rows");
  if (!x_f16 || !w_q4k || !y_f16) return fail(WQ_ERR_ARG, "gemv_q4k_noalloc: null pointer");
  if (!aligned16(x_f16) || !aligned16(w_q4k) || !aligned16(y_f16))
    return fail(WQ_ERR_ALIGN, "gemv_q4k_noalloc: device pointers must be 16-byte aligned");
  DeviceInfo di;
  if ((rc = device_info(&di))) return rc;
  uint8_t* scratch = nullptr;
  if ((rc = noalloc_scratch(&scratch))) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int n_bands = (N + 15) / 16;
  // counters start each call at zero (a call that gave up may have left some set)
  cudaError_t e = cudaMemsetAsync(scratch, 0, static_cast<size_t>(n_bands) * 4, st);
  if (e != cudaSuccess) return fail(WQ_ERR_CUDA, std::string("scratch clear: ") + cudaGetErrorString(e));
  std::string label;
  for (int m0 = 0; m0 < M; m0 += 8) {
    const int mc = std::min(8, M - m0);
    V1KPlan plan;
    if (!plan_v1k(Fmt::Q4K, mc, N, K, 0, di.sms, &plan))
      return fail(WQ_ERR_UNSUPPORTED, "gemv_q4k_noalloc: the activations of this call do not fit the kernel");
    plan.grid = std::min(plan.grid, kNaMaxCtas);
    plan.p.counters = reinterpret_cast<int*>(scratch);
    plan.p.partials = reinterpret_cast<float*>(scratch + static_cast<size_t>(kNaMaxBands) * 4);
    plan.p.x = static_cast<const uint8_t*>(x_f16) + static_cast<long long>(m0) * K * 2;
    plan.p.w = static_cast<const uint8_t*>(w_q4k);
    plan.p.y = static_cast<uint8_t*>(y_f16) + static_cast<long long>(m0) * N * 2;
    if ((rc = launch_v1k(plan, st, false))) return rc;
    char buf[64];
    std::snprintf(buf, sizeof(buf), "q4k.gemv.v1k.noalloc.m%d.g%d%s", mc, plan.grid, M > 8 ? ".chunked" : "");
    label = buf;
  }
  set_last_kernel(label);
  return WQ_OK;
}

int gemv_q4k_dsc(const void* x_f16, const void* w_q4k, const void* w_dsc, void* y_f16, int M, int N, int K,
                 int layout, void* stream) {
  int rc = check_dims(M, N, K);
  if (rc) return rc;
  if (layout != WQ_LAYOUT_CANONICAL) return fail(WQ_ERR_LAYOUT, "unknown q4_K layout version");
  if (K % 256) return fail(WQ_ERR_ARG, "gemv_q4k_dsc: K must be a multiple of 256");
  if (!x_f16 || !w_q4k || !w_dsc || !y_f16) return fail(WQ_ERR_ARG, "gemv_q4k_dsc: null pointer");
  if (!aligned16(x_f16) || !aligned16(w_q4k) || !aligned16(w_dsc) || !aligned16(y_f16))
    return fail(WQ_ERR_ALIGN, "gemv_q4k_dsc: device pointers must be 16-byte aligned");
  return run_gemv<Fmt::Q4KDsc>("q4k_dsc", x_f16, static_cast<const uint8_t*>(w_q4k), nullptr, nullptr,
                               static_cast<const uint8_t*>(w_dsc), y_f16, M, N, K,
                               static_cast<long long>(K / 256) * 144, 0, 0, 0, true,
                               static_cast<cudaStream_t>(stream));
}

int gemv_bf16(const void* x_bf16, const void* w_bf16, void* y_bf16, int M, int N, int K, void* stream) {
  int rc = check_dims(M, N, K);
  if (rc) return rc;
  if (!x_bf16 || !w_bf16 || !y_bf16) return fail(WQ_ERR_ARG, "gemv_bf16: null pointer");
  if (!aligned2(x_bf16) || !aligned2(w_bf16) || !aligned2(y_bf16))
    return fail(WQ_ERR_ARG, "gemv_bf16: pointers must be 2-byte aligned");
  const bool fast = aligned16(x_bf16) && aligned16(w_bf16) && (K % 8) == 0;
  return run_gemv<Fmt::BF16>("bf16", x_bf16, static_cast<const uint8_t*>(w_bf16), nullptr, nullptr, nullptr, y_bf16,
                             M, N, K, 2ll * K, 0, 0, 0, fast, static_cast<cudaStream_t>(stream));
}

int gemv_mxfp4(const void* x_f16, const void* w_packed, const void* scales_e8m0, void* y_f16, int M, int N, int K,
               void* stream) {
  int rc = check_dims(M, N, K);
  if (rc) return rc;
  if (K % 32) return fail(WQ_ERR_ARG, "gemv_mxfp4: K must be a multiple of 32");
  if (!x_f16 || !w_packed || !scales_e8m0 || !y_f16) return fail(WQ_ERR_ARG, "gemv_mxfp4: null pointer");
  if (!aligned16(x_f16) || !aligned16(w_packed) || !aligned2(y_f16))
    return fail(WQ_ERR_ALIGN, "gemv_mxfp4: x and w_packed must be 16-byte aligned, y 2-byte aligned");
  if (const char* force = forced_variant())
    if (std::strcmp(force, "mx") != 0)
      return fail(WQ_ERR_UNSUPPORTED, std::string("WQ_FORCE_KERNEL=") + force + ": mxfp4 has one kernel family (mx)");
  DeviceInfo di;
  if ((rc = device_info(&di))) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  for (int m0 = 0; m0 < M; m0 += 8) {  // batches past 8 rows run in chunks of 8 (W is read once per chunk)
    MXParams p{};
    p.x = static_cast<const uint8_t*>(x_f16) + static_cast<long long>(m0) * K * 2;
    p.w = static_cast<const uint8_t*>(w_packed);
    p.scales = static_cast<const uint8_t*>(scales_e8m0);
    p.y = static_cast<uint8_t*>(y_f16) + static_cast<long long>(m0) * N * 2;
    p.M = std::min(8, M - m0);
    p.N = N;
    p.K = K;
    gemv_mxfp4_kernel<<<(N + 15) / 16, kMXWarps * 32, 0, st>>>(p);
    if ((rc = launch_check("gemv_mxfp4 launch"))) return rc;
  }
  char buf[64];
  std::snprintf(buf, sizeof(buf), "mxfp4.gemv.mx.m%d%s", std::min(8, M), M > 8 ? ".chunked" : "");
  set_last_kernel(buf);
  return WQ_OK;
}

int wq_tp_rows(int N, int world, int rank, int align, int* n0, int* n1) {
  if (N <= 0 || world <= 0 || rank < 0 || rank >= world || align <= 0 || !n0 || !n1)
    return fail(WQ_ERR_ARG, "wq_tp_rows: need N, world, align > 0, 0 <= rank < world and output pointers");
  const long long units = (static_cast<long long>(N) + align - 1) / align;
  const long long base = units / world, extra = units % world;
  const long long u0 = rank * base + std::min<long long>(rank, extra);
  const long long cnt = base + (rank < extra ? 1 : 0);
  *n0 = static_cast<int>(std::min<long long>(N, u0 * align));
  *n1 = static_cast<int>(std::min<long long>(N, (u0 + cnt) * align));
  return WQ_OK;
}

int gemv_int4_tp(const void* x_f16, const void* w_shard, void* const* y_dsts, int n_dsts, int M, int N_shard, int K,
                 int block_size, int N_total, int n_offset, void* stream) {
  int rc = check_dims(M, N_shard, K);
  if (rc) return rc;
  if ((rc = check_int4(K, block_size, WQ_LAYOUT_B200_V1))) return rc;
  if (!x_f16 || !w_shard || !y_dsts) return fail(WQ_ERR_ARG, "gemv_int4_tp: null pointer");
  if (n_dsts < 1 || n_dsts > kV1MaxDst) return fail(WQ_ERR_ARG, "gemv_int4_tp: 1 to 8 destinations");
  if (n_offset < 0 || N_total < N_shard || n_offset > N_total - N_shard)
    return fail(WQ_ERR_ARG, "gemv_int4_tp: the shard's rows must lie inside the full output");
  for (int d = 0; d < n_dsts; ++d)
    if (!y_dsts[d] || !aligned2(y_dsts[d])) return fail(WQ_ERR_ALIGN, "gemv_int4_tp: destinations must be 2-byte aligned device pointers");
  if (!aligned16(x_f16) || !aligned16(w_shard)) return fail(WQ_ERR_ALIGN, "gemv_int4_tp: x and w_shard must be 16-byte aligned");
  if (const char* force = forced_variant())
    if (std::strcmp(force, "v1s") != 0)
      return fail(WQ_ERR_UNSUPPORTED, std::string("WQ_FORCE_KERNEL=") + force + ": the row-split GEMV runs the v1s kernel only");
  DeviceInfo di;
  if ((rc = device_info(&di))) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int mc_first = 0;
  for (int m0 = 0; m0 < M; m0 += 8) {  // batches past 8 rows in chunks of 8 (the shard is read once per chunk)
    const int mc = std::min(8, M - m0);
    if (m0 == 0) mc_first = mc;
    V1Plan vplan;
    if (!plan_v1(mc, N_shard, K, block_size, di.sms, &vplan))
      return fail(WQ_ERR_UNSUPPORTED, "gemv_int4_tp: needs blocks >= 128 and K % 128 == 0 (B200_V1 band kernel)");
    vplan.p.x = static_cast<const uint8_t*>(x_f16) + 2ll * m0 * K;
    vplan.p.w = static_cast<const uint8_t*>(w_shard);
    vplan.p.y = static_cast<uint8_t*>(y_dsts[0]) + 2ll * m0 * N_total;
    for (int d = 0; d < n_dsts; ++d) vplan.p.ydst[d] = static_cast<uint8_t*>(y_dsts[d]) + 2ll * m0 * N_total;
    vplan.p.n_dst = n_dsts;
    vplan.p.y_ld = N_total;
    vplan.p.y_off = n_offset;
    if ((rc = launch_v1(vplan, st))) return rc;
  }
  char buf[64];
  std::snprintf(buf, sizeof(buf), "int4.gemv.v1s.tp.m%d.d%d%s", mc_first, n_dsts, M > 8 ? ".chunked" : "");
  set_last_kernel(buf);
  return WQ_OK;
}

// cuMemGetAddressRange from the driver, looked up once (no link-time
// dependency on libcuda): the allocation an IPC handle stands for.
using MemRangeFn = CUresult (*)(CUdeviceptr*, size_t*, CUdeviceptr);
MemRangeFn mem_range_fn() {
  static MemRangeFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, []() {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<MemRangeFn>(f);
    else
      cudaGetLastError();
  });
  return fn;
}

int wq_ipc_handle(const void* dev_ptr, void* handle_out, unsigned long long* offset_out) {
  if (!dev_ptr || !handle_out || !offset_out) return fail(WQ_ERR_ARG, "wq_ipc_handle: null pointer");
  MemRangeFn range = mem_range_fn();
  if (!range) return fail(WQ_ERR_CUDA, "cuMemGetAddressRange is not available from the driver");
  CUdeviceptr base = 0;
  size_t size = 0;
  if (range(&base, &size, reinterpret_cast<CUdeviceptr>(dev_ptr)) != CUDA_SUCCESS)
    return fail(WQ_ERR_ARG, "wq_ipc_handle: not a device allocation");
  cudaIpcMemHandle_t h;
  cudaError_t e = cudaIpcGetMemHandle(&h, reinterpret_cast<void*>(base));
  if (e != cudaSuccess) return fail(WQ_ERR_CUDA, std::string("cudaIpcGetMemHandle: ") + cudaGetErrorString(e));
  std::memcpy(handle_out, &h, sizeof(h));
  *offset_out = static_cast<unsigned long long>(reinterpret_cast<CUdeviceptr>(dev_ptr) - base);
  return WQ_OK;
}

int wq_ipc_open(const void* handle, unsigned long long offset, void** dev_ptr_out) {
  if (!handle || !dev_ptr_out) return fail(WQ_ERR_ARG, "wq_ipc_open: null pointer");
  cudaIpcMemHandle_t h;
  std::memcpy(&h, handle, sizeof(h));
  void* base = nullptr;
  cudaError_t e = cudaIpcOpenMemHandle(&base, h, cudaIpcMemLazyEnablePeerAccess);
  if (e != cudaSuccess) return fail(WQ_ERR_CUDA, std::string("cudaIpcOpenMemHandle: ") + cudaGetErrorString(e));
  *dev_ptr_out = static_cast<uint8_t*>(base) + offset;
  return WQ_OK;
}

int wq_ipc_close(void* dev_ptr, unsigned long long offset) {
  if (!dev_ptr) return fail(WQ_ERR_ARG, "wq_ipc_close: null pointer");
  cudaError_t e = cudaIpcCloseMemHandle(static_cast<uint8_t*>(dev_ptr) - offset);
  if (e != cudaSuccess) return fail(WQ_ERR_CUDA, std::string("cudaIpcCloseMemHandle: ") + cudaGetErrorString(e));
  return WQ_OK;
}

size_t wq_q8_bytes(int M, int K) {
  if (M <= 0 || K <= 0 || K % 32) return 0;
  return static_cast<size_t>(M) * K;
}

size_t wq_q8_scale_bytes(int M, int K) {
  if (M <= 0 || K <= 0 || K % 32) return 0;
  return static_cast<size_t>(K / 32) * ((M + 15) / 16 * 16) * 8;
}

int quantize_q8(const void* x_f16, void* qa8, void* sda, int M, int K, void* stream) {
  int rc = check_dims(M, 1, K);
  if (rc) return rc;
  if (K % 32) return fail(WQ_ERR_ARG, "quantize_q8: K must be a multiple of 32");
  if (!x_f16 || !qa8 || !sda) return fail(WQ_ERR_ARG, "quantize_q8: null pointer");
  if (!aligned16(x_f16) || !aligned16(qa8) || !aligned16(sda))
    return fail(WQ_ERR_ALIGN, "quantize_q8: device pointers must be 16-byte aligned");
  DeviceInfo di;
  if ((rc = device_info(&di))) return rc;
  const int Mp = (M + 15) / 16 * 16;
  const long long items = static_cast<long long>(K / 32) * Mp;
  const int grid = static_cast<int>(std::min<long long>((items + 255) / 256, di.sms * 16ll));
  quantize_q8_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const __half*>(x_f16), static_cast<int8_t*>(qa8), static_cast<float2*>(sda), M, Mp, K);
  if ((rc = launch_check("quantize_q8 launch"))) return rc;
  set_last_kernel("q8.quantize");
  return WQ_OK;
}

int gemm_q4k_q8(const void* qa8, const void* sda, const void* w_q4k, const void* w_dsc, void* y_f16, int M, int N,
                int K, void* stream) {
  int rc = check_dims(M, N, K);
  if (rc) return rc;
  if (K % 256) return fail(WQ_ERR_ARG, "gemm_q4k_q8: q4_K needs K % 256 == 0");
  if (!qa8 || !sda || !w_q4k || !y_f16) return fail(WQ_ERR_ARG, "gemm_q4k_q8: null pointer");
  if (!aligned16(qa8) || !aligned16(sda) || !aligned16(w_q4k) || (w_dsc && !aligned16(w_dsc)) || !aligned2(y_f16))
    return fail(WQ_ERR_ALIGN, "gemm_q4k_q8: qa8, sda, w_q4k and w_dsc must be 16-byte aligned, y 2-byte aligned");
  if (const char* force = forced_variant())
    if (std::strcmp(force, "mmq") != 0)
      return fail(WQ_ERR_UNSUPPORTED, std::string("WQ_FORCE_KERNEL=") + force + ": the int8-activation GEMM has one kernel family (mmq)");
  DeviceInfo di;
  if ((rc = device_info(&di))) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  std::string label;
  const int bn = std::min(128, (M + 15) / 16 * 16);
  if (bn == 16)
    rc = launch_mmq_bn<16>(qa8, sda, w_q4k, w_dsc, y_f16, M, N, K, di.sms, st, &label);
  else if (bn == 32)
    rc = launch_mmq_bn<32>(qa8, sda, w_q4k, w_dsc, y_f16, M, N, K, di.sms, st, &label);
  else if (bn <= 64)
    rc = launch_mmq_bn<64>(qa8, sda, w_q4k, w_dsc, y_f16, M, N, K, di.sms, st, &label);
  else
    rc = launch_mmq_bn<128>(qa8, sda, w_q4k, w_dsc, y_f16, M, N, K, di.sms, st, &label);
  if (rc) return rc;
  set_last_kernel(label);
  return WQ_OK;
}

int dequant_mxfp4(const void* w_packed, const void* scales_e8m0, float* w_out, int N, int K, void* stream) {
  int rc = check_dims(1, N, K);
  if (rc) return rc;
  if (K % 32) return fail(WQ_ERR_ARG, "dequant_mxfp4: K must be a multiple of 32");
  if (!w_packed || !scales_e8m0 || !w_out) return fail(WQ_ERR_ARG, "dequant_mxfp4: null pointer");
  if (!aligned16(w_packed) || !aligned16(w_out))
    return fail(WQ_ERR_ALIGN, "dequant_mxfp4: w_packed and w_out must be 16-byte aligned");
  DeviceInfo di;
  if ((rc = device_info(&di))) return rc;
  const long long bytes = static_cast<long long>(N) * (K / 2);
  const int grid = static_cast<int>(std::min<long long>((bytes + 255) / 256, di.sms * 32ll));
  dequant_mxfp4_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint8_t*>(w_packed), static_cast<const uint8_t*>(scales_e8m0), w_out, N, K);
  if ((rc = launch_check("dequant_mxfp4 launch"))) return rc;
  set_last_kernel("mxfp4.dequant");
  return WQ_OK;
}

int dequant_int4_blockwise(const void* w_packed, const void* scales_f16, const void* zeros_u4, float* w_out, int N,
                           int K, int block_size, int layout, void* stream) {
  int rc = check_dims(1, N, K);
  if (rc) return rc;
  if ((rc = check_int4(K, block_size, layout))) return rc;
  const bool v1 = layout == WQ_LAYOUT_B200_V1;
  if (v1) {
    scales_f16 = nullptr;
    zeros_u4 = nullptr;
  }
  if (!w_packed || (!v1 && !scales_f16) || !w_out) return fail(WQ_ERR_ARG, "dequant_int4_blockwise: null pointer");
  if (!aligned16(w_packed) || (scales_f16 && !aligned16(scales_f16)) || (zeros_u4 && !aligned16(zeros_u4)) ||
      !aligned16(w_out))
    return fail(WQ_ERR_ALIGN, "dequant_int4_blockwise: device pointers must be 16-byte aligned");
  DeviceInfo di;
  if ((rc = device_info(&di))) return rc;
  const int nb = (K + block_size - 1) / block_size;
  const long long words = static_cast<long long>(N) * (K / 8);
  const int grid = static_cast<int>(std::min<long long>((words + 255) / 256, di.sms * 32ll));
  dequant_int4_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint8_t*>(w_packed), static_cast<const uint8_t*>(scales_f16),
      static_cast<const uint8_t*>(zeros_u4), w_out, N, K, nb, (nb + 1) / 2, ilog2_int(block_size), layout);
  if ((rc = launch_check("dequant_int4 launch"))) return rc;
  set_last_kernel(layout == WQ_LAYOUT_B200_V1 ? "int4.dequant.v1" : "int4.dequant");
  return WQ_OK;
}

int dequant_q4k(const void* w_q4k, const void* w_dsc, float* w_out, int N, int K, int layout, void* stream) {
  int rc = check_dims(1, N, K);
  if (rc) return rc;
  if (layout != WQ_LAYOUT_CANONICAL && layout != WQ_LAYOUT_B200_V1)
    return fail(WQ_ERR_LAYOUT, "unknown q4_K layout version");
  if (layout == WQ_LAYOUT_B200_V1 && w_dsc)
    return fail(WQ_ERR_LAYOUT, "dequant_q4k: the B200_V1 q4_K stream carries its coefficients; w_dsc must be NULL");
  if (K % 256) return fail(WQ_ERR_ARG, "dequant_q4k: K must be a multiple of 256");
  if (!w_q4k || !w_out) return fail(WQ_ERR_ARG, "dequant_q4k: null pointer");
  if (!aligned16(w_q4k) || (w_dsc && !aligned16(w_dsc)) || !aligned16(w_out))
    return fail(WQ_ERR_ALIGN, "dequant_q4k: device pointers must be 16-byte aligned");
  DeviceInfo di;
  if ((rc = device_info(&di))) return rc;
  if (layout == WQ_LAYOUT_B200_V1) {
    const long long vwords = static_cast<long long>(N) * (K / 8);
    const int vgrid = static_cast<int>(std::min<long long>((vwords + 255) / 256, di.sms * 32ll));
    dequant_q4k_v1_kernel<<<vgrid, 256, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<const uint8_t*>(w_q4k),
                                                                                w_out, N, K);
    if ((rc = launch_check("dequant_q4k_v1 launch"))) return rc;
    set_last_kernel("q4k.dequant.v1");
    return WQ_OK;
  }
  const long long words = static_cast<long long>(N) * (K / 256) * 32;
  const int grid = static_cast<int>(std::min<long long>((words + 255) / 256, di.sms * 32ll));
  dequant_q4k_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint8_t*>(w_q4k), static_cast<const uint8_t*>(w_dsc), w_out, N, K);
  if ((rc = launch_check("dequant_q4k launch"))) return rc;
  set_last_kernel(w_dsc ? "q4k_dsc.dequant" : "q4k.dequant");
  return WQ_OK;
}

int wq_repack_int4(const void* w_canonical, const void* scales_f16, const void* zeros_u4, void* w_out, int N, int K,
                   int block_size, int to_layout, void* stream) {
  if (N <= 0 || K <= 0) return fail(WQ_ERR_ARG, "wq_repack_int4: need N, K > 0");
  if (!w_canonical || !scales_f16 || !w_out) return fail(WQ_ERR_ARG, "wq_repack_int4: null pointer");
  if (to_layout != WQ_LAYOUT_B200_V1) return fail(WQ_ERR_LAYOUT, "wq_repack_int4: target layout must be B200_V1");
  if (block_size < 32 || block_size > 256 || (block_size & (block_size - 1)) || K % 128)
    return fail(WQ_ERR_ARG, "wq_repack_int4: B200_V1 needs a power-of-two block in [32, 256] and K % 128 == 0");
  if (!aligned16(w_canonical) || !aligned16(scales_f16) || (zeros_u4 && !aligned16(zeros_u4)) || !aligned16(w_out))
    return fail(WQ_ERR_ALIGN, "wq_repack_int4: device pointers must be 16-byte aligned");
  DeviceInfo di;
  int rc = device_info(&di);
  if (rc) return rc;
  const long long tiles = static_cast<long long>((N + 15) / 16) * (K / 128);
  const int g1 = static_cast<int>(std::min<long long>((tiles * 64 + 255) / 256, di.sms * 32ll));
  repack_int4_v1_codes_kernel<<<g1, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint8_t*>(w_canonical), static_cast<uint8_t*>(w_out), N, K, block_size);
  if ((rc = launch_check("repack_int4 codes launch"))) return rc;
  const long long items = tiles * int4_v1_bpt(block_size) * 8;
  const int g2 = static_cast<int>(std::min<long long>((items + 255) / 256, di.sms * 32ll));
  repack_int4_v1_meta_kernel<<<g2, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint8_t*>(scales_f16), static_cast<const uint8_t*>(zeros_u4), static_cast<uint8_t*>(w_out), N,
      K, block_size);
  if ((rc = launch_check("repack_int4 meta launch"))) return rc;
  set_last_kernel("int4.repack.v1");
  return WQ_OK;
}

int wq_repack_int4_gate_up(const void* w_gate, const void* scales_gate, const void* zeros_gate, const void* w_up,
                           const void* scales_up, const void* zeros_up, void* w_out, int N, int K, int block_size,
                           int to_layout, void* stream) {
  if (N <= 0 || K <= 0) return fail(WQ_ERR_ARG, "wq_repack_int4_gate_up: need N, K > 0");
  if (!w_gate || !scales_gate || !w_up || !scales_up || !w_out)
    return fail(WQ_ERR_ARG, "wq_repack_int4_gate_up: null pointer");
  if (to_layout != WQ_LAYOUT_B200_V1)
    return fail(WQ_ERR_LAYOUT, "wq_repack_int4_gate_up: target layout must be B200_V1");
  if (block_size < 128 || block_size > 256 || (block_size & (block_size - 1)) || K % 128)
    return fail(WQ_ERR_ARG, "wq_repack_int4_gate_up: needs block_size 128 or 256 and K % 128 == 0");
  if (!aligned16(w_gate) || !aligned16(scales_gate) || (zeros_gate && !aligned16(zeros_gate)) || !aligned16(w_up) ||
      !aligned16(scales_up) || (zeros_up && !aligned16(zeros_up)) || !aligned16(w_out))
    return fail(WQ_ERR_ALIGN, "wq_repack_int4_gate_up: device pointers must be 16-byte aligned");
  DeviceInfo di;
  int rc = device_info(&di);
  if (rc) return rc;
  const long long tiles = static_cast<long long>((N + 15) / 16) * (K / 128);
  const int g1 = static_cast<int>(std::min<long long>((tiles * 64 + 255) / 256, di.sms * 32ll));
  const int g2 = static_cast<int>(std::min<long long>((tiles * 8 + 255) / 256, di.sms * 32ll));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const void* ws[2] = {w_gate, w_up};
  const void* ss[2] = {scales_gate, scales_up};
  const void* zs[2] = {zeros_gate, zeros_up};
  for (int h = 0; h < 2; ++h) {  // gate tiles at even tile slots, up tiles at odd ones
    repack_int4_v1_codes_kernel<<<g1, 256, 0, st>>>(static_cast<const uint8_t*>(ws[h]), static_cast<uint8_t*>(w_out), N,
                                                    K, block_size, 2, h);
    if ((rc = launch_check("repack_int4_gate_up codes launch"))) return rc;
    repack_int4_v1_meta_kernel<<<g2, 256, 0, st>>>(static_cast<const uint8_t*>(ss[h]), static_cast<const uint8_t*>(zs[h]),
                                                   static_cast<uint8_t*>(w_out), N, K, block_size, 2, h);
    if ((rc = launch_check("repack_int4_gate_up meta launch"))) return rc;
  }
  set_last_kernel("int4.repack.gate_up.v1");
  return WQ_OK;
}

int gemv_int4_swiglu(const void* x_f16, const void* w_gate_up, void* y_f16, int M, int N, int K, int block_size,
                     int layout, void* stream) {
  int rc = check_dims(M, N, K);
  if (rc) return rc;
  if (layout != WQ_LAYOUT_B200_V1)
    return fail(WQ_ERR_LAYOUT, "gemv_int4_swiglu: the fused gate-up stream exists in the B200_V1 layout only");
  if (block_size < 128 || block_size > 256 || (block_size & (block_size - 1)) || K % 128)
    return fail(WQ_ERR_ARG, "gemv_int4_swiglu: needs block_size 128 or 256 and K % 128 == 0");
  if (!x_f16 || !w_gate_up || !y_f16) return fail(WQ_ERR_ARG, "gemv_int4_swiglu: null pointer");
  if (!aligned16(x_f16) || !aligned16(w_gate_up) || !aligned16(y_f16))
    return fail(WQ_ERR_ALIGN, "gemv_int4_swiglu: device pointers must be 16-byte aligned");
  DeviceInfo di;
  if ((rc = device_info(&di))) return rc;
  // rows of x per launch: at most 8, and few enough that they fit in shared memory
  const int mc_max = std::max(1, std::min(8, kV1KXBudget / (2 * K)));
  if (2 * K > kV1KXBudget) return fail(WQ_ERR_UNSUPPORTED, "gemv_int4_swiglu: K too large for resident activations");
  std::string label;
  for (int m0 = 0; m0 < M; m0 += mc_max) {
    const int mc = std::min(mc_max, M - m0);
    V1KPlan plan;
    if (!plan_v1k(Fmt::Int4, mc, N, K, block_size, di.sms, &plan, true))
      return fail(WQ_ERR_UNSUPPORTED, "gemv_int4_swiglu: no launch plan for this shape");
    plan.p.x = static_cast<const uint8_t*>(x_f16) + static_cast<long long>(m0) * K * 2;
    plan.p.w = static_cast<const uint8_t*>(w_gate_up);
    plan.p.y = static_cast<uint8_t*>(y_f16) + static_cast<long long>(m0) * N * 2;
    if ((rc = launch_v1k(plan, static_cast<cudaStream_t>(stream)))) return rc;
    char buf[64];
    std::snprintf(buf, sizeof(buf), "int4.swiglu.v1k.m%d.g%d%s", mc, plan.grid, M > mc_max ? ".chunked" : "");
    label = buf;
  }
  set_last_kernel(label);
  return WQ_OK;
}

int wq_repack_q4k(const void* w_q4k, void* w_out, int N, int K, int to_layout, void* stream) {
  if (N <= 0 || K <= 0 || K % 256) return fail(WQ_ERR_ARG, "wq_repack_q4k: need N > 0 and K % 256 == 0");
  if (!w_q4k || !w_out) return fail(WQ_ERR_ARG, "wq_repack_q4k: null pointer");
  if (to_layout != WQ_LAYOUT_B200_V1) return fail(WQ_ERR_LAYOUT, "wq_repack_q4k: target layout must be B200_V1");
  if (!aligned16(w_q4k) || !aligned16(w_out))
    return fail(WQ_ERR_ALIGN, "wq_repack_q4k: device pointers must be 16-byte aligned");
  DeviceInfo di;
  int rc = device_info(&di);
  if (rc) return rc;
  const long long tiles = static_cast<long long>((N + 15) / 16) * (K / 256);
  const int g1 = static_cast<int>(std::min<long long>((tiles * 128 + 255) / 256, di.sms * 32ll));
  repack_q4k_v1_codes_kernel<<<g1, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint8_t*>(w_q4k), static_cast<uint8_t*>(w_out), N, K);
  if ((rc = launch_check("repack_q4k codes launch"))) return rc;
  const int g2 = static_cast<int>(std::min<long long>((tiles * 16 + 255) / 256, di.sms * 32ll));
  repack_q4k_v1_meta_kernel<<<g2, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint8_t*>(w_q4k), static_cast<uint8_t*>(w_out), N, K);
  if ((rc = launch_check("repack_q4k meta launch"))) return rc;
  set_last_kernel("q4k.repack.v1");
  return WQ_OK;
}

int wq_build_q4k_dsc_device(const void* w_q4k, void* out, int N, int K, void* stream) {
  if (N <= 0 || K <= 0 || K % 256) return fail(WQ_ERR_ARG, "wq_build_q4k_dsc_device: need N > 0, K % 256 == 0");
  if (!w_q4k || !out) return fail(WQ_ERR_ARG, "wq_build_q4k_dsc_device: null pointer");
  if (!aligned16(w_q4k) || !aligned16(out))
    return fail(WQ_ERR_ALIGN, "wq_build_q4k_dsc_device: device pointers must be 16-byte aligned");
  DeviceInfo di;
  int rc = device_info(&di);
  if (rc) return rc;
  const long long total = static_cast<long long>(K / 32) * N;
  const int grid = static_cast<int>(std::min<long long>((total + 255) / 256, di.sms * 32ll));
  build_q4k_dsc_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<const uint8_t*>(w_q4k),
                                                                            static_cast<float2*>(out), N, K);
  if ((rc = launch_check("build_q4k_dsc launch"))) return rc;
  set_last_kernel("q4k.build_dsc");
  return WQ_OK;
}

const char* wq_last_error(void) { return t_last_error.c_str(); }
const char* wq_last_kernel(void) { return t_last_kernel.c_str(); }
int wq_layout_version(void) { return WQ_LAYOUT_B200_V1; }
const char* wq_build_info(void) {
  return "libwq sm_100a: decode GEMV M<=8 (B200_V1 int4 bulk-copy ring + warp MMA; warp-MMA GEMV for canonical "
         "int4, q4_K raw / W_dsc plane and bf16; CUDA-core and scalar GEMVs), tcgen05 dequant-then-MMA for M>=9 "
         "(int4 canonical, q4_K), device dequant exports, B200_V1 repack, W_dsc plane builders";
}

int wq_test_expire_wait(unsigned long long limit_ns, void* stream) {
  if (limit_ns < 1000ull || limit_ns > 1000000000ull)
    return fail(WQ_ERR_ARG, "wq_test_expire_wait: limit_ns must be in [1e3, 1e9]");
  DeviceInfo di;
  int rc = device_info(&di);
  if (rc) return rc;
  expire_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_ns);
  if ((rc = launch_check("expire_wait launch"))) return rc;
  set_last_kernel("test.expire_wait");
  return WQ_OK;
}

int wq_device_status(void) {
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return fail(WQ_ERR_CUDA, std::string("cudaDeviceSynchronize: ") + cudaGetErrorString(e));
  unsigned int v = 0, zero = 0;
  e = cudaMemcpyFromSymbol(&v, g_device_error, sizeof(v));
  if (e != cudaSuccess) return fail(WQ_ERR_CUDA, std::string("read device error word: ") + cudaGetErrorString(e));
  e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero));
  if (e != cudaSuccess) return fail(WQ_ERR_CUDA, std::string("clear device error word: ") + cudaGetErrorString(e));
  if (v & kDevErrTimeout) {
    reset_workspaces();  // a kernel that gave up may have left split-band counters set
    return fail(WQ_ERR_TIMEOUT, "a bounded device-side wait expired");
  }
  return WQ_OK;
}

}  // extern "C"
