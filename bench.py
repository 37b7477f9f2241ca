#!/usr/bin/env python3
"""Benchmark of the weight-only quantized decode GEMV on B200.

One step = one call of the decode linear layer y = x·Wᵀ (the whole hot path:
weight stream, unpack, dequantize, multiply-accumulate, reduce, epilogue)
over one batch of synthetic activations.  The default workload is the int4
MatMulNBits-style GEMV with block 128, uint4 zero-points, M = 1 and
N×K = 4096×14336 (the 4096×14336-class shape), its weights repacked once at
load time into the versioned B200_V1 stream layout; ``--workload`` picks
another (the canonical-layout, q4_K, bf16 and batched workloads).

Metric: achieved HBM GB/s (weight + scale + zero-point bytes ÷ device time)
and µs per call.  Timing: CUDA graphs of back-to-back calls, each call on the
next of R weight copies whose total exceeds 3× the L2, CUDA events on the
launching stream, barrier + synchronize on both sides, max over ranks; five
repetitions of at least 50 ms and 200 calls each (more when --steps asks for
more), reported as the median with its spread.  Decode workloads also get the
same measurement at M = 1, 2, 4 and 8 on their shape (``per_m``).

``--impl reference`` times the CPU oracle (test infrastructure) on the host
cores, on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from weight_only_quantized_q4_b200 import synth  # noqa: E402

# ---------------------------------------------------------------- workloads


def _int4(M, N, K, bs, zeros, workload, s_lo, s_hi, layout=0):
    return dict(fmt="int4", M=M, N=N, K=K, bs=bs, zeros=zeros, workload=workload, s_lo=s_lo, s_hi=s_hi,
                layout=layout)


WORKLOADS = {
    "int4_b128_zp_m1_4096x14336": _int4(1, 4096, 14336, 128, True, 3, 0.002, 0.01),
    "int4_b128_zp_m4_4096x14336": _int4(4, 4096, 14336, 128, True, 3, 0.002, 0.01),
    "int4_b128_zp_m1_14336x4096": _int4(1, 14336, 4096, 128, True, 3, 0.002, 0.01),
    "int4_b128_zp_m4_14336x4096": _int4(4, 14336, 4096, 128, True, 3, 0.002, 0.01),
    "int4_b128_zp_m1_4096x4096": _int4(1, 4096, 4096, 128, True, 3, 0.002, 0.01),
    "int4_b32_m1_256x1024": _int4(1, 256, 1024, 32, False, 1, 0.005, 0.02),
}
for _M in (1, 2, 4, 8):
    for _N, _K in ((4096, 4096), (11008, 4096), (4096, 11008)):
        WORKLOADS[f"q4k_m{_M}_{_N}x{_K}"] = dict(fmt="q4k", M=_M, N=_N, K=_K, dsc=False, workload=4)
        WORKLOADS[f"q4k_dsc_m{_M}_{_N}x{_K}"] = dict(fmt="q4k", M=_M, N=_N, K=_K, dsc=True, workload=4)
        WORKLOADS[f"q4k_v1_m{_M}_{_N}x{_K}"] = dict(fmt="q4k", M=_M, N=_N, K=_K, dsc=False, workload=4, layout=1)
for _M in (1, 3, 8):
    for _N, _K in ((1536, 1536), (256, 1536), (1536, 6912), (151936, 1536)):
        WORKLOADS[f"bf16_m{_M}_{_N}x{_K}"] = dict(fmt="bf16", M=_M, N=_N, K=_K, workload=2)
for _M in (2, 4, 8):
    WORKLOADS[f"int4_b128_zp_m{_M}_4096x14336"] = _int4(_M, 4096, 14336, 128, True, 3, 0.002, 0.01)
for _M in (1, 2, 4, 8):
    for _N, _K in ((4096, 4096), (14336, 4096), (4096, 14336)):
        WORKLOADS[f"int4_b128_zp_v1_m{_M}_{_N}x{_K}"] = _int4(_M, _N, _K, 128, True, 3, 0.002, 0.01, layout=1)

for _M in (1, 2, 4, 8):
    for _N, _K in ((4096, 4096), (14336, 4096), (4096, 14336)):
        WORKLOADS[f"mxfp4_m{_M}_{_N}x{_K}"] = dict(fmt="mxfp4", M=_M, N=_N, K=_K, workload=6)
    WORKLOADS[f"swiglu_b128_zp_m{_M}_14336x4096"] = dict(fmt="swiglu", M=_M, N=14336, K=4096, bs=128, workload=7)
for _M in (16, 32, 64, 128):
    for _N, _K in ((4096, 4096), (14336, 4096), (4096, 14336), (32000, 4096)):
        WORKLOADS[f"batched_int4_b128_zp_m{_M}_{_N}x{_K}"] = _int4(_M, _N, _K, 128, True, 5, 0.002, 0.01)
        WORKLOADS[f"batched_int4_b128_zp_v1_m{_M}_{_N}x{_K}"] = _int4(_M, _N, _K, 128, True, 5, 0.002, 0.01,
                                                                       layout=1)
        WORKLOADS[f"batched_q4k_m{_M}_{_N}x{_K}"] = dict(fmt="q4k", M=_M, N=_N, K=_K, dsc=False, workload=5)

# int8-activation q4_K (one step = the q8 prepass + the kind::i8 GEMM)
for _M in (16, 32, 64, 128, 512):
    for _N, _K in ((4096, 4096), (11008, 4096), (4096, 11008), (14336, 4096), (32000, 4096)):
        WORKLOADS[f"mmq_q4k_m{_M}_{_N}x{_K}"] = dict(fmt="mmq", M=_M, N=_N, K=_K, workload=5)

DEFAULT_WORKLOAD = "int4_b128_zp_v1_m1_4096x14336"
METRIC = "achieved HBM GB/s and \u00b5s/call per quantized GEMV at M=1..8 vs ~8 TB/s peak"
SWEEP_BATCHED = [f"batched_{f}_m{m}_{n}x{k}" for f in ("int4_b128_zp_v1", "int4_b128_zp", "q4k")
                 for m in (16, 32, 64, 128) for n, k in ((4096, 4096), (14336, 4096), (4096, 14336), (32000, 4096))]
SWEEP_BATCHED += [f"mmq_q4k_m{m}_{n}x{k}" for m in (16, 32, 64, 128, 512)
                  for n, k in ((4096, 4096), (11008, 4096), (4096, 11008), (32000, 4096))]
SWEEP = ["q4k_v1_m1_4096x11008", "q4k_v1_m4_4096x11008", "q4k_v1_m1_11008x4096", "int4_b128_zp_v1_m1_4096x14336", "int4_b128_zp_v1_m2_4096x14336", "int4_b128_zp_v1_m4_4096x14336", "int4_b128_zp_v1_m8_4096x14336",
         "int4_b128_zp_v1_m1_14336x4096", "int4_b128_zp_v1_m1_4096x4096",
         "int4_b128_zp_m1_4096x14336", "int4_b128_zp_m4_4096x14336", "int4_b128_zp_m1_14336x4096",
         "int4_b32_m1_256x1024", "q4k_m1_4096x11008", "q4k_dsc_m1_4096x11008", "q4k_m4_11008x4096",
         "q4k_m8_4096x4096", "mxfp4_m1_4096x14336", "mxfp4_m4_4096x14336", "bf16_m1_1536x6912", "bf16_m3_1536x6912", "bf16_m8_1536x6912", "bf16_m1_151936x1536"]


def weight_bytes(w) -> int:
    """Algorithmic bytes one call must read for the weights (x and y excluded)."""
    N, K = w["N"], w["K"]
    if w["fmt"] == "int4":
        nb = K // w["bs"]
        return N * K // 2 + 2 * N * nb + (N * ((nb + 1) // 2) if w["zeros"] else 0)
    if w["fmt"] == "q4k":
        return N * K // 2 + N * K // 4 if w["dsc"] else N * (K // 256) * 144
    if w["fmt"] == "mmq":
        return N * (K // 256) * 144
    if w["fmt"] == "mxfp4":
        return N * K // 2 + N * K // 32
    if w["fmt"] == "swiglu":  # gate and up: two int4 tensors of N x K
        nb = K // w["bs"]
        return 2 * (N * K // 2 + 2 * N * nb + N * ((nb + 1) // 2))
    return 2 * N * K


def dtype_of(w) -> str:
    return {"int4": "int4xf16->f32", "q4k": "q4kxf16->f32", "bf16": "bf16xbf16->f32",
            "mxfp4": "mxfp4xf16->f32", "swiglu": "int4xf16->f32", "mmq": "q4kxs8->s32->f32"}[w["fmt"]]


def host_inputs(w):
    """Seeded canonical arrays for one workload (numpy)."""
    M, N, K = w["M"], w["N"], w["K"]
    if w["fmt"] == "int4":
        t = synth.int4_weights(N, K, w["bs"], scale_lo=w["s_lo"], scale_hi=w["s_hi"], with_zeros=w["zeros"],
                               workload=w["workload"])
        return dict(x=synth.activations_f16(M, K, workload=w["workload"]), **t)
    if w["fmt"] == "q4k":
        return dict(x=synth.activations_f16(M, K, workload=w["workload"]),
                    raw=synth.q4k_weights(N, K, workload=w["workload"]))
    if w["fmt"] == "mxfp4":
        return dict(x=synth.activations_f16(M, K, workload=w["workload"]), **synth.mxfp4_weights(N, K, workload=w["workload"]))
    if w["fmt"] == "mmq":
        return dict(x=synth.activations_f16(M, K, workload=w["workload"]), raw=synth.q4k_weights(N, K, workload=w["workload"]))
    if w["fmt"] == "swiglu":
        g = synth.int4_weights(N, K, w["bs"], scale_lo=0.002, scale_hi=0.01, with_zeros=True, workload=w["workload"])
        u = synth.int4_weights(N, K, w["bs"], scale_lo=0.002, scale_hi=0.01, with_zeros=True, workload=w["workload"] + 50)
        return dict(x=synth.activations_f16(M, K, workload=w["workload"]), gate=g, up=u)
    return dict(x=synth.activations_bf16_bits(M, K, workload=w["workload"]),
                w=synth.bf16_weights_bits(N, K, workload=w["workload"]))


# ---------------------------------------------------------------- clocks (NVML, read-only)


class ClockSampler:
    """Samples SM clock and throttle reasons with NVML while the timed region runs."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4, "hw_slowdown": 0x8,
        "sync_boost": 0x10, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
        "hw_power_brake_slowdown": 0x80, "display_clock_setting": 0x100,
    }

    def __init__(self, index: int):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        try:
            import pynvml

            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:  # noqa: BLE001 - clocks are reported as unavailable
            self._nv = None
        self._t = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self._nv.nvmlDeviceGetClockInfo(self._h, self._nv.NVML_CLOCK_SM))
                r = self._nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for name, bit in self.REASONS.items():
                    if r & bit and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:  # noqa: BLE001
                pass
            time.sleep(0.005)

    def __enter__(self):
        if self._nv is not None:
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._nv is not None:
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ---------------------------------------------------------------- our arm


class DeviceWorkload:
    """Device buffers for one workload plus a callable that issues one call on copy i."""

    def __init__(self, w, host, torch, wq, l2_bytes, copies=0):
        self.w, self.torch, self.wq = w, torch, wq
        dev = torch.device("cuda", torch.cuda.current_device())
        M, N, K = w["M"], w["N"], w["K"]
        self.M, self.N, self.K = M, N, K
        self.bytes = weight_bytes(w)
        # enough weight copies that a round trip exceeds 3x L2
        self.R = max(1, -(-3 * l2_bytes // max(self.bytes, 1)))
        self.R = min(self.R, max(1, int(8e9 // max(self.bytes, 1))))
        if copies > 0:
            self.R = copies
        self.copies = []
        self.launches_per_call = 1
        if w["fmt"] == "int4":
            base = [torch.from_numpy(host["w_packed"]).to(dev), torch.from_numpy(host["scales"]).to(dev),
                    torch.from_numpy(host["zeros"]).to(dev) if host["zeros"] is not None else None]
            if w.get("layout", 0) == 1:  # offline repack to the B200_V1 stream (codes + scales + zero-points)
                packed = torch.empty(wq.wq_int4_packed_bytes(N, K, w["bs"], 1), dtype=torch.uint8, device=dev)
                wq.wq_repack_int4(base[0], base[1], base[2], packed, N, K, w["bs"], 1)
                base = [packed, None, None]
            for _ in range(self.R):
                self.copies.append([t.clone() if t is not None else None for t in base])
            self.x = torch.from_numpy(host["x"]).to(dev)
            self.y = torch.empty((M, N), dtype=torch.float16, device=dev)
        elif w["fmt"] == "q4k":
            raw = torch.from_numpy(host["raw"]).to(dev)
            if w.get("layout", 0) == 1:  # offline repack to the B200_V1 q4_K band stream
                packed = torch.empty(wq.wq_q4k_packed_bytes(N, K, 1), dtype=torch.uint8, device=dev)
                wq.wq_repack_q4k(raw, packed, N, K, 1)
                raw = packed
            for _ in range(self.R):
                c = [raw.clone()]
                if w["dsc"]:
                    P = torch.empty((K // 32, N, 2), dtype=torch.float32, device=dev)
                    wq.wq_build_q4k_dsc_device(c[0], P, N, K)
                    c.append(P)
                self.copies.append(c)
            self.x = torch.from_numpy(host["x"]).to(dev)
            self.y = torch.empty((M, N), dtype=torch.float16, device=dev)
        elif w["fmt"] == "mmq":
            raw = torch.from_numpy(host["raw"]).to(dev)
            for _ in range(self.R):
                self.copies.append([raw.clone()])
            self.x = torch.from_numpy(host["x"]).to(dev)
            self.y = torch.empty((M, N), dtype=torch.float16, device=dev)
            self.qa = torch.empty((M, K), dtype=torch.int8, device=dev)
            self.sd = torch.empty(wq.wq_q8_scale_bytes(M, K) // 4, dtype=torch.float32, device=dev)
            self.launches_per_call = 2
        elif w["fmt"] == "swiglu":
            d = {h: [torch.from_numpy(host[h][k]).to(dev) for k in ("w_packed", "scales", "zeros")] for h in ("gate", "up")}
            packed = torch.empty(wq.wq_int4_gate_up_packed_bytes(N, K, w["bs"]), dtype=torch.uint8, device=dev)
            wq.wq_repack_int4_gate_up(*d["gate"], *d["up"], packed, N, K, w["bs"])
            for _ in range(self.R):
                self.copies.append([packed.clone()])
            self.x = torch.from_numpy(host["x"]).to(dev)
            self.y = torch.empty((M, N), dtype=torch.float16, device=dev)
        elif w["fmt"] == "mxfp4":
            base = [torch.from_numpy(host["w_packed"]).to(dev), torch.from_numpy(host["scales"]).to(dev)]
            for _ in range(self.R):
                self.copies.append([t.clone() for t in base])
            self.x = torch.from_numpy(host["x"]).to(dev)
            self.y = torch.empty((M, N), dtype=torch.float16, device=dev)
        else:
            wt = torch.from_numpy(host["w"].view(np.int16)).to(dev).view(torch.bfloat16)
            for _ in range(self.R):
                self.copies.append([wt.clone()])
            self.x = torch.from_numpy(host["x"].view(np.int16)).to(dev).view(torch.bfloat16)
            self.y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        torch.cuda.synchronize()

    def batch_buffers(self, M):
        """Activations and output of batch M for the same weights (seeded like the workload's x)."""
        torch, w = self.torch, self.w
        dev = self.x.device
        if w["fmt"] == "bf16":
            x = torch.from_numpy(synth.activations_bf16_bits(M, self.K, workload=w["workload"]).view(np.int16))
            return x.to(dev).view(torch.bfloat16), torch.empty((M, self.N), dtype=torch.bfloat16, device=dev)
        x = torch.from_numpy(synth.activations_f16(M, self.K, workload=w["workload"])).to(dev)
        return x, torch.empty((M, self.N), dtype=torch.float16, device=dev)

    def call(self, i, x=None, y=None, stream=None, M=None):
        c = self.copies[i % self.R]
        x = self.x if x is None else x
        y = self.y if y is None else y
        M = self.M if M is None else M
        w, wq = self.w, self.wq
        if w["fmt"] == "int4":
            wq.gemv_int4_blockwise(x, c[0], c[1], c[2], y, M, self.N, self.K, w["bs"],
                                   layout=w.get("layout", 0), stream=stream)
        elif w["fmt"] == "q4k":
            if w["dsc"]:
                wq.gemv_q4k_dsc(x, c[0], c[1], y, M, self.N, self.K, stream=stream)
            else:
                wq.gemv_q4k(x, c[0], y, M, self.N, self.K, layout=w.get("layout", 0), stream=stream)
        elif w["fmt"] == "mxfp4":
            wq.gemv_mxfp4(x, c[0], c[1], y, M, self.N, self.K, stream=stream)
        elif w["fmt"] == "swiglu":
            wq.gemv_int4_swiglu(x, c[0], y, M, self.N, self.K, w["bs"], stream=stream)
        elif w["fmt"] == "mmq":
            wq.quantize_q8(x, self.qa, self.sd, M, self.K, stream=stream)
            wq.gemm_q4k_q8(self.qa, self.sd, c[0], None, y, M, self.N, self.K, stream=stream)
        else:
            wq.gemv_bf16(x, c[0], y, M, self.N, self.K, stream=stream)


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:  # noqa: BLE001
        return 6650.0, "fallback"


def _kernel_src_hash() -> str:
    """Hash of the kernel sources the committed DRAM counters must match: every
    file under csrc/ with its // comments and trailing blanks removed (a
    comment edit does not change the code the counters were taken on)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "weight_only_quantized_q4_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        path = os.path.join(csrc, name)
        if not os.path.isfile(path):
            continue
        with open(path, encoding="utf-8") as f:
            lines = [ln.split("//", 1)[0].rstrip() for ln in f]
        h.update(name.encode() + "\n".join(ln for ln in lines if ln).encode())
    return h.hexdigest()[:16]


def _traffic(workload: str):
    """Per-launch DRAM bytes from a committed ncu summary, if taken on the current kernel sources."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            t = json.load(f)
        e = t.get(workload)
        if e and e.get("kernel_src_sha") == _kernel_src_hash():
            return e.get("dram_bytes_per_launch")
    except Exception:  # noqa: BLE001
        pass
    return None


def max_over_ranks(vals, dist, device):
    """Each timing as the maximum over ranks (the slowest rank sets the job time)."""
    if dist is None:
        return [float(v) for v in vals]
    import torch

    t = torch.tensor([float(v) for v in vals], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.cpu()]


def job_gbs(world: int, bytes_per_call: int, calls: int, ms: float) -> float:
    """Whole-job GB/s: every rank streams its own weights (replicas), so the job
    moves world × bytes × calls in the max-over-ranks time."""
    return world * bytes_per_call * calls / (ms * 1e-3) / 1e9


def _timed_reps(torch, replay, calls_per_replay, stream, steps_req, reps, min_ms, warmup, barrier):
    """Replay a captured graph of back-to-back calls: `warmup` untimed replays,
    then `reps` timed repetitions, each of enough replays for at least
    `min_ms` milliseconds and 200 calls (and, over all repetitions, at least
    `steps_req` calls), bracketed by a barrier + synchronize on both sides and
    CUDA events on the launching stream.  Returns (replays per repetition,
    [ms per repetition])."""
    for _ in range(max(warmup, 3)):
        replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    replay()
    e1.record(stream)
    torch.cuda.synchronize()
    t_one = max(e0.elapsed_time(e1), 1e-3)
    per_rep = max(1, -(-200 // calls_per_replay), int(np.ceil(min_ms / t_one)),
                  -(-steps_req // (calls_per_replay * reps)))
    times = []
    for _ in range(reps):
        barrier()
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(per_rep):
            replay()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        times.append(e0.elapsed_time(e1))
    return per_rep, times


def _rep_summary(times_ms, calls_per_rep):
    us = sorted(t * 1e3 / calls_per_rep for t in times_ms)
    med = float(statistics.median(us))
    return {"us_per_call_median": round(med, 3), "us_per_call_min": round(us[0], 3),
            "us_per_call_max": round(us[-1], 3), "spread_pct": round(100.0 * (us[-1] - us[0]) / med, 2),
            "reps": len(us), "calls_per_rep": calls_per_rep}


def _capture(torch, d, stream, G, x=None, y=None):
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(G):
            d.call(i, x=x, y=y, stream=torch.cuda.current_stream())
    return g


def run_ours(args, w, wname, rank, world, dist):
    import torch

    import weight_only_quantized_q4_b200 as wq

    torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
    l2 = torch.cuda.get_device_properties(torch.cuda.current_device()).L2_cache_size
    host = host_inputs(w)
    d = DeviceWorkload(w, host, torch, wq, l2, copies=args.copies)
    stream = torch.cuda.Stream()

    def barrier():
        if dist is not None:
            dist.barrier()

    # configure every kernel once outside capture, then capture a graph of G
    # back-to-back calls (a whole number of passes over the R weight copies)
    with torch.cuda.stream(stream):
        d.call(0, stream=stream)
    torch.cuda.synchronize()
    label = wq.last_kernel()
    G = max(d.R, args.graph_calls)
    G = -(-G // d.R) * d.R
    g = _capture(torch, d, stream, G)
    # per-launch durations: events between consecutive calls in a second graph
    n_ev = min(G, 256)
    evs = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(n_ev + 1)]
    g_ev = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_ev, stream=stream):
        cs = torch.cuda.current_stream()
        for i in range(n_ev):
            evs[i].record(cs)
            d.call(i, stream=cs)
        evs[n_ev].record(cs)

    peak, peak_kind = _peaks()
    reps = max(4, args.reps)
    per_m = []
    with ClockSampler(torch.cuda.current_device()) as clk:
        with torch.cuda.stream(stream):
            per_rep, times = _timed_reps(torch, g.replay, G, stream, args.steps, reps, args.min_ms, args.warmup,
                                         barrier)
            # per-launch timing pass (same clocks window)
            for _ in range(3):
                g_ev.replay()
            torch.cuda.synchronize()
            # the same measurement for M = 1, 2, 4, 8 on this shape (decode GEMV workloads)
            if w["M"] <= 8 and not args.no_per_m:
                for Mb in (1, 2, 4, 8):
                    xb, yb = d.batch_buffers(Mb)
                    d.call(0, x=xb, y=yb, M=Mb, stream=stream)
                    torch.cuda.synchronize()
                    gb = torch.cuda.CUDAGraph()
                    with torch.cuda.graph(gb, stream=stream):
                        for i in range(G):
                            d.call(i, x=xb, y=yb, M=Mb, stream=torch.cuda.current_stream())
                    pr, tb = _timed_reps(torch, gb.replay, G, stream, 0, reps, args.min_ms, 3, barrier)
                    tb = max_over_ranks(tb, dist, "cuda")
                    sm_ = _rep_summary(tb, pr * G)
                    gbs = d.bytes / (sm_["us_per_call_median"] * 1e-6) / 1e9
                    per_m.append({"M": Mb, "us_per_call": sm_["us_per_call_median"], "gbs": round(gbs, 1),
                                  "frac": round(gbs / peak, 4), "spread_pct": sm_["spread_pct"],
                                  "calls_timed": pr * G * reps, "kernel": wq.last_kernel()})
                    del gb
    times = max_over_ranks(times, dist, "cuda")
    per_launch = [evs[i].elapsed_time(evs[i + 1]) for i in range(n_ev)]
    avg_launch_ms = float(np.mean(per_launch))
    calls_per_rep = per_rep * G
    rs = _rep_summary(times, calls_per_rep)

    # e2e: every step copies its x in from pinned host memory, runs the GEMV
    # through the API and copies its y out to pinned host memory.  Steps are
    # pipelined as a serving loop would: the host-to-device copy of step i+1
    # and the device-to-host copy of step i-1 run on two copy streams while the
    # GEMV of step i runs, with NB device buffers per tensor and events guarding
    # every reuse (x slot j is rewritten only after the GEMV that read it, y
    # slot j only after the copy that drained it).
    NB = 3
    xh = [torch.empty_like(d.x, device="cpu").pin_memory() for _ in range(NB)]
    for h in xh:
        h.copy_(d.x.cpu())
    yh = [torch.empty_like(d.y, device="cpu").pin_memory() for _ in range(NB)]
    xd = [torch.empty_like(d.x) for _ in range(NB)]
    yd = [torch.empty_like(d.y) for _ in range(NB)]
    Ge = min(G, 256)
    h2d_s, d2h_s = torch.cuda.Stream(), torch.cuda.Stream()
    ev_x = [torch.cuda.Event() for _ in range(Ge)]
    ev_k = [torch.cuda.Event() for _ in range(Ge)]
    ev_y = [torch.cuda.Event() for _ in range(Ge)]
    ge = torch.cuda.CUDAGraph()
    with torch.cuda.graph(ge, stream=stream):
        cs = torch.cuda.current_stream()
        fork = torch.cuda.Event()
        fork.record(cs)
        h2d_s.wait_event(fork)
        d2h_s.wait_event(fork)
        for i in range(Ge):
            j = i % NB
            with torch.cuda.stream(h2d_s):
                if i >= NB:
                    h2d_s.wait_event(ev_k[i - NB])  # the GEMV that read x slot j is done
                xd[j].copy_(xh[j], non_blocking=True)
                ev_x[i].record(h2d_s)
            cs.wait_event(ev_x[i])
            if i >= NB:
                cs.wait_event(ev_y[i - NB])  # y slot j has been copied out
            d.call(i, x=xd[j], y=yd[j], stream=cs)
            ev_k[i].record(cs)
            with torch.cuda.stream(d2h_s):
                d2h_s.wait_event(ev_k[i])
                yh[j].copy_(yd[j], non_blocking=True)
                ev_y[i].record(d2h_s)
        cs.wait_event(ev_x[Ge - 1])
        cs.wait_event(ev_y[Ge - 1])
    with torch.cuda.stream(stream):
        pe, te = _timed_reps(torch, ge.replay, Ge, stream, 0, reps, args.min_ms, 2, barrier)
    # the last step's result (same x, an identical weight copy) must have reached
    # host memory bit for bit: the kernels are deterministic, so a difference
    # would mean a missing dependency in the pipelined copies
    if not torch.equal(yh[(Ge - 1) % NB].view(torch.int16), d.y.cpu().view(torch.int16)):
        raise RuntimeError("e2e: host copy of y differs from the device result")
    te = max_over_ranks(te, dist, "cuda")
    es = _rep_summary(te, pe * Ge)

    bytes_call = d.bytes
    ms_step = rs["us_per_call_median"] * 1e-3
    steps = calls_per_rep * reps
    value = job_gbs(world, bytes_call, 1, ms_step)
    e2e_value = job_gbs(world, bytes_call, 1, es["us_per_call_median"] * 1e-3)
    # one launch of the kernel per step: its median duration over the timed region
    achieved = bytes_call / (ms_step * 1e-3) / 1e9
    out = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": steps,
        "steps_requested": args.steps,
        "warmup": max(args.warmup, 3),
        "ms_per_step": ms_step,
        "us_per_call": rs["us_per_call_median"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": dtype_of(w),
        "data": "synthetic (seeded; value distributions of the workload definition)",
        "config": {"workload": wname, "fmt": w["fmt"], "M": w["M"], "N": w["N"], "K": w["K"],
                   "layout": {0: "canonical", 1: "B200_V1 (offline repack)"}[w.get("layout", 0)],
                   "weight_bytes_per_call": bytes_call, "weight_copies_rotated": d.R,
                   "l2": f"inputs larger than L2: {d.R} rotating weight copies, {d.R * bytes_call / 1e6:.0f} MB "
                         f">= 3x L2 ({l2 / 1e6:.0f} MB)",
                   "timing": f"{reps} repetitions of {calls_per_rep} back-to-back calls (CUDA graph of {G} calls "
                             f"replayed {per_rep}x, >= {args.min_ms:g} ms and >= 200 calls per repetition), CUDA "
                             f"events on the launching stream; value and us_per_call from the median repetition",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU", "kernel": label},
        "timing": rs,
        "e2e": {"value": round(e2e_value, 2), "unit": "GB/s",
                "h2d_bytes_per_step": int(d.x.numel() * d.x.element_size()),
                "d2h_bytes_per_step": int(d.y.numel() * d.y.element_size()),
                "us_per_call": es["us_per_call_median"], "spread_pct": es["spread_pct"],
                "how": "per step: pinned x -> device, GEMV through the C ABI, y -> pinned host; steps pipelined over "
                       "two copy streams with 3 device buffers per tensor (copies of neighbouring steps overlap the "
                       "GEMV); graph-captured; median of the repetitions"},
        "gpu_launches": steps * d.launches_per_call,
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "traffic": _traffic(wname),
                     "peak_kind": f"{peak_kind} copy bandwidth", "avg_launch_us": rs["us_per_call_median"],
                     "isolated_launch_us": round(avg_launch_ms * 1e3, 3),
                     "how": "achieved = algorithmic bytes per launch / median launch duration over the timed "
                            "repetitions (one launch per step, CUDA events on the launching stream); "
                            "isolated_launch_us = events around single launches (no overlap with the next call)"},
        "clocks": clk.summary(),
    }
    if per_m:
        out["per_m"] = per_m
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(w, host, budget_s=args.cpu_budget)
    return out


# ---------------------------------------------------------------- oracle (CPU) arm


def cpu_baseline(w, host, budget_s=15.0):
    """Time the CPU oracle as it stands on the workload's rows, in blocks, cycling
    over the rows until about `budget_s` seconds of work are done; scale to GB/s
    of weights."""
    import oracle

    N, K, M = w["N"], w["K"], w["M"]
    rows = 8
    start, done_rows, t_total = 0, 0, 0.0
    x = host["x"]
    while t_total < budget_s:
        r = np.arange(start, min(start + rows, N))
        t0 = time.perf_counter()
        if w["fmt"] == "int4":
            z = host["zeros"][r] if host["zeros"] is not None else None
            W = oracle.dequant_int4(host["w_packed"][r], host["scales"][r], z, len(r), K, w["bs"])
            xv = x.astype(np.float64)
        elif w["fmt"] == "q4k":
            if w["dsc"]:
                P = oracle.q4k_plane(host["raw"][r], len(r), K)
                W = oracle.dequant_q4k_from_plane(host["raw"][r], P, len(r), K)
            else:
                W = oracle.dequant_q4k(host["raw"][r], len(r), K)
            xv = x.astype(np.float64)
        elif w["fmt"] == "mxfp4":
            W = oracle.dequant_mxfp4(host["w_packed"][r], host["scales"][r], len(r), K)
            xv = x.astype(np.float64)
        elif w["fmt"] == "mmq":
            qa, dq, sq = oracle.quantize_q8(x, M, K)
            oracle.mmq_q4k(host["raw"][r], qa, dq, sq, M, len(r), K)
            W = oracle.dequant_q4k(host["raw"][r], len(r), K)
            xv = oracle.dequant_q8(qa, dq, M, K)
        elif w["fmt"] == "swiglu":
            Wg = oracle.dequant_int4(host["gate"]["w_packed"][r], host["gate"]["scales"][r], host["gate"]["zeros"][r],
                                     len(r), K, w["bs"])
            W = oracle.dequant_int4(host["up"]["w_packed"][r], host["up"]["scales"][r], host["up"]["zeros"][r],
                                    len(r), K, w["bs"])
            xv = x.astype(np.float64)
            oracle.swiglu_gemv(Wg, W, xv)
        else:
            W = oracle.dequant_bf16(host["w"][r], len(r), K)
            xv = oracle.dequant_bf16(x, M, K)
        oracle.gemv(W, xv)
        oracle.bound(W, xv)
        t_total += time.perf_counter() - t0
        done_rows += len(r)
        start = r[-1] + 1 if r[-1] + 1 < N else 0
        rows = min(rows * 2, 4096)
    frac = done_rows / N
    bytes_done = weight_bytes(w) * frac
    gbs = bytes_done / t_total / 1e9
    try:
        cores = len(os.sched_getaffinity(0))
    except Exception:  # noqa: BLE001
        cores = os.cpu_count()
    return {"value": round(gbs, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
            "us_per_call_equiv": round(t_total / frac * 1e6, 1),
            "sample": f"{done_rows} rows of the {N}-row workload ({frac:.2f} passes over it, cycling), numpy fp64 "
                      f"dequant + GEMV + bound, {t_total:.1f} s; threads as numpy/BLAS uses them"}


def run_reference(args, w, wname):
    host = host_inputs(w)
    for _ in range(max(0, min(args.warmup, 1))):
        cpu_baseline(w, host, budget_s=0.5)
    budget = max(1.0, min(args.cpu_budget, 120.0 / max(1, args.steps)))
    vals = [cpu_baseline(w, host, budget_s=budget) for _ in range(max(1, min(args.steps, 8)))]
    v = float(np.median([c["value"] for c in vals]))
    cb = dict(vals[0])
    cb["value"] = round(v, 4)
    return {
        "metric": METRIC,
        "value": round(v, 4), "unit": "GB/s", "n_gpus": 1, "steps": len(vals), "warmup": args.warmup,
        "ms_per_step": float(np.median([c["us_per_call_equiv"] for c in vals])) / 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded)", "impl": "reference",
        "config": {"workload": wname, "fmt": w["fmt"], "M": w["M"], "N": w["N"], "K": w["K"]},
        "cpu_baseline": cb,
        "e2e": {"value": round(v, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ---------------------------------------------------------------- main


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--sweep", action="store_true", help="one JSON line per workload of the sweep list")
    ap.add_argument("--sweep-batched", action="store_true", help="one JSON line per batched (M >= 16) workload")
    ap.add_argument("--graph-calls", type=int, default=200, help="calls captured in one graph (rounded up to "
                    "whole passes over the weight copies)")
    ap.add_argument("--reps", type=int, default=5, help="timed repetitions (at least 4)")
    ap.add_argument("--min-ms", type=float, default=50.0, help="minimum duration of one timed repetition")
    ap.add_argument("--no-per-m", action="store_true", help="skip the M = 1, 2, 4, 8 record")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--copies", type=int, default=0,
                    help="weight copies to rotate (0: enough to exceed 3x L2); small values only for profiling")
    args = ap.parse_args()

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    dist = None
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, WORKLOADS[args.workload], args.workload)), flush=True)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as tdist

        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist = tdist
    names = SWEEP if args.sweep else (SWEEP_BATCHED if args.sweep_batched else [args.workload])
    for name in names:
        out = run_ours(args, WORKLOADS[name], name, rank, world, dist)
        if rank == 0:
            print(json.dumps(out), flush=True)
    if dist is not None:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
