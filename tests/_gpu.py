"""Helpers for the GPU parity tests: seeded inputs on the device, calls through
the C ABI binding, and oracle comparisons (whole outputs or sampled rows)."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import weight_only_quantized_q4_b200 as wq
from weight_only_quantized_q4_b200 import synth

DEV = "cuda:0"


def dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def f16_of(t: torch.Tensor) -> np.ndarray:
    return t.cpu().numpy()


def bf16_bits_of(t: torch.Tensor) -> np.ndarray:
    return t.cpu().view(torch.int16).numpy().view(np.uint16)


GUARD = 256       # canary bytes on each side of every output buffer
CANARY = 0xA5


class Guarded:
    """A device output buffer with GUARD canary bytes on each side.

    compute-sanitizer is not available on the GPU pool, so out-of-bounds
    stores are caught this way instead: every kernel output in the tests
    lives between two bands of known bytes, and check() asserts the bands
    are untouched after the call.  `lead` extra bytes before the tensor
    (part of the front band) give a tensor an odd 2-byte offset."""

    def __init__(self, shape, dtype, lead: int = 0):
        n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        self.lead, self.n = GUARD + lead, n
        self.buf = torch.full((self.lead + n + GUARD,), CANARY, dtype=torch.uint8, device=DEV)
        self.ptr = self.buf.data_ptr() + self.lead
        self.t = self.buf[self.lead:self.lead + n].view(dtype).view(shape) if lead % 16 == 0 else None

    def check(self, what: str = "output") -> None:
        b = self.buf.cpu().numpy()
        head, tail = b[:self.lead], b[self.lead + self.n:]
        if (head != CANARY).any() or (tail != CANARY).any():
            hb = np.flatnonzero(head != CANARY)
            tb = np.flatnonzero(tail != CANARY)
            raise AssertionError(f"{what}: store outside the output buffer (bytes before: {hb[:8].tolist()}, "
                                 f"bytes after: {tb[:8].tolist()})")


def guarded_empty(shape, dtype):
    return Guarded(shape, dtype)


def check(y_dev: np.ndarray, W: np.ndarray, x: np.ndarray, what: str) -> None:
    """Accept iff |y − y_ref| ≤ 2e-3·Σ|w·x| + 1e-3 for every element."""
    y_ref = oracle.gemv(W, x)
    B = oracle.bound(W, x)
    bad = oracle.violations(y_dev, y_ref, B)
    if bad.any():
        idx = np.argwhere(bad)[:5]
        detail = [(tuple(i), float(y_dev[tuple(i)]), float(y_ref[tuple(i)]), float(B[tuple(i)])) for i in idx]
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} outside tolerance; first: {detail}")


# ----------------------------------------------------------------- int4

class Int4Case:
    def __init__(self, M, N, K, bs, zeros, workload=3, s_lo=0.002, s_hi=0.01, layout=0):
        self.M, self.N, self.K, self.bs, self.layout = M, N, K, bs, layout
        t = synth.int4_weights(N, K, bs, scale_lo=s_lo, scale_hi=s_hi, with_zeros=zeros, workload=workload)
        self.w, self.s, self.z = t["w_packed"], t["scales"], t["zeros"]
        self.x = synth.activations_f16(M, K, workload=workload)
        self.dw, self.ds = dev(self.w), dev(self.s)
        self.dz = dev(self.z) if self.z is not None else None
        if layout == wq.WQ_LAYOUT_B200_V1:
            g = Guarded((wq.wq_int4_packed_bytes(N, K, bs, layout),), torch.uint8)
            g.buf[g.lead:g.lead + g.n] = 0x5A
            wq.wq_repack_int4(self.dw, self.ds, self.dz, g.t, N, K, bs, layout)
            torch.cuda.synchronize()
            g.check("B200_V1 repack output")
            self._packed_guard = g
            self.dw = g.t
        self.dx = dev(self.x)

    def run(self, stream=None) -> np.ndarray:
        g = Guarded((self.M, self.N), torch.float16)
        wq.gemv_int4_blockwise(self.dx, self.dw, self.ds, self.dz, g.t, self.M, self.N, self.K, self.bs,
                               layout=self.layout, stream=stream)
        torch.cuda.synchronize()
        g.check(f"int4 y M={self.M} N={self.N} K={self.K}")
        return f16_of(g.t).astype(np.float64)

    def W(self, rows=None):
        r = slice(None) if rows is None else rows
        z = None if self.z is None else self.z[r]
        n = self.N if rows is None else len(rows)
        return oracle.dequant_int4(self.w[r], self.s[r], z, n, self.K, self.bs)


# ----------------------------------------------------------------- q4_K

class Q4KCase:
    def __init__(self, M, N, K, workload=4, layout=0):
        self.M, self.N, self.K, self.layout = M, N, K, layout
        self.raw = synth.q4k_weights(N, K, workload=workload)
        self.x = synth.activations_f16(M, K, workload=workload)
        self.draw, self.dx = dev(self.raw), dev(self.x)
        self._plane = None
        self.dw = self.draw
        if layout == wq.WQ_LAYOUT_B200_V1:
            g = Guarded((wq.wq_q4k_packed_bytes(N, K, layout),), torch.uint8)
            wq.wq_repack_q4k(self.draw, g.t, N, K, layout)
            torch.cuda.synchronize()
            g.check("q4_K B200_V1 repack output")
            self._packed_guard = g
            self.dw = g.t

    def plane_dev(self):
        if self._plane is None:
            g = Guarded((self.K // 32, self.N, 2), torch.float32)
            wq.wq_build_q4k_dsc_device(self.draw, g.t, self.N, self.K)
            torch.cuda.synchronize()
            g.check("W_dsc plane")
            self._plane_guard = g
            self._plane = g.t
        return self._plane

    def run(self, dsc: bool, stream=None) -> np.ndarray:
        g = Guarded((self.M, self.N), torch.float16)
        if dsc:
            wq.gemv_q4k_dsc(self.dx, self.draw, self.plane_dev(), g.t, self.M, self.N, self.K, stream=stream)
        else:
            wq.gemv_q4k(self.dx, self.dw, g.t, self.M, self.N, self.K, layout=self.layout, stream=stream)
        torch.cuda.synchronize()
        g.check(f"q4k y dsc={dsc} M={self.M} N={self.N} K={self.K}")
        return f16_of(g.t).astype(np.float64)

    def W(self, rows=None):
        if rows is None:
            return oracle.dequant_q4k(self.raw, self.N, self.K)
        return oracle.dequant_q4k(self.raw[rows], len(rows), self.K)


# ----------------------------------------------------------------- bf16

class BF16Case:
    def __init__(self, M, N, K, offset=0, workload=2):
        self.M, self.N, self.K, self.offset = M, N, K, offset
        self.wb = synth.bf16_weights_bits(N, K, workload=workload)
        self.xb = synth.activations_bf16_bits(M, K, workload=workload)
        wbuf, _ = synth.with_element_offset(self.wb, offset)
        xbuf, _ = synth.with_element_offset(self.xb, offset)
        self.dwbuf = dev(wbuf.view(np.int16)).view(torch.bfloat16)
        self.dxbuf = dev(xbuf.view(np.int16)).view(torch.bfloat16)

    def run(self, stream=None) -> np.ndarray:
        g = Guarded((self.M * self.N,), torch.bfloat16, lead=2 * self.offset)
        wq.gemv_bf16(self.dxbuf.data_ptr() + 2 * self.offset, self.dwbuf.data_ptr() + 2 * self.offset, g.ptr,
                     self.M, self.N, self.K, stream=stream)
        torch.cuda.synchronize()
        g.check(f"bf16 y M={self.M} N={self.N} K={self.K} offset={self.offset}")
        raw = g.buf[g.lead:g.lead + g.n].cpu().numpy()
        bits = raw.view(np.uint16).reshape(self.M, self.N)
        return oracle.q4.bf16_bits_to_f64(bits)

    def W(self, rows=None):
        wb = self.wb if rows is None else self.wb[rows]
        return oracle.dequant_bf16(wb, wb.shape[0], self.K)

    def X(self):
        return oracle.dequant_bf16(self.xb, self.M, self.K)


VARIANTS = ("tc", "cc", "simple", "tc5", "v1s", "v1r", "v1k", "v1tc", "v1w", None)


def each_variant(run, W, x, what):
    """Run `run()` under every forced GEMV variant (and the default); check each
    against the oracle; return the liveness labels seen.  A forced family that
    cannot run the call must say so (WQ_ERR_UNSUPPORTED, label "unsupported");
    one that runs must be the family that was asked for."""
    import os

    labels = {}
    old = os.environ.get("WQ_FORCE_KERNEL")
    try:
        for v in VARIANTS:
            if v is None:
                os.environ.pop("WQ_FORCE_KERNEL", None)
            else:
                os.environ["WQ_FORCE_KERNEL"] = v
            try:
                y = run()
            except wq.WQError as e:
                if v is None or e.code != wq.WQ_ERR_UNSUPPORTED:
                    raise
                labels[v] = "unsupported"
                continue
            labels[v or "default"] = wq.last_kernel()
            if v is not None:
                assert f".{v}." in labels[v], (what, v, labels[v])
            check(y, W, x, f"{what} [{v or 'default'} -> {labels[v or 'default']}]")
    finally:
        if old is None:
            os.environ.pop("WQ_FORCE_KERNEL", None)
        else:
            os.environ["WQ_FORCE_KERNEL"] = old
    return labels


def sample_rows(N: int, count: int = 48, seed: int = 0) -> np.ndarray:
    rng = np.random.default_rng(seed)
    rows = set(rng.integers(0, N, count).tolist())
    rows.update({0, 1, N - 1, N - 2, N // 2})
    return np.array(sorted(r for r in rows if 0 <= r < N))
