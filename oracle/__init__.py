"""CPU oracle for the W4A16 group-128 linear layer (TEST INFRASTRUCTURE ONLY).

Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package.  The CUDA library never calls it, links it or
shares code with it.

The arithmetic lives in ``w4a16_oracle.c`` (plain C, FP32 with separate
roundings, sequential over k).  This wrapper only builds it with gcc and
marshals numpy arrays; BF16 travels as uint16 bit patterns.

Every oracle function is pinned by ``tests/test_oracle_pins.py``; the pins
are in turn shown to reject deliberately broken copies of the C source by
``tests/test_oracle_mutants.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(HERE, "w4a16_oracle.c")
LIBRARY = os.path.join(HERE, "libw4a16_oracle.so")
CFLAGS = ["-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-fPIC", "-shared",
          "-std=c11", "-Wall", "-Wextra", "-Werror"]
LIBS = ["-lm"]


def compile_source(src: str, out: str) -> str:
    tmp = out + f".tmp{os.getpid()}"
    subprocess.run(["gcc", *CFLAGS, src, "-o", tmp, *LIBS], check=True)
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    """Compile the oracle with gcc if the shared object is missing or stale."""
    stale = (not os.path.exists(LIBRARY)) or os.path.getmtime(LIBRARY) < os.path.getmtime(SOURCE)
    if force or stale:
        compile_source(SOURCE, LIBRARY)
    return LIBRARY


def _c(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a, a.ctypes.data_as(ctypes.c_void_p)


class Oracle:
    """ctypes view of one build of ``w4a16_oracle.c``."""

    def __init__(self, path: str):
        lib = ctypes.CDLL(path)
        p, i64 = ctypes.c_void_p, ctypes.c_int64
        for name in ("w4a16_oracle_matmul", "w4a16_oracle_matmul_f32"):
            fn = getattr(lib, name)
            fn.argtypes = [p, p, p, p, p, i64, i64, i64]
            fn.restype = ctypes.c_int
        lib.w4a16_oracle_unpack.argtypes = [p, p, i64, i64]
        lib.w4a16_oracle_unpack.restype = ctypes.c_int
        lib.w4a16_oracle_round_bf16.argtypes = [p, p, i64]
        lib.w4a16_oracle_round_bf16.restype = None
        lib.w4a16_oracle_threads.argtypes = []
        lib.w4a16_oracle_threads.restype = ctypes.c_int
        lib.w4a16_oracle_set_threads.argtypes = [ctypes.c_int]
        lib.w4a16_oracle_set_threads.restype = None
        lib.w4a16_oracle_gate_up.argtypes = [p, p, p, p, p, i64, i64, i64]
        lib.w4a16_oracle_gate_up.restype = ctypes.c_int
        lib.w4a16_oracle_matmul_bits.argtypes = [p, p, p, p, p, i64, i64, i64, ctypes.c_int]
        lib.w4a16_oracle_matmul_bits.restype = ctypes.c_int
        lib.w4a16_oracle_unpack_bits.argtypes = [p, p, i64, i64, ctypes.c_int]
        lib.w4a16_oracle_unpack_bits.restype = ctypes.c_int
        for name in ("w4a16_oracle_quantize", "w4a16_oracle_quantize_bf16"):
            fn = getattr(lib, name)
            fn.argtypes = [p, p, p, p, i64, i64]
            fn.restype = ctypes.c_int
        self.lib = lib
        self.path = path

    @staticmethod
    def _inputs(x, wq, scales, biases):
        x, px = _c(x, np.uint16)
        wq, pw = _c(wq, np.uint32)
        s, ps = _c(scales, np.uint16)
        b, pb = _c(biases, np.uint16)
        M, K = x.shape
        N = wq.shape[0]
        G = K // 128 if K % 128 == 0 else -1
        if wq.shape != (N, K // 8) or s.shape != (N, G) or b.shape != (N, G):
            raise ValueError("shape mismatch between x, wq, scales and biases")
        return (x, wq, s, b), (px, pw, ps, pb), M, N, K

    def matmul(self, x, wq, scales, biases) -> np.ndarray:
        """y [M,N] BF16 bits = x . dequant(wq)^T (FP32 sequential accumulation)."""
        keep, ptrs, M, N, K = self._inputs(x, wq, scales, biases)
        y = np.empty((M, N), dtype=np.uint16)
        if self.lib.w4a16_oracle_matmul(*ptrs, y.ctypes.data_as(ctypes.c_void_p), M, N, K):
            raise ValueError("oracle rejected its arguments")
        return y

    def matmul_f32(self, x, wq, scales, biases) -> np.ndarray:
        """The FP32 accumulator before the final BF16 rounding."""
        keep, ptrs, M, N, K = self._inputs(x, wq, scales, biases)
        acc = np.empty((M, N), dtype=np.float32)
        if self.lib.w4a16_oracle_matmul_f32(*ptrs, acc.ctypes.data_as(ctypes.c_void_p), M, N, K):
            raise ValueError("oracle rejected its arguments")
        return acc

    def matmul_bits(self, x, wq, scales, biases, bits: int) -> np.ndarray:
        """y [M,N] BF16 bits with b-bit codes (wq [N, K b / 32], 32 / b codes per word, low first)."""
        x, px = _c(x, np.uint16)
        wq, pw = _c(wq, np.uint32)
        s, ps = _c(scales, np.uint16)
        b, pb = _c(biases, np.uint16)
        M, K = x.shape
        N = wq.shape[0]
        G = K // 128 if K % 128 == 0 else -1
        if bits not in (2, 4, 8) or wq.shape != (N, K * bits // 32) or s.shape != (N, G) or b.shape != (N, G):
            raise ValueError("shape mismatch between x, wq, scales and biases (or bits not 2, 4, 8)")
        y = np.empty((M, N), dtype=np.uint16)
        if self.lib.w4a16_oracle_matmul_bits(px, pw, ps, pb, y.ctypes.data_as(ctypes.c_void_p), M, N, K, bits):
            raise ValueError("oracle rejected its arguments")
        return y

    def unpack_bits(self, wq, K: int, bits: int) -> np.ndarray:
        wq, pw = _c(wq, np.uint32)
        N = wq.shape[0]
        q = np.empty((N, K), dtype=np.uint8)
        if self.lib.w4a16_oracle_unpack_bits(pw, q.ctypes.data_as(ctypes.c_void_p), N, K, bits):
            raise ValueError("oracle rejected its arguments")
        return q

    def gate_up(self, x, wq, scales, biases) -> np.ndarray:
        """h [M, N2] BF16 bits = silu(gate) * up over interleaved gate/up rows (2 N2 rows)."""
        keep, ptrs, M, N, K = self._inputs(x, wq, scales, biases)
        if N % 16:
            raise ValueError("gate/up rows come in blocks of 16")
        h = np.empty((M, N // 2), dtype=np.uint16)
        if self.lib.w4a16_oracle_gate_up(*ptrs, h.ctypes.data_as(ctypes.c_void_p), M, N // 2, K):
            raise ValueError("oracle rejected its arguments")
        return h

    def unpack(self, wq, K: int) -> np.ndarray:
        wq, pw = _c(wq, np.uint32)
        N = wq.shape[0]
        q = np.empty((N, K), dtype=np.uint8)
        if self.lib.w4a16_oracle_unpack(pw, q.ctypes.data_as(ctypes.c_void_p), N, K):
            raise ValueError("oracle rejected its arguments")
        return q

    def round_bf16(self, a) -> np.ndarray:
        a, pa = _c(a, np.float32)
        out = np.empty(a.shape, dtype=np.uint16)
        self.lib.w4a16_oracle_round_bf16(pa, out.ctypes.data_as(ctypes.c_void_p), a.size)
        return out

    def quantize(self, w):
        """W [N,K] (float32 values, or uint16 BF16 bit patterns) -> (wq uint32 [N,K/8],
        scales uint16 [N,K/128], biases uint16 [N,K/128]) by the min/max recipe."""
        w = np.asarray(w)
        if w.ndim != 2:
            raise ValueError("W must be [N, K]")
        if w.dtype == np.uint16:
            fn, w = self.lib.w4a16_oracle_quantize_bf16, np.ascontiguousarray(w)
        else:
            fn, w = self.lib.w4a16_oracle_quantize, np.ascontiguousarray(w, dtype=np.float32)
        N, K = w.shape
        G = K // 128 if K % 128 == 0 else 0
        wq = np.empty((N, K // 8), dtype=np.uint32)
        s = np.empty((N, G), dtype=np.uint16)
        b = np.empty((N, G), dtype=np.uint16)
        vp = ctypes.c_void_p
        if fn(w.ctypes.data_as(vp), wq.ctypes.data_as(vp), s.ctypes.data_as(vp), b.ctypes.data_as(vp), N, K):
            raise ValueError("oracle rejected its arguments")
        return wq, s, b

    def threads(self) -> int:
        return self.lib.w4a16_oracle_threads()

    def set_threads(self, n: int) -> None:
        self.lib.w4a16_oracle_set_threads(int(n))


_lock = threading.Lock()
_default = None


def default() -> Oracle:
    global _default
    with _lock:
        if _default is None:
            _default = Oracle(build())
    return _default


def matmul(x, wq, scales, biases):
    return default().matmul(x, wq, scales, biases)


def matmul_f32(x, wq, scales, biases):
    return default().matmul_f32(x, wq, scales, biases)


def gate_up(x, wq, scales, biases):
    return default().gate_up(x, wq, scales, biases)


def matmul_bits(x, wq, scales, biases, bits):
    return default().matmul_bits(x, wq, scales, biases, bits)


def unpack_bits(wq, K, bits):
    return default().unpack_bits(wq, K, bits)


def unpack(wq, K):
    return default().unpack(wq, K)


def round_bf16(a):
    return default().round_bf16(a)


def quantize(w):
    return default().quantize(w)


def threads():
    return default().threads()


def set_threads(n):
    default().set_threads(n)
