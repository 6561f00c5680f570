"""CPU oracle for the weight-only low-bit GEMM -- TEST INFRASTRUCTURE ONLY.

Thin ctypes wrapper around ``lowbit_oracle.c`` (plain C, fp64). Only the tests, the
package's ``smoke()`` check and the benchmark's CPU-baseline leg may import this
module; the CUDA library never does. See the C file's header for the definitions it
follows and the passages of the pages they come from.

Parity status: pack / unpack / decode / GEMM are pinned by the tests in
``tests/test_oracle_pins.py`` (closed forms, hand-derived golden words, invariants,
exact rational brute force and a numpy matmul reduction).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "lowbit_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liblowbit_oracle.so")
_lock = threading.Lock()
_lib = None

CFLAGS = ["-O2", "-fopenmp", "-shared", "-fPIC"]


def compile_oracle(src: str, out: str) -> str:
    """Compile an oracle source file to a shared library (used by build() and tests)."""
    tmp = out + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, src, "-lm"])
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        compile_oracle(_SRC, _LIB_PATH)
    return _LIB_PATH


def bind(lib: ctypes.CDLL) -> ctypes.CDLL:
    p, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    lib.oracle_threads.argtypes = [i32]
    lib.oracle_threads.restype = i32
    lib.oracle_bf16_to_f64.argtypes = [ctypes.c_uint16]
    lib.oracle_bf16_to_f64.restype = ctypes.c_double
    lib.oracle_f16_to_f64.argtypes = [ctypes.c_uint16]
    lib.oracle_f16_to_f64.restype = ctypes.c_double
    lib.oracle_f64_to_bf16.argtypes = [ctypes.c_double]
    lib.oracle_f64_to_bf16.restype = ctypes.c_uint16
    lib.oracle_pack.argtypes = [p, i64, i64, i32, p]
    lib.oracle_pack.restype = i64
    lib.oracle_unpack.argtypes = [p, i64, i64, i32, p]
    lib.oracle_unpack.restype = i64
    lib.oracle_decode.argtypes = [p, p, p, i64, i64, i32, i64, p]
    lib.oracle_decode.restype = i32
    lib.oracle_gemm.argtypes = [p, i64, i64, p, p, p, i64, i32, i64, p, i32]
    lib.oracle_gemm.restype = i32
    lib.oracle_gemm_entries.argtypes = [p, i64, i64, p, p, p, i64, i32, i64, p, p, i64, p, i32]
    lib.oracle_gemm_entries.restype = i32
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = bind(ctypes.CDLL(build()))
    return _lib


def _c(a: Optional[np.ndarray], dtype) -> Optional[np.ndarray]:
    if a is None:
        return None
    return np.ascontiguousarray(a).view(dtype) if a.dtype != dtype else np.ascontiguousarray(a)


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data


class Oracle:
    """The oracle's functions bound to one compiled library (the default one, or a
    variant compiled by a test)."""

    def __init__(self, lib: Optional[ctypes.CDLL] = None):
        self.lib = lib if lib is not None else _load()

    def threads(self, t: int = 0) -> int:
        return int(self.lib.oracle_threads(t))

    def bf16_to_f64(self, h: int) -> float:
        return float(self.lib.oracle_bf16_to_f64(h))

    def f16_to_f64(self, h: int) -> float:
        return float(self.lib.oracle_f16_to_f64(h))

    def f64_to_bf16(self, v: float) -> int:
        return int(self.lib.oracle_f64_to_bf16(v))

    def pack(self, codes: np.ndarray, bits: int):
        """codes int8 [N][K] -> (packed uint32 [N][K*bits/32], number of invalid codes)."""
        codes = np.ascontiguousarray(codes, dtype=np.int8)
        N, K = codes.shape
        out = np.zeros((N, K * bits // 32), dtype=np.uint32)
        bad = self.lib.oracle_pack(_p(codes), N, K, bits, _p(out))
        if bad < 0:
            raise ValueError("invalid shape for pack")
        return out, int(bad)

    def unpack(self, packed: np.ndarray, N: int, K: int, bits: int):
        packed = np.ascontiguousarray(packed, dtype=np.uint32)
        out = np.zeros((N, K), dtype=np.int8)
        bad = self.lib.oracle_unpack(_p(packed), N, K, bits, _p(out))
        if bad < 0:
            raise ValueError("invalid shape for unpack")
        return out, int(bad)

    def decode(self, packed, scales, zeros, N: int, K: int, bits: int, g: int) -> np.ndarray:
        packed = np.ascontiguousarray(packed, dtype=np.uint32)
        s = _c(scales, np.uint16)
        z = _c(zeros, np.uint16)
        W = np.zeros((N, K), dtype=np.float64)
        if self.lib.oracle_decode(_p(packed), _p(s), _p(z), N, K, bits, g, _p(W)) != 0:
            raise ValueError("invalid arguments for decode")
        return W

    def gemm(self, x_bf16, packed, scales, zeros, N: int, bits: int, g: int, threads: int = 0) -> np.ndarray:
        """fp64 reference Y [M][N] for X (bf16 bit patterns, uint16 [M][K])."""
        x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
        M, K = x.shape
        packed = np.ascontiguousarray(packed, dtype=np.uint32)
        s = _c(scales, np.uint16)
        z = _c(zeros, np.uint16)
        ref = np.zeros((M, N), dtype=np.float64)
        rc = self.lib.oracle_gemm(_p(x), M, K, _p(packed), _p(s), _p(z), N, bits, g, _p(ref), threads)
        if rc != 0:
            raise ValueError("invalid arguments for gemm")
        return ref

    def gemm_entries(self, x_bf16, packed, scales, zeros, N: int, bits: int, g: int,
                     ms: np.ndarray, ns: np.ndarray, threads: int = 0) -> np.ndarray:
        x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
        M, K = x.shape
        packed = np.ascontiguousarray(packed, dtype=np.uint32)
        s = _c(scales, np.uint16)
        z = _c(zeros, np.uint16)
        ms = np.ascontiguousarray(ms, dtype=np.int64)
        ns = np.ascontiguousarray(ns, dtype=np.int64)
        out = np.zeros(len(ms), dtype=np.float64)
        rc = self.lib.oracle_gemm_entries(_p(x), M, K, _p(packed), _p(s), _p(z), N, bits, g,
                                          _p(ms), _p(ns), len(ms), _p(out), threads)
        if rc != 0:
            raise ValueError("invalid arguments for gemm_entries")
        return out


_default: Optional[Oracle] = None


def default() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle()
    return _default


def pack(codes, bits):
    return default().pack(codes, bits)


def unpack(packed, N, K, bits):
    return default().unpack(packed, N, K, bits)


def decode(packed, scales, zeros, N, K, bits, g):
    return default().decode(packed, scales, zeros, N, K, bits, g)


def gemm(x_bf16, packed, scales, zeros, N, bits, g, threads=0):
    return default().gemm(x_bf16, packed, scales, zeros, N, bits, g, threads)


def gemm_entries(x_bf16, packed, scales, zeros, N, bits, g, ms, ns, threads=0):
    return default().gemm_entries(x_bf16, packed, scales, zeros, N, bits, g, ms, ns, threads)
