"""Seeded synthetic inputs shared by the tests, the oracle's callers and the benchmark.

Nothing here computes any part of the low-bit GEMM: it only draws random numbers
(see ``synth.c`` for the generator's definition) and describes the workload
shapes. The C helper is compiled with gcc on first use if it is not built yet.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB_PATH = os.path.join(_HERE, "libsynth.so")
_lock = threading.Lock()
_lib = None

# Per-tensor stream ids: one independent random stream per input tensor.
STREAM_X = 1
STREAM_CODES = 2
STREAM_SCALES = 3
STREAM_ZEROS = 4


def build(force: bool = False) -> str:
    """Compile libsynth.so next to its source (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            u64, p = ctypes.c_uint64, ctypes.c_void_p
            lib.synth_raw_u64.argtypes = [u64, u64, u64]
            lib.synth_raw_u64.restype = u64
            lib.synth_uniform_f64.argtypes = [u64, u64, u64, p]
            lib.synth_normal_f64.argtypes = [u64, u64, u64, p]
            lib.synth_normal_bf16.argtypes = [u64, u64, u64, p]
            lib.synth_uniform_f16.argtypes = [u64, u64, u64, ctypes.c_double, ctypes.c_double, p]
            lib.synth_codes.argtypes = [u64, u64, u64, ctypes.c_int, ctypes.c_double, p]
            lib.synth_codes.restype = ctypes.c_int
            _lib = lib
    return _lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def raw_u64(seed: int, stream: int, index: int) -> int:
    return int(_load().synth_raw_u64(seed, stream, index))


def uniform_f64(seed: int, stream: int, n: int) -> np.ndarray:
    out = np.empty(n, dtype=np.float64)
    _load().synth_uniform_f64(seed, stream, n, _ptr(out))
    return out


def normal_f64(seed: int, stream: int, n: int) -> np.ndarray:
    out = np.empty(n, dtype=np.float64)
    _load().synth_normal_f64(seed, stream, n, _ptr(out))
    return out


def normal_bf16(seed: int, stream: int, shape) -> np.ndarray:
    """N(0,1) draws rounded to bf16, returned as raw uint16 bit patterns."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)
    _load().synth_normal_bf16(seed, stream, n, _ptr(out))
    return out.reshape(shape)


def uniform_f16(seed: int, stream: int, shape, lo: float, hi: float) -> np.ndarray:
    """U[lo, hi) draws rounded to fp16, returned as a numpy float16 array."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)
    _load().synth_uniform_f16(seed, stream, n, lo, hi, _ptr(out))
    return out.view(np.float16).reshape(shape)


def codes(seed: int, stream: int, shape, bits: int, p0: float = 1.0 / 3.0) -> np.ndarray:
    """Weight codes: bits 1 -> {-1,+1}; bits 2 -> {-1,0,+1} with P(0)=p0; bits 4 -> 0..15."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.int8)
    rc = _load().synth_codes(seed, stream, n, bits, p0, _ptr(out))
    if rc != 0:
        raise ValueError(f"unsupported bits={bits}")
    return out.reshape(shape)


from .workloads import LinearSpec, Problem, make_problem, WORKLOADS, chain_linears  # noqa: E402,F401
