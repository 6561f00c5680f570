"""Python binding of liblowbit.so: weight-only low-bit GEMM for B200 (sm_100a).

Argument marshalling only: every step of the computation runs in the library's CUDA
kernels. PyTorch provides device memory and streams. The binding raises if the library
is missing; there is no fallback.

    Y = gemm(x, packed, scales, zeros, bits, group_size)   # Y[M][N] = X[M][K] W^T

Layouts (see include/lowbit.h): x bf16 [M][K]; packed int32 view of uint32 words
[N][K*bits/32]; scales / zeros fp16 [K/group_size][N]; y bf16 [M][N].
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblowbit.so")
DEBUG_LIB_PATH = os.path.join(_HERE, "liblowbit_debug.so")

STATUS = {
    0: "LOWBIT_OK", 1: "LOWBIT_ERR_INVALID_ARG", 2: "LOWBIT_ERR_ALIGNMENT", 3: "LOWBIT_ERR_UNSUPPORTED",
    4: "LOWBIT_ERR_UNSUPPORTED_DEVICE", 5: "LOWBIT_ERR_BAD_CODE", 6: "LOWBIT_ERR_TIMEOUT", 7: "LOWBIT_ERR_CUDA",
    8: "LOWBIT_ERR_WORKSPACE", 9: "LOWBIT_ERR_DEVICE_CHECK",
}


class LowbitError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS.get(status, status)}")


class GemmDesc(ctypes.Structure):
    _fields_ = [("M", ctypes.c_int64), ("N", ctypes.c_int64), ("K", ctypes.c_int64),
                ("bits", ctypes.c_int), ("group_size", ctypes.c_int),
                ("X", ctypes.c_void_p), ("Wp", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("zeros", ctypes.c_void_p), ("Y", ctypes.c_void_p)]


_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load liblowbit.so (raises FileNotFoundError if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    _lib = open_library(path)
    return _lib


_debug_lib = None


def load_debug() -> ctypes.CDLL:
    """Load liblowbit_debug.so: the same library built with device-side index checks."""
    global _debug_lib
    if _debug_lib is None:
        _debug_lib = open_library(DEBUG_LIB_PATH)
    return _debug_lib


def open_library(path: str) -> ctypes.CDLL:
    """Open a build of the library at `path` and declare its C signatures."""
    if not os.path.exists(path):
        raise FileNotFoundError(f"{path} is missing: build it with `python -m bit_weight_only_w2_b200.build`")
    lib = ctypes.CDLL(path)
    i64, i32, p = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p
    lib.lowbit_status_string.argtypes = [i32]
    lib.lowbit_status_string.restype = ctypes.c_char_p
    lib.lowbit_version.restype = i32
    lib.lowbit_packed_words.argtypes = [i64, i64, i32]
    lib.lowbit_packed_words.restype = ctypes.c_size_t
    lib.lowbit_pack.argtypes = [p, i64, i64, i32, p, p]
    lib.lowbit_pack.restype = i32
    lib.lowbit_unpack.argtypes = [p, i64, i64, i32, p, p]
    lib.lowbit_unpack.restype = i32
    sz = ctypes.c_size_t
    lib.lowbit_gemm_workspace_size.argtypes = [i64, i64]
    lib.lowbit_gemm_workspace_size.restype = sz
    lib.lowbit_gemm.argtypes = [i64, i64, i64, i32, i32, p, p, p, p, p, p, sz, p]
    lib.lowbit_gemm.restype = i32
    lib.lowbit_gemm_ex.argtypes = [i64, i64, i64, i32, i32, p, p, p, p, p, p, sz, i32, i32, i32, p]
    lib.lowbit_gemm_ex.restype = i32
    lib.lowbit_gemm_batch.argtypes = [ctypes.POINTER(GemmDesc), i32, p, sz, p]
    lib.lowbit_gemm_batch.restype = i32
    lib.lowbit_device_status.argtypes = [i32]
    lib.lowbit_device_status.restype = i32
    lib.lowbit_selftest_bounded_wait.argtypes = [ctypes.c_longlong, p]
    lib.lowbit_selftest_bounded_wait.restype = i32
    lib.lowbit_last_device_status.argtypes = [p]
    lib.lowbit_last_device_status.restype = i32
    lib.lowbit_test_fail_next.argtypes = [i32]
    lib.lowbit_test_fail_next.restype = i32
    lib.lowbit_debug_checks_enabled.argtypes = []
    lib.lowbit_debug_checks_enabled.restype = i32
    lib.lowbit_selftest_index_check.argtypes = [p]
    lib.lowbit_selftest_index_check.restype = i32
    lib.lowbit_gemm_noalloc.argtypes = [i64, i64, i64, i32, i32, p, p, p, p, p, p]
    lib.lowbit_gemm_noalloc.restype = i32
    return lib


def _check(st: int, what: str) -> None:
    if st != 0:
        raise LowbitError(st, what)


def _stream(t: Optional[torch.Tensor] = None) -> int:
    dev = t.device if t is not None else None
    return torch.cuda.current_stream(dev).cuda_stream


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _need(t: torch.Tensor, dtype, name: str, ndim: int = 2):
    if t.dtype != dtype or not t.is_contiguous() or t.dim() != ndim:
        raise ValueError(f"{name}: expected a contiguous {ndim}-D {dtype} tensor, got {t.dtype} "
                         f"{tuple(t.shape)} (contiguous={t.is_contiguous()})")


def _need_cuda(*named):
    for name, t in named:
        if t is not None and not t.is_cuda:
            raise ValueError(f"{name}: expected a CUDA tensor, got one on {t.device}")


def _check_gemm_args(x, packed, scales, zeros, out, bits: int, group_size: int):
    """Shapes, dtypes and devices of a GEMM's tensors against each other, before any library call:
    the tensor maps are built from M, N and K, so a buffer smaller than its shape implies would be
    read or written past its end on the GPU. Bits and group sizes the library rejects anyway are
    left to it (it returns LOWBIT_ERR_INVALID_ARG / _UNSUPPORTED)."""
    _need(x, torch.bfloat16, "x")
    _need(packed, torch.int32, "packed")
    _need(scales, torch.float16, "scales")
    if zeros is not None:
        _need(zeros, torch.float16, "zeros")
    if out is not None:
        _need(out, torch.bfloat16, "out")
    M, K = x.shape
    N = scales.shape[1]
    if group_size > 0 and K % group_size == 0 and scales.shape[0] != K // group_size:
        raise ValueError(f"scales: expected shape ({K // group_size}, N) (group-major [K/g][N]), "
                         f"got {tuple(scales.shape)}")
    if bits in (1, 2, 4) and K * bits % 32 == 0 and tuple(packed.shape) != (N, K * bits // 32):
        raise ValueError(f"packed: expected shape {(N, K * bits // 32)} for N={N}, K={K}, bits={bits}, "
                         f"got {tuple(packed.shape)}")
    if zeros is not None and tuple(zeros.shape) != tuple(scales.shape):
        raise ValueError(f"zeros: expected the scales' shape {tuple(scales.shape)}, got {tuple(zeros.shape)}")
    if out is not None and tuple(out.shape) != (M, N):
        raise ValueError(f"out: expected shape {(M, N)}, got {tuple(out.shape)}")
    for name, t in (("packed", packed), ("scales", scales), ("zeros", zeros), ("out", out)):
        if t is not None and t.device != x.device:
            raise ValueError(f"{name}: on {t.device}, but x is on {x.device}")
    _need_cuda(("x", x))
    return M, N, K


def version() -> int:
    return int(load().lowbit_version())


def packed_words(N: int, K: int, bits: int) -> int:
    return int(load().lowbit_packed_words(N, K, bits))


def pack(codes: torch.Tensor, bits: int) -> torch.Tensor:
    """int8 codes [N][K] (binary -1/+1, ternary -1/0/+1, uint4 0..15) -> packed words
    [N][K*bits/32] (int32 storage of uint32 words). Synchronous."""
    _need(codes, torch.int8, "codes")
    _need_cuda(("codes", codes))
    N, K = codes.shape
    out = torch.empty((N, K * bits // 32), dtype=torch.int32, device=codes.device)
    with torch.cuda.device(codes.device):
        _check(load().lowbit_pack(_ptr(codes), N, K, bits, _ptr(out), _stream(codes)), "lowbit_pack")
    return out


def unpack(packed: torch.Tensor, N: int, K: int, bits: int) -> torch.Tensor:
    """Inverse of pack: packed words [N][K*bits/32] -> int8 codes [N][K]. Synchronous."""
    _need(packed, torch.int32, "packed")
    if bits in (1, 2, 4) and N >= 0 and K >= 0 and K * bits % 32 == 0 and packed.numel() != N * K * bits // 32:
        raise ValueError(f"packed: {packed.numel()} words, but N={N}, K={K}, bits={bits} needs {N * K * bits // 32}")
    _need_cuda(("packed", packed))
    out = torch.empty((N, K), dtype=torch.int8, device=packed.device)
    with torch.cuda.device(packed.device):
        _check(load().lowbit_unpack(_ptr(packed), N, K, bits, _ptr(out), _stream(packed)), "lowbit_unpack")
    return out


def workspace_size(M: int, K: int) -> int:
    return int(load().lowbit_gemm_workspace_size(M, K))


def _workspace_size_fast(M: int, K: int) -> int:
    # the closed form lowbit_gemm_workspace_size returns (fp16 X copy + fp32 row factors, each
    # rounded up to 256 bytes); tests check the two agree
    return ((M * K * 2 + 255) // 256 + (M * 4 + 255) // 256) * 256


_workspaces = {}


def workspace(device: torch.device, nbytes: int) -> torch.Tensor:
    """A cached per-device workspace buffer of at least `nbytes` (grown on demand). Work that
    uses it is ordered on the current stream; callers running GEMMs on several streams at once
    should pass their own buffers."""
    dev = torch.device(device)
    key = dev.index if dev.index is not None else torch.cuda.current_device()
    buf = _workspaces.get(key)
    if buf is None or buf.numel() < nbytes:
        buf = torch.empty(max(nbytes, 1 << 20), dtype=torch.uint8, device=torch.device("cuda", key))
        _workspaces[key] = buf
    return buf


def gemm(x: torch.Tensor, packed: torch.Tensor, scales: torch.Tensor, zeros: Optional[torch.Tensor],
         bits: int, group_size: int, out: Optional[torch.Tensor] = None, tile_tokens: int = 0,
         ksplit: int = 0, ws: Optional[torch.Tensor] = None, tile_rows: int = 0) -> torch.Tensor:
    """Y[M][N] = X[M][K] * W^T with W decoded from `packed`, `scales` (and `zeros`)."""
    M, N, K = _check_gemm_args(x, packed, scales, zeros, out, bits, group_size)
    if ws is not None:
        _need(ws, torch.uint8, "ws", ndim=1)
        if ws.device != x.device:
            raise ValueError(f"ws: on {ws.device}, but x is on {x.device}")
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    dev = x.get_device()
    if dev != torch.cuda.current_device():
        with torch.cuda.device(dev):
            return _gemm_call(x, packed, scales, zeros, bits, group_size, out, tile_tokens, ksplit, ws, tile_rows,
                              M, N, K, dev)
    return _gemm_call(x, packed, scales, zeros, bits, group_size, out, tile_tokens, ksplit, ws, tile_rows, M, N, K,
                      dev)


def _gemm_call(x, packed, scales, zeros, bits, group_size, out, tile_tokens, ksplit, ws, tile_rows, M, N, K, dev):
    lib = _lib if _lib is not None else load()
    if ws is None:
        ws = workspace(x.device, _workspace_size_fast(M, K))
    stream = torch.cuda.current_stream().cuda_stream
    zp = None if zeros is None else zeros.data_ptr()
    if tile_tokens or ksplit or tile_rows:
        st = lib.lowbit_gemm_ex(M, N, K, bits, group_size, x.data_ptr(), packed.data_ptr(), scales.data_ptr(), zp,
                                out.data_ptr(), ws.data_ptr(), ws.numel(), tile_tokens, tile_rows, ksplit, stream)
    else:
        st = lib.lowbit_gemm(M, N, K, bits, group_size, x.data_ptr(), packed.data_ptr(), scales.data_ptr(), zp,
                             out.data_ptr(), ws.data_ptr(), ws.numel(), stream)
    if st != 0:
        raise LowbitError(st, "lowbit_gemm")
    return out


def make_desc(x, packed, scales, zeros, y, bits: int, group_size: int) -> GemmDesc:
    """One linear of a lowbit_gemm_batch call (the tensors must outlive the call)."""
    if y is None:
        raise ValueError("y: a batch descriptor needs its output tensor")
    M, N, K = _check_gemm_args(x, packed, scales, zeros, y, bits, group_size)
    return GemmDesc(M, N, K, bits, group_size, _ptr(x), _ptr(packed), _ptr(scales), _ptr(zeros), _ptr(y))


def gemm_batch(descs: Sequence[GemmDesc], device: Optional[torch.device] = None,
               ws: Optional[torch.Tensor] = None) -> None:
    """Run the descriptors in order on the current stream (see lowbit_gemm_batch)."""
    arr = (GemmDesc * len(descs))(*descs)
    dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
    with torch.cuda.device(dev):
        if ws is None:
            need = max((workspace_size(d.M, d.K) for d in descs), default=0)
            ws = workspace(dev, need)
        _check(load().lowbit_gemm_batch(arr, len(descs), _ptr(ws), ws.numel(), _stream()), "lowbit_gemm_batch")


def device_status(clear: bool = True) -> int:
    """The device status word (0 = OK, LOWBIT_ERR_TIMEOUT if a kernel wait gave up)."""
    return int(load().lowbit_device_status(1 if clear else 0))


def last_device_status(stream: Optional[torch.cuda.Stream] = None) -> int:
    """The device status word read (and cleared) in the order of `stream` (default: the current
    stream), waiting for that stream only (see lowbit_last_device_status)."""
    st = stream if stream is not None else torch.cuda.current_stream()
    return int(load().lowbit_last_device_status(st.cuda_stream))


def selftest_bounded_wait(limit_cycles: int = 50_000_000) -> None:
    """Launch the bounded-wait self-test kernel (see lowbit_selftest_bounded_wait)."""
    _check(load().lowbit_selftest_bounded_wait(limit_cycles, _stream()), "lowbit_selftest_bounded_wait")
