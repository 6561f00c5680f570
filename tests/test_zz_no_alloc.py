"""lowbit_gemm_noalloc: the GEMM for callers that cannot allocate device memory.

Such callers (a plug-in whose host engine owns all device memory, a latency-critical loop that
cannot afford cudaMalloc's synchronisation) cannot pass lowbit_gemm a workspace; this entry
point keeps its scratch in static device memory instead. The test calls it through the C ABI
twice in a row, on two different problems, and checks each result against lowbit_gemm's within
the parity tolerance used everywhere else. This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import synth
import bit_weight_only_w2_b200 as lb
from synth.workloads import LinearSpec
from tests import _gpu

pytestmark = pytest.mark.gpu

LOWBIT_ERR_WORKSPACE = 8


def noalloc_fn():
    f = lb.load().lowbit_gemm_noalloc
    i64, i32, p = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p
    f.argtypes = [i64, i64, i64, i32, i32, p, p, p, p, p, p]
    f.restype = i32
    return f


def call_noalloc(f, spec, x, packed, s, z, y):
    return f(spec.M, spec.N, spec.K, spec.bits, spec.group_size, x.data_ptr(), packed.data_ptr(), s.data_ptr(),
             None if z is None else z.data_ptr(), y.data_ptr(), torch.cuda.current_stream().cuda_stream)


def test_noalloc_matches_gemm_on_two_calls_in_a_row():
    f = noalloc_fn()
    specs = [LinearSpec("noalloc_a", 300, 512, 520, bits=2, group_size=128, p0=0.4, seed=41),
             LinearSpec("noalloc_b", 96, 1024, 264, bits=4, group_size=64, scale_lo=0.002, scale_hi=0.01, seed=42),
             LinearSpec("noalloc_c", 16, 2048, 1032, bits=1, group_size=128, seed=43)]   # small-M kernel
    for spec in specs:
        prob = synth.make_problem(spec)
        x, packed, s, z = _gpu.dev_problem(prob)
        want = lb.gemm(x, packed, s, z, spec.bits, spec.group_size)
        got = torch.full_like(want, float("nan"))
        assert call_noalloc(f, spec, x, packed, s, z, got) == 0
        torch.cuda.synchronize()
        assert lb.device_status() == 0
        _gpu.check_close(_gpu.y_to_f64(got), _gpu.y_to_f64(want), what=spec.name)


def test_noalloc_rejects_problems_beyond_its_scratch():
    f = noalloc_fn()
    fake = 1 << 20   # never dereferenced: the size check fails before any CUDA call
    st = f(4608, 3072, 12288, 2, 128, fake, fake, fake, None, fake, None)
    assert st == LOWBIT_ERR_WORKSPACE
    assert lb.workspace_size(4608, 12288) > 32 * 1024 * 1024
