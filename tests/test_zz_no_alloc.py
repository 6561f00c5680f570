"""lowbit_gemm_noalloc: the GEMM for callers that cannot allocate device memory.

Such callers -- a plug-in whose host engine owns all device memory and forbids allocations once
it is running, or a latency-critical loop that cannot afford cudaMalloc's implicit device
synchronisation -- cannot hand lowbit_gemm a workspace, so this entry point keeps its scratch (the
fp16 copy of X and the row factors) in a fixed array of static device memory instead.

The tests call it through the C ABI:
  * two calls in a row on each of three problems (large-M ternary, large-M uint4, small-M
    binary), each result against lowbit_gemm's within the parity tolerance and against the CPU
    oracle;
  * all problems queued back to back on one stream with separate outputs and no synchronisation
    in between (a small-M call followed by large-M ones and the reverse), so that the calls
    share the scratch while the next call's kernels may already be starting; then device free
    memory is compared before and after, to show that the calls allocate nothing;
  * a problem whose scratch would exceed the array is rejected before any CUDA call.
This file is collected last on purpose, so that a run stopping at the first failure has already
run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synth
import bit_weight_only_w2_b200 as lb
from synth.workloads import LinearSpec
from tests import _gpu

pytestmark = pytest.mark.gpu

LOWBIT_ERR_WORKSPACE = 8
SCRATCH_BYTES = 32 * 1024 * 1024

SPECS = [LinearSpec("noalloc_a", 300, 512, 520, bits=2, group_size=128, p0=0.4, seed=41),
         LinearSpec("noalloc_b", 96, 1024, 264, bits=4, group_size=64, scale_lo=0.002, scale_hi=0.01, seed=42),
         LinearSpec("noalloc_c", 16, 2048, 1032, bits=1, group_size=128, seed=43)]   # small-M kernel


def noalloc_fn():
    f = lb.load().lowbit_gemm_noalloc
    i64, i32, p = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p
    f.argtypes = [i64, i64, i64, i32, i32, p, p, p, p, p, p]
    f.restype = i32
    return f


def call_noalloc(f, spec, x, packed, s, z, y):
    return f(spec.M, spec.N, spec.K, spec.bits, spec.group_size, x.data_ptr(), packed.data_ptr(), s.data_ptr(),
             None if z is None else z.data_ptr(), y.data_ptr(), torch.cuda.current_stream().cuda_stream)


def problems():
    out = []
    for spec in SPECS:
        prob = synth.make_problem(spec)
        ref = oracle.gemm(prob.x_bf16, _gpu.oracle_packed(prob), prob.scales, prob.zeros, spec.N, spec.bits,
                          spec.group_size)
        out.append((spec, _gpu.dev_problem(prob), ref))
    return out


def test_noalloc_matches_gemm_and_oracle_on_two_calls_in_a_row():
    f = noalloc_fn()
    for spec, (x, packed, s, z), ref in problems():
        want = lb.gemm(x, packed, s, z, spec.bits, spec.group_size)
        for call in range(2):
            got = torch.full_like(want, float("nan"))
            assert call_noalloc(f, spec, x, packed, s, z, got) == 0
            torch.cuda.synchronize()
            assert lb.device_status() == 0
            _gpu.check_close(_gpu.y_to_f64(got), _gpu.y_to_f64(want), what=f"{spec.name} call {call} vs lowbit_gemm")
            _gpu.check_close(_gpu.y_to_f64(got), ref, what=f"{spec.name} call {call} vs oracle")


@pytest.mark.parametrize("order", [(2, 0, 1), (0, 1, 2, 0)], ids=["small_first", "large_first"])
def test_noalloc_back_to_back_allocates_nothing(order):
    f = noalloc_fn()
    probs = problems()
    # first use on this device: the library looks up the scratch array's address and the kernels'
    # modules are loaded; nothing after this point may take device memory
    for spec, (x, packed, s, z), _ in probs:
        warm = torch.empty((spec.M, spec.N), dtype=torch.bfloat16, device="cuda")
        assert call_noalloc(f, spec, x, packed, s, z, warm) == 0
    outs = [torch.full((probs[i][0].M, probs[i][0].N), float("nan"), dtype=torch.bfloat16, device="cuda")
            for i in order]
    torch.cuda.synchronize()
    free_before, _ = torch.cuda.mem_get_info()
    for i, y in zip(order, outs):
        spec, (x, packed, s, z), _ = probs[i]
        assert call_noalloc(f, spec, x, packed, s, z, y) == 0      # no synchronisation in between
    torch.cuda.synchronize()
    free_after, _ = torch.cuda.mem_get_info()
    assert lb.device_status() == 0
    assert free_after >= free_before, f"device free memory fell by {free_before - free_after} bytes"
    for i, y in zip(order, outs):
        spec, _, ref = probs[i]
        _gpu.check_close(_gpu.y_to_f64(y), ref, what=f"{spec.name} queued vs oracle")


def test_noalloc_rejects_problems_beyond_its_scratch():
    f = noalloc_fn()
    fake = 1 << 20   # never dereferenced: the size check fails before any CUDA call
    st = f(4608, 3072, 12288, 2, 128, fake, fake, fake, None, fake, None)
    assert st == LOWBIT_ERR_WORKSPACE
    assert lb.workspace_size(4608, 12288) > SCRATCH_BYTES
    # the cap is on the workspace arithmetic, not on M or K alone: a shorter X with the same K fits
    m_fit = (SCRATCH_BYTES - 512) // (12288 * 2 + 4)
    assert lb.workspace_size(m_fit, 12288) <= SCRATCH_BYTES
