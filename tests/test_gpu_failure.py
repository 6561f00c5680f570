"""Failure detection without a GPU fault: injected host-side failures surface as
LOWBIT_ERR_CUDA, the stream-ordered status read reports a kernel's bounded-wait timeout, and the
debug build's device-side index checks record LOWBIT_ERR_DEVICE_CHECK instead of trapping. No
test here faults, traps or hangs the GPU: the injected failures stop a call on the host before
its kernel is launched, the timeout is the bounded-wait self-test, and the index check skips the
store it rejects."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synth
import bit_weight_only_w2_b200 as lb
from tests import _gpu
from tests.test_gpu_gemm import spec_for

pytestmark = pytest.mark.gpu

LOWBIT_ERR_TIMEOUT, LOWBIT_ERR_CUDA, LOWBIT_ERR_DEVICE_CHECK = 6, 7, 9


def gemm_via(lib, x, packed, s, z, y, ws, spec):
    return lib.lowbit_gemm(spec.M, spec.N, spec.K, spec.bits, spec.group_size, x.data_ptr(), packed.data_ptr(),
                           s.data_ptr(), None if z is None else z.data_ptr(), y.data_ptr(), ws.data_ptr(), ws.numel(),
                           torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("what", [1, 2])
@pytest.mark.parametrize("M", [64, 9])   # tensor-memory kernel (two launches), small-M kernel (one)
def test_injected_failure_returns_cuda_error(what, M):
    spec = spec_for(2, 128, M, 512, 264, seed=what + M)
    prob = synth.make_problem(spec)
    x, packed, s, z = _gpu.dev_problem(prob)
    y = torch.full((M, spec.N), float("nan"), dtype=torch.bfloat16, device="cuda")
    ws = lb.workspace(x.device, lb.workspace_size(M, spec.K))
    lib = lb.load()
    assert lib.lowbit_test_fail_next(what) == 0
    assert gemm_via(lib, x, packed, s, z, y, ws, spec) == LOWBIT_ERR_CUDA
    torch.cuda.synchronize()
    assert torch.isnan(y.float()).all()          # nothing ran
    # the injection fired once: the same call now succeeds
    assert gemm_via(lib, x, packed, s, z, y, ws, spec) == 0
    torch.cuda.synchronize()
    assert lb.device_status() == 0
    ref = oracle.gemm(prob.x_bf16, _gpu.oracle_packed(prob), prob.scales, None, spec.N, 2, 128)
    _gpu.check_close(_gpu.y_to_f64(y), ref, what=f"after injected failure {what}")


def test_injected_failure_stops_a_batch():
    specs = [spec_for(2, 128, 64, 256, 128, seed=1), spec_for(2, 128, 64, 256, 128, seed=2)]
    dev = [_gpu.dev_problem(synth.make_problem(sp)) for sp in specs]
    outs = [torch.zeros((64, 128), dtype=torch.bfloat16, device="cuda") for _ in specs]
    descs = [lb.make_desc(x, w, s, z, y, 2, 128) for (x, w, s, z), y in zip(dev, outs)]
    assert lb.load().lowbit_test_fail_next(1) == 0
    with pytest.raises(lb.LowbitError) as e:
        lb.gemm_batch(descs)
    assert e.value.status == LOWBIT_ERR_CUDA
    lb.gemm_batch(descs)
    torch.cuda.synchronize()
    assert lb.device_status() == 0


def test_stream_ordered_status_reports_timeout():
    side = torch.cuda.Stream()
    assert lb.last_device_status(side) == 0
    with torch.cuda.stream(side):
        lb.selftest_bounded_wait(20_000_000)
    assert lb.last_device_status(side) == LOWBIT_ERR_TIMEOUT
    assert lb.last_device_status(side) == 0        # read and cleared
    assert lb.device_status() == 0


def test_debug_build_index_checks():
    """liblowbit_debug.so: same results as the release build on both kernels (no check fires on
    valid problems), and its self-test records LOWBIT_ERR_DEVICE_CHECK without a fault."""
    dbg = lb.load_debug()
    rel = lb.load()
    assert dbg.lowbit_debug_checks_enabled() == 1 and rel.lowbit_debug_checks_enabled() == 0
    assert rel.lowbit_selftest_index_check(None) == 3                   # release: not built in
    stream = torch.cuda.current_stream().cuda_stream
    assert dbg.lowbit_last_device_status(stream) == 0
    for spec in (spec_for(4, 64, 200, 768, 264, seed=3), spec_for(2, 128, 16, 2048, 1032, seed=4),
                 spec_for(1, 128, 40, 1024, 264, seed=5)):
        prob = synth.make_problem(spec)
        x, packed, s, z = _gpu.dev_problem(prob)
        ws = torch.empty(lb.workspace_size(spec.M, spec.K), dtype=torch.uint8, device="cuda")
        y_rel = torch.empty((spec.M, spec.N), dtype=torch.bfloat16, device="cuda")
        y_dbg = torch.empty_like(y_rel)
        assert gemm_via(rel, x, packed, s, z, y_rel, ws, spec) == 0
        assert gemm_via(dbg, x, packed, s, z, y_dbg, ws, spec) == 0
        torch.cuda.synchronize()
        assert dbg.lowbit_last_device_status(stream) == 0, spec.name
        assert torch.equal(y_rel.view(torch.int16), y_dbg.view(torch.int16)), spec.name
    assert dbg.lowbit_selftest_index_check(stream) == 0
    assert dbg.lowbit_last_device_status(stream) == LOWBIT_ERR_DEVICE_CHECK
    assert dbg.lowbit_last_device_status(stream) == 0


# (bits, gs, M, K, N, tile_tokens, tile_rows, ksplit): CTA-pair tiles (several per pair, and a
# ragged token tile), K split 2, 3 and 7 ways (the push reduction), flat row tiles, 16- to
# 128-token tiles, single-tile launches (the last tile's TMA store) with ragged N, and the
# small-M kernel in both orientations.
DEBUG_CASES = [(2, 128, 2304, 256, 2560, 0, 256, 0), (4, 64, 300, 384, 768, 0, 256, 0),
               (1, 128, 300, 1024, 512, 0, 256, 0), (2, 128, 512, 3072, 264, 256, 128, 2),
               (4, 64, 200, 768, 264, 256, 0, 3), (2, 64, 300, 1792, 520, 128, 0, 7),
               (2, 128, 40, 768, 264, 32, 72, 1), (1, 64, 70, 1024, 136, 16, 0, 0), (4, 128, 129, 512, 1032, 0, 0, 0),
               # the small-M kernel: X as the 16-row operand (automatic tiles, a forced 3-way split
               # with ragged N) and weights as the 16-row operand (split 2)
               (4, 64, 16, 2560, 9728, 1, 0, 0), (4, 64, 16, 9728, 2560, 1, 0, 0), (1, 128, 12, 1536, 1032, 1, 48, 3),
               (2, 128, 5, 3072, 264, 8, 16, 2), (4, 64, 3, 2048, 520, 8, 0, 0)]


@pytest.mark.parametrize("case", DEBUG_CASES, ids=lambda c: "b{}g{}_{}x{}x{}_bt{}_rows{}_ks{}".format(*c))
def test_debug_build_checks_every_tile_path(case):
    """The debug build's index checks stay silent on the CTA-pair, split-K (push reduction), flat,
    staged-store and small-M paths, and its results equal the release build's and match the
    oracle."""
    bits_, gs, M, K, N, bt, rows, ks = case
    spec = spec_for(bits_, gs, M, K, N, seed=sum(case))
    prob = synth.make_problem(spec)
    x, packed, s, z = _gpu.dev_problem(prob)
    ws = torch.empty(lb.workspace_size(M, K), dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    outs = []
    for lib in (lb.load(), lb.load_debug()):
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        st = lib.lowbit_gemm_ex(M, N, K, bits_, gs, x.data_ptr(), packed.data_ptr(), s.data_ptr(),
                                None if z is None else z.data_ptr(), y.data_ptr(), ws.data_ptr(), ws.numel(), bt,
                                rows, ks, stream)
        assert st == 0
        torch.cuda.synchronize()
        assert lib.lowbit_last_device_status(stream) == 0, spec.name
        outs.append(y)
    assert torch.equal(outs[0].view(torch.int16), outs[1].view(torch.int16)), spec.name
    ref = oracle.gemm(prob.x_bf16, _gpu.oracle_packed(prob), prob.scales, prob.zeros, N, bits_, gs)
    _gpu.check_close(_gpu.y_to_f64(outs[1]), ref, what=spec.name)
