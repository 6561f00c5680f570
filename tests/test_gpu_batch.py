"""lowbit_gemm_batch with runs of small-M linears (the text encoder at a handful of tokens):
independent linears of several shapes, dependent chains (a linear reading the previous one's
output, and one overwriting an earlier linear's input), formats and orientations mixed with
tensor-memory linears, and repeatability. Each output is compared with the fp64 oracle on the
inputs that linear actually read (for a linear that reads an earlier one's output, that output
as the GPU wrote it)."""
import numpy as np
import pytest
import torch

import oracle
import synth
import bit_weight_only_w2_b200 as lb
from tests import _gpu
from tests.test_gpu_gemm import spec_for

pytestmark = pytest.mark.gpu


def bits16(t: torch.Tensor) -> np.ndarray:
    """bf16 device tensor -> host uint16 bit patterns (the oracle's X format)."""
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def weights(spec):
    prob = synth.make_problem(spec)
    _, packed, s, z = _gpu.dev_problem(prob)
    return prob, packed, s, z


def check(spec, prob, x_bits, y):
    ref = oracle.gemm(x_bits, _gpu.oracle_packed(prob), prob.scales, prob.zeros, spec.N, spec.bits,
                      spec.group_size)
    return _gpu.check_close(_gpu.y_to_f64(y), ref, what=spec.name)


@pytest.mark.parametrize("bits,gs,M", [(4, 64, 16), (4, 64, 5), (2, 128, 16), (2, 128, 1), (1, 128, 8),
                                        (1, 64, 12)])
def test_independent_small_m_linears(bits, gs, M):
    """Five independent linears with different K and N (ragged N, K not a multiple of 512) in one
    batch; every output matches the oracle."""
    shapes = [(2560, 9728), (9728, 2560), (1024, 1032), (768, 264), (3072, 3072)]
    specs = [spec_for(bits, gs, M, k, n, seed=100 + i) for i, (k, n) in enumerate(shapes)
             if not (bits == 1 and k % 128)]
    items = []
    for sp in specs:
        prob, packed, s, z = weights(sp)
        x = torch.from_numpy(prob.x_bf16.view(np.int16)).cuda().view(torch.bfloat16)
        y = torch.full((sp.M, sp.N), float("nan"), dtype=torch.bfloat16, device="cuda")
        items.append((sp, prob, x, packed, s, z, y))
    lb.gemm_batch([lb.make_desc(x, w, s, z, y, sp.bits, sp.group_size) for sp, _, x, w, s, z, y in items])
    torch.cuda.synchronize()
    assert lb.device_status() == 0
    for sp, prob, x, _, _, _, y in items:
        check(sp, prob, prob.x_bf16, y)


@pytest.mark.parametrize("bits,gs,M", [(4, 64, 16), (2, 128, 4)])
def test_dependent_small_m_chain(bits, gs, M):
    """Text-encoder-like chain: up (2560 -> 9728), down reads up's output (9728 -> 2560), the next
    up reads down's output, and a last linear overwrites the first one's input (a write after
    read): the batch keeps stream order between the launches."""
    K0, K1 = 2560, 9728
    sp = [spec_for(bits, gs, M, K0, K1, seed=201), spec_for(bits, gs, M, K1, K0, seed=202),
          spec_for(bits, gs, M, K0, K1, seed=203), spec_for(bits, gs, M, K1, K0, seed=204)]
    w = [weights(s) for s in sp]
    x0 = torch.from_numpy(w[0][0].x_bf16.view(np.int16)).cuda().view(torch.bfloat16)
    x0_before = bits16(x0)
    y0 = torch.empty((M, K1), dtype=torch.bfloat16, device="cuda")
    y1 = torch.empty((M, K0), dtype=torch.bfloat16, device="cuda")
    y2 = torch.empty((M, K1), dtype=torch.bfloat16, device="cuda")
    # linear 3 reads y2 and writes x0 (read by linear 0: write after read)
    descs = [lb.make_desc(x0, w[0][1], w[0][2], w[0][3], y0, bits, gs),
             lb.make_desc(y0, w[1][1], w[1][2], w[1][3], y1, bits, gs),
             lb.make_desc(y1, w[2][1], w[2][2], w[2][3], y2, bits, gs),
             lb.make_desc(y2, w[3][1], w[3][2], w[3][3], x0, bits, gs)]
    lb.gemm_batch(descs)
    torch.cuda.synchronize()
    assert lb.device_status() == 0
    check(sp[0], w[0][0], x0_before, y0)
    check(sp[1], w[1][0], bits16(y0), y1)
    check(sp[2], w[2][0], bits16(y1), y2)
    check(sp[3], w[3][0], bits16(y2), x0)


def test_mixed_small_and_large_m_batch():
    """Small-M linears of both orientations around tensor-memory linears, with format changes:
    [uint4 M=16 x2, ternary M=300 (X copied to the workspace), uint4 M=4 x2, binary M=16, ternary
    M=300 on the same X as the first ternary one, which may reuse its fp16 copy: the small-M
    linears in between leave the workspace untouched]."""
    specs = [spec_for(4, 64, 16, 2560, 2048, seed=301), spec_for(4, 64, 16, 2048, 1032, seed=302),
             spec_for(2, 128, 300, 512, 264, seed=303),
             spec_for(4, 64, 4, 1024, 520, seed=304), spec_for(4, 64, 4, 512, 136, seed=305),
             spec_for(1, 128, 16, 1024, 1024, seed=306),
             spec_for(2, 128, 300, 512, 136, seed=307)]
    items = []
    for sp in specs:
        prob, packed, s, z = weights(sp)
        x = torch.from_numpy(prob.x_bf16.view(np.int16)).cuda().view(torch.bfloat16)
        items.append([sp, prob, x, packed, s, z, torch.empty((sp.M, sp.N), dtype=torch.bfloat16, device="cuda")])
    items[6][2] = items[2][2]                       # same X as linear 2
    items[6][1].x_bf16 = items[2][1].x_bf16
    lb.gemm_batch([lb.make_desc(x, w, s, z, y, sp.bits, sp.group_size) for sp, _, x, w, s, z, y in items])
    torch.cuda.synchronize()
    assert lb.device_status() == 0
    for sp, prob, _, _, _, _, y in items:
        check(sp, prob, prob.x_bf16, y)


def test_small_m_batch_is_deterministic():
    specs = [spec_for(4, 64, 16, 9728, 2560, seed=401), spec_for(4, 64, 16, 2560, 9728, seed=402),
             spec_for(4, 64, 16, 2560, 9728, seed=403)]
    items = []
    for sp in specs:
        prob, packed, s, z = weights(sp)
        x = torch.from_numpy(prob.x_bf16.view(np.int16)).cuda().view(torch.bfloat16)
        items.append((sp, x, packed, s, z))
    outs = []
    for _ in range(3):
        ys = [torch.empty((sp.M, sp.N), dtype=torch.bfloat16, device="cuda") for sp, *_ in items]
        lb.gemm_batch([lb.make_desc(x, w, s, z, y, 4, 64) for (sp, x, w, s, z), y in zip(items, ys)])
        outs.append(ys)
    torch.cuda.synchronize()
    for ys in outs[1:]:
        for a, b in zip(outs[0], ys):
            assert torch.equal(a.view(torch.int16), b.view(torch.int16))
