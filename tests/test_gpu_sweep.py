"""A seeded sweep of shapes and launch configurations against the fp64 oracle.

Each case draws a format, a shape (1 to 700 tokens, K a multiple of the group, N a multiple of
8) and one of the launch configurations the C ABI accepts: automatic, a forced token tile with a
forced K split and row count, the small-M kernel in either orientation with forced rows and
splits, or CTA-pair tiles. Every case runs first on the debug build, whose device-side index
checks record an out-of-range access instead of making it, then on the release build; the two
outputs must be bit-identical and match the oracle within the bound of `tests/_gpu.py`.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import bit_weight_only_w2_b200 as lb
from tests import _gpu
from tests.test_gpu_gemm import FORMATS, spec_for


def sweep_cases(n=200, seed=2026):
    """(bits, gs, M, K, N, tile_tokens, tile_rows, ksplit) tuples, every one a configuration the
    ABI documents as supported (no case is expected to be refused)."""
    rng = np.random.default_rng(seed)
    cases = []
    while len(cases) < n:
        bits, gs = FORMATS[rng.integers(len(FORMATS))]
        band = int(rng.integers(4))
        M = int([rng.integers(1, 17), rng.integers(17, 65), rng.integers(65, 301), rng.integers(301, 701)][band])
        kunit = 128 if bits == 1 else gs
        K = kunit * int(rng.integers(1, 2560 // kunit + 1))
        N = 8 * int(rng.integers(1, 201))
        modes = ["auto", "forced"] + (["smallm"] if M <= 16 else []) + (["swapped"] if M <= 8 else []) + \
                (["pair"] if M > 128 else [])
        mode = modes[rng.integers(len(modes))]
        if mode == "auto":
            bt, rows, ks = 0, 0, 0
        elif mode == "forced":      # the tensor-memory kernel: token tile, rows per CTA, K split
            bt = int(rng.choice([16, 32, 64, 128, 256]))
            rows = 8 * int(rng.integers(0, 17))
            ks = int(rng.integers(1, 5))
        elif mode == "smallm":      # warp-MMA kernel, X as the 16-row operand
            bt, rows, ks = 1, 8 * int(rng.integers(0, 17)), int(rng.integers(0, 4))
        elif mode == "swapped":     # warp-MMA kernel, weights as the 16-row operand
            bt, rows, ks = 8, 16 * int(rng.integers(1, 9)), int(rng.integers(0, 3))
        else:                       # CTA-pair tiles: 256 weight rows x 256 tokens
            N = 256 * int(rng.integers(1, 7))
            bt, rows, ks = 256, 256, 0
        if M * K * N > 300_000_000:
            continue
        cases.append((bits, gs, M, K, N, bt, rows, ks))
    return cases


def _mode(c):
    return "auto" if c[5] == 0 else "pair" if c[6] == 256 else {1: "smallm", 8: "swapped"}.get(c[5], "forced")


def test_sweep_covers_every_mode():
    """The seeded draw reaches every launch mode, each more than once."""
    counts = {}
    for c in sweep_cases():
        counts[_mode(c)] = counts.get(_mode(c), 0) + 1
    assert set(counts) == {"auto", "forced", "smallm", "swapped", "pair"}
    assert min(counts.values()) >= 2, counts


@pytest.mark.gpu
@pytest.mark.parametrize("case", sweep_cases(), ids=lambda c: "b{}g{}_{}x{}x{}_bt{}_rows{}_ks{}".format(*c))
def test_sweep_against_oracle(case):
    bits, gs, M, K, N, bt, rows, ks = case
    spec = spec_for(bits, gs, M, K, N, seed=sum(case))
    prob = synth.make_problem(spec)
    x, packed, s, z = _gpu.dev_problem(prob)
    ws = torch.empty(lb.workspace_size(M, K), dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    outs = []
    for lib in (lb.load_debug(), lb.load()):
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        st = lib.lowbit_gemm_ex(M, N, K, bits, gs, x.data_ptr(), packed.data_ptr(), s.data_ptr(),
                                None if z is None else z.data_ptr(), y.data_ptr(), ws.data_ptr(), ws.numel(), bt,
                                rows, ks, stream)
        assert st == 0, f"{spec.name}: status {st}"
        torch.cuda.synchronize()
        assert lib.lowbit_last_device_status(stream) == 0, spec.name
        outs.append(y)
    assert torch.equal(outs[0].view(torch.int16), outs[1].view(torch.int16)), spec.name
    ref = oracle.gemm(prob.x_bf16, _gpu.oracle_packed(prob), prob.scales, prob.zeros, N, bits, gs)
    _gpu.check_close(_gpu.y_to_f64(outs[1]), ref, what=spec.name)
