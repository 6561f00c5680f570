"""Tiles of 256 weight rows x 256 tokens computed by a CTA pair (cta_group::2 MMAs, each CTA
holding 128 weight rows in its tensor memory and half of the tile's X rows in its shared memory)
against the fp64 oracle: every format, ragged token tiles, more pair tiles than resident pairs,
integer problems bit-exact, and agreement with single-CTA tiles within the same bound.

`tile_rows = 256` forces the pair tiles; `tile_rows = 128` forces single-CTA tiles of the same
256-token width. The automatic choice takes pairs for unsplit 256-token grids with N % 256 == 0,
which the full-size and chain tests elsewhere exercise."""
import numpy as np
import pytest
import torch

import oracle
import synth
import bit_weight_only_w2_b200 as lb
from tests import _gpu
from tests.test_gpu_gemm import FORMATS, integer_problem, spec_for

pytestmark = pytest.mark.gpu


def ref_of(prob, spec):
    return oracle.gemm(prob.x_bf16, _gpu.oracle_packed(prob), prob.scales, prob.zeros, spec.N, spec.bits,
                       spec.group_size)


def run(prob, spec, tile_rows):
    x, packed, s, z = _gpu.dev_problem(prob)
    y = lb.gemm(x, packed, s, z, spec.bits, spec.group_size, tile_rows=tile_rows)
    torch.cuda.synchronize()
    assert lb.device_status() == 0
    return y


@pytest.mark.parametrize("bits,gs", FORMATS)
def test_pair_tiles_every_format(bits, gs):
    """300 tokens (a full and a ragged 256-token tile) x 384 -> 768 (three pair tiles); the
    pair and the single-CTA tiles both match the oracle."""
    spec = spec_for(bits, gs, 300, 384, 768, seed=31)
    prob = synth.make_problem(spec)
    ref = ref_of(prob, spec)
    yp = run(prob, spec, 256)
    worst = _gpu.check_close(_gpu.y_to_f64(yp), ref, what=f"pair {spec.name}")
    ys = run(prob, spec, 128)
    _gpu.check_close(_gpu.y_to_f64(ys), ref, what=f"single {spec.name}")
    same = torch.equal(yp.view(torch.int16), ys.view(torch.int16))
    print(f"\n{spec.name}: pair max err/bound {worst:.3f}; bit-identical to single-CTA tiles: {same}")


@pytest.mark.parametrize("bits,gs", [(2, 128), (1, 128), (4, 64)])
def test_pair_tiles_persistent_loop(bits, gs):
    """2304 tokens x 256 -> 2560: 9 x 10 = 90 pair tiles on at most 74 resident pairs, so pairs
    run a second tile after their accumulator is drained. Every output against the oracle."""
    spec = spec_for(bits, gs, 2304, 256, 2560, seed=33)
    prob = synth.make_problem(spec)
    ref = ref_of(prob, spec)
    y = run(prob, spec, 256)
    _gpu.check_close(_gpu.y_to_f64(y), ref, what=f"pair persistent {spec.name}")


@pytest.mark.parametrize("bits", [1, 2, 4])
def test_pair_integer_exact(bits):
    """Unit scales, integer zeros, x in {-1,0,1}, |y| <= 256: the pair tiles' bf16 output equals
    the oracle exactly (ragged token tile, two pair tiles along N, long K)."""
    M, N, K, g = 300, 512, 1024, 64
    prob = integer_problem(bits, M, K, N, g, seed=40 + bits, nonzeros=256)
    ref = oracle.gemm(prob.x_bf16, _gpu.oracle_packed(prob), prob.scales, prob.zeros, N, bits, g)
    xd, packed, sd, zd = _gpu.dev_problem(prob)
    y = lb.gemm(xd, packed, sd, zd, bits, g, tile_rows=256)
    torch.cuda.synchronize()
    assert lb.device_status() == 0
    assert np.array_equal(_gpu.y_to_f64(y), ref)


def test_pair_tiles_deterministic_and_automatic():
    """Repeated pair launches give identical bits, and the automatic configuration of an unsplit
    256-token grid with N % 256 == 0 gives the same bits as the forced pair tiles."""
    spec = spec_for(2, 128, 600, 1024, 1024, seed=35)
    prob = synth.make_problem(spec)
    x, packed, s, z = _gpu.dev_problem(prob)
    outs = [lb.gemm(x, packed, s, z, 2, 128, tile_rows=256) for _ in range(3)]
    auto = lb.gemm(x, packed, s, z, 2, 128)
    torch.cuda.synchronize()
    assert lb.device_status() == 0
    for o in outs[1:] + [auto]:
        assert torch.equal(outs[0].view(torch.int16), o.view(torch.int16))
    _gpu.check_close(_gpu.y_to_f64(outs[0]), ref_of(prob, spec), what="pair 600x1024x1024")


@pytest.mark.parametrize("M,N,tile_tokens,ksplit", [(300, 520, 0, 0), (100, 512, 0, 0), (300, 512, 128, 0),
                                                     (300, 512, 0, 2)])
def test_pair_tiles_unsupported_shapes(M, N, tile_tokens, ksplit):
    """Pair tiles need 256-token tiles, N % 256 == 0 and no K split: anything else is refused."""
    spec = spec_for(2, 128, M, 256, N, seed=37)
    prob = synth.make_problem(spec)
    x, packed, s, z = _gpu.dev_problem(prob)
    with pytest.raises(lb.LowbitError) as e:
        lb.gemm(x, packed, s, z, 2, 128, tile_tokens=tile_tokens, tile_rows=256, ksplit=ksplit)
    assert e.value.status == 3   # LOWBIT_ERR_UNSUPPORTED
