"""GPU packer / unpacker against the oracle: bit-exact."""
import numpy as np
import pytest
import torch

import oracle
import synth
import bit_weight_only_w2_b200 as lb
from tests import _pins

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("bits", [1, 2, 4])
@pytest.mark.parametrize("N,K", [(1, 32), (7, 96), (33, 256), (300, 384), (1000, 3072)])
def test_pack_unpack_bit_exact(bits, N, K):
    codes = _pins.random_codes(N, K, bits, seed=N + K + bits)
    want, bad = oracle.pack(codes, bits)
    assert bad == 0
    got = lb.pack(torch.from_numpy(codes).cuda(), bits)
    assert np.array_equal(got.cpu().numpy().view(np.uint32), want)
    back = lb.unpack(got, N, K, bits)
    assert np.array_equal(back.cpu().numpy(), codes)


@pytest.mark.parametrize("bits,K", [(4, 40), (4, 104), (2, 80), (2, 112), (2, 48)])
def test_pack_rows_with_plain_tail_words(bits, K):
    """Rows whose word count is not a multiple of four: whole blocks in block order, then the
    remaining words in plain order."""
    N = 11
    codes = _pins.random_codes(N, K, bits, seed=K + 7 * bits)
    want, bad = oracle.pack(codes, bits)
    assert bad == 0
    got = lb.pack(torch.from_numpy(codes).cuda(), bits)
    assert np.array_equal(got.cpu().numpy().view(np.uint32), want)
    assert np.array_equal(lb.unpack(got, N, K, bits).cpu().numpy(), codes)


def test_pack_golden_words():
    for bits, K, N, codes, words in _pins.load_golden_pack():
        got = lb.pack(torch.from_numpy(codes).cuda(), bits).cpu().numpy().view(np.uint32)
        assert np.array_equal(got, words), (bits, K)


@pytest.mark.parametrize("bits,badv", [(1, 0), (2, 2), (2, -2), (4, 16), (4, -1)])
def test_pack_rejects_invalid_codes(bits, badv):
    codes = _pins.random_codes(64, 128, bits, seed=1)
    codes[63, 127] = badv
    with pytest.raises(lb.LowbitError) as e:
        lb.pack(torch.from_numpy(codes).cuda(), bits)
    assert e.value.status == 5
    # a valid call right after succeeds (the error counter is reset per call)
    codes[63, 127] = 1 if bits != 4 else 3
    lb.pack(torch.from_numpy(codes).cuda(), bits)


def test_unpack_rejects_ternary_field_3():
    words = torch.full((2, 4), -1, dtype=torch.int32, device="cuda")
    with pytest.raises(lb.LowbitError) as e:
        lb.unpack(words, 2, 64, 2)
    assert e.value.status == 5


def test_pack_full_size_weights():
    spec = synth.WORKLOADS["mlp_1024sq_binary_g128"][0]
    codes = synth.codes(spec.seed, synth.STREAM_CODES, (spec.N, spec.K), spec.bits)
    want, _ = oracle.pack(codes, spec.bits)
    got = lb.pack(torch.from_numpy(codes).cuda(), spec.bits)
    assert np.array_equal(got.cpu().numpy().view(np.uint32), want)
