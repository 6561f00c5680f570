"""The shared input generator against its published definitions and library routines."""
import numpy as np
import torch

import synth


def test_splitmix64_first_output():
    # splitmix64 seeded with 0: the first output is 0xE220A8397B1DCDAF.
    assert synth.raw_u64(0, 0, 0) == 0xE220A8397B1DCDAF


def test_counter_mixing():
    a = synth.raw_u64(0, 1, 5)
    assert a == synth.raw_u64(0, 1, 5)
    assert a != synth.raw_u64(1, 1, 5) and a != synth.raw_u64(0, 2, 5) and a != synth.raw_u64(0, 1, 6)


def test_uniform_and_normal_moments():
    u = synth.uniform_f64(0, 1, 200000)
    assert 0.0 <= u.min() and u.max() < 1.0
    assert abs(u.mean() - 0.5) < 0.005
    z = synth.normal_f64(0, 2, 200000)
    assert abs(z.mean()) < 0.01 and abs(z.std() - 1.0) < 0.01


def test_bf16_rounding_matches_torch():
    z = synth.normal_f64(3, 1, 50000)
    got = synth.normal_bf16(3, 1, (50000,))
    want = torch.tensor(z.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, want)


def test_fp16_rounding_matches_numpy():
    u = synth.uniform_f64(4, 3, 50000)
    got = synth.uniform_f16(4, 3, (50000,), 0.005, 0.02)
    want = (0.005 + (0.02 - 0.005) * u).astype(np.float16)
    assert np.array_equal(got.view(np.uint16), want.view(np.uint16))


def test_codes_distributions():
    t = synth.codes(0, 2, (400000,), 2, 0.4)
    assert set(np.unique(t)) == {-1, 0, 1}
    assert abs((t == 0).mean() - 0.4) < 0.005 and abs((t == 1).mean() - 0.3) < 0.005
    b = synth.codes(0, 2, (400000,), 1)
    assert set(np.unique(b)) == {-1, 1} and abs((b == 1).mean() - 0.5) < 0.005
    q = synth.codes(0, 2, (400000,), 4)
    assert q.min() == 0 and q.max() == 15 and abs(q.mean() - 7.5) < 0.05


def test_workloads_shapes():
    chain = synth.chain_linears()
    assert len(chain) == 80
    flops = sum(s.flops for s in chain)
    assert abs(flops / 1e12 - 21.743) < 0.01
    # packed ternary codes plus fp16 group scales: about 752 MB per step
    wbytes = sum(s.N * s.K * s.bits // 8 + (s.K // s.group_size) * s.N * 2 for s in chain)
    assert abs(wbytes / 1e6 - 752) < 1.0
    for specs in synth.WORKLOADS.values():
        for s in specs:
            assert s.K % s.group_size == 0


def test_unfused_projection_layout_has_100_linears():
    """Separate Q/K/V and add-Q/K/V per double block: 5 x 12 + 20 x 2 = 100 linears, the same
    work and weights as the fused layout."""
    sep = synth.WORKLOADS["klein_step_linears100_1024sq_ternary_g128"]
    fused = synth.chain_linears()
    assert len(sep) == 100
    assert sum(s.flops for s in sep) == sum(s.flops for s in fused)
    wb = lambda specs: sum(s.N * s.K * s.bits // 8 + (s.K // s.group_size) * s.N * 2 for s in specs)  # noqa: E731
    assert wb(sep) == wb(fused)
    q = [s for s in sep if s.name.endswith(".q")]
    assert len(q) == 10 and all((s.K, s.N) == (3072, 3072) for s in q)


def test_text_encoder_layer_workloads():
    for tokens in (512, 16):
        specs = synth.WORKLOADS[f"te_mlp4_m{tokens}_uint4_g64"]
        assert len(specs) == 12
        assert all(s.M == tokens and s.bits == 4 and s.group_size == 64 for s in specs)
        assert sorted({(s.K, s.N) for s in specs}) == [(2560, 9728), (9728, 2560)]
        # every linear draws its own weights
        assert len({(s.seed, s.stream_base) for s in specs}) == 12
