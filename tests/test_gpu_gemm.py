"""GPU GEMM against the fp64 CPU oracle.

Bound per element: |gpu - ref| <= 1e-2 |ref| + 1e-2 rms(ref) (ref = oracle, fp64). Small and
ragged shapes are compared whole; full workload sizes are compared on sampled entries (4096
random ones plus 16 full rows and 16 full columns) in the configuration the benchmark runs.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import bit_weight_only_w2_b200 as lb
from synth.workloads import LinearSpec
from tests import _gpu, _pins

pytestmark = pytest.mark.gpu

FORMATS = [(1, 128), (1, 64), (2, 128), (2, 64), (4, 64), (4, 128)]


def spec_for(bits, gs, M, K, N, seed=0, p0=0.4):
    kw = dict(bits=bits, group_size=gs, p0=p0, seed=seed)
    if bits == 4:
        kw.update(scale_lo=0.002, scale_hi=0.01)
    return LinearSpec(f"b{bits}g{gs}_{M}x{K}x{N}", M, K, N, **kw)


def run_and_compare(spec, tile_tokens=0, ksplit=0, prob=None, ref=None):
    prob = prob or synth.make_problem(spec)
    x, packed, s, z = _gpu.dev_problem(prob)
    y = lb.gemm(x, packed, s, z, spec.bits, spec.group_size, tile_tokens=tile_tokens, ksplit=ksplit)
    torch.cuda.synchronize()
    assert lb.device_status() == 0
    if ref is None:
        ref = oracle.gemm(prob.x_bf16, _gpu.oracle_packed(prob), prob.scales, prob.zeros, spec.N, spec.bits,
                          spec.group_size)
    _gpu.check_close(_gpu.y_to_f64(y), ref, what=f"{spec.name} bt={tile_tokens} split={ksplit}")
    return y, ref


@pytest.mark.parametrize("bits,gs", FORMATS)
@pytest.mark.parametrize("M,K,N", [(64, 256, 512), (300, 512, 520), (1, 256, 128), (129, 384, 136)])
def test_gemm_auto_config(bits, gs, M, K, N):
    if bits == 1 and K % 128:
        pytest.skip("binary needs K % 128 == 0")
    run_and_compare(spec_for(bits, gs, M, K, N, seed=M + N))


def test_tiny_ternary_workload():
    spec = synth.WORKLOADS["tiny_ternary_g64"][0]
    run_and_compare(spec)


_ref_cache = {}


@pytest.mark.parametrize("bits,gs", FORMATS)
@pytest.mark.parametrize("tile_tokens", [16, 32, 64, 128, 256])
@pytest.mark.parametrize("ksplit", [1, 2, 3, 7])
def test_gemm_every_tile_config(bits, gs, tile_tokens, ksplit):
    spec = spec_for(bits, gs, 200, 768, 264, seed=7)
    key = (bits, gs)
    if key not in _ref_cache:
        prob = synth.make_problem(spec)
        ref = oracle.gemm(prob.x_bf16, _gpu.oracle_packed(prob), prob.scales, prob.zeros, spec.N, bits, gs)
        _ref_cache[key] = (prob, ref)
    prob, ref = _ref_cache[key]
    run_and_compare(spec, tile_tokens, ksplit, prob=prob, ref=ref)


_flat_cache = {}


@pytest.mark.parametrize("bits,gs", FORMATS)
@pytest.mark.parametrize("tile_tokens", [16, 32, 64])
@pytest.mark.parametrize("tile_rows", [8, 40, 72, 120])
def test_gemm_flat_row_tiles(bits, gs, tile_tokens, tile_rows):
    """Small-M "flat" tiles: fewer than 128 weight rows per CTA, whole K per CTA, ragged N."""
    spec = spec_for(bits, gs, 40, 768, 264, seed=9)
    key = (bits, gs)
    if key not in _flat_cache:
        prob = synth.make_problem(spec)
        ref = oracle.gemm(prob.x_bf16, _gpu.oracle_packed(prob), prob.scales, prob.zeros, spec.N, bits, gs)
        _flat_cache[key] = (prob, ref)
    prob, ref = _flat_cache[key]
    x, packed, s, z = _gpu.dev_problem(prob)
    y = lb.gemm(x, packed, s, z, bits, gs, tile_tokens=tile_tokens, tile_rows=tile_rows, ksplit=1)
    torch.cuda.synchronize()
    assert lb.device_status() == 0
    _gpu.check_close(_gpu.y_to_f64(y), ref, what=f"flat rows={tile_rows} bt={tile_tokens}")


@pytest.mark.parametrize("bits,gs", FORMATS)
@pytest.mark.parametrize("M", [1, 5, 16])
@pytest.mark.parametrize("K,N,rows,ksplit", [
    (256, 520, 0, 1),       # one step, half of it past K
    (768, 264, 0, 3),       # a request for 3 slices served with 2 (slices are whole 512-wide steps)
    (2560, 1032, 0, 0),     # automatic choice
    (9728, 256, 0, 0),      # long K, few rows: split over a cluster
    (640, 136, 56, 0),      # 7 octets: a partial batch of four
    (1152, 1000, 120, 2),   # the second slice holds one 128-wide group of K
    (1024, 2376, 8, 1),     # more row blocks than SMs: persistent tiles, no cluster
    (2048, 1352, 8, 2),     # persistent tiles with the cross-rank reduction on every tile
])
def test_gemm_small_m_warp_mma(bits, gs, M, K, N, rows, ksplit):
    """The small-M kernel (warp-level MMAs on X as stored), ragged N and K, forced tilings."""
    if bits == 1 and K % 128:
        pytest.skip("binary needs K % 128 == 0")
    spec = spec_for(bits, gs, M, K, N, seed=M * 7 + K)
    prob = synth.make_problem(spec)
    ref = oracle.gemm(prob.x_bf16, _gpu.oracle_packed(prob), prob.scales, prob.zeros, N, bits, gs)
    x, packed, s, z = _gpu.dev_problem(prob)
    y = lb.gemm(x, packed, s, z, bits, gs, tile_tokens=1, tile_rows=rows, ksplit=ksplit)
    torch.cuda.synchronize()
    assert lb.device_status() == 0
    _gpu.check_close(_gpu.y_to_f64(y), ref, what=f"warp-mma M={M} K={K} N={N} rows={rows} split={ksplit}")


def test_gemm_small_m_deterministic():
    """Repeated small-M runs with a cluster split give bit-identical outputs (fixed summation order)."""
    spec = spec_for(4, 64, 16, 9728, 2560, seed=5)
    prob = synth.make_problem(spec)
    x, packed, s, z = _gpu.dev_problem(prob)
    ys = [lb.gemm(x, packed, s, z, 4, 64, tile_tokens=1, ksplit=4).clone() for _ in range(3)]
    torch.cuda.synchronize()
    assert all(torch.equal(ys[0].view(torch.int16), y.view(torch.int16)) for y in ys[1:])


def test_gemm_small_m_k_partial_block():
    """K a multiple of 64 but not of 128 on the small-M kernel (last k-block half out of range)."""
    spec = spec_for(2, 64, 9, 192, 136, seed=2)
    run_and_compare(spec, tile_tokens=1)


@pytest.mark.parametrize("bits,gs", [(2, 64), (4, 64)])
def test_k_single_group_partial_stage(bits, gs):
    # K = 64: one half-filled stage of 128; the other half reads out of bounds (zero-filled)
    run_and_compare(spec_for(bits, gs, 40, 64, 24, seed=3))


def test_n_minimum_and_m_one():
    run_and_compare(spec_for(2, 128, 1, 256, 8, seed=5))
    run_and_compare(spec_for(1, 128, 17, 128, 8, seed=6))


def test_all_zero_ternary_gives_zero():
    spec = spec_for(2, 128, 100, 512, 256)
    prob = synth.make_problem(spec)
    prob.codes[:] = 0
    x, packed, s, z = _gpu.dev_problem(prob)
    y = lb.gemm(x, packed, s, z, 2, 128)
    assert torch.count_nonzero(y.float()) == 0


@pytest.mark.parametrize("bits", [1, 2, 4])
def test_integer_exact(bits):
    """Unit scales, integer zeros, x in {-1,0,1}, |y| <= 256: bf16 output equals the oracle."""
    M, N, K, g = 70, 136, 256, 64
    codes = _pins.random_codes(N, K, bits, seed=bits)
    if bits == 4:
        codes = np.random.default_rng(bits).integers(7, 10, size=(N, K)).astype(np.int8)
    x = _pins.small_int_x(M, K, seed=bits)
    s = np.ones((K // g, N), dtype=np.float16)
    z = np.full((K // g, N), 8.0, dtype=np.float16) if bits == 4 else None
    prob = synth.Problem(spec_for(bits, g, M, K, N), x, codes, s, z)
    ref = oracle.gemm(x, _gpu.oracle_packed(prob), s, z, N, bits, g)
    xd, packed, sd, zd = _gpu.dev_problem(prob)
    y = _gpu.y_to_f64(lb.gemm(xd, packed, sd, zd, bits, g))
    assert np.array_equal(y, ref)


def test_orientation_square():
    """K = N with a non-symmetric W: the GPU result matches W, not W^T (layout-orientation guard)."""
    spec = spec_for(2, 128, 64, 512, 512, seed=11)
    prob = synth.make_problem(spec)
    y, ref = run_and_compare(spec, prob=prob)
    codes_t = np.ascontiguousarray(prob.codes.T)
    ref_t = oracle.gemm(prob.x_bf16, oracle.pack(codes_t, 2)[0], prob.scales, None, spec.N, 2, 128)
    assert not np.allclose(_gpu.y_to_f64(y), ref_t, rtol=1e-2, atol=1e-2)


def test_binary_all_plus_one_group_sums():
    spec = spec_for(1, 128, 96, 1024, 256, seed=12)
    prob = synth.make_problem(spec)
    prob.codes[:] = 1
    x, packed, s, z = _gpu.dev_problem(prob)
    y = _gpu.y_to_f64(lb.gemm(x, packed, s, None, 1, 128))
    xf = _pins.x_as_f64(prob.x_bf16)
    want = xf.reshape(96, 8, 128).sum(axis=2) @ prob.scales.astype(np.float64)
    _gpu.check_close(y, want, what="group row sums")


# ------------------------------------------------------------------ full workload sizes (sampled)
def sampled_check(spec, seed=0, n_random=4096, n_rows=16, n_cols=16):
    prob = synth.make_problem(spec)
    x, packed, s, z = _gpu.dev_problem(prob)
    y = _gpu.y_to_f64(lb.gemm(x, packed, s, z, spec.bits, spec.group_size))
    assert lb.device_status() == 0
    r = np.random.default_rng(seed)
    ms = [r.integers(0, spec.M, n_random)]
    ns = [r.integers(0, spec.N, n_random)]
    rows = r.choice(spec.M, size=min(n_rows, spec.M), replace=False)
    cols = r.choice(spec.N, size=min(n_cols, spec.N), replace=False)
    for m in rows:
        ms.append(np.full(spec.N, m))
        ns.append(np.arange(spec.N))
    for n in cols:
        ms.append(np.arange(spec.M))
        ns.append(np.full(spec.M, n))
    ms = np.concatenate(ms)
    ns = np.concatenate(ns)
    ref = oracle.gemm_entries(prob.x_bf16, _gpu.oracle_packed(prob), prob.scales, prob.zeros, spec.N, spec.bits,
                              spec.group_size, ms, ns)
    rms = float(np.sqrt(np.mean(ref * ref)))
    return _gpu.check_close(y[ms, ns], ref, rms=rms, what=spec.name)


FULL = [s for w in ("qkv_512sq_ternary_g128", "mlp_1024sq_binary_g128", "te_m512_uint4_g64", "te_m16_uint4_g64")
        for s in synth.WORKLOADS[w]]


@pytest.mark.parametrize("spec", FULL, ids=lambda s: s.name)
def test_full_size_sampled(spec):
    worst = sampled_check(spec)
    print(f"\n{spec.name} M={spec.M} K={spec.K} N={spec.N}: max err/bound {worst:.3f}")


@pytest.mark.parametrize("bits,gs", [(4, 64), (2, 128), (1, 128)])
def test_second_wave_tiles(bits, gs):
    """512 x 2048 -> 9728: 2 x 76 = 152 tiles of 256 tokens x 128 rows. On a 148-SM B200 the
    persistent grid gives the last 4 tiles (tokens 256.., rows 9216..) to CTAs that already
    finished one, after their accumulator is drained; every output of those tiles is checked,
    plus random outputs elsewhere."""
    spec = spec_for(bits, gs, 512, 2048, 9728, seed=7)
    prob = synth.make_problem(spec)
    x, packed, s, z = _gpu.dev_problem(prob)
    y = _gpu.y_to_f64(lb.gemm(x, packed, s, z, bits, gs))
    assert lb.device_status() == 0
    tm, tn = np.meshgrid(np.arange(256, 512), np.arange(9216, 9728), indexing="ij")
    r = np.random.default_rng(3)
    ms = np.concatenate([tm.ravel(), r.integers(0, 512, 8192)])
    ns = np.concatenate([tn.ravel(), r.integers(0, 9728, 8192)])
    ref = oracle.gemm_entries(prob.x_bf16, _gpu.oracle_packed(prob), prob.scales, prob.zeros, spec.N, bits, gs,
                              ms, ns)
    rms = float(np.sqrt(np.mean(ref * ref)))
    _gpu.check_close(y[ms, ns], ref, rms=rms, what=f"second-wave tiles bits={bits}")


def chain_distinct():
    seen = {}
    for s in synth.chain_linears():
        seen.setdefault((s.M, s.K, s.N), s)
    return list(seen.values())


@pytest.mark.parametrize("spec", chain_distinct(), ids=lambda s: s.name)
def test_chain_shapes_sampled(spec):
    worst = sampled_check(spec, n_random=2048, n_rows=4, n_cols=4)
    print(f"\n{spec.name} M={spec.M} K={spec.K} N={spec.N}: max err/bound {worst:.3f}")


def test_batch_matches_single_calls():
    specs = [spec_for(2, 128, m, k, n, seed=i) for i, (m, k, n) in
             enumerate([(300, 384, 264), (64, 256, 512), (16, 1024, 520), (513, 256, 136)])]
    probs = [synth.make_problem(sp) for sp in specs]
    dev = [_gpu.dev_problem(p) for p in probs]
    singles = [lb.gemm(x, w, s, z, sp.bits, sp.group_size) for sp, (x, w, s, z) in zip(specs, dev)]
    outs = [torch.empty_like(y) for y in singles]
    descs = [lb.make_desc(x, w, s, z, o, sp.bits, sp.group_size) for sp, (x, w, s, z), o in zip(specs, dev, outs)]
    lb.gemm_batch(descs)
    torch.cuda.synchronize()
    for y1, y2 in zip(singles, outs):
        assert torch.equal(y1, y2)
    for sp, p, y in zip(specs, probs, outs):
        ref = oracle.gemm(p.x_bf16, _gpu.oracle_packed(p), p.scales, p.zeros, sp.N, sp.bits, sp.group_size)
        _gpu.check_close(_gpu.y_to_f64(y), ref, what=sp.name)


def test_batch_chain_dependency():
    """A descriptor may read the previous descriptor's output (stream order is kept)."""
    a = spec_for(2, 128, 128, 256, 256, seed=21)
    b = spec_for(2, 128, 128, 256, 128, seed=22)
    pa, pb = synth.make_problem(a), synth.make_problem(b)
    xa, wa, sa, _ = _gpu.dev_problem(pa)
    _, wb, sb, _ = _gpu.dev_problem(pb)
    ya = torch.empty((128, 256), dtype=torch.bfloat16, device="cuda")
    yb = torch.empty((128, 128), dtype=torch.bfloat16, device="cuda")
    lb.gemm_batch([lb.make_desc(xa, wa, sa, None, ya, 2, 128), lb.make_desc(ya, wb, sb, None, yb, 2, 128)])
    want = lb.gemm(lb.gemm(xa, wa, sa, None, 2, 128), wb, sb, None, 2, 128)
    torch.cuda.synchronize()
    assert torch.equal(yb, want)


def test_bounded_wait_timeout_is_reported():
    """A kernel wait that nothing completes gives up, reports LOWBIT_ERR_TIMEOUT, and the
    context stays usable."""
    assert lb.device_status() == 0
    lb.selftest_bounded_wait(20_000_000)
    assert lb.device_status(clear=True) == 6
    assert lb.device_status() == 0
    run_and_compare(spec_for(2, 128, 64, 256, 128, seed=1))


def test_extreme_row_magnitudes():
    """Rows far outside fp16's range (huge, tiny, zero, near the bf16 maximum) still match the
    oracle row by row: X is converted with a per-row power-of-two factor."""
    spec = spec_for(2, 128, 64, 512, 256, seed=31)
    prob = synth.make_problem(spec)
    x = _pins.x_as_f64(prob.x_bf16)
    x[0] *= 2.0 ** 20
    x[1] *= 2.0 ** -30
    x[2] = 0.0
    x[3] *= 2.0 ** -100
    x[4, 7] = 1.5 * 2.0 ** 127          # near the bf16 maximum
    x[5] *= 2.0 ** 60
    prob.x_bf16 = _pins.bf16_bits_from_f32(x.astype(np.float32))
    ref = oracle.gemm(prob.x_bf16, _gpu.oracle_packed(prob), prob.scales, None, spec.N, 2, 128)
    xd, packed, s, z = _gpu.dev_problem(prob)
    y = _gpu.y_to_f64(lb.gemm(xd, packed, s, z, 2, 128))
    assert np.all(y[2] == 0.0)
    for m in range(spec.M):
        if m == 2:
            continue
        _gpu.check_close(y[m], ref[m], what=f"row {m}")


@pytest.mark.parametrize("bits,gs", [(1, 128), (2, 128), (4, 64)])
def test_small_m_row_magnitudes(bits, gs):
    """The small-M kernel sums unscaled codes times X in fp32 per group, so it is exact for
    |x| up to about 2^114; rows scaled by 2^100 and 2^-100, tiny and zero rows match the oracle
    row by row."""
    spec = spec_for(bits, gs, 9, 1024, 264, seed=41)
    prob = synth.make_problem(spec)
    x = _pins.x_as_f64(prob.x_bf16)
    x[0] *= 2.0 ** 100
    x[1] *= 2.0 ** -60
    x[2] = 0.0
    x[3] *= 2.0 ** -100
    x[4, 5] = 1.5 * 2.0 ** 104          # one huge entry in an otherwise ordinary row
    prob.x_bf16 = _pins.bf16_bits_from_f32(x.astype(np.float32))
    ref = oracle.gemm(prob.x_bf16, _gpu.oracle_packed(prob), prob.scales, prob.zeros, spec.N, bits, gs)
    xd, packed, s, z = _gpu.dev_problem(prob)
    y = _gpu.y_to_f64(lb.gemm(xd, packed, s, z, bits, gs, tile_tokens=1))
    torch.cuda.synchronize()
    assert np.all(y[2] == 0.0)
    for m in range(spec.M):
        if m == 2:
            continue
        _gpu.check_close(y[m:m + 1], ref[m:m + 1], what=f"row {m}")
