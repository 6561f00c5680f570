"""GPU GEMM against the fp64 CPU oracle.

Bound per element: |gpu - ref| <= 1e-2 |ref| + 1e-2 rms(ref) (ref = oracle, fp64). Small and
ragged shapes are compared whole, and so are the full-size ternary QKV linear at a 512x512 image
and the text-encoder linears at 512 and 16 tokens. The 1024x1024 binary MLP linears and the
denoise-step chain are compared on sampled entries (4096 random ones plus 16 full rows and 16
full columns per shape), and the step's 80-linear batch call is sampled linear by linear as the
benchmark runs it.
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


@pytest.mark.parametrize("bits,gs", FORMATS)
@pytest.mark.parametrize("M", [1, 3, 8])
@pytest.mark.parametrize("K,N,rows,ksplit", [
    (256, 520, 0, 1),       # one step, half of it past K
    (768, 264, 0, 3),       # a request for 3 slices served with 2
    (2560, 1032, 0, 0),     # automatic choice
    (9728, 256, 0, 0),      # long K, few rows: split over a cluster
    (640, 136, 48, 0),      # 3 units of 16 rows, the last tile half past N
    (1152, 1000, 112, 2),   # the second slice holds one 128-wide group of K
    (1024, 2376, 16, 1),    # more row blocks than SMs: persistent tiles, no cluster
    (2048, 1352, 16, 2),    # persistent tiles with the cross-rank reduction on every tile
])
def test_gemm_small_m_weights_as_16_row_operand(bits, gs, M, K, N, rows, ksplit):
    """The small-M kernel with weights as the MMA's 16-row operand and at most 8 tokens as its n8
    operand (tile_tokens = 8, the automatic choice for M <= 8): ragged N and K, forced tilings."""
    if bits == 1 and K % 128:
        pytest.skip("binary needs K % 128 == 0")
    spec = spec_for(bits, gs, M, K, N, seed=M * 11 + K)
    prob = synth.make_problem(spec)
    ref = oracle.gemm(prob.x_bf16, _gpu.oracle_packed(prob), prob.scales, prob.zeros, N, bits, gs)
    x, packed, s, z = _gpu.dev_problem(prob)
    y = lb.gemm(x, packed, s, z, bits, gs, tile_tokens=8, tile_rows=rows, ksplit=ksplit)
    torch.cuda.synchronize()
    assert lb.device_status() == 0
    _gpu.check_close(_gpu.y_to_f64(y), ref, what=f"weights-as-A M={M} K={K} N={N} rows={rows} split={ksplit}")


@pytest.mark.parametrize("bits,gs", [(2, 128), (4, 64)])
def test_small_m_orientations_agree_and_auto_picks_weights_as_a(bits, gs):
    """At M <= 8 both orientations compute the same products; the automatic configuration is the
    weights-as-A kernel (bit-identical to tile_tokens = 8)."""
    spec = spec_for(bits, gs, 6, 3072, 1032, seed=81)
    prob = synth.make_problem(spec)
    ref = oracle.gemm(prob.x_bf16, _gpu.oracle_packed(prob), prob.scales, prob.zeros, spec.N, bits, gs)
    x, packed, s, z = _gpu.dev_problem(prob)
    y_auto = lb.gemm(x, packed, s, z, bits, gs)
    y8 = lb.gemm(x, packed, s, z, bits, gs, tile_tokens=8)
    y16 = lb.gemm(x, packed, s, z, bits, gs, tile_tokens=1)
    torch.cuda.synchronize()
    assert torch.equal(y_auto.view(torch.int16), y8.view(torch.int16))
    for y in (y8, y16):
        _gpu.check_close(_gpu.y_to_f64(y), ref, what="orientation")


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


def integer_problem(bits, M, K, N, g, seed, nonzeros=None):
    """Unit scales, integer zeros (8), codes with |w| <= 1 and x in {-1,0,1} with at most
    `nonzeros` (default K) nonzero entries per row: every product and partial sum is an integer
    and |y| <= 256, so the exact result is a bf16 value."""
    codes = _pins.random_codes(N, K, bits, seed=seed)
    if bits == 4:
        codes = np.random.default_rng(seed).integers(7, 10, size=(N, K)).astype(np.int8)
    x = _pins.x_as_f64(_pins.small_int_x(M, K, seed=seed))
    if nonzeros is not None:
        r = np.random.default_rng(seed + 1)
        for m in range(M):
            x[m, r.permutation(K)[nonzeros:]] = 0.0
    x = _pins.bf16_bits_from_f32(x.astype(np.float32))
    s = np.ones((K // g, N), dtype=np.float16)
    z = np.full((K // g, N), 8.0, dtype=np.float16) if bits == 4 else None
    return synth.Problem(spec_for(bits, g, M, K, N), x, codes, s, z)


@pytest.mark.parametrize("bits", [1, 2, 4])
def test_integer_exact(bits):
    """Unit scales, integer zeros, x in {-1,0,1}, |y| <= 256: bf16 output equals the oracle."""
    M, N, K, g = 70, 136, 256, 64
    prob = integer_problem(bits, M, K, N, g, seed=bits)
    ref = oracle.gemm(prob.x_bf16, _gpu.oracle_packed(prob), prob.scales, prob.zeros, N, bits, g)
    xd, packed, sd, zd = _gpu.dev_problem(prob)
    y = _gpu.y_to_f64(lb.gemm(xd, packed, sd, zd, bits, g))
    assert np.array_equal(y, ref)


@pytest.mark.parametrize("bits", [1, 2, 4])
@pytest.mark.parametrize("M,tile_tokens", [(1, 1), (5, 1), (16, 1), (1, 8), (5, 8), (8, 8)])
@pytest.mark.parametrize("K,nonzeros,ksplit", [(256, None, 1), (2048, 256, 2), (1024, 200, 0)])
def test_integer_exact_small_m(bits, M, tile_tokens, K, nonzeros, ksplit):
    """The small-M kernel on integer problems: it decodes codes without their scale (+-1, 128 + f,
    128 + q), sums one group at a time in fp32 and subtracts c * Sx, so every intermediate is an
    exact integer and the bf16 output must equal the oracle bit for bit -- also across the
    cluster's K split (ksplit 2) and the automatic tiling, in both orientations (X or the weights
    as the 16-row MMA operand)."""
    N, g = 264, 64
    if bits == 1 and K % 128:
        pytest.skip("binary needs K % 128 == 0")
    prob = integer_problem(bits, M, K, N, g, seed=10 * bits + M, nonzeros=nonzeros)
    ref = oracle.gemm(prob.x_bf16, _gpu.oracle_packed(prob), prob.scales, prob.zeros, N, bits, g)
    assert np.abs(ref).max() <= 256
    xd, packed, sd, zd = _gpu.dev_problem(prob)
    y = _gpu.y_to_f64(lb.gemm(xd, packed, sd, zd, bits, g, tile_tokens=tile_tokens, ksplit=ksplit))
    torch.cuda.synchronize()
    assert lb.device_status() == 0
    assert np.array_equal(y, ref)


@pytest.mark.parametrize("M,tile_tokens", [(96, 0), (300, 0), (16, 1), (16, 16), (5, 1), (5, 8)])
def test_uint4_codes_at_their_zero_point(M, tile_tokens):
    """uint4 codes equal or next to their group's zero point, with zero points that are not
    integers: each weight (q - z) * s is a small difference of two large terms. The
    tensor-memory kernel rounds every weight once to fp16 from its exact value (the small-M
    kernel sums exact codes and subtracts (128 + z) * s * Sx in fp32), so the outputs stay
    inside the tolerance although every |w| is far below |z * s|."""
    N, K, g = 264, 1024, 64
    r = np.random.default_rng(M + tile_tokens)
    q0 = r.integers(6, 10, size=(K // g, N))                           # per group
    dz = r.choice([-3, -2, -1, 1, 2, 3], size=(K // g, N)) / 128.0      # z = q0 + dz, fp16-exact
    z = (q0 + dz).astype(np.float16)
    assert np.array_equal(z.astype(np.float64), q0 + dz)
    step = r.choice([-1, 0, 0, 0, 1], size=(N, K))                      # codes mostly equal to q0
    codes = np.clip(np.repeat(q0.T, g, axis=1) + step, 0, 15).astype(np.int8)
    spec = spec_for(4, g, M, K, N, seed=77)
    prob = synth.make_problem(spec)
    prob = synth.Problem(spec, prob.x_bf16, codes, prob.scales, z)
    run_and_compare(spec, tile_tokens=tile_tokens, prob=prob)


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


FULL_WHOLE = [s for w in ("qkv_512sq_ternary_g128", "te_m512_uint4_g64", "te_m16_uint4_g64", "smallm_steady_m16_uint4_g64",
                           *(f"klein_linears_m{m}_{f}_g128" for f in ("ternary", "binary") for m in (1, 4, 16)))
              for s in synth.WORKLOADS[w]]
FULL_SAMPLED = synth.WORKLOADS["mlp_1024sq_binary_g128"]


@pytest.mark.parametrize("spec", FULL_WHOLE, ids=lambda s: s.name)
def test_full_size_whole(spec):
    """The ternary QKV linear at a 512x512 image (1536 x 3072 -> 9216), the uint4 text-encoder
    linears at 512 and 16 tokens and the transformer's ternary / binary linear shapes at 1, 4 and
    16 tokens, every output element against the oracle."""
    y, ref = run_and_compare(spec)
    worst = _gpu.check_close(_gpu.y_to_f64(y), ref, what=spec.name)
    print(f"\n{spec.name} M={spec.M} K={spec.K} N={spec.N}: max err/bound {worst:.3f} over all {ref.size}")


@pytest.mark.parametrize("spec", FULL_SAMPLED, ids=lambda s: s.name)
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
    worst = sampled_check(spec)
    print(f"\n{spec.name} M={spec.M} K={spec.K} N={spec.N}: max err/bound {worst:.3f}")


def sample_entries(M, N, r, n_random, n_rows, n_cols):
    """Random (m, n) entries plus every entry of a few full rows and full columns."""
    ms = [r.integers(0, M, n_random)]
    ns = [r.integers(0, N, n_random)]
    for m in r.choice(M, size=min(n_rows, M), replace=False):
        ms.append(np.full(N, m))
        ns.append(np.arange(N))
    for n in r.choice(N, size=min(n_cols, N), replace=False):
        ms.append(np.arange(M))
        ns.append(np.full(M, n))
    return np.concatenate(ms), np.concatenate(ns)


def test_chain_batch_as_run_sampled():
    """The headline call as the benchmark makes it: one lowbit_gemm_batch over the 80 linears of
    a denoise step at a 1024x1024 image (weights packed on the GPU, outputs pre-filled with NaN),
    then every linear's output sampled against the oracle (1024 random entries, 2 full rows and
    2 full columns each; each distinct shape is also checked more densely above)."""
    specs = synth.chain_linears()
    dev = []
    for sp in specs:
        x, packed, s, z = _gpu.dev_problem(synth.make_problem(sp))
        y = torch.full((sp.M, sp.N), float("nan"), dtype=torch.bfloat16, device="cuda")
        dev.append((x, packed, s, z, y))
    descs = [lb.make_desc(x, w, s, z, y, sp.bits, sp.group_size) for sp, (x, w, s, z, y) in zip(specs, dev)]
    lb.gemm_batch(descs)
    torch.cuda.synchronize()
    assert lb.device_status() == 0
    r = np.random.default_rng(80)
    worst = 0.0
    for sp, (_, _, _, _, y) in zip(specs, dev):
        prob = synth.make_problem(sp)
        ms, ns = sample_entries(sp.M, sp.N, r, 1024, 2, 2)
        got = y[torch.from_numpy(ms).cuda(), torch.from_numpy(ns).cuda()].float().cpu().numpy().astype(np.float64)
        ref = oracle.gemm_entries(prob.x_bf16, _gpu.oracle_packed(prob), prob.scales, prob.zeros, sp.N, sp.bits,
                                  sp.group_size, ms, ns)
        rms = float(np.sqrt(np.mean(ref * ref)))
        worst = max(worst, _gpu.check_close(got, ref, rms=rms, what=sp.name))
    print(f"\n80-linear batch: max err/bound {worst:.3f}")


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


def test_batch_reuses_x_copy_only_while_x_is_unchanged():
    """Q, K and V of one input in one batch: the X conversion runs once and every output matches
    its single call bit for bit. Then a linear whose output overwrites that X sits between two
    readers of it: the second reader must see the new contents (the copy is made again)."""
    M, K = 96, 512
    specs = [spec_for(2, 128, M, K, n, seed=60 + i) for i, n in enumerate((264, 136, 512))]
    probs = [synth.make_problem(sp) for sp in specs]
    x, _, _, _ = _gpu.dev_problem(probs[0])
    ws = [_gpu.dev_problem(p)[1:] for p in probs]
    outs = [torch.empty((M, sp.N), dtype=torch.bfloat16, device="cuda") for sp in specs]
    descs = [lb.make_desc(x, w, s, z, y, 2, 128) for (w, s, z), y in zip(ws, outs)]
    lb.gemm_batch(descs)
    singles = [lb.gemm(x, w, s, z, 2, 128) for (w, s, z) in ws]
    torch.cuda.synchronize()
    for sp, y1, y2 in zip(specs, outs, singles):
        assert torch.equal(y1.view(torch.int16), y2.view(torch.int16)), sp.name
    # reader, writer of X (K -> N = K, so its output has X's shape), reader again
    wspec = spec_for(2, 128, M, K, K, seed=70)
    wprob = synth.make_problem(wspec)
    x2, w2, s2, _ = _gpu.dev_problem(wprob)
    xa = x.clone()
    ya, yb = torch.empty_like(outs[0]), torch.empty_like(outs[0])
    (w0, s0, _) = ws[0]
    lb.gemm_batch([lb.make_desc(xa, w0, s0, None, ya, 2, 128), lb.make_desc(x2, w2, s2, None, xa, 2, 128),
                   lb.make_desc(xa, w0, s0, None, yb, 2, 128)])
    want_x = lb.gemm(x2, w2, s2, None, 2, 128)
    want_b = lb.gemm(want_x, w0, s0, None, 2, 128)
    torch.cuda.synchronize()
    assert torch.equal(ya.view(torch.int16), singles[0].view(torch.int16))
    assert torch.equal(xa.view(torch.int16), want_x.view(torch.int16))
    assert torch.equal(yb.view(torch.int16), want_b.view(torch.int16))


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
@pytest.mark.parametrize("M,tile_tokens", [(9, 1), (8, 8)])
def test_small_m_row_magnitudes(bits, gs, M, tile_tokens):
    """The small-M kernel sums unscaled codes times X in fp32 per group, so it is exact for
    |x| up to about 2^114; rows scaled by 2^100 and 2^-100, tiny and zero rows match the oracle
    row by row."""
    spec = spec_for(bits, gs, M, 1024, 264, seed=41)
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
    y = _gpu.y_to_f64(lb.gemm(xd, packed, s, z, bits, gs, tile_tokens=tile_tokens))
    torch.cuda.synchronize()
    assert np.all(y[2] == 0.0)
    for m in range(spec.M):
        if m == 2:
            continue
        _gpu.check_close(y[m:m + 1], ref[m:m + 1], what=f"row {m}")


def test_concurrent_host_threads_match_sequential_calls():
    """Four host threads, each with its own stream and workspace, run linears of every kernel
    path at once (the binding releases the GIL in the C calls): the library's host caches --
    tensor maps, cluster capacities, shared-memory opt-ins -- are shared by the threads, and every
    output equals the sequential call's bit for bit."""
    from concurrent.futures import ThreadPoolExecutor
    shapes = [(2, 128, 2304, 256, 2560), (4, 64, 16, 2560, 1032), (1, 128, 300, 1024, 520), (4, 64, 200, 768, 264),
              (2, 128, 5, 3072, 264), (2, 64, 40, 768, 264), (1, 64, 513, 512, 768), (4, 128, 1024, 512, 1024)]
    items = []
    for i, (b, g, m, k, n) in enumerate(shapes):
        sp = spec_for(b, g, m, k, n, seed=900 + i)
        items.append((sp, _gpu.dev_problem(synth.make_problem(sp))))
    want = [lb.gemm(x, w, s, z, sp.bits, sp.group_size) for sp, (x, w, s, z) in items]
    torch.cuda.synchronize()

    def worker(t):
        stream = torch.cuda.Stream()
        ws = torch.empty(max(lb.workspace_size(sp.M, sp.K) for sp, _ in items), dtype=torch.uint8, device="cuda")
        outs = []
        with torch.cuda.stream(stream):
            for r in range(3):
                for j in range(len(items)):
                    sp, (x, w, s, z) = items[(j + t) % len(items)]
                    outs.append(((j + t) % len(items), lb.gemm(x, w, s, z, sp.bits, sp.group_size, ws=ws)))
        stream.synchronize()
        return outs

    with ThreadPoolExecutor(4) as pool:
        results = list(pool.map(worker, range(4)))
    torch.cuda.synchronize()
    assert lb.device_status() == 0
    for outs in results:
        for j, y in outs:
            assert torch.equal(y.view(torch.int16), want[j].view(torch.int16)), items[j][0].name
