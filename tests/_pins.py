"""Pins for the CPU oracle: checks against facts that do not come from the oracle itself.

Each ``pin_*`` function takes an ``oracle.Oracle`` and raises AssertionError on a
mismatch. ``test_oracle_pins.py`` runs them against the real oracle;
``test_oracle_mutants.py`` runs them against deliberately broken copies of the oracle
to show that each plausible mistake is caught by at least one pin.

What pins what:
- scalar formats: torch's bf16 -> float and numpy's fp16 -> float64 conversions
  (library routines), over every bit pattern;
- packed layout: hand-derived golden words (tests/golden/pack_words.txt) and closed
  forms (all-zero / all-+1 words), plus the round trip;
- storage size: the model card's b_eff = 1 + 16/128 = 1.125 bits per weight and its
  14.2x reduction versus FP16 (bonsai-image-binary-4B-gemlite-1bit model card,
  "Binary Weight Representation: 1-bit g128");
- decode: closed forms (all +1 binary gives the group scales; ternary zeros give 0;
  4-bit with z = q gives 0), one-hot codes and one-hot scales (index mapping);
- GEMM: exact rational brute force (fractions), integer exactness, scaled group row
  sums, bit-flip negation, linearity, group permutation invariance, orientation, and
  a numpy float64 matmul reduction.
"""
from __future__ import annotations

import os
from fractions import Fraction

import numpy as np
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
GOLDEN = os.path.join(HERE, "golden")


# ---------------------------------------------------------------------------------------
# helpers (test-side; they use only numpy / torch library routines and the data)
# ---------------------------------------------------------------------------------------
def rng(seed):
    return np.random.default_rng(seed)


def f16(a):
    return np.asarray(a, dtype=np.float16)


def bf16_bits_from_f32(vals):
    """bf16 bit patterns of float32 values that are exactly representable in bf16."""
    t = torch.tensor(np.asarray(vals, dtype=np.float32)).to(torch.bfloat16)
    assert torch.equal(t.float(), torch.tensor(np.asarray(vals, dtype=np.float32))), "not bf16-exact"
    return t.view(torch.int16).numpy().view(np.uint16)


def small_int_x(M, K, seed, lo=-1, hi=1):
    return bf16_bits_from_f32(rng(seed).integers(lo, hi + 1, size=(M, K)).astype(np.float32))


def random_x(M, K, seed):
    v = rng(seed).standard_normal((M, K)).astype(np.float32)
    t = torch.tensor(v).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def x_as_f64(x_bits):
    return torch.tensor(x_bits.view(np.int16)).view(torch.bfloat16).double().numpy()


def random_codes(N, K, bits, seed):
    r = rng(seed)
    if bits == 1:
        return r.choice(np.array([-1, 1], dtype=np.int8), size=(N, K))
    if bits == 2:
        return r.choice(np.array([-1, 0, 1], dtype=np.int8), size=(N, K))
    return r.integers(0, 16, size=(N, K)).astype(np.int8)


def code_values(codes, bits):
    """The integer each code stands for (t or b; q for 4-bit), straight from the codes."""
    return codes.astype(np.int64)


def load_golden_pack():
    cases = []
    with open(os.path.join(GOLDEN, "pack_words.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            head, codes_s, words_s = [p.strip() for p in line.split("|")]
            bits, K, N = (int(v) for v in head.split())
            rows = [[int(v) for v in r.split()] for r in codes_s.split("/")]
            codes = np.array(rows, dtype=np.int8)
            assert codes.shape == (N, K), line
            words = np.array([int(w, 16) for w in words_s.split()], dtype=np.uint32)
            cases.append((bits, K, N, codes, words.reshape(N, K * bits // 32)))
    return cases


# ---------------------------------------------------------------------------------------
# scalar formats
# ---------------------------------------------------------------------------------------
def pin_bf16_widening(orc):
    pats = np.arange(0, 1 << 16, 97, dtype=np.uint32).astype(np.uint16)
    want = torch.tensor(pats.view(np.int16)).view(torch.bfloat16).double().numpy()
    got = np.array([orc.bf16_to_f64(int(p)) for p in pats])
    same = (got == want) | (np.isnan(got) & np.isnan(want))
    assert same.all(), f"bf16 widening differs at {pats[~same][:4]}"


def pin_f16_widening(orc):
    pats = np.arange(0, 1 << 16, 1, dtype=np.uint32).astype(np.uint16)
    want = pats.view(np.float16).astype(np.float64)
    got = np.array([orc.f16_to_f64(int(p)) for p in pats[::13]])
    w = want[::13]
    same = (got == w) | (np.isnan(got) & np.isnan(w))
    assert same.all(), f"fp16 widening differs at {pats[::13][~same][:4]}"


def pin_bf16_rounding(orc):
    vals = rng(5).standard_normal(2000).astype(np.float32) * np.float32(3.0)
    vals = np.concatenate([vals, np.float32([0.0, -0.0, 1.0, 1.00390625, 1.01171875, 3.0e-39, 1e38])])
    want = torch.tensor(vals).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([orc.f64_to_bf16(float(v)) for v in vals], dtype=np.uint16)
    assert np.array_equal(got, want), "bf16 rounding differs from torch"


# ---------------------------------------------------------------------------------------
# packing
# ---------------------------------------------------------------------------------------
def pin_pack_golden(orc):
    for bits, K, N, codes, words in load_golden_pack():
        got, bad = orc.pack(codes, bits)
        assert bad == 0
        assert np.array_equal(got, words), f"bits={bits} K={K}: {[hex(v) for v in got.ravel()]} != " \
                                           f"{[hex(v) for v in words.ravel()]}"
        back, bad = orc.unpack(words, N, K, bits)
        assert bad == 0 and np.array_equal(back, codes), f"unpack of golden words, bits={bits}"


def pin_pack_closed_forms(orc):
    for bits, code, word in ((2, 0, 0x55555555), (2, 1, 0xAAAAAAAA), (2, -1, 0), (1, 1, 0xFFFFFFFF),
                             (1, -1, 0), (4, 5, 0x55555555), (4, 15, 0xFFFFFFFF), (4, 10, 0xAAAAAAAA)):
        N, K = 3, 64 * 3
        got, bad = orc.pack(np.full((N, K), code, dtype=np.int8), bits)
        assert bad == 0 and (got == word).all(), f"bits={bits} code={code}"


def pin_pack_roundtrip(orc):
    for bits in (1, 2, 4):
        for (N, K) in ((1, 32), (7, 96), (33, 256), (64, 128)):
            c = random_codes(N, K, bits, seed=N * 1000 + K + bits)
            p, bad = orc.pack(c, bits)
            assert bad == 0 and p.shape == (N, K * bits // 32)
            back, bad = orc.unpack(p, N, K, bits)
            assert bad == 0 and np.array_equal(back, c), f"round trip bits={bits} N={N} K={K}"


def pin_pack_rejects_invalid(orc):
    for bits, badv in ((1, 0), (1, 2), (2, 2), (2, -2), (4, 16), (4, -1)):
        c = random_codes(4, 64, bits, seed=3)
        c[2, 17] = badv
        c[3, 63] = badv
        _, bad = orc.pack(c, bits)
        assert bad == 2, f"bits={bits} value {badv}: {bad} invalid codes reported"
    # ternary field 3 is not a code
    _, bad = orc.unpack(np.full((1, 2), 0xFFFFFFFF, dtype=np.uint32), 1, 32, 2)
    assert bad == 32


def pin_storage_size(orc):
    # binary g128: K*N one-bit codes + (K/128)*N fp16 scales -> 1 + 16/128 bits per weight
    N, K, g = 256, 1024, 128
    p, _ = orc.pack(np.ones((N, K), dtype=np.int8), 1)
    bits_total = p.nbytes * 8 + (K // g) * N * 16
    b_eff = bits_total / (N * K)
    assert b_eff == 1.125
    assert round(16 / b_eff, 1) == 14.2


# ---------------------------------------------------------------------------------------
# decode
# ---------------------------------------------------------------------------------------
def pin_decode_closed_forms(orc):
    N, K, g = 24, 256, 64
    G = K // g
    s = f16(rng(1).uniform(0.005, 0.02, (G, N)))
    s_full = np.repeat(s.astype(np.float64).T, g, axis=1)          # [N][K]
    for bits, code, factor in ((1, 1, 1.0), (1, -1, -1.0), (2, 1, 1.0), (2, -1, -1.0), (2, 0, 0.0)):
        p, _ = orc.pack(np.full((N, K), code, dtype=np.int8), bits)
        W = orc.decode(p, s, None, N, K, bits, g)
        assert np.array_equal(W, factor * s_full), f"bits={bits} code={code}"
    # 4-bit: z = q in every group gives 0; z = 0 gives q * s
    q = rng(2).integers(0, 16, size=(N, G)).astype(np.int8)
    codes = np.repeat(q, g, axis=1)
    p, _ = orc.pack(codes, 4)
    W = orc.decode(p, s, f16(q.T), N, K, 4, g)
    assert np.array_equal(W, np.zeros((N, K)))
    W = orc.decode(p, s, f16(np.zeros((G, N))), N, K, 4, g)
    assert np.array_equal(W, codes.astype(np.float64) * s_full)


def pin_decode_invalid_ternary_field(orc):
    # reading r2: ternary field 3 is not a code, so it must never decode to a finite weight; it
    # poisons exactly the weights it occupies (and the outputs that use them), nothing else
    N, K, g = 2, 64, 64
    p, _ = orc.pack(np.zeros((N, K), dtype=np.int8), 2)       # all fields 1 (t = 0)
    p[1, 1] = 0xFFFFFFFF                                        # row 1: one word of fields 3
    s = f16(np.full((1, N), 0.5))
    W = orc.decode(p, s, None, N, K, 2, g)
    bad = np.isnan(W)
    assert bad[1].sum() == 16 and not bad[0].any(), "exactly the 16 fields of the word are poisoned"
    assert np.array_equal(W[~bad], np.zeros(int((~bad).sum())))
    x = bf16_bits_from_f32(np.ones((1, K)))
    y = orc.gemm(x, p, s, None, N, 2, g)
    assert y[0, 0] == 0.0 and np.isnan(y[0, 1])


def pin_decode_one_hot(orc):
    N, K, g = 20, 128, 64
    G = K // g
    s = f16(rng(4).uniform(0.5, 2.0, (G, N)))
    for (n0, k0) in ((0, 0), (19, 127), (3, 64), (7, 1), (12, 33)):
        c = np.zeros((N, K), dtype=np.int8)
        c[n0, k0] = 1
        p, _ = orc.pack(c, 2)
        W = orc.decode(p, s, None, N, K, 2, g)
        want = np.zeros((N, K))
        want[n0, k0] = float(s[k0 // g, n0])
        assert np.array_equal(W, want), f"one-hot code at (n={n0}, k={k0})"
    # one-hot scale: every code +1, scale 1 except (group g0, row n0) = 2
    for (g0, n0) in ((0, 5), (1, 19), (1, 0)):
        sc = f16(np.ones((G, N)))
        sc[g0, n0] = 2.0
        p, _ = orc.pack(np.ones((N, K), dtype=np.int8), 2)
        W = orc.decode(p, sc, None, N, K, 2, g)
        want = np.ones((N, K))
        want[n0, g0 * g:(g0 + 1) * g] = 2.0
        assert np.array_equal(W, want), f"one-hot scale at (group={g0}, n={n0})"
    # 4-bit one-hot zero point
    q = np.full((N, K), 8, dtype=np.int8)
    p, _ = orc.pack(q, 4)
    z = f16(np.full((G, N), 8.0))
    z[1, 4] = 6.0
    W = orc.decode(p, f16(np.ones((G, N))), z, N, K, 4, g)
    want = np.zeros((N, K))
    want[4, g:2 * g] = 2.0
    assert np.array_equal(W, want), "one-hot zero point"


# ---------------------------------------------------------------------------------------
# GEMM
# ---------------------------------------------------------------------------------------
def _exact_dot(xrow, wrow):
    return sum((Fraction(float(a)) * Fraction(float(b)) for a, b in zip(xrow, wrow)), Fraction(0))


def pin_gemm_fraction_bruteforce(orc):
    """Exact rational sum on tiny shapes; the oracle's fp64 result must agree to ~1e-13."""
    for bits, K, g in ((1, 64, 32), (2, 64, 32), (4, 64, 32), (2, 128, 64)):
        M, N = 3, 3
        c = random_codes(N, K, bits, seed=K + bits)
        s = f16(rng(bits).uniform(0.005, 0.02, (K // g, N)))
        z = f16(rng(bits + 9).uniform(6, 9, (K // g, N))) if bits == 4 else None
        x = random_x(M, K, seed=bits * 7 + K)
        p, _ = orc.pack(c, bits)
        ref = orc.gemm(x, p, s, z, N, bits, g, threads=1)
        xf = x_as_f64(x)
        for m in range(M):
            for n in range(N):
                wrow = []
                for k in range(K):
                    sv = Fraction(float(s[k // g, n]))
                    if bits == 4:
                        wrow.append((Fraction(int(c[n, k])) - Fraction(float(z[k // g, n]))) * sv)
                    else:
                        wrow.append(Fraction(int(c[n, k])) * sv)
                exact = sum((Fraction(float(xf[m, k])) * wrow[k] for k in range(K)), Fraction(0))
                scale = sum(abs(Fraction(float(xf[m, k])) * wrow[k]) for k in range(K))
                err = abs(Fraction(ref[m, n]) - exact)
                assert err <= scale * Fraction(1, 10 ** 13), f"bits={bits} ({m},{n}): err {float(err)}"


def pin_gemm_integer_exact(orc):
    """Unit scales, integer zeros and x in {-1,0,1}: every value is an integer."""
    for bits in (1, 2, 4):
        M, N, K, g = 9, 13, 256, 64
        c = random_codes(N, K, bits, seed=40 + bits)
        s = f16(np.ones((K // g, N)))
        z = f16(np.full((K // g, N), 8.0)) if bits == 4 else None
        x = small_int_x(M, K, seed=bits)
        p, _ = orc.pack(c, bits)
        ref = orc.gemm(x, p, s, z, N, bits, g)
        wint = code_values(c, bits) - (8 if bits == 4 else 0)
        xint = x_as_f64(x).astype(np.int64)
        want = xint @ wint.T
        assert np.array_equal(ref, want.astype(np.float64)), f"bits={bits}"


def pin_gemm_group_row_sums(orc):
    """All +1 binary weights: y[m,n] = sum_g s[g,n] * sum_{k in g} x[m,k]."""
    M, N, K, g = 11, 17, 512, 128
    s = f16(rng(8).uniform(0.005, 0.02, (K // g, N)))
    x = random_x(M, K, seed=8)
    xf = x_as_f64(x)
    gsum = xf.reshape(M, K // g, g).sum(axis=2)            # [M][G]
    want = gsum @ s.astype(np.float64)                      # [M][N]
    for bits, code, sign in ((1, 1, 1.0), (1, -1, -1.0), (2, 1, 1.0)):
        p, _ = orc.pack(np.full((N, K), code, dtype=np.int8), bits)
        ref = orc.gemm(x, p, s, None, N, bits, g)
        assert np.allclose(ref, sign * want, rtol=1e-12, atol=1e-12), f"bits={bits} code={code}"


def pin_gemm_bitflip_negates(orc):
    M, N, K, g = 5, 40, 256, 128
    c = random_codes(N, K, 1, seed=12)
    s = f16(rng(12).uniform(0.005, 0.02, (K // g, N)))
    x = random_x(M, K, seed=12)
    p, _ = orc.pack(c, 1)
    a = orc.gemm(x, p, s, None, N, 1, g)
    b = orc.gemm(x, ~p, s, None, N, 1, g)
    assert np.array_equal(b, -a)


def pin_gemm_linearity(orc):
    M, N, K, g = 6, 21, 192, 64
    for bits in (2, 4):
        c = random_codes(N, K, bits, seed=20 + bits)
        s = f16(rng(21).uniform(0.005, 0.02, (K // g, N)))
        z = f16(rng(22).uniform(6, 9, (K // g, N))) if bits == 4 else None
        p, _ = orc.pack(c, bits)
        xa = x_as_f64(random_x(M, K, seed=23))
        mask = rng(24).random((M, K)) < 0.5
        x1 = np.where(mask, xa, 0.0)
        x2 = np.where(mask, 0.0, xa)
        to_bits = lambda v: bf16_bits_from_f32(v.astype(np.float32))
        y = orc.gemm(to_bits(xa), p, s, z, N, bits, g)
        y1 = orc.gemm(to_bits(x1), p, s, z, N, bits, g)
        y2 = orc.gemm(to_bits(x2), p, s, z, N, bits, g)
        y3 = orc.gemm(to_bits(2 * xa), p, s, z, N, bits, g)
        assert np.allclose(y, y1 + y2, rtol=1e-12, atol=1e-12)
        assert np.array_equal(y3, 2 * y)


def pin_gemm_group_permutation(orc):
    M, N, K, g = 4, 19, 256, 64
    G = K // g
    for bits in (1, 2, 4):
        c = random_codes(N, K, bits, seed=30 + bits)
        s = f16(rng(31).uniform(0.005, 0.02, (G, N)))
        z = f16(rng(32).uniform(6, 9, (G, N))) if bits == 4 else None
        x = random_x(M, K, seed=33)
        perm = np.array([2, 0, 3, 1])
        cols = np.concatenate([np.arange(gi * g, (gi + 1) * g) for gi in perm])
        p, _ = orc.pack(c, bits)
        pp, _ = orc.pack(np.ascontiguousarray(c[:, cols]), bits)
        y = orc.gemm(x, p, s, z, N, bits, g)
        yp = orc.gemm(np.ascontiguousarray(x[:, cols]), pp, f16(s[perm]), None if z is None else f16(z[perm]),
                      N, bits, g)
        assert np.allclose(y, yp, rtol=1e-12, atol=1e-12), f"bits={bits}"


def pin_gemm_orientation(orc):
    """Square K = N: one-hot weights pick one input column into one output column, and a
    non-symmetric W gives a different result from its transpose."""
    M, K, g = 7, 64, 32
    N = K
    s = f16(np.ones((K // g, N)))
    x = random_x(M, K, seed=40)
    xf = x_as_f64(x)
    for (n0, k0) in ((0, 63), (63, 0), (5, 40), (40, 5)):
        c = np.zeros((N, K), dtype=np.int8)
        c[n0, k0] = 1
        p, _ = orc.pack(c, 2)
        y = orc.gemm(x, p, s, None, N, 2, g)
        want = np.zeros((M, N))
        want[:, n0] = xf[:, k0]
        assert np.array_equal(y, want), f"one-hot (n={n0}, k={k0})"
    c = random_codes(N, K, 2, seed=41)
    assert not np.array_equal(c, c.T)
    p, _ = orc.pack(c, 2)
    pt, _ = orc.pack(np.ascontiguousarray(c.T), 2)
    y = orc.gemm(x, p, s, None, N, 2, g)
    yt = orc.gemm(x, pt, s, None, N, 2, g)
    assert not np.allclose(y, yt)
    assert np.allclose(y, xf @ c.T.astype(np.float64), rtol=1e-12, atol=1e-12)


def pin_gemm_matmul_reduction(orc):
    """Decoded weights times X via numpy's float64 matmul."""
    for bits, g in ((1, 128), (2, 64), (2, 128), (4, 64)):
        M, N, K = 37, 70, 512
        c = random_codes(N, K, bits, seed=50 + bits)
        s = f16(rng(51).uniform(0.005, 0.02, (K // g, N)))
        z = f16(rng(52).uniform(6, 9, (K // g, N))) if bits == 4 else None
        x = random_x(M, K, seed=53)
        p, _ = orc.pack(c, bits)
        W = orc.decode(p, s, z, N, K, bits, g)
        y = orc.gemm(x, p, s, z, N, bits, g)
        assert np.allclose(y, x_as_f64(x) @ W.T, rtol=1e-12, atol=1e-12), f"bits={bits}"
        # the sampled-entry path gives the same sums
        ms = np.array([0, 36, 5, 17])
        ns = np.array([69, 0, 33, 1])
        e = orc.gemm_entries(x, p, s, z, N, bits, g, ms, ns)
        assert np.array_equal(e, y[ms, ns])


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
