"""Pins for the oracle's other bit widths (CPU only).

RotaryQuant's KV path is 3-bit; its system quantizes weights at 2, 4 and 8
bits as well (Abstract).  The library offers 2 and 4 bits for K/V with the
same construction: 2^bits fp16-rounded Lloyd-Max levels for N(0,1),
midpoint thresholds, floor(32 / bits) codes per 32-bit word (16 and 8).
Pinned by Max (1960) Table I (the levels for N = 4 and N = 16), an
independent Lloyd iteration for the 16-level distortion, hand-worked packed
words,
the threshold rule, the measured distortion against the distortion under
the exact marginal of one coordinate of a uniform unit vector in R^128, and
compressed-space attention against brute force.
"""
import numpy as np
import pytest
from scipy.special import softmax

import oracle
from tests.test_oracle_quantize import rand_params, sphere_marginal_distortion

D = 128


def test_formats():
    assert oracle.WORDS_FOR == {2: 8, 3: 13, 4: 16}
    for bits, words in oracle.WORDS_FOR.items():
        lv, th = oracle.codebook(bits)
        assert lv.shape == (1 << bits,) and th.shape == ((1 << bits) - 1,)
        assert np.all(np.diff(lv) > 0) and np.allclose(lv, -lv[::-1])
        np.testing.assert_array_equal(th, 0.5 * (lv[:-1] + lv[1:]))


def test_codebooks_match_max_1960():
    # N = 4: levels +-0.4528, +-1.510 (four printed digits; fp16 rounding
    # moves them by < 5e-4)
    lv, _ = oracle.codebook(2)
    np.testing.assert_allclose(lv[2:], [0.4528, 1.510], atol=1e-3)
    # N = 16: the eight positive levels of the table (four printed digits)
    lv, _ = oracle.codebook(4)
    np.testing.assert_allclose(lv[8:], [0.1284, 0.3881, 0.6568, 0.9424, 1.256, 1.618, 2.069, 2.733], atol=1.5e-3)
    # and the distortion of the fp64 optimum against an independent Lloyd
    # iteration (scipy normal cdf/pdf for the cell centroids, quadrature for
    # the error)
    l64, t64, dist, _ = oracle.lloyd_max(16)
    assert dist == pytest.approx(independent_lloyd_distortion(16), abs=1e-12)
    # the 3-bit codebook is unchanged by the generalisation
    a, b = oracle.codebook()
    c, d = oracle.codebook(3)
    np.testing.assert_array_equal(a, c)
    np.testing.assert_array_equal(b, d)


def independent_lloyd_distortion(nlev, iters=4000):
    from scipy import integrate, stats
    lv = np.linspace(-2, 2, nlev)
    for _ in range(iters):
        e = np.concatenate([[-np.inf], 0.5 * (lv[:-1] + lv[1:]), [np.inf]])
        lv = np.array([(stats.norm.pdf(e[i]) - stats.norm.pdf(e[i + 1])) /
                       (stats.norm.cdf(e[i + 1]) - stats.norm.cdf(e[i])) for i in range(nlev)])
    e = np.concatenate([[-np.inf], 0.5 * (lv[:-1] + lv[1:]), [np.inf]])
    return sum(integrate.quad(lambda z, c=lv[i]: (z - c) ** 2 * stats.norm.pdf(z), e[i], e[i + 1],
                              epsabs=1e-15)[0] for i in range(nlev))


def test_unpack_hand_worked_words():
    # 2-bit: codes 0, 1, 2, 3 repeating -> every byte 0b11100100 = 0xE4
    w2 = np.full(8, 0xE4E4E4E4, dtype=np.uint32)
    np.testing.assert_array_equal(oracle.unpack(w2, bits=2)[0], np.arange(D) % 4)
    # 4-bit: codes 0..15 repeating -> words 0x76543210, 0xFEDCBA98
    w4 = np.tile(np.array([0x76543210, 0xFEDCBA98], dtype=np.uint32), 8)
    np.testing.assert_array_equal(oracle.unpack(w4, bits=4)[0], np.arange(D) % 16)
    # 2-bit: only coordinate 17 set to code 3 -> word 1, bits 2..3
    w = np.zeros(8, dtype=np.uint32)
    w[1] = 0xC
    c = oracle.unpack(w, bits=2)[0]
    assert c[17] == 3 and c.sum() == 3


@pytest.mark.parametrize("bits", [2, 4])
def test_codes_follow_threshold_rule(bits):
    signs, quats = rand_params(7 + bits)
    rng = np.random.default_rng(bits)
    x = rng.standard_normal((300, D)) * np.exp(rng.uniform(-3, 3, (300, 1)))
    codes, norms, z, sat = oracle.compress(signs, quats, x, want_z=True, bits=bits)
    assert codes.shape == (300, oracle.WORDS_FOR[bits]) and sat == 0
    _, th = oracle.codebook(bits)
    np.testing.assert_array_equal(oracle.unpack(codes, bits=bits), (z[..., None] > th).sum(-1))
    np.testing.assert_array_equal(norms, np.linalg.norm(x, axis=1).astype(np.float16).view(np.uint16))


@pytest.mark.parametrize("bits,published", [(2, 0.1175), (4, 0.009501)])
def test_mse_matches_lloyd_max_distortion(bits, published):
    signs, quats = rand_params(20 + bits)
    rng = np.random.default_rng(30 + bits)
    n = 20000
    x = rng.standard_normal((n, D))
    codes, norms, _, _ = oracle.compress(signs, quats, x, bits=bits)
    xh = oracle.dequantize(signs, quats, codes, norms, bits=bits)
    ratio = np.sum((x - xh) ** 2, axis=1) / np.sum(x * x, axis=1)
    mean, se = ratio.mean(), ratio.std(ddof=1) / np.sqrt(n)
    l16, t16 = oracle.codebook(bits)
    # the exact marginal integral over the 2^bits cells
    d_sphere = sphere_marginal_distortion_n(l16, t16)
    assert abs(mean - d_sphere) < 3 * se + 1e-7, (mean, d_sphere, se)
    assert mean == pytest.approx(published, rel=0.03)


def sphere_marginal_distortion_n(levels, thresholds, d=D):
    from scipy import integrate
    from scipy.special import gammaln
    logc = gammaln(d / 2) - gammaln((d - 1) / 2) - 0.5 * np.log(np.pi * d)
    f = lambda z: np.exp(logc + (d - 3) / 2 * np.log1p(-z * z / d))
    r = np.sqrt(d)
    edges = np.concatenate([[-r], thresholds, [r]])
    n = len(levels)
    mass = sum(integrate.quad(f, edges[i], edges[i + 1], epsabs=1e-14)[0] for i in range(n))
    assert mass == pytest.approx(1.0, abs=1e-10)
    return sum(integrate.quad(lambda z, c=levels[i]: (z - c) ** 2 * f(z), edges[i], edges[i + 1],
                              epsabs=1e-14, epsrel=1e-12)[0] for i in range(n))


@pytest.mark.parametrize("bits", [2, 4])
def test_attention_equals_bruteforce(bits):
    rng = np.random.default_rng(40 + bits)
    signs, quats = rand_params(50 + bits)
    L, R = 40, 5
    scale_c = np.exp(rng.uniform(np.log(0.1), np.log(10), D))
    k = rng.standard_normal((L, D)) * scale_c
    v = rng.standard_normal((L, D)) * scale_c
    q = rng.standard_normal((R, D))
    kc, kn, _, _ = oracle.compress(signs, quats, k, bits=bits)
    vc, vn, _, _ = oracle.compress(signs, quats, v, bits=bits)
    limits = np.array([L, 1, 0, 17, L])
    for scale in (1 / np.sqrt(D), 0.02):
        got = oracle.attend(signs, quats, q, kc, kn, vc, vn, limits, scale, bits=bits)
        brute = oracle.attend(signs, quats, q, kc, kn, vc, vn, limits, scale, brute=True, bits=bits)
        kx = oracle.dequantize(signs, quats, kc, kn, bits=bits)
        vx = oracle.dequantize(signs, quats, vc, vn, bits=bits)
        ref = np.zeros((R, D))
        for r in range(R):
            if limits[r]:
                ref[r] = softmax(scale * (kx[:limits[r]] @ q[r])) @ vx[:limits[r]]
        den = np.abs(ref).max()
        assert np.abs(got - ref).max() <= 1e-12 * den
        assert np.abs(brute - ref).max() <= 1e-12 * den
        assert not got[2].any()
