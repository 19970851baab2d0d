"""Pins for the oracle's norm, quantizer and packing (CPU only).

RotaryQuant, Abstract: "3-bit scalar quantization" of the isotropized
vectors into "packed 3-bit tensors".  The library fixes the open parts: an
fp16 L2 norm per vector, Lloyd-Max levels for N(0, 1/d), ten codes per
32-bit word.  Pinned by hand-worked packed words, the zero vector, and the
measured distortion against the distortion integrated under the exact
marginal of one coordinate of a uniformly random unit vector in R^128.
"""
import numpy as np
import pytest
from scipy import integrate
from scipy.special import gammaln

import oracle
from tests.golden.loader import packing

D = 128


def rand_params(seed):
    rng = np.random.default_rng(seed)
    return (rng.choice(np.array([-1, 1], dtype=np.int8), D),
            rng.standard_normal((32, 2, 4)).astype(np.float32))


def test_unpack_golden():
    g = packing()
    np.testing.assert_array_equal(oracle.unpack(np.array(g["all7"], dtype=np.uint32)), 7)
    np.testing.assert_array_equal(oracle.unpack(np.array(g["all1"], dtype=np.uint32)), 1)
    np.testing.assert_array_equal(oracle.unpack(np.array(g["all3"], dtype=np.uint32)), 3)
    words = np.zeros(13, dtype=np.uint32)
    words[:2] = g["mod8_w0_w1"]
    c = oracle.unpack(words)[0]
    np.testing.assert_array_equal(c[:20], np.arange(20) % 8)


def test_compress_zero_vector():
    signs, quats = rand_params(1)
    codes, norms, z, sat = oracle.compress(signs, quats, np.zeros((1, D)), want_z=True)
    assert norms[0] == 0 and sat == 0
    np.testing.assert_array_equal(codes[0], packing()["all3"])
    np.testing.assert_array_equal(z, 0.0)
    # and it dequantizes to exactly zero
    np.testing.assert_array_equal(oracle.dequantize(signs, quats, codes, norms), 0.0)


def test_compress_hand_worked_pattern():
    """z chosen cell by cell (norm sqrt(128)); packed words worked by hand."""
    signs, quats = rand_params(2)
    z = np.empty(D)
    z[:8] = [-2.0, -1.4, -0.75, -0.25, 0.25, 0.75, 1.4, 2.0]
    a = np.sqrt((D - np.sum(z[:8] ** 2)) / (D - 8))
    z[8::2] = a
    z[9::2] = -a
    assert np.sum(z ** 2) == pytest.approx(D)
    x = oracle.unrotate(signs, quats, z[None, :])   # so that R x = z and ||x|| = sqrt(128)
    codes, norms, zz, _ = oracle.compress(signs, quats, x, want_z=True)
    np.testing.assert_allclose(zz[0], z, atol=1e-12)
    np.testing.assert_array_equal(codes[0], packing()["pattern_a"])
    assert norms[0] == np.float16(np.sqrt(D)).view(np.uint16)


def test_codes_follow_threshold_rule_and_norms_round_to_nearest():
    signs, quats = rand_params(3)
    rng = np.random.default_rng(4)
    x = rng.standard_normal((300, D)) * np.exp(rng.uniform(-4, 4, (300, 1)))
    codes, norms, z, sat = oracle.compress(signs, quats, x, want_z=True)
    assert sat == 0
    _, th = oracle.codebook()
    expect = (z[..., None] > th).sum(-1)
    np.testing.assert_array_equal(oracle.unpack(codes), expect)
    # z is the rotated vector over its norm, times sqrt(128)
    y = oracle.rotate(signs, quats, x)
    np.testing.assert_allclose(z, np.sqrt(D) * y / np.linalg.norm(x, axis=1, keepdims=True), atol=1e-12)
    np.testing.assert_array_equal(norms, np.linalg.norm(x, axis=1).astype(np.float16).view(np.uint16))
    # the top 2 bits of every word and the top 8 bits of word 12 are zero
    assert np.all(codes[:, :12] >> 30 == 0) and np.all(codes[:, 12] >> 24 == 0)


def test_norm_saturation_is_counted():
    signs, quats = rand_params(5)
    x = np.zeros((2, D))
    x[0, 0] = 70000.0
    x[1, 0] = 1.0
    codes, norms, _, sat = oracle.compress(signs, quats, x)
    assert sat == 1
    assert norms[0] == 0x7BFF and norms[1] == np.float16(1.0).view(np.uint16)


def sphere_marginal_distortion(levels, thresholds, d=D):
    """E[(z - Q(z))^2] for z = sqrt(d) u_1, u uniform on the unit sphere:
    density proportional to (1 - z^2/d)^((d-3)/2) on |z| < sqrt(d)."""
    logc = gammaln(d / 2) - gammaln((d - 1) / 2) - 0.5 * np.log(np.pi * d)
    f = lambda z: np.exp(logc + (d - 3) / 2 * np.log1p(-z * z / d))
    r = np.sqrt(d)
    edges = np.concatenate([[-r], thresholds, [r]])
    mass = sum(integrate.quad(f, edges[i], edges[i + 1], epsabs=1e-14)[0] for i in range(8))
    assert mass == pytest.approx(1.0, abs=1e-10)
    return sum(integrate.quad(lambda z, c=levels[i]: (z - c) ** 2 * f(z), edges[i], edges[i + 1],
                              epsabs=1e-14, epsrel=1e-12)[0] for i in range(8))


def test_mse_matches_lloyd_max_distortion():
    """Gaussian input: E||x - x_hat||^2 / ||x||^2 ~ 0.0345 (Lloyd-Max D)."""
    signs, quats = rand_params(6)
    rng = np.random.default_rng(11)
    n = 30000
    x = rng.standard_normal((n, D))
    codes, norms, _, _ = oracle.compress(signs, quats, x)
    xh = oracle.dequantize(signs, quats, codes, norms)
    ratio = np.sum((x - xh) ** 2, axis=1) / np.sum(x * x, axis=1)
    mean, se = ratio.mean(), ratio.std(ddof=1) / np.sqrt(n)
    l16, t16 = oracle.codebook()
    d_sphere = sphere_marginal_distortion(l16, t16)
    assert abs(mean - d_sphere) < 3 * se + 1e-7, (mean, d_sphere, se)
    assert mean == pytest.approx(0.03454, rel=0.02)
