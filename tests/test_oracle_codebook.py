"""Pins for the oracle's codebook (CPU only).

The pages leave the quantizer open; the library fixes it as the 8-level
Lloyd-Max quantizer for N(0, 1/d), applied in z = sqrt(d) * u space, with the
levels rounded to fp16.  These tests pin the oracle's Lloyd iteration to the
published Max (1960) table, to its own optimality conditions evaluated with
scipy's adaptive quadrature, and its fp16 rounding to numpy's.
"""
import numpy as np
import pytest
from scipy import integrate, stats

import oracle
from tests.golden.loader import max1960


def test_levels_match_max_1960_table():
    lv, th, dist, it = oracle.lloyd_max(8)
    assert it > 0
    ref = max1960()
    pos_levels = lv[4:]
    for i in range(4):
        assert pos_levels[i] == pytest.approx(ref["level"][i + 1], abs=6e-4)
    pos_th = th[3:]
    for i in range(4):
        assert pos_th[i] == pytest.approx(ref["threshold"][i + 1], abs=6e-4)
    # the table prints four digits and truncates the last one (0.034548 ->
    # 0.03454), so allow one unit in the last printed place
    assert dist == pytest.approx(ref["mse"], abs=1.0e-5)


def test_symmetric_and_sorted():
    lv, th, _, _ = oracle.lloyd_max(8)
    assert np.all(np.diff(lv) > 0)
    np.testing.assert_allclose(lv, -lv[::-1], atol=1e-14)
    np.testing.assert_allclose(th, 0.5 * (lv[1:] + lv[:-1]), atol=0)


def test_fixed_point_by_quadrature():
    """Each level is the N(0,1) conditional mean of its cell (scipy quad)."""
    lv, th, dist, _ = oracle.lloyd_max(8)
    edges = np.concatenate([[-np.inf], th, [np.inf]])
    phi = stats.norm.pdf
    for i in range(8):
        a, b = edges[i], edges[i + 1]
        mass = integrate.quad(phi, a, b, epsabs=1e-14, epsrel=1e-13)[0]
        mom = integrate.quad(lambda z: z * phi(z), a, b, epsabs=1e-14, epsrel=1e-13)[0]
        assert mom / mass == pytest.approx(lv[i], abs=1e-9)
    d_quad = sum(integrate.quad(lambda z, c=lv[i]: (z - c) ** 2 * phi(z), edges[i], edges[i + 1],
                                epsabs=1e-14, epsrel=1e-13)[0] for i in range(8))
    assert dist == pytest.approx(d_quad, abs=1e-10)


def test_other_sizes_reduce_to_known_cases():
    # 2 levels: +-sqrt(2/pi), distortion 1 - 2/pi (closed form)
    lv, th, dist, _ = oracle.lloyd_max(2)
    assert lv[1] == pytest.approx(np.sqrt(2 / np.pi), abs=1e-12)
    assert dist == pytest.approx(1 - 2 / np.pi, abs=1e-12)
    # 4 levels: Max (1960) Table I, N = 4: levels 0.4528, 1.510; MSE 0.1175
    lv, th, dist, _ = oracle.lloyd_max(4)
    assert lv[2] == pytest.approx(0.4528, abs=6e-5)
    assert lv[3] == pytest.approx(1.510, abs=6e-4)
    assert dist == pytest.approx(0.1175, abs=6e-5)


def test_fp16_rounding_matches_numpy():
    rng = np.random.default_rng(7)
    vals = np.concatenate([
        np.clip(rng.standard_normal(3000) * 10.0 ** rng.uniform(-9, 5, 3000), -65500, 65500),
        [0.0, -0.0, 1.0, 65504.0, 65519.99, 2.0 ** -24, 2.0 ** -25, 3 * 2.0 ** -26,
         2.0 ** -14, 2.0 ** -14 * (1 - 2 ** -12), 1 + 2 ** -11, 1 + 3 * 2 ** -11, 2048 + 1.0],
    ])
    bits, sat = oracle.f64_to_f16_bits(vals)
    assert sat == 0
    ref = vals.astype(np.float16).view(np.uint16)
    np.testing.assert_array_equal(bits, ref)
    back = oracle.f16_bits_to_f64(bits)
    np.testing.assert_array_equal(back, ref.view(np.float16).astype(np.float64))


def test_fp16_saturates_instead_of_overflowing():
    bits, sat = oracle.f64_to_f16_bits([65520.0, 1e9])
    assert sat == 1 or sat == 2
    assert list(bits) == [0x7BFF, 0x7BFF]


def test_codebook_is_fp16_rounded_lloyd_max():
    lv, _, _, _ = oracle.lloyd_max(8)
    l16, t16 = oracle.codebook()
    np.testing.assert_array_equal(l16, lv.astype(np.float16).astype(np.float64))
    np.testing.assert_array_equal(t16, 0.5 * (l16[1:] + l16[:-1]))
    # midpoints of fp16 values are exact in fp32
    np.testing.assert_array_equal(t16.astype(np.float32).astype(np.float64), t16)
    # rounding the levels moves the distortion by far less than the 4th digit
    d16 = oracle.gauss_distortion(l16, t16)
    assert d16 == pytest.approx(max1960()["mse"], abs=1.0e-5)
    assert abs(d16 - oracle.lloyd_max(8)[2]) < 1e-6
