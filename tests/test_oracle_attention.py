"""Pins for the oracle's compressed-space attention (CPU only).

RotaryQuant, Abstract: attention "directly on packed 3-bit tensors without
materializing full-precision KV state".  Because R is orthogonal, attention
computed in the rotated space on the codes must equal ordinary softmax
attention over the explicitly dequantized, un-rotated K/V with the
un-rotated query.  Checked on tiny inputs against a plain numpy/scipy
softmax attention and against closed-form special cases.
"""
import numpy as np
import pytest
from scipy.special import softmax

import oracle

D = 128


def setup(seed, L, R, heavy=True):
    rng = np.random.default_rng(seed)
    signs = rng.choice(np.array([-1, 1], dtype=np.int8), D)
    quats = rng.standard_normal((32, 2, 4)).astype(np.float32)
    scale = np.exp(rng.uniform(np.log(0.1), np.log(10), D)) if heavy else np.ones(D)
    k = rng.standard_normal((L, D)) * scale
    v = rng.standard_normal((L, D)) * scale
    q = rng.standard_normal((R, D))
    kc, kn, _, _ = oracle.compress(signs, quats, k)
    vc, vn, _, _ = oracle.compress(signs, quats, v)
    return signs, quats, q, kc, kn, vc, vn


def reference(signs, quats, q, kc, kn, vc, vn, limits, scale):
    kx = oracle.dequantize(signs, quats, kc, kn)
    vx = oracle.dequantize(signs, quats, vc, vn)
    out = np.zeros((q.shape[0], D))
    for r in range(q.shape[0]):
        lim = limits[r]
        if lim == 0:
            continue
        p = softmax(scale * (kx[:lim] @ q[r]))
        out[r] = p @ vx[:lim]
    return out


@pytest.mark.parametrize("L,R,seed", [(1, 1, 0), (17, 3, 1), (64, 4, 2), (50, 8, 3)])
def test_compressed_space_equals_bruteforce(L, R, seed):
    signs, quats, q, kc, kn, vc, vn = setup(seed, L, R)
    rng = np.random.default_rng(100 + seed)
    limits = rng.integers(0, L + 1, R)
    limits[0] = L
    for scale in (1 / np.sqrt(D), 0.02):
        got = oracle.attend(signs, quats, q, kc, kn, vc, vn, limits, scale)
        brute = oracle.attend(signs, quats, q, kc, kn, vc, vn, limits, scale, brute=True)
        ref = reference(signs, quats, q, kc, kn, vc, vn, limits, scale)
        denom = np.abs(ref).max()
        assert np.abs(got - ref).max() <= 1e-12 * denom
        assert np.abs(brute - ref).max() <= 1e-12 * denom


def test_causal_rows_and_empty_rows():
    signs, quats, q, kc, kn, vc, vn = setup(4, 40, 4)
    limits = np.array([40 - 3, 40 - 2, 40 - 1, 40])  # causal within a 4-query chunk
    got = oracle.attend(signs, quats, q, kc, kn, vc, vn, limits)
    ref = reference(signs, quats, q, kc, kn, vc, vn, limits, 1 / np.sqrt(D))
    np.testing.assert_allclose(got, ref, atol=1e-12 * np.abs(ref).max())
    got0 = oracle.attend(signs, quats, q[:1], kc, kn, vc, vn, [0])
    np.testing.assert_array_equal(got0, 0.0)


def test_single_token_returns_its_value():
    signs, quats, q, kc, kn, vc, vn = setup(5, 1, 2)
    got = oracle.attend(signs, quats, q, kc, kn, vc, vn, [1, 1])
    vx = oracle.dequantize(signs, quats, vc, vn)
    np.testing.assert_allclose(got, np.repeat(vx, 2, axis=0), atol=1e-13 * np.abs(vx).max())


def test_identical_keys_give_mean_of_values():
    signs, quats, q, kc, kn, vc, vn = setup(6, 12, 2)
    kc = np.repeat(kc[:1], 12, axis=0)
    kn = np.repeat(kn[:1], 12)
    got = oracle.attend(signs, quats, q, kc, kn, vc, vn, [12, 12])
    vx = oracle.dequantize(signs, quats, vc, vn)
    np.testing.assert_allclose(got, np.tile(vx.mean(0), (2, 1)), atol=1e-13 * np.abs(vx).max())


def test_large_scale_picks_argmax_key():
    signs, quats, q, kc, kn, vc, vn = setup(7, 30, 1, heavy=False)
    kx = oracle.dequantize(signs, quats, kc, kn)
    best = int(np.argmax(kx @ q[0]))
    got = oracle.attend(signs, quats, q, kc, kn, vc, vn, [30], scale=1e4)
    vx = oracle.dequantize(signs, quats, vc, vn)
    np.testing.assert_allclose(got[0], vx[best], atol=1e-9 * np.abs(vx).max())
