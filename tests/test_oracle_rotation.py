"""Pins for the oracle's rotation R = B * Hn * D (CPU only).

RotaryQuant, Abstract: a Walsh-Hadamard transform followed by block-diagonal
SO(4) rotations, 256 stored parameters per head versus 16,384 for a dense
rotation.  Checked against scipy's Hadamard matrix and scipy's quaternion
rotation, the quaternion algebra's defining relations, orthogonality,
determinant and the round trip.
"""
import numpy as np
import pytest
from scipy.linalg import hadamard
from scipy.spatial.transform import Rotation

import oracle

D = 128
IDENT = np.tile(np.array([1.0, 0, 0, 0], dtype=np.float32), (32, 2, 1))
PLUS = np.ones(D, dtype=np.int8)


def rand_params(seed):
    rng = np.random.default_rng(seed)
    signs = rng.choice(np.array([-1, 1], dtype=np.int8), D)
    quats = rng.standard_normal((32, 2, 4)).astype(np.float32)
    return signs, quats


def rotation_matrix(signs, quats, inverse=False):
    eye = np.eye(D)
    fn = oracle.unrotate if inverse else oracle.rotate
    return fn(signs, quats, eye).T  # column k = image of e_k


def test_quaternion_relations():
    one, i, j, k = np.eye(4)
    np.testing.assert_array_equal(oracle.qmul(i, i), -one)
    np.testing.assert_array_equal(oracle.qmul(j, j), -one)
    np.testing.assert_array_equal(oracle.qmul(k, k), -one)
    np.testing.assert_array_equal(oracle.qmul(oracle.qmul(i, j), k), -one)
    np.testing.assert_array_equal(oracle.qmul(i, j), k)
    np.testing.assert_array_equal(oracle.qmul(j, k), i)
    np.testing.assert_array_equal(oracle.qmul(k, i), j)
    rng = np.random.default_rng(0)
    a, b, c = rng.standard_normal((3, 4))
    np.testing.assert_allclose(oracle.qmul(oracle.qmul(a, b), c), oracle.qmul(a, oracle.qmul(b, c)),
                               atol=1e-14)
    assert np.linalg.norm(oracle.qmul(a, b)) == pytest.approx(np.linalg.norm(a) * np.linalg.norm(b),
                                                              rel=1e-14)


def test_hadamard_matches_scipy():
    H = hadamard(D)
    for i in range(0, D, 7):
        for j in range(D):
            assert oracle.hadamard_entry(i, j) == H[i, j]
    # identity blocks and + signs: R = H / sqrt(128)
    R = rotation_matrix(PLUS, IDENT)
    np.testing.assert_allclose(R, H / np.sqrt(D), atol=1e-15)


def test_signs_come_first():
    signs, _ = rand_params(1)
    R = rotation_matrix(signs, IDENT)
    np.testing.assert_allclose(R, (hadamard(D) / np.sqrt(D)) @ np.diag(signs.astype(float)), atol=1e-15)


def block_of(quats, b):
    """4x4 matrix of block b, read off R (H_n^-1 = H_n, + signs)."""
    Hn = hadamard(D) / np.sqrt(D)
    B = rotation_matrix(PLUS, quats) @ Hn  # = B
    return B[4 * b:4 * b + 4, 4 * b:4 * b + 4], B


def test_conjugation_block_is_scipy_rotation():
    rng = np.random.default_rng(3)
    quats = np.zeros((32, 2, 4), dtype=np.float32)
    for b in range(32):
        q = rng.standard_normal(4)
        q /= np.linalg.norm(q)
        quats[b, 0] = q
        quats[b, 1] = q
    uq = oracle.normalise_quats(quats)
    for b in (0, 5, 31):
        M, _ = block_of(quats, b)
        w, x, y, z = uq[b, 0]
        R3 = Rotation.from_quat([x, y, z, w]).as_matrix()
        assert M[0, 0] == pytest.approx(1.0, abs=1e-13)
        np.testing.assert_allclose(M[0, 1:], 0, atol=1e-13)
        np.testing.assert_allclose(M[1:, 0], 0, atol=1e-13)
        np.testing.assert_allclose(M[1:, 1:], R3, atol=1e-13)


def test_left_and_right_factors():
    rng = np.random.default_rng(4)
    quats = np.tile(np.array([1.0, 0, 0, 0], dtype=np.float32), (32, 2, 1))
    a = rng.standard_normal(4).astype(np.float32)
    c = rng.standard_normal(4).astype(np.float32)
    quats[2, 0] = a          # block 2: v -> a v
    quats[3, 1] = c          # block 3: v -> v conj(c)
    uq = oracle.normalise_quats(quats)
    M2, B = block_of(quats, 2)
    M3, _ = block_of(quats, 3)
    # image of the real unit 1 is a itself, resp. conj(c)
    np.testing.assert_allclose(M2[:, 0], uq[2, 0], atol=1e-14)
    cc = uq[3, 1] * np.array([1, -1, -1, -1])
    np.testing.assert_allclose(M3[:, 0], cc, atol=1e-14)
    # left multiplication is isoclinic: <M v, v> = a_w |v|^2 for every v
    v = rng.standard_normal(4)
    assert v @ M2 @ v == pytest.approx(uq[2, 0, 0] * (v @ v), rel=1e-12)
    # block-diagonal: nothing leaks between blocks
    off = B.copy()
    for b in range(32):
        off[4 * b:4 * b + 4, 4 * b:4 * b + 4] = 0
    assert np.abs(off).max() < 1e-13


def test_block_composition_homomorphism():
    """block(a1,c1) block(a2,c2) = block(a1 a2, c1 c2)."""
    rng = np.random.default_rng(5)
    q1 = rng.standard_normal((32, 2, 4))
    q2 = rng.standard_normal((32, 2, 4))
    q1 /= np.linalg.norm(q1, axis=-1, keepdims=True)
    q2 /= np.linalg.norm(q2, axis=-1, keepdims=True)
    q12 = np.zeros((32, 2, 4))
    for b in range(32):
        for s in range(2):
            q12[b, s] = oracle.qmul(q1[b, s], q2[b, s])
    for b in (0, 17):
        M1, _ = block_of(q1.astype(np.float32), b)
        M2, _ = block_of(q2.astype(np.float32), b)
        M12, _ = block_of(q12.astype(np.float32), b)
        np.testing.assert_allclose(M1 @ M2, M12, atol=2e-7)  # float32 parameter rounding


def test_orthogonal_det_plus_one():
    signs, quats = rand_params(6)
    R = rotation_matrix(signs, quats)
    assert np.abs(R.T @ R - np.eye(D)).max() < 1e-14
    Hn = hadamard(D) / np.sqrt(D)
    sgn, logdet = np.linalg.slogdet(Hn)
    assert sgn == 1.0 and abs(logdet) < 1e-10
    _, B = block_of(quats, 0)
    for b in range(32):
        M = B[4 * b:4 * b + 4, 4 * b:4 * b + 4]
        assert np.abs(M.T @ M - np.eye(4)).max() < 1e-14
        assert np.linalg.det(M) == pytest.approx(1.0, abs=1e-14)
    Rinv = rotation_matrix(signs, quats, inverse=True)
    assert np.abs(Rinv @ R - np.eye(D)).max() < 1e-14


def test_round_trip_and_dot_invariance():
    signs, quats = rand_params(8)
    rng = np.random.default_rng(9)
    x = rng.standard_normal((20, D)) * np.exp(rng.uniform(-3, 3, (20, 1)))
    y = oracle.rotate(signs, quats, x)
    back = oracle.unrotate(signs, quats, y)
    assert np.abs(back - x).max() / np.abs(x).max() < 1e-12
    q = rng.standard_normal((20, D))
    k = rng.standard_normal((20, D)) * 30
    dq = np.einsum("ij,ij->i", oracle.rotate(signs, quats, q), oracle.rotate(signs, quats, k))
    d0 = np.einsum("ij,ij->i", q, k)
    assert np.abs(dq - d0).max() / np.abs(np.linalg.norm(q, axis=1) * np.linalg.norm(k, axis=1)).max() < 1e-12


def test_parameter_count():
    """256 stored parameters per head versus 16,384 for a dense 128x128 rotation."""
    _, quats = rand_params(10)
    assert quats.size == 256
    assert D * D == 16384
    # the sign vector is 128 bits, not parameters in the count; the
    # transform only needs O(d log d) work: 7 butterfly stages of d adds
    # plus 32 4x4 products = 896 + 512 operations versus d^2 = 16,384
    assert 7 * D + 32 * 16 < D * D // 10
