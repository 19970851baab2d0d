"""fp64 CPU oracle for IsoQuant compressed-space attention.

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py`` may import this package.  It shares
no code with the CUDA library: the arithmetic lives in ``isoquant_oracle.c``
(plain C, fp64), and this module only marshals numpy arrays.

Method source: "RotaryQuant: Fitting 120B MoE Models on Consumer Hardware
via Fused Compressed-Space Attention", Abstract.  The readings of what the
pages leave open are listed in ``isoquant_oracle.h``.

Every function below is pinned by ``tests/test_oracle_*.py`` against
closed forms, published tables, library routines or brute force.
"""
import ctypes
import os

import numpy as np

from . import build as _build

D = 128
BLOCKS = 32
WORDS = 13
LEVELS = 8
# other bit widths: words per vector (floor(32 / bits) codes per word)
WORDS_FOR = {2: 8, 3: 13, 4: 16}

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        dp = ctypes.POINTER(ctypes.c_double)
        L.orc_lloyd_max_gauss.restype = ctypes.c_int
        L.orc_lloyd_max_gauss.argtypes = [ctypes.c_int, dp, dp, dp]
        L.orc_gauss_distortion.restype = ctypes.c_double
        L.orc_gauss_distortion.argtypes = [ctypes.c_int, dp, dp]
        L.orc_f64_to_f16.restype = ctypes.c_uint16
        L.orc_f64_to_f16.argtypes = [ctypes.c_double, ctypes.POINTER(ctypes.c_int)]
        L.orc_f16_to_f64.restype = ctypes.c_double
        L.orc_f16_to_f64.argtypes = [ctypes.c_uint16]
        L.orc_hadamard_entry.restype = ctypes.c_int
        L.orc_hadamard_entry.argtypes = [ctypes.c_int, ctypes.c_int]
        L.orc_compress.restype = ctypes.c_int
        L.orc_compress_b.restype = ctypes.c_int
        L.orc_attend.restype = None
        L.orc_attend_bruteforce.restype = None
        L.orc_attend_b.restype = None
        L.orc_attend_bruteforce_b.restype = None
        L.orc_format.restype = ctypes.c_int
        _lib = L
    return _lib


def _p(a, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


# ------------------------------------------------------------------ codebook
def lloyd_max(nlev=LEVELS):
    """Lloyd-Max levels/thresholds/distortion for N(0,1) (fp64)."""
    lv = np.zeros(nlev)
    th = np.zeros(nlev - 1)
    dist = np.zeros(1)
    it = lib().orc_lloyd_max_gauss(nlev, _p(lv, ctypes.c_double), _p(th, ctypes.c_double),
                                   _p(dist, ctypes.c_double))
    return lv, th, float(dist[0]), it


def gauss_distortion(levels, thresholds):
    lv = _f64(levels)
    th = _f64(thresholds)
    return lib().orc_gauss_distortion(len(lv), _p(lv, ctypes.c_double), _p(th, ctypes.c_double))


def codebook(bits=3):
    """(levels16 [2^bits], thresholds [2^bits - 1]): fp16-rounded Lloyd-Max
    levels and midpoints (bits 3: the method's codebook; 2 and 4: the other
    widths)."""
    n = 1 << bits
    lv = np.zeros(n)
    th = np.zeros(n - 1)
    lib().orc_codebook_b(ctypes.c_int(bits), _p(lv, ctypes.c_double), _p(th, ctypes.c_double))
    return lv, th


def f64_to_f16_bits(x):
    """fp64 -> fp16 bits (RNE, saturating).  Returns (uint16 array, n_saturated)."""
    x = np.asarray(x, dtype=np.float64)
    out = np.zeros(x.shape, dtype=np.uint16)
    sat = ctypes.c_int(0)
    L = lib()
    flat = x.ravel()
    o = out.ravel()
    for i in range(flat.size):
        o[i] = L.orc_f64_to_f16(float(flat[i]), ctypes.byref(sat))
    return out, sat.value


def f16_bits_to_f64(h):
    h = np.asarray(h, dtype=np.uint16)
    L = lib()
    return np.array([L.orc_f16_to_f64(int(v)) for v in h.ravel()]).reshape(h.shape)


# ------------------------------------------------------------------ rotation
def hadamard_entry(i, j):
    return lib().orc_hadamard_entry(int(i), int(j))


def normalise_quats(raw):
    """raw float32 [32][2][4] -> unit quaternions fp64 [32][2][4]."""
    raw = np.ascontiguousarray(raw, dtype=np.float32)
    assert raw.shape == (BLOCKS, 2, 4)
    out = np.zeros((BLOCKS, 2, 4))
    lib().orc_normalise_quats(_p(raw, ctypes.c_float), _p(out, ctypes.c_double))
    return out


def qmul(a, b):
    a = _f64(a)
    b = _f64(b)
    out = np.zeros(4)
    lib().orc_qmul(_p(a, ctypes.c_double), _p(b, ctypes.c_double), _p(out, ctypes.c_double))
    return out


def _signs(signs):
    s = np.ascontiguousarray(signs, dtype=np.int8)
    assert s.shape == (D,)
    return s


def rotate(signs, quats_raw, x):
    """y = B Hn D x for each row of x [..., 128]."""
    s = _signs(signs)
    uq = normalise_quats(quats_raw)
    x = _f64(x)
    flat = x.reshape(-1, D)
    out = np.zeros_like(flat)
    L = lib()
    for r in range(flat.shape[0]):
        xr = np.ascontiguousarray(flat[r])
        yr = np.zeros(D)
        L.orc_rotate(_p(s, ctypes.c_int8), _p(uq, ctypes.c_double), _p(xr, ctypes.c_double),
                     _p(yr, ctypes.c_double))
        out[r] = yr
    return out.reshape(x.shape)


def unrotate(signs, quats_raw, y):
    """x = D Hn B^T y for each row."""
    s = _signs(signs)
    uq = normalise_quats(quats_raw)
    y = _f64(y)
    flat = y.reshape(-1, D)
    out = np.zeros_like(flat)
    L = lib()
    for r in range(flat.shape[0]):
        yr = np.ascontiguousarray(flat[r])
        xr = np.zeros(D)
        L.orc_unrotate(_p(s, ctypes.c_int8), _p(uq, ctypes.c_double), _p(yr, ctypes.c_double),
                       _p(xr, ctypes.c_double))
        out[r] = xr
    return out.reshape(y.shape)


# ------------------------------------------------------- quantize and pack
def compress(signs, quats_raw, x, want_z=False, bits=3):
    """Compress vectors x [n][128] (any float dtype, read as fp64).

    Returns codes uint32 [n][WORDS_FOR[bits]], norms uint16 [n] (fp16 bits),
    z [n][128] (or None) and the number of saturated norms.
    """
    s = _signs(signs)
    uq = normalise_quats(quats_raw)
    x = _f64(np.asarray(x, dtype=np.float64).reshape(-1, D))
    n = x.shape[0]
    codes = np.zeros((n, WORDS_FOR[bits]), dtype=np.uint32)
    norms = np.zeros(n, dtype=np.uint16)
    z = np.zeros((n, D)) if want_z else None
    sat = lib().orc_compress_b(ctypes.c_int(bits), ctypes.c_int(n), _p(x, ctypes.c_double), _p(s, ctypes.c_int8),
                               _p(uq, ctypes.c_double), _p(codes, ctypes.c_uint32),
                               _p(norms, ctypes.c_uint16),
                               _p(z, ctypes.c_double) if want_z else None)
    return codes, norms, z, sat


def unpack(words, bits=3):
    words = np.ascontiguousarray(words, dtype=np.uint32).reshape(-1, WORDS_FOR[bits])
    out = np.zeros((words.shape[0], D), dtype=np.uint8)
    L = lib()
    for r in range(words.shape[0]):
        w = np.ascontiguousarray(words[r])
        c = np.zeros(D, dtype=np.uint8)
        L.orc_unpack_b(ctypes.c_int(bits), _p(w, ctypes.c_uint32), _p(c, ctypes.c_uint8))
        out[r] = c
    return out


def dequantize(signs, quats_raw, words, norms, bits=3):
    s = _signs(signs)
    uq = normalise_quats(quats_raw)
    words = np.ascontiguousarray(words, dtype=np.uint32).reshape(-1, WORDS_FOR[bits])
    norms = np.ascontiguousarray(norms, dtype=np.uint16).reshape(-1)
    out = np.zeros((words.shape[0], D))
    L = lib()
    for r in range(words.shape[0]):
        w = np.ascontiguousarray(words[r])
        xr = np.zeros(D)
        L.orc_dequantize_b(ctypes.c_int(bits), _p(w, ctypes.c_uint32), ctypes.c_uint16(int(norms[r])),
                           _p(s, ctypes.c_int8), _p(uq, ctypes.c_double), _p(xr, ctypes.c_double))
        out[r] = xr
    return out


# ------------------------------------------------------------------ attention
def _attend_args(signs, quats_raw, q, kcodes, knorms, vcodes, vnorms, limits, bits=3):
    s = _signs(signs)
    uq = normalise_quats(quats_raw)
    q = _f64(np.asarray(q, dtype=np.float64).reshape(-1, D))
    kc = np.ascontiguousarray(kcodes, dtype=np.uint32).reshape(-1, WORDS_FOR[bits])
    vc = np.ascontiguousarray(vcodes, dtype=np.uint32).reshape(-1, WORDS_FOR[bits])
    kn = np.ascontiguousarray(knorms, dtype=np.uint16).reshape(-1)
    vn = np.ascontiguousarray(vnorms, dtype=np.uint16).reshape(-1)
    assert kc.shape[0] == vc.shape[0] == kn.shape[0] == vn.shape[0]
    lim = np.ascontiguousarray(limits, dtype=np.int32).reshape(-1)
    assert lim.shape[0] == q.shape[0]
    return s, uq, q, kc, kn, vc, vn, lim


def attend(signs, quats_raw, q, kcodes, knorms, vcodes, vnorms, limits, scale=None, brute=False, bits=3):
    """Attention of rows q [R][128] (un-rotated) over one KV head's packed cache.

    limits[r] = number of leading tokens row r sees.  scale defaults to
    1/sqrt(128).  Returns out [R][128] in the un-rotated space.
    """
    s, uq, q, kc, kn, vc, vn, lim = _attend_args(signs, quats_raw, q, kcodes, knorms, vcodes, vnorms,
                                                 limits, bits)
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    R, L = q.shape[0], kc.shape[0]
    out = np.zeros((R, D))
    fn = lib().orc_attend_bruteforce_b if brute else lib().orc_attend_b
    fn(ctypes.c_int(bits), ctypes.c_int(R), ctypes.c_int(L), _p(q, ctypes.c_double), _p(kc, ctypes.c_uint32),
       _p(kn, ctypes.c_uint16), _p(vc, ctypes.c_uint32), _p(vn, ctypes.c_uint16),
       _p(lim, ctypes.c_int32), ctypes.c_double(scale), _p(s, ctypes.c_int8),
       _p(uq, ctypes.c_double), _p(out, ctypes.c_double))
    return out


def near_boundary(z, band=1e-6, bits=3):
    """Mask of coordinates whose fp64 z lies within `band` of a threshold."""
    _, th = codebook(bits)
    z = np.asarray(z, dtype=np.float64)
    return (np.abs(z[..., None] - th) < band).any(axis=-1)
