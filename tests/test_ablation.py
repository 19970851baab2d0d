"""Isotropization ablation (RotaryQuant, Abstract): the WHT followed by
block-diagonal SO(4) rotations is claimed to isotropize KV vectors at
O(d log d) cost with 256 parameters per head, against 16,384 for a dense
rotation, before 3-bit scalar quantization.

On seeded heavy-tailed K vectors (Student-t(4) per channel, log-uniform
channel scales in [0.1, 10], 4 outlier channels x20: the workloads' recipe)
four rotations are compared, all in fp64 through the oracle:

  none     z = sqrt(128) x / |x|
  wht      signs + Walsh-Hadamard (identity quaternions: B = I)
  wht_so4  signs + Walsh-Hadamard + the 32 SO(4) blocks (the method)
  haar     a dense Haar-random 128 x 128 orthogonal matrix (seeded)

and, for each, the kurtosis and per-coordinate variance spread of z, the
relative reconstruction error E|x - x^|^2 / |x|^2 with 2-, 3- and 4-bit
Lloyd-Max codebooks for N(0, 1), and the attention output error of 64
query rows over 1024 tokens with V, or K and V, quantized to 3 bits, at a
softmax temperature that spreads the weight over many tokens (score
spread about 2; at the default 1/sqrt(128) these K norms make the softmax
one-hot and the error measures argmax flips only).  The table is printed;
the assertions are the claims the pages make or the mathematics implies.

What the numbers show (and the assertions check): the raw coordinates are
heavy-tailed (kurtosis ~39) with variances spanning >10^4; after the WHT
every coordinate has the same variance (all |H_jk| are equal), and with a
few dominant outlier channels the coordinates are no heavier-tailed than a
Gaussian, so the 3-bit error falls to or below the Gaussian Lloyd-Max
distortion and matches a dense Haar rotation's with 64x fewer parameters.
The GPU test checks that the library's codes give the same errors for the
two rotations it implements (identity quaternions = WHT only).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from compressed_space_decode_b200 import synthetic

D = 128
SEED = 4321
N_VEC = 4096


def _heavy_tailed(n, which=0, stream=0):
    sc = synthetic.channel_scales(SEED, which, 1)
    x = synthetic.heavy_tailed(SEED + which, stream, n, sc, dtype=torch.float32)
    return x[:, 0].double().numpy()


def _haar(seed):
    rng = np.random.default_rng(seed)
    q, r = np.linalg.qr(rng.standard_normal((D, D)))
    return q * np.sign(np.diag(r))[None, :]


def _rotations():
    signs, quats = synthetic.rotation_params(SEED, 1)
    s, qt = signs[0].numpy(), quats[0].numpy()
    ident = np.zeros((32, 2, 4), dtype=np.float32)
    ident[:, :, 0] = 1.0
    Q = _haar(SEED)
    return {
        "none": (lambda x: x, lambda y: y),
        "wht": (lambda x: oracle.rotate(s, ident, x), lambda y: oracle.unrotate(s, ident, y)),
        "wht_so4": (lambda x: oracle.rotate(s, qt, x), lambda y: oracle.unrotate(s, qt, y)),
        "haar": (lambda x: x @ Q.T, lambda y: y @ Q),
    }


def _codebooks():
    books = {}
    for bits in (2, 4):
        lv, th, dist, _ = oracle.lloyd_max(1 << bits)
        books[bits] = (lv, th, dist)
    lv3, th3 = oracle.codebook()  # the method's fp16-rounded 3-bit codebook
    books[3] = (lv3, th3, oracle.gauss_distortion(lv3, th3))
    return books


def _quantize(z, levels, thresholds):
    code = (z[..., None] > thresholds).sum(-1)
    return levels[code]


def _reconstruct(x, fwd, inv, levels, thresholds):
    n = np.linalg.norm(x, axis=1, keepdims=True)
    z = math.sqrt(D) * fwd(x) / n
    y_hat = _quantize(z, levels, thresholds) * n / math.sqrt(D)
    return inv(y_hat), z


def _attention(q, k, v, scale):
    s = scale * (q @ k.T)
    s -= s.max(axis=1, keepdims=True)
    p = np.exp(s)
    p /= p.sum(axis=1, keepdims=True)
    return p @ v


def _kurtosis(z):
    z = z.ravel()
    return float(np.mean(z ** 4) / np.mean(z ** 2) ** 2)


def ablation_table():
    x = _heavy_tailed(N_VEC)
    books = _codebooks()
    k = _heavy_tailed(1024, 0, 1)
    v = _heavy_tailed(1024, 1, 2)
    q = synthetic.gaussian(SEED, 7, (64, D), dtype=torch.float64).numpy()
    # temperature: scores of the unquantized K spread with standard deviation 2
    scale = 2.0 / float(np.std(q @ k.T))
    ref = _attention(q, k, v, scale)
    rows = {}
    for name, (fwd, inv) in _rotations().items():
        row = {}
        _, z = _reconstruct(x, fwd, inv, books[3][0], books[3][1])
        row["kurtosis"] = _kurtosis(z)
        var = z.var(axis=0)
        row["var_spread"] = float(var.max() / var.min())
        for bits, (lv, th, _) in books.items():
            xh, _ = _reconstruct(x, fwd, inv, lv, th)
            row[f"mse{bits}"] = float(np.mean(np.sum((x - xh) ** 2, 1) / np.sum(x ** 2, 1)))
        kh, _ = _reconstruct(k, fwd, inv, books[3][0], books[3][1])
        vh, _ = _reconstruct(v, fwd, inv, books[3][0], books[3][1])
        for key, (kk, vv) in (("attn_v", (k, vh)), ("attn_kv", (kh, vh))):
            out = _attention(q, kk, vv, scale)
            row[key] = float(np.mean(np.abs(out - ref).max(1) / np.abs(ref).max(1)))
        rows[name] = row
    return rows, {b: books[b][2] for b in books}


@pytest.fixture(scope="module")
def table():
    rows, dist = ablation_table()
    hdr = f"{'rotation':9s} {'kurt':>7s} {'varspr':>8s} {'mse2':>8s} {'mse3':>8s} {'mse4':>8s} {'attn V':>8s} {'attn KV':>8s}"
    print("\n" + hdr)
    for name, r in rows.items():
        print(f"{name:9s} {r['kurtosis']:7.3f} {r['var_spread']:8.2f} {r['mse2']:8.5f} {r['mse3']:8.5f} "
              f"{r['mse4']:8.5f} {r['attn_v']:8.4f} {r['attn_kv']:8.4f}")
    print("Lloyd-Max Gaussian distortion:", {b: round(d, 5) for b, d in dist.items()})
    return rows, dist


def test_rotation_isotropizes_heavy_tails(table):
    rows, _ = table
    # the raw vectors are far from isotropic: heavy tails, variances spanning >10^4
    assert rows["none"]["kurtosis"] > 10 and rows["none"]["var_spread"] > 1e3
    # the WHT gives every coordinate the same variance (|H_jk| = 1/sqrt(128)
    # for all j, k): the spread left is sampling noise; the SO(4) blocks mix
    # within 4 coordinates only, so it stays small
    assert rows["wht"]["var_spread"] < 1.3
    assert rows["wht_so4"]["var_spread"] < 4
    # tails: no heavier than a Gaussian's (kurtosis 3) after the WHT, as after
    # a dense Haar rotation
    for name in ("wht", "wht_so4", "haar"):
        assert rows[name]["kurtosis"] < 3.2, (name, rows[name]["kurtosis"])


def test_quantization_error_matches_gaussian_lloyd_max(table):
    rows, dist = table
    for bits in (2, 3, 4):
        m = rows["wht_so4"][f"mse{bits}"]
        # coordinates no heavier-tailed than N(0,1): at most the Lloyd-Max
        # distortion of the Gaussian the codebook was designed for
        assert m < 1.02 * dist[bits], (bits, m, dist[bits])
        # at least as good as a dense rotation with 64x the parameters
        assert m < 1.02 * rows["haar"][f"mse{bits}"], bits
        # and far better than quantizing the raw coordinates
        assert rows["none"][f"mse{bits}"] > 3 * m, bits
    assert rows["wht_so4"]["mse2"] > rows["wht_so4"]["mse3"] > rows["wht_so4"]["mse4"]


def test_attention_error_falls_with_rotation(table):
    rows, _ = table
    # quantized V alone: the output error falls several-fold with the
    # rotation (mean row-normwise error over the 64 query rows)
    assert rows["wht_so4"]["attn_v"] < 0.3 * rows["none"]["attn_v"]
    assert rows["wht_so4"]["attn_v"] < 1.2 * rows["haar"]["attn_v"]
    # quantized K too: 3-bit K moves these random-direction scores by ~0.2
    # of their spread whatever the rotation, so the error is O(1) for all;
    # the rotation does not make it worse
    assert rows["wht_so4"]["attn_kv"] < 1.05 * rows["none"]["attn_kv"]


def test_parameter_counts():
    # 32 blocks x (left, right) unit quaternions x 4 floats, against a dense
    # 128 x 128 rotation
    signs, quats = synthetic.rotation_params(SEED, 1)
    assert quats[0].numel() == 256 and D * D == 16384


@pytest.mark.gpu
def test_gpu_codes_reproduce_ablation(cuda_lib):
    """The library's codes (WHT only via identity quaternions, and WHT +
    SO(4)) are the oracle's, so their reconstruction errors agree with the
    oracle's compress + dequantize to rounding."""
    csd = cuda_lib
    x = _heavy_tailed(N_VEC)
    signs, quats = synthetic.rotation_params(SEED, 1)
    ident = torch.zeros_like(quats)
    ident[..., 0] = 1.0
    for qt in (ident, quats):
        ctx = csd.isoquant_init(signs, qt)
        cache = csd.PagedCache.allocate(1, N_VEC // 256, 256)
        xt = torch.from_numpy(x).float().reshape(N_VEC, 1, D).cuda()
        slots = torch.arange(N_VEC, dtype=torch.int64, device="cuda")
        csd.isoquant_compress_kv(ctx, cache, xt, xt, slots)
        torch.cuda.synchronize()
        # page layout [page][K/V][head][13][256] -> canonical [n][13]
        codes = cache.codes.view(N_VEC // 256, 2, 1, 13, 256)[:, 0, 0].permute(0, 2, 1).reshape(N_VEC, 13)
        norms = cache.norms.view(torch.int16).view(N_VEC // 256, 2, 1, 256)[:, 0, 0].reshape(N_VEC)
        gpu = oracle.dequantize(signs[0].numpy(), qt[0].numpy(), codes.cpu().numpy().view(np.uint32),
                                norms.cpu().numpy().view(np.uint16))
        oc, on, _, _ = oracle.compress(signs[0].numpy(), qt[0].numpy(), xt.cpu().numpy()[:, 0])
        ref = oracle.dequantize(signs[0].numpy(), qt[0].numpy(), oc, on)
        xf = xt.cpu().double().numpy()[:, 0]
        e_gpu = np.mean(np.sum((xf - gpu) ** 2, 1) / np.sum(xf ** 2, 1))
        e_ref = np.mean(np.sum((xf - ref) ** 2, 1) / np.sum(xf ** 2, 1))
        assert abs(e_gpu / e_ref - 1) < 1e-6, (e_gpu, e_ref)
        ctx.close()
