"""Comparison helpers for the GPU-vs-oracle parity tests.

Acceptance rules (the spec of this library):
  * packed codes and fp16 norms are bit-exact, except coordinates whose fp64
    z lies within 1e-6 of a decision threshold (and norms within 1e-6
    relative of an fp16 rounding midpoint), which are counted and reported;
  * attention outputs: per output row, max_j |o_j - r_j| / max_j |r_j|
    <= 2e-3 (fp32 accumulation against the fp64 oracle on the same codes).
"""
import numpy as np
import torch

import oracle

ATTN_TOL = 2e-3
BOUNDARY_BAND = 1e-6


def near_f16_midpoint(n, rel=BOUNDARY_BAND):
    n = np.asarray(n, dtype=np.float64)
    h = n.astype(np.float16).astype(np.float64)
    up = np.nextafter(h.astype(np.float16), np.float16(np.inf)).astype(np.float64)
    dn = np.nextafter(h.astype(np.float16), np.float16(-np.inf)).astype(np.float64)
    mids = np.stack([(h + up) / 2, (h + dn) / 2])
    return (np.abs(mids - n) <= rel * np.abs(n)).any(axis=0)


def compare_compressed(x64, signs, quats, gpu_codes, gpu_norms, bits=3):
    """Oracle-compress x64 [n][128] and compare with the GPU's canonical words.

    Returns a dict of counts; raises AssertionError on any non-exempt mismatch."""
    codes, norms, z, _ = oracle.compress(signs, quats, x64, want_z=True, bits=bits)
    gpu_codes = np.asarray(gpu_codes, dtype=np.uint32).reshape(codes.shape)
    gpu_norms = np.asarray(gpu_norms, dtype=np.uint16).reshape(norms.shape)
    near = oracle.near_boundary(z, BOUNDARY_BAND, bits=bits)
    stats = {"vectors": codes.shape[0], "coords": codes.shape[0] * 128, "near_boundary": int(near.sum())}
    word_diff = codes != gpu_codes
    if word_diff.any():
        oc = oracle.unpack(codes[word_diff.any(1)], bits=bits)
        gc = oracle.unpack(gpu_codes[word_diff.any(1)], bits=bits)
        bad = (oc != gc) & ~near[word_diff.any(1)]
        stats["code_mismatch"] = int((oc != gc).sum())
        assert not bad.any(), f"{int(bad.sum())} code mismatches outside the boundary band"
    else:
        stats["code_mismatch"] = 0
    n64 = np.linalg.norm(np.asarray(x64, dtype=np.float64), axis=1)
    nd = norms != gpu_norms
    stats["norm_mismatch"] = int(nd.sum())
    stats["norm_near_midpoint"] = int(near_f16_midpoint(n64).sum())
    assert not (nd & ~near_f16_midpoint(n64)).any(), "norm mismatch outside the midpoint band"
    stats["max_abs_z"] = float(np.abs(z).max()) if z.size else 0.0
    return stats, codes, norms


def rowwise_rel_err(got, ref):
    got = np.asarray(got, dtype=np.float64).reshape(-1, 128)
    ref = np.asarray(ref, dtype=np.float64).reshape(-1, 128)
    den = np.abs(ref).max(axis=1)
    num = np.abs(got - ref).max(axis=1)
    zero = den == 0
    err = np.where(zero, num, num / np.where(zero, 1.0, den))
    return err


def oracle_rows(state, b, h, q_cpu, limits_fn, ora, scale=None):
    """Oracle attention for all rows of KV head h of sequence b, on the
    oracle's own codes ``ora`` (from oracle_codes_for: compressed by the
    oracle from the same seeded K/V, never read back from the GPU path).

    q_cpu: [B][nq][Hq][128] (the queries fed to the GPU).
    Returns (out [R][128], list of (i, hq) per row)."""
    G, nq = state.G, q_cpu.shape[1]
    L = state.seq_lens[b]
    kc, kn, vc, vn = ora[:4]
    rows, idx, lims = [], [], []
    for i in range(nq):
        for g in range(G):
            hq = h * G + g
            rows.append(np.asarray(q_cpu[b, i, hq], dtype=np.float64))
            idx.append((i, hq))
            lims.append(limits_fn(L, i))
    out = oracle.attend(state.signs[h].numpy(), state.quats[h].numpy(), np.stack(rows), kc, kn, vc, vn,
                        np.array(lims), scale, bits=getattr(state, "bits", 3))
    return out, idx


def oracle_codes_for(state, b, h, t0, t1):
    """Oracle compression of sequence b, head h, tokens [t0, t1) from the
    same seeded inputs (raw K/V regenerated, never read from the GPU path)."""
    k, v = state.kv_tokens(b, t0, t1)
    k64 = k[:, h].to(torch.float64).cpu().numpy()
    v64 = v[:, h].to(torch.float64).cpu().numpy()
    s, q = state.signs[h].numpy(), state.quats[h].numpy()
    kc, kn, _, _ = oracle.compress(s, q, k64)
    vc, vn, _, _ = oracle.compress(s, q, v64)
    return kc, kn, vc, vn, k64, v64
