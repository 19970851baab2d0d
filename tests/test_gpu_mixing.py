"""GPU parity with the softmax weights spread over many tokens.

With the heavy-tailed synthetic keys (norms of a few hundred) and the default
scale 1/sqrt(128), nearly every row's softmax is one-hot, so the other parity
tests barely exercise the online-softmax rescaling, the merge of split
records (the log-sum-exp combine across CTAs), or the rescale of the
accumulators held in tensor memory.  Here the softmax scale is chosen per
workload so that the weights of a row really mix: a score standard deviation
of 2 is not enough with these keys (a few outlier keys dominate the spread),
so the scale is found by bisection on the oracle's fp64 scores until the
median row spreads its weight over a few hundred tokens, measured as the
effective token count exp(entropy); each test asserts that spread.

Kernels reached: the mma.sync split kernel at the full B = 16 x 32768
decode, the ragged 64K..128K long-context decode and the 2- and 4-bit
decode; the 64-row tcgen05 kernel on the verification workload; the
128-row tcgen05 kernel on a causal prefill.  Each compares every row of the
sampled (sequence, KV head) pairs with the oracle at 2e-3 (row-normwise).
Source: RotaryQuant, Abstract (attention directly on the packed codes).
"""
import numpy as np
import pytest
import torch

import oracle
from tests.parity import ATTN_TOL, compare_compressed, oracle_rows, rowwise_rel_err
from tests.test_gpu_parity import _ws, limits

pytestmark = pytest.mark.gpu
D = 128
TARGET_TOKENS = 300.0


def _pair_codes(st, b, h):
    """GPU codes of (b, h) checked against the oracle's; returns the
    oracle's own codes (never the GPU's) for the attention reference."""
    L = st.seq_lens[b]
    k, v = st.kv_tokens(b, 0, L)
    s, qt = st.signs[h].numpy(), st.quats[h].numpy()
    gkc, gkn = st.gather(b, h, 0, 0, L)
    gvc, gvn = st.gather(b, h, 1, 0, L)
    _, kc, kn = compare_compressed(k[:, h].double().cpu().numpy(), s, qt, gkc.numpy(), gkn.numpy(), bits=st.bits)
    _, vc, vn = compare_compressed(v[:, h].double().cpu().numpy(), s, qt, gvc.numpy(), gvn.numpy(), bits=st.bits)
    return kc, kn, vc, vn


def _scores(st, b, h, q_cpu, kc, kn):
    """fp64 scores q . k_hat (unscaled) of the rows of (b, h) over the
    oracle's dequantized, un-rotated keys; shape [rows][L], with the row
    limits applied as -inf."""
    khat = oracle.dequantize(st.signs[h].numpy(), st.quats[h].numpy(), kc, kn, bits=st.bits)
    lim = limits(st.wl)
    L = st.seq_lens[b]
    rows, lims = [], []
    for i in range(st.wl.nq):
        for g in range(st.G):
            rows.append(np.asarray(q_cpu[b, i, h * st.G + g], dtype=np.float64))
            lims.append(lim(L, i))
    s = np.stack(rows) @ khat.T
    for r, n in enumerate(lims):
        s[r, n:] = -np.inf
    return s


def _pick_scale(s, target=TARGET_TOKENS):
    """Softmax scale at which the median row of the score matrix `s` (rows
    of every sampled pair) spreads its weight over about `target` tokens
    (bisection in log scale; the effective token count falls as the scale
    grows)."""
    vis = s[np.isfinite(s)]
    lo, hi = 1e-3 / vis.std(), 1e3 / vis.std()
    for _ in range(40):
        mid = np.sqrt(lo * hi)
        if np.median(_effective_tokens(s, mid)) > target:
            lo = mid
        else:
            hi = mid
    return float(np.sqrt(lo * hi))


def _effective_tokens(s, scale):
    """exp(entropy) of each row's softmax (rows that see no token skipped)."""
    s = s[np.isfinite(s).any(axis=1)] * scale
    z = s - s.max(axis=1, keepdims=True)
    p = np.where(np.isfinite(z), np.exp(z), 0.0)
    p /= p.sum(axis=1, keepdims=True)
    ent = -(p * np.log(np.where(p > 0, p, 1.0))).sum(axis=1)
    return np.exp(ent)


def _run(csd, st, scale):
    q = st.queries(0)
    q_rot = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    csd.isoquant_rotate_q(st.ctx, q.reshape(-1, st.Hq, D), q_rot.view(-1, st.Hq, D))
    out = torch.full(q.shape, float("nan"), dtype=torch.float32, device="cuda")
    csd.isoquant_attend_decode(st.ctx, st.cache, q_rot, st.page_table, st.seq_lens_dev, _ws(csd, st), out,
                               causal=st.wl.causal, scale=scale)
    torch.cuda.synchronize()
    assert csd.isoquant_get_status(st.ctx) == 0
    return q.float().cpu(), out.cpu()


def _check_mixed(csd, st, pairs, min_tokens):
    """Pick the scale on the first pair, run the whole workload at it and
    compare every row of `pairs` with the oracle; assert that the weights
    really spread (median effective token count >= min_tokens)."""
    q_cpu = st.queries(0).float().cpu()
    codes = {p: _pair_codes(st, *p) for p in pairs}
    # one scale for the whole call, chosen on the rows of all sampled pairs
    # (pairs of different heads have different score scales); rows padded to
    # a common length with -inf
    mats = [_scores(st, b, h, q_cpu, codes[(b, h)][0], codes[(b, h)][1]) for (b, h) in pairs]
    width = max(m.shape[1] for m in mats)
    allrows = np.concatenate([np.pad(m, ((0, 0), (0, width - m.shape[1])), constant_values=-np.inf) for m in mats])
    scale = _pick_scale(allrows)
    q_cpu, out = _run(csd, st, scale)
    assert torch.isfinite(out).all()
    worst, eff_all = 0.0, []
    for (b, h) in pairs:
        kc, kn, vc, vn = codes[(b, h)]
        eff = _effective_tokens(_scores(st, b, h, q_cpu, kc, kn), scale)
        eff_all.append(eff)
        ref, idx = oracle_rows(st, b, h, q_cpu, limits(st.wl), (kc, kn, vc, vn), scale=scale)
        got = np.stack([out[b, i, hq].numpy() for (i, hq) in idx])
        err = rowwise_rel_err(got, ref)
        assert err.max() <= ATTN_TOL, f"b={b} h={h} max row rel err {err.max():.3e}"
        worst = max(worst, float(err.max()))
    eff = np.concatenate(eff_all)
    print(f"{st.wl.name} bits={st.bits}: scale {scale:.3e}, effective tokens per row median "
          f"{np.median(eff):.0f} (min {eff.min():.1f}), worst row rel err {worst:.2e}")
    assert np.median(eff) >= min_tokens, np.median(eff)
    return worst


def _state(name, bits=3):
    import compressed_space_decode_b200.synthetic as syn
    from compressed_space_decode_b200.workload import DecodeState
    return DecodeState(syn.workloads()[name], bits=bits)


@pytest.mark.parametrize("bits", [3, 2, 4])
def test_mixing_full_decode(cuda_lib, bits):
    """B = 16 x 32768 decode (mma.sync split kernel, ~5 records per row
    merged by the combine): two sampled sequences."""
    st = _state("gqa_b16_q32_kv4_L32768_paged", bits)
    pairs = [(3, 1), (12, 2)] if bits == 3 else [(7, 3)]
    _check_mixed(cuda_lib, st, pairs, min_tokens=50)


def test_mixing_long_ragged(cuda_lib):
    """B = 4, ragged 64K..128K contexts, 64 q / 8 KV heads: the shortest
    sequence, one KV head (its rows merge records of several CTAs)."""
    st = _state("long_b4_q64_kv8_L64k_128k_ragged")
    b = int(np.argmin(st.seq_lens))
    _check_mixed(cuda_lib, st, [(b, 5)], min_tokens=50)


def test_mixing_verify_tiles_kernel(cuda_lib):
    """Verification (nq = 16, causal, G = 4: 64 rows per KV head) on the
    64-row tcgen05 kernel, whose output rows are rescaled in tensor memory
    when a row maximum moves."""
    st = _state("verify_b8_nq16_q32_kv8_L16384")
    rows = st.wl.nq * st.G
    assert 64 <= rows < 128
    _check_mixed(cuda_lib, st, [(2, 6), (5, 1)], min_tokens=50)


def test_mixing_prefill_wide_kernel(cuda_lib):
    """Causal prefill of a 1536-token prompt (6144 rows per KV head) on the
    128-row tcgen05 kernel: every row of one KV head."""
    from compressed_space_decode_b200.synthetic import Workload
    from compressed_space_decode_b200.workload import DecodeState
    wl = Workload("prefill_mix_L1536", 1, 8, 2, [1536], nq=1536, page_size=64, causal=True, seed=91)
    st = DecodeState(wl)
    assert st.wl.nq * st.G >= 128
    # early query positions see few tokens: judge the spread on the rows that see 512 or more
    q_cpu = st.queries(0).float().cpu()
    codes = _pair_codes(st, 0, 1)
    scale = _pick_scale(_scores(st, 0, 1, q_cpu, codes[0], codes[1]))
    q_cpu, out = _run(cuda_lib, st, scale)
    assert torch.isfinite(out).all()
    kc, kn, vc, vn = codes
    s = _scores(st, 0, 1, q_cpu, kc, kn)
    eff = _effective_tokens(s[512 * st.G:], scale)
    ref, idx = oracle_rows(st, 0, 1, q_cpu, limits(st.wl), (kc, kn, vc, vn), scale=scale)
    got = np.stack([out[0, i, hq].numpy() for (i, hq) in idx])
    err = rowwise_rel_err(got, ref)
    print(f"prefill L=1536: scale {scale:.3e}, effective tokens median {np.median(eff):.0f}, "
          f"worst row rel err {err.max():.2e}")
    assert err.max() <= ATTN_TOL
    assert np.median(eff) >= 30
