"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Bit-exact packed codes and fp16 norms (coordinates within 1e-6 of a decision
threshold counted and exempt), and attention outputs within 2e-3 normwise
per row, on every workload at sizes the oracle finishes in seconds, plus
full-size runs checked on sampled (sequence, KV head) pairs.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from tests.parity import ATTN_TOL, compare_compressed, oracle_rows, rowwise_rel_err

pytestmark = pytest.mark.gpu

D = 128


def _ws(csd, st):
    # NaN-filled so that reading a record nobody wrote shows up as NaN
    return csd.alloc_workspace(st.ctx, st.B, st.wl.nq, st.Hq, page_size=st.ps).fill_(0x7FC00000)


def run_attend(csd, st, step=0, scale=0.0, q=None):
    wl = st.wl
    nq = wl.nq
    if q is None:
        q = st.queries(step)
    q_rot = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    csd.isoquant_rotate_q(st.ctx, q.reshape(st.B * nq, st.Hq, D), q_rot.view(st.B * nq, st.Hq, D))
    out = torch.full(q.shape, float("nan"), dtype=torch.float32, device="cuda")
    ws = _ws(csd, st)
    csd.isoquant_attend_decode(st.ctx, st.cache, q_rot, st.page_table, st.seq_lens_dev, ws, out,
                               causal=wl.causal, scale=scale)
    torch.cuda.synchronize()
    assert csd.isoquant_get_status(st.ctx) == 0
    return q.float().cpu(), q_rot.cpu(), out.cpu()


def limits(wl):
    if wl.causal:
        return lambda L, i: max(L - wl.nq + i + 1, 0)
    return lambda L, i: L


def check_pair(st, b, h, q_cpu, out, scale=None, report=None):
    L = st.seq_lens[b]
    k, v = st.kv_tokens(b, 0, L) if L > 0 else (None, None)
    s, qt = st.signs[h].numpy(), st.quats[h].numpy()
    if L > 0:
        gkc, gkn = st.gather(b, h, 0, 0, L)
        gvc, gvn = st.gather(b, h, 1, 0, L)
        k64 = k[:, h].to(torch.float64).cpu().numpy()
        v64 = v[:, h].to(torch.float64).cpu().numpy()
        ks, kc, kn = compare_compressed(k64, s, qt, gkc.numpy(), gkn.numpy())
        vs, vc, vn = compare_compressed(v64, s, qt, gvc.numpy(), gvn.numpy())
        if report is not None:
            report.append((b, h, ks, vs))
    else:
        kc = vc = np.zeros((0, 13), np.uint32)
        kn = vn = np.zeros(0, np.uint16)
    ref, idx = oracle_rows(st, b, h, q_cpu, limits(st.wl), (kc, kn, vc, vn), scale=scale)
    got = np.stack([out[b, i, hq].numpy() for (i, hq) in idx])
    err = rowwise_rel_err(got, ref)
    assert np.isfinite(got).all()
    assert err.max() <= ATTN_TOL, f"b={b} h={h} max row rel err {err.max():.3e}"
    return err.max()


SMALL = ["single_head_d128_L1024", "gqa_b1_q32_kv8_L4096", "gqa_b16_q32_kv4_L32768_paged",
         "long_b4_q64_kv8_L64k_128k_ragged", "verify_b8_nq16_q32_kv8_L16384"]


@pytest.mark.parametrize("name", SMALL)
def test_attend_small(cuda_lib, name):
    from compressed_space_decode_b200.workload import DecodeState
    wl = cuda_lib.synthetic.workloads(small=True)[name]
    st = DecodeState(wl)
    q, _, out = run_attend(cuda_lib, st)
    rng = np.random.default_rng(0)
    pairs = [(b, h) for b in range(st.B) for h in range(st.H)]
    if len(pairs) > 6:
        pairs = [pairs[i] for i in rng.choice(len(pairs), 6, replace=False)]
    worst = max(check_pair(st, b, h, q, out) for b, h in pairs)
    print(f"{name}: worst row rel err {worst:.2e}")


def test_compress_bit_exact_all_dtypes(cuda_lib):
    """Heavy-tailed, Gaussian, zero, tiny and huge vectors; fp32/bf16/fp16 inputs."""
    from compressed_space_decode_b200 import synthetic
    H, n = 2, 3000
    signs, quats = synthetic.rotation_params(77, H)
    ctx = cuda_lib.isoquant_init(signs, quats)
    cache = cuda_lib.PagedCache.allocate(H, (n + 255) // 256, 256)
    sc = synthetic.channel_scales(78, 0, H)
    base = synthetic.heavy_tailed(79, 0, n, sc, device="cuda", dtype=torch.float32)
    base[:200] = synthetic.gaussian(80, 0, (200, H, D), device="cuda")
    base[200] = 0.0
    base[201] = 1e-3 * base[202]
    base[203, :, 5] = 70000.0  # saturating norm
    for dtype in (torch.float32, torch.bfloat16, torch.float16):
        x = base.to(dtype)
        if dtype == torch.float16:
            x = torch.nan_to_num(x, posinf=60000.0, neginf=-60000.0).clamp(-60000, 60000)
        slots = torch.arange(n, dtype=torch.int64, device="cuda")
        cuda_lib.isoquant_compress_kv(ctx, cache, x, x.flip(0).contiguous(), slots)
        torch.cuda.synchronize()
        assert cuda_lib.isoquant_get_status(ctx) == 0
        for h in range(H):
            codes = cache.codes[:, 0, h].permute(0, 2, 1).reshape(-1, 13)[:n]
            norms = cache.norms[:, 0, h].reshape(-1)[:n]
            gc = codes.cpu().numpy().view(np.uint32)
            gn = norms.cpu().numpy().view(np.uint16)
            x64 = x[:, h].to(torch.float64).cpu().numpy()
            stats, _, _ = compare_compressed(x64, signs[h].numpy(), quats[h].numpy(), gc, gn)
            print(dtype, h, stats)


def test_compress_norms_at_fp16_midpoints(cuda_lib):
    """Vectors scaled so that their norm sits on an fp16 rounding midpoint
    (and a few fp32 units either side of it), across binades from 2^-13 to
    2^15: the fp16 norm must still round as the oracle's fp64 norm does, so
    these must take the re-check path where the fp32 norm cannot decide."""
    from compressed_space_decode_b200 import synthetic
    H, n = 1, 768
    signs, quats = synthetic.rotation_params(81, H)
    ctx = cuda_lib.isoquant_init(signs, quats)
    cache = cuda_lib.PagedCache.allocate(H, (n + 255) // 256, 256)
    rng = np.random.default_rng(82)
    v = rng.standard_normal((n, D))
    v /= np.linalg.norm(v, axis=1, keepdims=True)
    # midpoint between two adjacent fp16 values of binade 2^e, nudged by k fp64 steps of 2^-24 relative
    e = rng.integers(-13, 15, n)
    m = rng.integers(0, 1023, n)
    mid = (1.0 + (m + 0.5) / 1024.0) * np.exp2(e)
    k = rng.integers(-12, 13, n)
    target = mid * (1.0 + k * 2.0 ** -24)
    x = torch.tensor((v * target[:, None])[:, None, :], dtype=torch.float32, device="cuda")
    slots = torch.arange(n, dtype=torch.int64, device="cuda")
    cuda_lib.isoquant_compress_kv(ctx, cache, x, x, slots)
    torch.cuda.synchronize()
    assert cuda_lib.isoquant_get_status(ctx) == 0
    codes = cache.codes[:, 0, 0].permute(0, 2, 1).reshape(-1, 13)[:n]
    norms = cache.norms[:, 0, 0].reshape(-1)[:n]
    gc = codes.cpu().numpy().view(np.uint32)
    gn = norms.cpu().numpy().view(np.uint16)
    stats, _, _ = compare_compressed(x[:, 0].double().cpu().numpy(), signs[0].numpy(), quats[0].numpy(), gc, gn)
    print(stats)
    # the exemption band of compare_compressed is not needed: the re-check
    # decides every one of them as the fp64 norm does
    assert stats["norm_near_midpoint"] > n // 4 and stats["norm_mismatch"] == 0, stats


def test_compress_slot_rules(cuda_lib):
    from compressed_space_decode_b200 import synthetic
    H = 1
    signs, quats = synthetic.rotation_params(5, H)
    ctx = cuda_lib.isoquant_init(signs, quats)
    cache = cuda_lib.PagedCache.allocate(H, 2, 32)
    cache.codes.fill_(-1)
    x = synthetic.gaussian(6, 0, (3, H, D), device="cuda")
    slots = torch.tensor([-1, 5, 64], dtype=torch.int64, device="cuda")  # skip, write, out of range
    cuda_lib.isoquant_compress_kv(ctx, cache, x, x, slots)
    torch.cuda.synchronize()
    st = cuda_lib.isoquant_get_status(ctx)
    assert st & cuda_lib.DEVERR_SLOT_RANGE
    written = (cache.codes[0, 0, 0, :, :] != -1).any(dim=0).cpu()
    assert written.tolist() == [i == 5 for i in range(32)]
    assert cuda_lib.isoquant_get_status(ctx) == 0  # cleared by the read


def test_rotate_q_matches_oracle(cuda_lib):
    from compressed_space_decode_b200 import synthetic
    H, Hq = 4, 16
    signs, quats = synthetic.rotation_params(11, H)
    ctx = cuda_lib.isoquant_init(signs, quats)
    q = synthetic.gaussian(12, 0, (5, Hq, D), device="cuda") * 7.0
    out = torch.empty_like(q)
    cuda_lib.isoquant_rotate_q(ctx, q, out)
    torch.cuda.synchronize()
    qc, oc = q.double().cpu().numpy(), out.double().cpu().numpy()
    for hq in range(Hq):
        h = hq // (Hq // H)
        ref = oracle.rotate(signs[h].numpy(), quats[h].numpy(), qc[:, hq])
        err = np.abs(oc[:, hq] - ref).max() / np.abs(ref).max()
        assert err < 2e-6, (hq, err)


@pytest.mark.parametrize("ps", [32, 64, 128, 256])
def test_attend_edge_lengths(cuda_lib, ps):
    """Empty, single-token, ragged, page-multiple and split-boundary lengths."""
    from compressed_space_decode_b200.synthetic import Workload
    from compressed_space_decode_b200.workload import DecodeState
    lens = [0, 1, 31, 32, 33, ps - 1, ps, ps + 1, 3 * ps + 17, 700]
    wl = Workload(f"edge_ps{ps}", len(lens), 8, 2, lens, page_size=ps, seed=4242)
    st = DecodeState(wl)
    q, _, out = run_attend(cuda_lib, st)
    for b in range(len(lens)):
        for h in range(2):
            if lens[b] == 0:
                assert torch.all(out[b] == 0)
                continue
            check_pair(st, b, h, q, out)


def test_attend_mixing_softmax(cuda_lib):
    """Scale chosen so the score spread is O(1): many tokens share the weight."""
    from compressed_space_decode_b200.workload import DecodeState
    wl = cuda_lib.synthetic.workloads(small=True)["gqa_b1_q32_kv8_L4096"]
    st = DecodeState(wl)
    # the heavy-tailed keys have norms of a few hundred: a scale of 1e-3
    # brings the scores to a spread of about 2
    q, _, out = run_attend(cuda_lib, st, scale=1e-3)
    for h in range(st.H):
        check_pair(st, 0, h, q, out, scale=1e-3)


def test_append_steps_then_attend(cuda_lib):
    """Decode steps: append one token per sequence via compress_kv, attend."""
    from compressed_space_decode_b200.workload import DecodeState
    wl = cuda_lib.synthetic.workloads(small=True)["gqa_b16_q32_kv4_L32768_paged"]
    st = DecodeState(wl, growth=40)
    for step in range(40):
        k = torch.stack([st.kv_tokens(b, st.seq_lens[b], st.seq_lens[b] + 1)[0][0] for b in range(st.B)])
        v = torch.stack([st.kv_tokens(b, st.seq_lens[b], st.seq_lens[b] + 1)[1][0] for b in range(st.B)])
        slots = torch.cat([st.slots(b, st.seq_lens[b], st.seq_lens[b] + 1) for b in range(st.B)])
        cuda_lib.isoquant_compress_kv(st.ctx, st.cache, k.contiguous(), v.contiguous(), slots)
        st.seq_lens = [L + 1 for L in st.seq_lens]
        st.seq_lens_dev += 1
        q, _, out = run_attend(cuda_lib, st, step=step)
    for b, h in [(0, 0), (7, 3), (15, 1)]:
        check_pair(st, b, h, q, out)


def test_attend_allocates_nothing(cuda_lib):
    from compressed_space_decode_b200.workload import DecodeState
    wl = cuda_lib.synthetic.workloads(small=True)["gqa_b1_q32_kv8_L4096"]
    st = DecodeState(wl)
    q = st.queries(0)
    q_rot = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    out = torch.empty_like(q_rot)
    ws = _ws(cuda_lib, st)
    torch.cuda.synchronize()
    before = torch.cuda.memory_allocated()
    cuda_lib.isoquant_rotate_q(st.ctx, q.reshape(-1, st.Hq, D), q_rot.view(-1, st.Hq, D))
    cuda_lib.isoquant_attend_decode(st.ctx, st.cache, q_rot, st.page_table, st.seq_lens_dev, ws, out)
    torch.cuda.synchronize()
    assert torch.cuda.memory_allocated() == before
    # the workspace holds partial (m, l, o) records only: far smaller than the
    # fp16 K/V this cache stands for (no full-precision KV is materialised)
    assert ws.numel() * 4 < sum(st.seq_lens) * st.H * 2 * D * 2


@pytest.mark.parametrize("name,pairs", [
    ("gqa_b1_q32_kv8_L4096", "all"),
    ("gqa_b16_q32_kv4_L32768_paged", 2),
    ("long_b4_q64_kv8_L64k_128k_ragged", 1),
    ("verify_b8_nq16_q32_kv8_L16384", 2),
])
def test_attend_full_size_sampled(cuda_lib, name, pairs):
    from compressed_space_decode_b200.workload import DecodeState
    wl = cuda_lib.synthetic.workloads()[name]
    st = DecodeState(wl)
    q, _, out = run_attend(cuda_lib, st)
    assert torch.isfinite(out).all()
    allp = [(b, h) for b in range(st.B) for h in range(st.H)]
    rng = np.random.default_rng(1)
    sel = allp if pairs == "all" else [allp[i] for i in rng.choice(len(allp), pairs, replace=False)]
    if name.startswith("long"):
        b_short = int(np.argmin(st.seq_lens))
        sel = [(b_short, int(rng.integers(st.H)))]
    for b, h in sel:
        check_pair(st, b, h, q, out)


def _split_attend(csd, st, q_rot, scale=0.0):
    """Records (isoquant_attend_partial), then merge and inverse rotation
    (isoquant_attend_combine), as two calls."""
    out = torch.full(q_rot.shape, float("nan"), dtype=torch.float32, device="cuda")
    ws = _ws(csd, st)
    csd.isoquant_attend_partial(st.ctx, st.cache, q_rot, st.page_table, st.seq_lens_dev, ws,
                                causal=st.wl.causal, scale=scale)
    csd.isoquant_attend_combine(st.ctx, st.B, st.wl.nq, st.Hq, st.seq_lens_dev, st.ps, ws, out)
    torch.cuda.synchronize()
    assert csd.isoquant_get_status(st.ctx) == 0
    return out.cpu()


@pytest.mark.parametrize("name", ["edge_ps64", "gqa_b16_q32_kv4_L32768_paged", "verify_b8_nq16_q32_kv8_L16384"])
def test_decode_equals_partial_then_combine(cuda_lib, name):
    """isoquant_attend_decode is the partial and combine halves back to back:
    the two routes agree exactly, zero rows of empty sequences included,
    and match the oracle."""
    from compressed_space_decode_b200.synthetic import Workload
    from compressed_space_decode_b200.workload import DecodeState
    if name == "edge_ps64":
        # few pages in all: fewer pages than CTAs, empty sequences between
        lens = [0, 1, 63, 64, 0, 65, 209, 700, 0]
        wl = Workload(name, len(lens), 8, 2, lens, page_size=64, seed=77)
    else:
        wl = cuda_lib.synthetic.workloads(small=True)[name]
    st = DecodeState(wl)
    q, q_rot_cpu, whole = run_attend(cuda_lib, st)
    halves = _split_attend(cuda_lib, st, q_rot_cpu.cuda())
    assert torch.isfinite(whole).all()
    assert torch.equal(whole, halves)
    for b in range(st.B):
        if st.seq_lens[b] == 0:
            assert torch.all(whole[b] == 0)
    b = max(range(st.B), key=lambda i: st.seq_lens[i])
    check_pair(st, b, st.H - 1, q, whole)


def test_decode_step_graph_replay(cuda_lib):
    """rotate_q + attend_decode captured once in a CUDA graph (the kernels
    are programmatic dependent launches, so the graph holds programmatic
    edges) and replayed on new queries gives the eager result bit for bit."""
    from compressed_space_decode_b200.workload import DecodeState
    csd = cuda_lib
    wl = csd.synthetic.workloads(small=True)["gqa_b1_q32_kv8_L4096"]
    st = DecodeState(wl)
    q_in = st.queries(0).reshape(st.B * wl.nq, st.Hq, D).contiguous()
    q_rot = torch.empty((st.B, wl.nq, st.Hq, D), dtype=torch.float32, device="cuda")
    out = torch.empty_like(q_rot)
    ws = _ws(csd, st)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        csd.isoquant_rotate_q(st.ctx, q_in, q_rot.view(-1, st.Hq, D), stream=s)
        csd.isoquant_attend_decode(st.ctx, st.cache, q_rot, st.page_table, st.seq_lens_dev, ws, out, stream=s)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        csd.isoquant_rotate_q(st.ctx, q_in, q_rot.view(-1, st.Hq, D), stream=s)
        csd.isoquant_attend_decode(st.ctx, st.cache, q_rot, st.page_table, st.seq_lens_dev, ws, out, stream=s)
    for step in range(1, 5):
        q_in.copy_(st.queries(step).reshape(q_in.shape))
        out.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        got = out.cpu()
        # the same step through eager calls into fresh buffers
        _, _, ref = run_attend(csd, st, q=st.queries(step))
        assert torch.equal(got, ref), step
    assert csd.isoquant_get_status(st.ctx) == 0
    del g


def test_decode_prep_equals_separate_calls(cuda_lib):
    """isoquant_decode_prep (append + rotate q in one launch) writes the same
    cache bytes as isoquant_compress_kv and the same q_rot as
    isoquant_rotate_q, bit for bit, for every input dtype."""
    from compressed_space_decode_b200.workload import DecodeState
    csd = cuda_lib
    wl = csd.synthetic.workloads(small=True)["gqa_b16_q32_kv4_L32768_paged"]
    for dt in (torch.bfloat16, torch.float16, torch.float32):
        sa, sb = DecodeState(wl, growth=8), DecodeState(wl, growth=8)
        k = torch.stack([sa.kv_tokens(b, sa.seq_lens[b], sa.seq_lens[b] + 3)[0] for b in range(sa.B)], 1)
        v = torch.stack([sa.kv_tokens(b, sa.seq_lens[b], sa.seq_lens[b] + 3)[1] for b in range(sa.B)], 1)
        k = k.reshape(-1, sa.H, D).to(dt).contiguous()
        v = v.reshape(-1, sa.H, D).to(dt).contiguous()
        slots = sa.slot_matrix(sa.seq_lens, 3).reshape(-1).contiguous()
        q = sa.queries(0).reshape(-1, sa.Hq, D).to(dt).contiguous()
        qa = torch.empty(q.shape, dtype=torch.float32, device="cuda")
        qb = torch.full(q.shape, float("nan"), dtype=torch.float32, device="cuda")
        csd.isoquant_compress_kv(sa.ctx, sa.cache, k, v, slots)
        csd.isoquant_rotate_q(sa.ctx, q, qa)
        csd.isoquant_decode_prep(sb.ctx, sb.cache, k, v, slots, q, qb)
        assert csd.isoquant_last_launch_count(sb.ctx) == 1
        torch.cuda.synchronize()
        assert csd.isoquant_get_status(sb.ctx) == 0
        assert torch.equal(qa, qb), dt
        assert torch.equal(sa.cache.codes, sb.cache.codes), dt
        assert torch.equal(sa.cache.norms.view(torch.int16), sb.cache.norms.view(torch.int16)), dt


def test_decode_step_matches_separate_calls_and_oracle(cuda_lib):
    """isoquant_decode_step over several steps: the same outputs and cache as
    compress_kv + rotate_q + attend_decode, and the oracle's attention."""
    from compressed_space_decode_b200.workload import DecodeState
    csd = cuda_lib
    for name in ("gqa_b16_q32_kv4_L32768_paged", "verify_b8_nq16_q32_kv8_L16384"):
        wl = csd.synthetic.workloads(small=True)[name]
        nq = wl.nq
        sa, sb = DecodeState(wl, growth=3 * nq), DecodeState(wl, growth=3 * nq)
        ws_a = _ws(csd, sa)
        ws_b = csd.alloc_step_workspace(sb.ctx, sb.B, nq, sb.Hq).fill_(0x7FC00000)
        for step in range(3):
            k = torch.stack([sa.kv_tokens(b, sa.seq_lens[b], sa.seq_lens[b] + nq)[0] for b in range(sa.B)], 1)
            v = torch.stack([sa.kv_tokens(b, sa.seq_lens[b], sa.seq_lens[b] + nq)[1] for b in range(sa.B)], 1)
            k = k.reshape(-1, sa.H, D).contiguous()
            v = v.reshape(-1, sa.H, D).contiguous()
            slots = sa.slot_matrix(sa.seq_lens, nq).reshape(-1).contiguous()
            for st in (sa, sb):
                st.seq_lens = [L + nq for L in st.seq_lens]
                st.seq_lens_dev += nq
            q = sa.queries(step)
            # separate calls
            q_rot = torch.empty(q.shape, dtype=torch.float32, device="cuda")
            out_a = torch.empty(q.shape, dtype=torch.float32, device="cuda")
            csd.isoquant_compress_kv(sa.ctx, sa.cache, k, v, slots)
            csd.isoquant_rotate_q(sa.ctx, q.reshape(-1, sa.Hq, D), q_rot.view(-1, sa.Hq, D))
            csd.isoquant_attend_decode(sa.ctx, sa.cache, q_rot, sa.page_table, sa.seq_lens_dev, ws_a, out_a,
                                       causal=wl.causal)
            # one call
            out_b = torch.full(q.shape, float("nan"), dtype=torch.float32, device="cuda")
            csd.isoquant_decode_step(sb.ctx, sb.cache, k, v, slots, q.contiguous(), sb.page_table, sb.seq_lens_dev,
                                     ws_b, out_b, causal=wl.causal)
            assert csd.isoquant_last_launch_count(sb.ctx) == 3
            torch.cuda.synchronize()
            assert csd.isoquant_get_status(sa.ctx) == 0 and csd.isoquant_get_status(sb.ctx) == 0
            assert torch.equal(out_a, out_b), (name, step)
        assert torch.equal(sa.cache.codes, sb.cache.codes)
        b = sb.B - 1
        check_pair(sb, b, sb.H - 1, q.float().cpu(), out_b.cpu())


@pytest.mark.parametrize("case", ["prefill_b1_L600", "chunk_b2", "rows128_noncausal", "rows200_ragged_ps64",
                                  "prefill_nq_gt_L"])
def test_tcgen05_wide_kernel_matches_mma_path_and_oracle(cuda_lib, case):
    """128 or more query rows per KV head (causal prefill, long chunks) run
    on the warp-specialised 128-row tcgen05 kernel, each stream walking only
    the pages inside its causal horizon.  It matches the oracle on every
    query row of sampled (sequence, head) pairs and the mma.sync kernel (the
    minimum workspace) on all rows."""
    from compressed_space_decode_b200.synthetic import Workload
    from compressed_space_decode_b200.workload import DecodeState
    csd = cuda_lib
    if case == "prefill_b1_L600":
        # a 600-token prompt attends to itself: 2400 rows per KV head, 19
        # streams (the last of 96 rows), 64-token pages
        wl = Workload(case, 1, 8, 2, [600], nq=600, page_size=64, causal=True, seed=41)
    elif case == "chunk_b2":
        # chunked prefill: the last 200 positions of two ragged contexts
        wl = Workload(case, 2, 16, 4, [1500, 900], nq=200, page_size=128, causal=True, seed=42)
    elif case == "rows128_noncausal":
        wl = Workload(case, 3, 32, 1, [2000, 517, 130], nq=4, page_size=256, causal=False, seed=43)
    elif case == "rows200_ragged_ps64":
        wl = Workload(case, 5, 16, 2, [3000, 1, 700, 64, 1234], nq=25, page_size=64, causal=True, seed=44)
    else:
        # more query positions than tokens: the first positions see nothing
        wl = Workload(case, 2, 8, 2, [40, 300], nq=100, page_size=64, causal=True, seed=45)
    st = DecodeState(wl)
    q = st.queries(0)
    q_rot = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    csd.isoquant_rotate_q(st.ctx, q.reshape(-1, st.Hq, D), q_rot.view(-1, st.Hq, D))
    outs = []
    n_sms = torch.cuda.get_device_properties(0).multi_processor_count
    pairs = ((wl.nq * st.G + 7) // 8) * st.B * st.H
    ws_min = (256 + (2 * n_sms + pairs) * 4160) // 4
    for ws in (_ws(csd, st), torch.empty(ws_min, dtype=torch.int32, device="cuda").fill_(0x7FC00000)):
        out = torch.full(q.shape, float("nan"), dtype=torch.float32, device="cuda")
        csd.isoquant_attend_decode(st.ctx, st.cache, q_rot, st.page_table, st.seq_lens_dev, ws, out,
                                   causal=wl.causal)
        torch.cuda.synchronize()
        assert csd.isoquant_get_status(st.ctx) == 0
        outs.append(out.cpu())
    wide, mma = outs
    assert torch.isfinite(wide).all()
    err = rowwise_rel_err(wide.numpy(), mma.numpy())
    assert err.max() <= 2 * ATTN_TOL, err.max()
    if wl.causal:
        # rows that see no token are zero
        for b in range(st.B):
            for i in range(wl.nq):
                if st.seq_lens[b] - wl.nq + i + 1 <= 0:
                    assert not wide[b, i].any()
    qc = q.float().cpu()
    for b in range(st.B):
        if st.seq_lens[b] == 0:
            continue
        check_pair(st, b, (b * 3 + 1) % st.H, qc, wide)


@pytest.mark.parametrize("case", ["verify", "ragged_ps64", "rows96_ps128", "short"])
def test_tcgen05_rows_kernel_matches_mma_path(cuda_lib, case):
    """64 or more query rows per KV head run on the tcgen05 kernel (one
    decode of each KV tile for 64 rows, products in tensor memory) when the
    workspace has its records; a workspace of the minimum size runs the
    mma.sync kernel.  Both match the oracle and each other."""
    from compressed_space_decode_b200.synthetic import Workload
    from compressed_space_decode_b200.workload import DecodeState
    csd = cuda_lib
    if case == "verify":
        wl = csd.synthetic.workloads(small=True)["verify_b8_nq16_q32_kv8_L16384"]
    elif case == "ragged_ps64":
        # 16 positions x 4 heads = 64 rows, causal, ragged lengths, 64-token pages
        wl = Workload(case, 5, 16, 4, [3000, 1, 700, 64, 1234], nq=16, page_size=64, causal=True, seed=31)
    elif case == "rows96_ps128":
        # 3 positions x 32 heads = 96 rows: a full stream and one of 32 rows
        wl = Workload(case, 3, 32, 1, [2000, 517, 130], nq=3, page_size=128, causal=True, seed=32)
    else:
        wl = Workload(case, 4, 16, 2, [17, 64, 65, 200], nq=16, page_size=256, causal=True, seed=33)
    st = DecodeState(wl)
    q = st.queries(0)
    q_rot = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    csd.isoquant_rotate_q(st.ctx, q.reshape(-1, st.Hq, D), q_rot.view(-1, st.Hq, D))
    outs = []
    n_sms = torch.cuda.get_device_properties(0).multi_processor_count
    pairs = ((wl.nq * st.G + 7) // 8) * st.B * st.H
    ws_min = (256 + (2 * n_sms + pairs) * 4160) // 4
    for ws in (_ws(csd, st), torch.empty(ws_min, dtype=torch.int32, device="cuda").fill_(0x7FC00000)):
        out = torch.full(q.shape, float("nan"), dtype=torch.float32, device="cuda")
        csd.isoquant_attend_decode(st.ctx, st.cache, q_rot, st.page_table, st.seq_lens_dev, ws, out,
                                   causal=wl.causal)
        torch.cuda.synchronize()
        assert csd.isoquant_get_status(st.ctx) == 0
        outs.append(out.cpu())
    tiles, mma = outs
    assert torch.isfinite(tiles).all()
    err = rowwise_rel_err(tiles.numpy(), mma.numpy())
    # each path is within ATTN_TOL of the exact result
    assert err.max() <= 2 * ATTN_TOL, err.max()
    qc = q.float().cpu()
    for b in range(st.B):
        if st.seq_lens[b] == 0:
            continue
        check_pair(st, b, (b * 3) % st.H, qc, tiles)


@pytest.mark.parametrize("hq,h,nq,L", [(32, 8, 300, 400), (32, 4, 300, 350), (16, 8, 600, 700)])
def test_combine_grouped_rows(cuda_lib, hq, h, nq, L):
    """With many output rows (at least 64 per SM) the combine kernel merges
    the rows of a GQA group (8, 4 or 2 of them) in one warp; every row still
    matches the oracle."""
    from compressed_space_decode_b200.synthetic import Workload
    from compressed_space_decode_b200.workload import DecodeState
    csd = cuda_lib
    n_sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert nq * hq >= 64 * n_sms
    wl = Workload("grouped", 1, hq, h, [L], nq=nq, page_size=64, causal=True, seed=70 + hq // h)
    st = DecodeState(wl)
    q, _, out = run_attend(csd, st)
    assert torch.isfinite(out).all()
    for hh in (0, st.H - 1):
        check_pair(st, 0, hh, q, out)
