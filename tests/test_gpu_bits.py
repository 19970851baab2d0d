"""Other code widths on the GPU: 2- and 4-bit contexts (isoquant_init_bits).

The codes and norms the library writes are the oracle's bit for bit
(outside the 1e-6 boundary band), and attention over them matches the
oracle's compressed-space attention on every row of sampled (sequence, KV
head) pairs at decode, verification and prefill shapes: below 64 query rows
per KV head or with 32-token pages on the mma.sync kernel, from 64 rows on
the tcgen05 kernels.
"""
import numpy as np
import pytest
import torch

from tests.parity import ATTN_TOL, compare_compressed, oracle_rows, rowwise_rel_err
from tests.test_gpu_parity import _ws, limits

pytestmark = pytest.mark.gpu
D = 128


def _state(csd, case, bits):
    from compressed_space_decode_b200.synthetic import Workload
    from compressed_space_decode_b200.workload import DecodeState
    if case == "decode":
        wl = Workload(case, 3, 32, 8, [700, 65, 1], nq=1, page_size=256, seed=61)
    elif case == "decode_p32":
        wl = Workload(case, 2, 8, 2, [100, 37], nq=1, page_size=32, seed=66)
    elif case == "verify_p32":
        wl = Workload(case, 2, 32, 8, [300, 45], nq=16, page_size=32, causal=True, seed=67)
    elif case == "decode_full":
        # the decode bench's workload (B = 16, 32 q / 4 KV heads, 32768 tokens, shuffled pages); two
        # sequences are checked against the oracle
        import compressed_space_decode_b200.synthetic as syn
        wl = syn.workloads()["gqa_b16_q32_kv4_L32768_paged"]
    elif case == "verify":
        wl = Workload(case, 2, 32, 8, [600, 130], nq=16, page_size=128, causal=True, seed=62)
    else:
        wl = Workload(case, 1, 8, 2, [500], nq=500, page_size=64, causal=True, seed=63)
    return DecodeState(wl, bits=bits)


@pytest.mark.parametrize("bits", [2, 4])
def test_codebook_matches_oracle(cuda_lib, bits):
    import oracle
    lv, th = cuda_lib.isoquant_codebook(bits)
    olv, oth = oracle.codebook(bits)
    np.testing.assert_array_equal(np.array(lv, dtype=np.float64), olv)
    np.testing.assert_allclose(np.array(th, dtype=np.float64), oth, rtol=0, atol=6e-8)


@pytest.mark.parametrize("bits", [2, 4])
@pytest.mark.parametrize("case", ["decode", "verify", "prefill", "decode_p32", "verify_p32", "decode_full"])
def test_codes_and_attention_match_oracle(cuda_lib, bits, case):
    csd = cuda_lib
    st = _state(csd, case, bits)
    wl = st.wl
    assert st.cache.codes.shape[3] == csd.WORDS_FOR[bits]
    q = st.queries(0)
    q_rot = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    csd.isoquant_rotate_q(st.ctx, q.reshape(-1, st.Hq, D), q_rot.view(-1, st.Hq, D))
    out = torch.full(q.shape, float("nan"), dtype=torch.float32, device="cuda")
    csd.isoquant_attend_decode(st.ctx, st.cache, q_rot, st.page_table, st.seq_lens_dev, _ws(csd, st), out,
                               causal=wl.causal)
    torch.cuda.synchronize()
    assert csd.isoquant_get_status(st.ctx) == 0
    out = out.cpu()
    assert torch.isfinite(out).all()
    qc = q.float().cpu()
    for b in (range(st.B) if case != "decode_full" else (3, 12)):
        L = st.seq_lens[b]
        h = (3 * b + 1) % st.H
        k, v = st.kv_tokens(b, 0, L)
        s, qt = st.signs[h].numpy(), st.quats[h].numpy()
        gkc, gkn = st.gather(b, h, 0, 0, L)
        gvc, gvn = st.gather(b, h, 1, 0, L)
        _, kc, kn = compare_compressed(k[:, h].double().cpu().numpy(), s, qt, gkc.numpy(), gkn.numpy(), bits=bits)
        _, vc, vn = compare_compressed(v[:, h].double().cpu().numpy(), s, qt, gvc.numpy(), gvn.numpy(), bits=bits)
        ref, idx = oracle_rows(st, b, h, qc, limits(wl), (kc, kn, vc, vn))
        got = np.stack([out[b, i, hq].numpy() for (i, hq) in idx])
        err = rowwise_rel_err(got, ref)
        assert err.max() <= ATTN_TOL, (bits, case, b, err.max())


@pytest.mark.parametrize("bits", [2, 4])
def test_decode_step_and_static_entry(cuda_lib, bits):
    """The one-call step (append + rotate in one launch, then attention) and
    the allocation-free entry give the separate calls' results at 2 and 4
    bits."""
    from compressed_space_decode_b200.synthetic import Workload
    from compressed_space_decode_b200.workload import DecodeState
    csd = cuda_lib
    wl = Workload("step", 2, 16, 4, [300, 129], nq=16, page_size=64, causal=True, seed=65)
    sa, sb = DecodeState(wl, growth=16, bits=bits), DecodeState(wl, growth=16, bits=bits)
    k = torch.stack([sa.kv_tokens(b, sa.seq_lens[b], sa.seq_lens[b] + 16)[0] for b in range(sa.B)], 1)
    v = torch.stack([sa.kv_tokens(b, sa.seq_lens[b], sa.seq_lens[b] + 16)[1] for b in range(sa.B)], 1)
    k, v = k.reshape(-1, sa.H, D).contiguous(), v.reshape(-1, sa.H, D).contiguous()
    slots = sa.slot_matrix(sa.seq_lens, 16).reshape(-1).contiguous()
    for st in (sa, sb):
        st.seq_lens = [L + 16 for L in st.seq_lens]
        st.seq_lens_dev += 16
    q = sa.queries(0)
    q_rot = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    out_a = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    csd.isoquant_compress_kv(sa.ctx, sa.cache, k, v, slots)
    csd.isoquant_rotate_q(sa.ctx, q.reshape(-1, sa.Hq, D), q_rot.view(-1, sa.Hq, D))
    csd.isoquant_attend_decode(sa.ctx, sa.cache, q_rot, sa.page_table, sa.seq_lens_dev, _ws(csd, sa), out_a,
                               causal=True)
    out_b = torch.full(q.shape, float("nan"), dtype=torch.float32, device="cuda")
    ws_b = csd.alloc_step_workspace(sb.ctx, sb.B, 16, sb.Hq).fill_(0x7FC00000)
    csd.isoquant_decode_step(sb.ctx, sb.cache, k, v, slots, q.contiguous(), sb.page_table, sb.seq_lens_dev, ws_b,
                             out_b, causal=True)
    out_c = torch.full(q.shape, float("nan"), dtype=torch.float32, device="cuda")
    csd.isoquant_attend_decode_static(sa.ctx, sa.cache, q_rot, sa.page_table, sa.seq_lens_dev, out_c, causal=True)
    torch.cuda.synchronize()
    assert csd.isoquant_get_status(sa.ctx) == 0 and csd.isoquant_get_status(sb.ctx) == 0
    assert torch.equal(sa.cache.codes, sb.cache.codes) and torch.equal(sa.cache.norms, sb.cache.norms)
    assert torch.equal(out_a, out_b)
    assert torch.equal(out_a, out_c)


def test_init_bits_rejects_other_widths(cuda_lib):
    from compressed_space_decode_b200 import synthetic
    csd = cuda_lib
    signs, quats = synthetic.rotation_params(3, 2)
    for bits in (1, 5, 8):
        with pytest.raises(csd.IsoquantError) as e:
            csd.isoquant_init(signs, quats, bits=bits)
        assert e.value.status == -2
    ctx = csd.isoquant_init(signs, quats, bits=2)
    code_bytes, norm_bytes = csd.isoquant_cache_bytes(ctx, 3, 64)
    assert code_bytes == 3 * 2 * 2 * 8 * 64 * 4 and norm_bytes == 3 * 2 * 2 * 64 * 2
    ctx.close()
