"""Other code widths on the GPU: 2- and 4-bit contexts (isoquant_init_bits).

The codes and norms the library writes are the oracle's bit for bit
(outside the 1e-6 boundary band), and attention over them matches the
oracle's compressed-space attention on every row of sampled (sequence, KV
head) pairs at decode, verification and prefill shapes (2- and 4-bit
attention runs on the tcgen05 kernels at every shape).
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
@pytest.mark.parametrize("case", ["decode", "verify", "prefill"])
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
    for b in range(st.B):
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


def test_small_pages_are_unsupported_below_3_bits(cuda_lib):
    from compressed_space_decode_b200.synthetic import Workload
    from compressed_space_decode_b200.workload import DecodeState
    csd = cuda_lib
    wl = Workload("p32", 1, 8, 2, [100], nq=1, page_size=32, seed=64)
    st = DecodeState(wl, bits=2)
    q_rot = torch.zeros((1, 1, 8, D), dtype=torch.float32, device="cuda")
    out = torch.empty_like(q_rot)
    with pytest.raises(csd.IsoquantError) as e:
        csd.isoquant_attend_decode(st.ctx, st.cache, q_rot, st.page_table, st.seq_lens_dev, _ws(csd, st), out)
    assert e.value.status == -2
