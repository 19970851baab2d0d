"""Failure path on the GPU without a fault: the pipelines' bounded wait.

A kernel thread waits, through the same bounded wait the attention
pipelines use, on a barrier that nothing completes.  The wait must give up
after its limit, raise the timeout bit of the status word and return, and
the context must serve a correct attention call right after.
"""
import pytest
import torch

from tests.test_gpu_parity import _ws, check_pair

pytestmark = pytest.mark.gpu
D = 128


def test_bounded_wait_times_out_and_context_survives(cuda_lib):
    from compressed_space_decode_b200.synthetic import Workload
    from compressed_space_decode_b200.workload import DecodeState
    csd = cuda_lib
    st = DecodeState(Workload("wait", 2, 16, 4, [300, 40], nq=1, page_size=64, seed=71))
    limit = 20_000_000  # 20 ms
    elapsed = torch.zeros(1, dtype=torch.int64, device="cuda")
    csd.isoquant_selftest_wait(st.ctx, limit, elapsed)
    torch.cuda.synchronize()
    assert csd.isoquant_get_status(st.ctx) == csd.DEVERR_WAIT_TIMEOUT
    waited = int(elapsed.item())
    assert limit <= waited < limit + 50_000_000, waited
    assert csd.isoquant_get_status(st.ctx) == 0  # cleared by the read

    # the same context right after: attention matches the oracle, no error bit
    q = st.queries(0)
    q_rot = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    csd.isoquant_rotate_q(st.ctx, q.reshape(-1, st.Hq, D), q_rot.view(-1, st.Hq, D))
    out = torch.full(q.shape, float("nan"), dtype=torch.float32, device="cuda")
    csd.isoquant_attend_decode(st.ctx, st.cache, q_rot, st.page_table, st.seq_lens_dev, _ws(csd, st), out)
    torch.cuda.synchronize()
    assert csd.isoquant_get_status(st.ctx) == 0
    out, qc = out.cpu(), q.float().cpu()
    for b in range(st.B):
        check_pair(st, b, (b + 1) % st.H, qc, out)


def test_selftest_wait_rejects_unbounded_limits(cuda_lib):
    from compressed_space_decode_b200 import synthetic
    signs, quats = synthetic.rotation_params(3, 1)
    ctx = cuda_lib.isoquant_init(signs, quats)
    for bad in (0, 10_000_000_001):
        with pytest.raises(cuda_lib.IsoquantError):
            cuda_lib.isoquant_selftest_wait(ctx, bad)
