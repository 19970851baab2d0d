"""The allocation-free attention entry point (collected last on purpose).

isoquant_attend_decode_static serves callers that cannot allocate device
memory or lend the library a workspace (a serving process whose pool owns
all device memory, or a decode loop that must avoid cudaMalloc's device-wide
synchronisation).  Its split records live in a fixed array inside the
library.  It must give the same output as isoquant_attend_decode, call
after call: the array keeps the previous call's records, so a second call
with different inputs checks that nothing stale leaks through.  Both entry
points pick their kernel by the shape and the room for its records (the
16 MiB array holds the tcgen05 plan of the verification shape here), so the
two outputs are identical bit for bit, which also pins the kernel the static
path chose; each workload is checked against the oracle as well.
"""
import pytest
import torch

from tests.parity import ATTN_TOL, rowwise_rel_err
from tests.test_gpu_parity import check_pair

pytestmark = pytest.mark.gpu


def _rotated(csd, st, step):
    q = st.queries(step)
    q_rot = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    csd.isoquant_rotate_q(st.ctx, q.reshape(-1, st.Hq, 128), q_rot.view(-1, st.Hq, 128))
    return q_rot


def test_static_entry_matches_workspace_entry_twice(cuda_lib):
    csd = cuda_lib
    from compressed_space_decode_b200.workload import DecodeState
    wls = csd.synthetic.workloads(small=True)
    for name, steps in (("gqa_b16_q32_kv4_L32768_paged", (0, 1)), ("verify_b8_nq16_q32_kv8_L16384", (2, 3))):
        wl = wls[name]
        st = DecodeState(wl)
        ws = csd.alloc_workspace(st.ctx, st.B, wl.nq, st.Hq)
        for step in steps:  # two calls in a row, different queries
            q_rot = _rotated(csd, st, step)
            ref = torch.empty_like(q_rot)
            got = torch.full_like(q_rot, float("nan"))
            csd.isoquant_attend_decode(st.ctx, st.cache, q_rot, st.page_table, st.seq_lens_dev, ws, ref,
                                       causal=wl.causal)
            csd.isoquant_attend_decode_static(st.ctx, st.cache, q_rot, st.page_table, st.seq_lens_dev, got,
                                              causal=wl.causal)
            torch.cuda.synchronize()
            assert csd.isoquant_get_status(st.ctx) == 0
            err = rowwise_rel_err(got.cpu().numpy(), ref.cpu().numpy())
            assert err.max() <= ATTN_TOL, (name, step, err.max())
            # same kernel and plan as the workspace entry: identical output
            assert torch.equal(got, ref), (name, step)
        # the last call's output against the oracle on one sampled pair
        q = st.queries(steps[-1]).float().cpu()
        check_pair(st, st.B - 1, st.H - 1, q, got.cpu())


def test_static_entry_rejects_oversized_shapes(cuda_lib):
    csd = cuda_lib
    from compressed_space_decode_b200 import synthetic
    signs, quats = synthetic.rotation_params(3, 8)
    ctx = csd.isoquant_init(signs, quats)
    cache = csd.PagedCache.allocate(8, 1, 256)
    # 2048 sequences x 8 KV heads of records need far more than 16 MiB
    q_rot = torch.zeros((2048, 1, 8, 128), dtype=torch.float32, device="cuda")
    pt = torch.zeros((2048, 1), dtype=torch.int32, device="cuda")
    lens = torch.ones(2048, dtype=torch.int32, device="cuda")
    out = torch.empty_like(q_rot)
    with pytest.raises(csd.IsoquantError) as e:
        csd.isoquant_attend_decode_static(ctx, cache, q_rot, pt, lens, out)
    assert e.value.status == -4
