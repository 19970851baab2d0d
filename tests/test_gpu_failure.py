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


def test_argument_errors_with_a_live_context(cuda_lib):
    """Checks that need a context: each bad argument returns its status from
    the host, launches nothing and leaves the status word clear; the same
    context then serves a correct call."""
    import ctypes
    from compressed_space_decode_b200.synthetic import Workload
    from compressed_space_decode_b200.workload import DecodeState
    csd = cuda_lib
    L = csd.lib()
    st = DecodeState(Workload("args", 2, 16, 4, [300, 40], nq=1, page_size=64, seed=72))
    ctx = st.ctx.handle
    s0 = csd._stream(None)
    q = st.queries(0)
    n_rows = q.shape[0] * q.shape[1]
    q_rot = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    spare = torch.empty(q_rot.numel() + 4, dtype=torch.float32, device="cuda")
    off4 = ctypes.c_void_p(spare.data_ptr() + 4)  # 4 bytes past a 16-byte boundary
    p = csd._ptr
    dt = csd._dtype(q)
    # rotate_q: misaligned output, unknown dtype, q heads not a multiple of the KV heads
    assert L.isoquant_rotate_q(ctx, p(q), dt, n_rows, st.Hq, off4, s0) == -6
    assert L.isoquant_rotate_q(ctx, p(q), 99, n_rows, st.Hq, p(q_rot), s0) == -2
    assert L.isoquant_rotate_q(ctx, p(q), dt, n_rows, st.Hq + 1, p(q_rot), s0) == -1
    assert L.isoquant_last_launch_count(ctx) == 0
    csd.isoquant_rotate_q(st.ctx, q.reshape(-1, st.Hq, D), q_rot.view(-1, st.Hq, D))
    ws = _ws(csd, st)
    out = torch.empty_like(q_rot)
    cs = st.cache.c_struct()
    B, nq, Hq, maxp = st.B, 1, st.Hq, st.page_table.shape[1]

    def attend(cache_struct=cs, ws_ptr=None, ws_bytes=None, out_ptr=None, scale=0.0):
        return L.isoquant_attend_decode(ctx, ctypes.byref(cache_struct), p(q_rot), B, nq, Hq, p(st.page_table), maxp,
                                        p(st.seq_lens_dev), 0, scale, ws_ptr if ws_ptr is not None else p(ws),
                                        ws.numel() * 4 if ws_bytes is None else ws_bytes,
                                        out_ptr if out_ptr is not None else p(out), s0)
    assert attend(ws_bytes=64) == -4                      # workspace too small
    assert attend(ws_ptr=ctypes.c_void_p(ws.data_ptr() + 4)) == -6
    assert attend(out_ptr=off4) == -6
    assert attend(scale=-1.0) == -1
    bad = csd._Cache(st.cache.codes.data_ptr(), st.cache.norms.data_ptr(), st.cache.num_pages, 48)
    assert attend(cache_struct=bad) == -2                 # page size 48
    none = csd._Cache(0, st.cache.norms.data_ptr(), st.cache.num_pages, st.ps)
    assert attend(cache_struct=none) == -1
    assert L.isoquant_last_launch_count(ctx) == 0
    torch.cuda.synchronize()
    assert csd.isoquant_get_status(st.ctx) == 0
    assert attend() == 0
    torch.cuda.synchronize()
    assert csd.isoquant_get_status(st.ctx) == 0
    out_c, qc = out.cpu(), q.float().cpu()
    for b in range(st.B):
        check_pair(st, b, b % st.H, qc, out_c)


def test_combine_with_another_plan_is_flagged(cuda_lib):
    """The partial half writes the tag of its plan into the workspace
    header.  A combine given another workspace size (so another kernel's
    record layout) sees the mismatch: it merges nothing, writes zeros and
    raises DEVERR_PLAN_MISMATCH; with matching sizes the halves agree with
    the one-call entry."""
    from compressed_space_decode_b200.synthetic import Workload
    from compressed_space_decode_b200.workload import DecodeState
    csd = cuda_lib
    # 16 positions x 4 heads = 64 rows per KV head: the tcgen05 plan with the
    # full workspace, the mma.sync plan with the minimum one
    st = DecodeState(Workload("plan", 3, 16, 4, [700, 300, 65], nq=16, page_size=64, causal=True, seed=73))
    q = st.queries(0)
    q_rot = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    csd.isoquant_rotate_q(st.ctx, q.reshape(-1, st.Hq, D), q_rot.view(-1, st.Hq, D))
    ws = _ws(csd, st)
    n_sms = torch.cuda.get_device_properties(0).multi_processor_count
    pairs = ((16 * st.G + 7) // 8) * st.B * st.H
    small = (256 + (2 * n_sms + pairs) * 4160)
    assert small < ws.numel() * 4
    out = torch.full(q.shape, float("nan"), dtype=torch.float32, device="cuda")
    csd.isoquant_attend_partial(st.ctx, st.cache, q_rot, st.page_table, st.seq_lens_dev, ws, causal=True)
    # combine told the workspace is the small one: the mma.sync layout
    csd.isoquant_attend_combine(st.ctx, st.B, 16, st.Hq, st.seq_lens_dev, st.ps, ws[:small // 4], out)
    torch.cuda.synchronize()
    assert csd.isoquant_get_status(st.ctx) == csd.DEVERR_PLAN_MISMATCH
    assert torch.all(out == 0)
    # matching sizes: no flag, and the same output as the one-call entry
    csd.isoquant_attend_partial(st.ctx, st.cache, q_rot, st.page_table, st.seq_lens_dev, ws, causal=True)
    csd.isoquant_attend_combine(st.ctx, st.B, 16, st.Hq, st.seq_lens_dev, st.ps, ws, out)
    ref = torch.empty_like(out)
    csd.isoquant_attend_decode(st.ctx, st.cache, q_rot, st.page_table, st.seq_lens_dev, _ws(csd, st), ref,
                               causal=True)
    torch.cuda.synchronize()
    assert csd.isoquant_get_status(st.ctx) == 0
    assert torch.equal(out, ref)


def test_oversized_shapes_are_refused(cuda_lib):
    """Shapes whose row or unit counts would overflow the kernels' 32-bit
    indexing are refused on the host (INVALID_ARG), before any launch."""
    import ctypes
    from compressed_space_decode_b200 import synthetic
    csd = cuda_lib
    L = csd.lib()
    signs, quats = synthetic.rotation_params(9, 8)
    ctx = csd.isoquant_init(signs, quats)
    sz = ctypes.c_size_t()
    # 2^31 query rows per KV head (nq * G)
    assert L.isoquant_workspace_size(ctx.handle, 1, 1 << 28, 64, ctypes.byref(sz)) == -1
    # 2^28 row groups x 16 sequences x 8 KV heads
    assert L.isoquant_workspace_size(ctx.handle, 16, 1 << 28, 64, ctypes.byref(sz)) == -1
    # a modest shape still works
    assert L.isoquant_workspace_size(ctx.handle, 16, 1, 64, ctypes.byref(sz)) == 0


def test_workspace_sized_by_the_kernel_that_runs(cuda_lib):
    """isoquant_workspace_size reports the records of the kernel the shape
    runs on: the mma.sync records below 64 query rows per KV head, the
    tcgen05 plan (16 or 8 records per CTA and per stream, plus the unit
    prefix) from there, and the mma.sync records again for 32-token pages."""
    from compressed_space_decode_b200 import synthetic
    csd = cuda_lib
    n_sms = torch.cuda.get_device_properties(0).multi_processor_count
    rec = 4160
    signs, quats = synthetic.rotation_params(10, 8)
    ctx = csd.isoquant_init(signs, quats)
    # decode, 16 sequences, 8 rows per KV head
    assert csd.isoquant_workspace_size(ctx, 16, 1, 64) == 256 + (2 * n_sms + 16 * 8) * rec
    # verification, 8 sequences, 16 positions x 4 heads = 64 rows: one 64-row stream
    tiles = 256 + (2 * n_sms + 1 * 8 * 8) * 8 * rec + (1 * 8 + 1) * 8
    assert csd.isoquant_workspace_size(ctx, 8, 16, 32) == tiles
    # causal prefill of 4096 positions, 32 q heads: 128-row streams
    streams = 4096 * 4 // 128
    wide = 256 + (n_sms + streams * 8) * 16 * rec + (streams + 1) * 8
    assert csd.isoquant_workspace_size(ctx, 1, 4096, 32) == wide
    # 32-token pages: the mma.sync records whatever the rows
    assert csd.isoquant_workspace_size_paged(ctx, 8, 16, 32, 32) == 256 + (2 * n_sms + 8 * 8 * 8) * rec
