"""IsoQuant compressed-space attention on B200 (sm_100a).

Thin Python binding over the C ABI of ``libisoquant.so`` (declared in
``include/isoquant.h``).  Each function here has the name of the C entry point
it calls and only marshals arguments: every step of the path runs in the
library's CUDA kernels.  PyTorch provides device memory and streams.

There is no CPU fallback: if the native library is missing or fails to load,
every call raises.
"""
import ctypes
import os

import torch

from . import synthetic  # noqa: F401  (seeded inputs; no method arithmetic)

HEAD_DIM = 128
WORDS = 13
WORDS_FOR = {2: 8, 3: 13, 4: 16}  # code words per vector by code width

F32, BF16, F16 = 0, 1, 2
_DTYPES = {torch.float32: F32, torch.bfloat16: BF16, torch.float16: F16}

DEVERR_WAIT_TIMEOUT = 1
DEVERR_PAGE_RANGE = 2
DEVERR_SLOT_RANGE = 4
DEVERR_PLAN_MISMATCH = 8

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libisoquant.so")
_lib = None

SYMBOLS = [
    "isoquant_init", "isoquant_destroy", "isoquant_strerror", "isoquant_codebook", "isoquant_cache_bytes",
    "isoquant_compress_kv", "isoquant_rotate_q", "isoquant_workspace_size", "isoquant_attend_decode",
    "isoquant_attend_partial", "isoquant_attend_combine", "isoquant_get_status", "isoquant_last_launch_count",
    "isoquant_attend_decode_static", "isoquant_decode_prep", "isoquant_step_workspace_size",
    "isoquant_decode_step", "isoquant_init_bits", "isoquant_codebook_bits", "isoquant_selftest_wait",
    "isoquant_workspace_size_paged", "isoquant_debug_export_z",
]


class IsoquantError(RuntimeError):
    def __init__(self, status, what):
        super().__init__(f"{what}: {strerror(status)} (status {status})")
        self.status = status


class _Cache(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("norms", ctypes.c_void_p),
                ("num_pages", ctypes.c_int32), ("page_size", ctypes.c_int32)]


def lib():
    """Load libisoquant.so (raises if it is missing: no fallback path)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing; build it with "
                               "`python compressed_space_decode_b200/build.py` (no CPU fallback exists)")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        cp = ctypes.POINTER(_Cache)
        sig = {
            "isoquant_init": ([ctypes.POINTER(vp), i32, i32, vp, vp], i32),
            "isoquant_init_bits": ([ctypes.POINTER(vp), i32, i32, vp, vp, i32], i32),
            "isoquant_codebook_bits": ([i32, vp, vp], i32),
            "isoquant_destroy": ([vp], None),
            "isoquant_strerror": ([i32], ctypes.c_char_p),
            "isoquant_codebook": ([vp, vp], i32),
            "isoquant_cache_bytes": ([vp, i32, i32, ctypes.POINTER(sz), ctypes.POINTER(sz)], i32),
            "isoquant_compress_kv": ([vp, cp, vp, vp, i32, i32, vp, vp], i32),
            "isoquant_rotate_q": ([vp, vp, i32, i32, i32, vp, vp], i32),
            "isoquant_workspace_size": ([vp, i32, i32, i32, ctypes.POINTER(sz)], i32),
            "isoquant_workspace_size_paged": ([vp, i32, i32, i32, i32, ctypes.POINTER(sz)], i32),
            "isoquant_attend_decode": ([vp, cp, vp, i32, i32, i32, vp, i32, vp, i32, ctypes.c_float, vp, sz, vp, vp],
                                       i32),
            "isoquant_attend_partial": ([vp, cp, vp, i32, i32, i32, vp, i32, vp, i32, ctypes.c_float, vp, sz, vp],
                                        i32),
            "isoquant_attend_combine": ([vp, i32, i32, i32, vp, i32, vp, sz, vp, vp], i32),
            "isoquant_get_status": ([vp, ctypes.POINTER(ctypes.c_uint32), vp], i32),
            "isoquant_last_launch_count": ([vp], i32),
            "isoquant_attend_decode_static": ([vp, cp, vp, i32, i32, i32, vp, i32, vp, i32, ctypes.c_float, vp, vp],
                                              i32),
            "isoquant_decode_prep": ([vp, cp, vp, vp, i32, vp, vp, i32, i32, i32, vp, vp], i32),
            "isoquant_step_workspace_size": ([vp, i32, i32, i32, ctypes.POINTER(sz)], i32),
            "isoquant_decode_step": ([vp, cp, vp, vp, i32, vp, vp, i32, i32, i32, i32, vp, i32, vp, i32,
                                      ctypes.c_float, vp, sz, vp, vp], i32),
            "isoquant_selftest_wait": ([vp, ctypes.c_uint64, vp, vp], i32),
            "isoquant_debug_export_z": ([vp, vp, i32, i32, vp, vp], i32),
        }
        for name, (args, res) in sig.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _lib = L
    return _lib


def strerror(status):
    return lib().isoquant_strerror(int(status)).decode()


def _check(status, what):
    if status != 0:
        raise IsoquantError(status, what)


def _stream(stream):
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _dtype(t):
    try:
        return _DTYPES[t.dtype]
    except KeyError:
        raise TypeError(f"unsupported dtype {t.dtype}")


class Context:
    """An isoquant_ctx*: per-head rotation parameters on one device."""

    def __init__(self, handle, num_kv_heads, device, bits=3):
        self.handle = handle
        self.num_kv_heads = num_kv_heads
        self.device = device
        self.bits = bits

    def close(self):
        if self.handle:
            lib().isoquant_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class PagedCache:
    """Caller-owned packed cache: codes int32 [pages][2][H][W][page_size]
    (bit patterns of uint32 words; W = 13 at 3 bits, 8 at 2, 16 at 4),
    norms float16 [pages][2][H][page_size]."""

    def __init__(self, codes, norms, page_size):
        assert codes.dtype == torch.int32 and norms.dtype == torch.float16
        self.codes = codes
        self.norms = norms
        self.num_pages = codes.shape[0]
        self.page_size = page_size

    @staticmethod
    def allocate(num_kv_heads, num_pages, page_size, device="cuda", bits=3):
        codes = torch.zeros((num_pages, 2, num_kv_heads, WORDS_FOR[bits], page_size), dtype=torch.int32,
                            device=device)
        norms = torch.zeros((num_pages, 2, num_kv_heads, page_size), dtype=torch.float16, device=device)
        return PagedCache(codes, norms, page_size)

    def c_struct(self):
        return _Cache(self.codes.data_ptr(), self.norms.data_ptr(), self.num_pages, self.page_size)


# ----------------------------------------------------------------- C ABI calls
def isoquant_init(signs, quats, head_dim=HEAD_DIM, bits=3):
    """signs: int8 [H][128] (+-1); quats: float32 [H][32][2][4] (host arrays);
    bits: code width, 3 (the method's) or 2 / 4 (isoquant_init_bits)."""
    signs = torch.as_tensor(signs, dtype=torch.int8).contiguous().cpu()
    quats = torch.as_tensor(quats, dtype=torch.float32).contiguous().cpu()
    H = signs.shape[0]
    h = ctypes.c_void_p()
    if bits == 3:
        _check(lib().isoquant_init(ctypes.byref(h), H, head_dim, _ptr(signs), _ptr(quats)), "isoquant_init")
    else:
        _check(lib().isoquant_init_bits(ctypes.byref(h), H, head_dim, _ptr(signs), _ptr(quats), bits),
               "isoquant_init_bits")
    return Context(h, H, torch.cuda.current_device(), bits)


def isoquant_codebook(bits=3):
    n = 1 << bits
    lv = (ctypes.c_float * n)()
    th = (ctypes.c_float * (n - 1))()
    if bits == 3:
        _check(lib().isoquant_codebook(lv, th), "isoquant_codebook")
    else:
        _check(lib().isoquant_codebook_bits(bits, lv, th), "isoquant_codebook_bits")
    return list(lv), list(th)


def isoquant_cache_bytes(ctx, num_pages, page_size):
    cb, nb = ctypes.c_size_t(), ctypes.c_size_t()
    _check(lib().isoquant_cache_bytes(ctx.handle, num_pages, page_size, ctypes.byref(cb), ctypes.byref(nb)),
           "isoquant_cache_bytes")
    return cb.value, nb.value


def isoquant_compress_kv(ctx, cache, k, v, slot_mapping, stream=None):
    """k, v: [n_tok][H][128] (fp32/bf16/fp16, device); slot_mapping int64 [n_tok]."""
    assert k.is_contiguous() and v.is_contiguous() and slot_mapping.dtype == torch.int64
    cs = cache.c_struct()
    _check(lib().isoquant_compress_kv(ctx.handle, ctypes.byref(cs), _ptr(k), _ptr(v), _dtype(k), k.shape[0],
                                      _ptr(slot_mapping), _stream(stream)), "isoquant_compress_kv")


def isoquant_rotate_q(ctx, q, q_rot, stream=None):
    """q: [n_rows][Hq][128] (device); q_rot float32 same shape."""
    assert q.is_contiguous() and q_rot.is_contiguous() and q_rot.dtype == torch.float32
    _check(lib().isoquant_rotate_q(ctx.handle, _ptr(q), _dtype(q), q.shape[0], q.shape[1], _ptr(q_rot),
                                   _stream(stream)), "isoquant_rotate_q")


def isoquant_decode_prep(ctx, cache, k, v, slot_mapping, q, q_rot, stream=None):
    """Append k, v ([n_tok][H][128], device) at slot_mapping (int64 [n_tok])
    and rotate q ([n_rows][Hq][128], same dtype) into q_rot (float32, same
    shape), in one launch."""
    assert k.is_contiguous() and v.is_contiguous() and slot_mapping.dtype == torch.int64
    assert q.is_contiguous() and q_rot.is_contiguous() and q_rot.dtype == torch.float32
    assert k.dtype == v.dtype == q.dtype
    cs = cache.c_struct()
    _check(lib().isoquant_decode_prep(ctx.handle, ctypes.byref(cs), _ptr(k), _ptr(v), k.shape[0], _ptr(slot_mapping),
                                      _ptr(q), _dtype(q), q.shape[0], q.shape[1], _ptr(q_rot), _stream(stream)),
           "isoquant_decode_prep")


def isoquant_step_workspace_size(ctx, batch, nq, num_q_heads):
    n = ctypes.c_size_t()
    _check(lib().isoquant_step_workspace_size(ctx.handle, batch, nq, num_q_heads, ctypes.byref(n)),
           "isoquant_step_workspace_size")
    return n.value


def alloc_step_workspace(ctx, batch, nq, num_q_heads, device="cuda"):
    n = isoquant_step_workspace_size(ctx, batch, nq, num_q_heads)
    return torch.empty(((n + 15) // 16) * 4, dtype=torch.int32, device=device)


def isoquant_decode_step(ctx, cache, k, v, slot_mapping, q, page_table, seq_lens, workspace, out, causal=False,
                         scale=0.0, stream=None):
    """One decode step: append k, v (as isoquant_compress_kv), rotate q
    ([B][nq][Hq][128], same dtype as k), attend over seq_lens tokens (which
    count the appended ones) and write out (float32 [B][nq][Hq][128])."""
    assert k.is_contiguous() and v.is_contiguous() and slot_mapping.dtype == torch.int64
    assert q.is_contiguous() and q.dim() == 4 and k.dtype == v.dtype == q.dtype
    assert page_table.dtype == torch.int32 and page_table.is_contiguous() and seq_lens.dtype == torch.int32
    B, nq, Hq, _ = q.shape
    cs = cache.c_struct()
    _check(lib().isoquant_decode_step(ctx.handle, ctypes.byref(cs), _ptr(k), _ptr(v), k.shape[0], _ptr(slot_mapping),
                                      _ptr(q), _dtype(q), B, nq, Hq, _ptr(page_table), page_table.shape[1],
                                      _ptr(seq_lens), int(bool(causal)), float(scale), _ptr(workspace),
                                      workspace.numel() * workspace.element_size(), _ptr(out), _stream(stream)),
           "isoquant_decode_step")


def isoquant_workspace_size(ctx, batch, nq, num_q_heads):
    n = ctypes.c_size_t()
    _check(lib().isoquant_workspace_size(ctx.handle, batch, nq, num_q_heads, ctypes.byref(n)),
           "isoquant_workspace_size")
    return n.value


def isoquant_workspace_size_paged(ctx, batch, nq, num_q_heads, page_size):
    n = ctypes.c_size_t()
    _check(lib().isoquant_workspace_size_paged(ctx.handle, batch, nq, num_q_heads, page_size, ctypes.byref(n)),
           "isoquant_workspace_size_paged")
    return n.value


def alloc_workspace(ctx, batch, nq, num_q_heads, device="cuda", page_size=256):
    n = isoquant_workspace_size_paged(ctx, batch, nq, num_q_heads, page_size)
    return torch.empty(((n + 15) // 16) * 4, dtype=torch.int32, device=device)


def _attend_args(q_rot, page_table, seq_lens):
    assert q_rot.dtype == torch.float32 and q_rot.is_contiguous() and q_rot.dim() == 4
    assert page_table.dtype == torch.int32 and page_table.is_contiguous()
    assert seq_lens.dtype == torch.int32
    B, nq, Hq, _ = q_rot.shape
    return B, nq, Hq, page_table.shape[1]


def isoquant_attend_decode(ctx, cache, q_rot, page_table, seq_lens, workspace, out, causal=False, scale=0.0,
                           stream=None):
    """q_rot float32 [B][nq][Hq][128]; page_table int32 [B][max_pages];
    seq_lens int32 [B]; out float32 [B][nq][Hq][128]."""
    B, nq, Hq, maxp = _attend_args(q_rot, page_table, seq_lens)
    cs = cache.c_struct()
    _check(lib().isoquant_attend_decode(ctx.handle, ctypes.byref(cs), _ptr(q_rot), B, nq, Hq, _ptr(page_table), maxp,
                                        _ptr(seq_lens), int(bool(causal)), float(scale), _ptr(workspace),
                                        workspace.numel() * workspace.element_size(), _ptr(out), _stream(stream)),
           "isoquant_attend_decode")


def isoquant_attend_decode_static(ctx, cache, q_rot, page_table, seq_lens, out, causal=False, scale=0.0,
                                  stream=None):
    """isoquant_attend_decode for callers that cannot allocate device memory
    or lend a workspace: the split records go to a fixed 16 MiB array inside
    the library.  Its first call on a device must precede any stream
    capture; calls that overlap on the GPU race on the shared array."""
    B, nq, Hq, maxp = _attend_args(q_rot, page_table, seq_lens)
    cs = cache.c_struct()
    _check(lib().isoquant_attend_decode_static(ctx.handle, ctypes.byref(cs), _ptr(q_rot), B, nq, Hq,
                                               _ptr(page_table), maxp, _ptr(seq_lens), int(bool(causal)),
                                               float(scale), _ptr(out), _stream(stream)),
           "isoquant_attend_decode_static")


def isoquant_attend_partial(ctx, cache, q_rot, page_table, seq_lens, workspace, causal=False, scale=0.0,
                            stream=None):
    B, nq, Hq, maxp = _attend_args(q_rot, page_table, seq_lens)
    cs = cache.c_struct()
    _check(lib().isoquant_attend_partial(ctx.handle, ctypes.byref(cs), _ptr(q_rot), B, nq, Hq, _ptr(page_table),
                                         maxp, _ptr(seq_lens), int(bool(causal)), float(scale), _ptr(workspace),
                                         workspace.numel() * workspace.element_size(), _stream(stream)),
           "isoquant_attend_partial")


def isoquant_attend_combine(ctx, batch, nq, num_q_heads, seq_lens, page_size, workspace, out, stream=None):
    _check(lib().isoquant_attend_combine(ctx.handle, batch, nq, num_q_heads, _ptr(seq_lens), page_size,
                                         _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(out),
                                         _stream(stream)), "isoquant_attend_combine")


def isoquant_get_status(ctx, stream=None):
    s = ctypes.c_uint32()
    _check(lib().isoquant_get_status(ctx.handle, ctypes.byref(s), _stream(stream)), "isoquant_get_status")
    return s.value


def isoquant_selftest_wait(ctx, limit_ns, elapsed=None, stream=None):
    """Run the bounded-wait self-test: one device thread waits on a barrier
    that nothing completes and gives up after limit_ns, raising the timeout
    bit of the status word.  elapsed: optional int64 device tensor of one
    element that receives the measured wait in nanoseconds."""
    ptr = ctypes.c_void_p(0)
    if elapsed is not None:
        assert elapsed.dtype == torch.int64 and elapsed.numel() >= 1
        ptr = _ptr(elapsed)
    _check(lib().isoquant_selftest_wait(ctx.handle, int(limit_ns), ptr, _stream(stream)),
           "isoquant_selftest_wait")


def isoquant_debug_export_z(ctx, x, z, stream=None):
    """x: [n_tok][H][128] (fp32/bf16/fp16, device); z float32 same shape:
    the compress kernels' fp32 z = sqrt(128) (R x) / ||x|| (debug only)."""
    assert x.is_contiguous() and z.is_contiguous() and z.dtype == torch.float32 and z.shape == x.shape
    _check(lib().isoquant_debug_export_z(ctx.handle, _ptr(x), _dtype(x), x.shape[0], _ptr(z), _stream(stream)),
           "isoquant_debug_export_z")


def isoquant_last_launch_count(ctx):
    return lib().isoquant_last_launch_count(ctx.handle)
