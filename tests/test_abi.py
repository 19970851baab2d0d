"""The C-ABI library loads on a machine without a GPU, exports every symbol
declared in include/isoquant.h, and its host-only parts behave (CPU only:
no device work is started here)."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    with open(os.path.join(ROOT, "include", "isoquant.h")) as f:
        text = f.read()
    return sorted(set(re.findall(r"^\s*(?:int|void|const char \*)\s*\*?\s*(isoquant_\w+)\s*\(", text, re.M)))


@pytest.fixture(scope="module")
def native():
    from compressed_space_decode_b200 import build
    build.build()
    import compressed_space_decode_b200 as csd
    return csd


def test_header_declares_the_four_calls():
    syms = declared_symbols()
    for name in ("isoquant_init", "isoquant_compress_kv", "isoquant_rotate_q", "isoquant_attend_decode"):
        assert name in syms


def test_library_exports_every_declared_symbol(native):
    L = native.lib()
    for name in declared_symbols():
        assert hasattr(L, name), name
    assert sorted(native.SYMBOLS) == declared_symbols()


def test_codebook_matches_oracle(native):
    lv, th = native.isoquant_codebook()
    ol, ot = oracle.codebook()
    np.testing.assert_array_equal(np.array(lv, dtype=np.float64), ol)
    np.testing.assert_array_equal(np.array(th, dtype=np.float64), ot)


def test_strerror_and_argument_errors(native):
    L = native.lib()
    assert native.strerror(0) == "ok"
    assert "workspace" in native.strerror(-4)
    h = ctypes.c_void_p()
    signs = np.ones((1, 128), np.int8)
    quats = np.zeros((1, 32, 2, 4), np.float32)
    quats[..., 0] = 1
    # rejected on the host before any CUDA call
    assert L.isoquant_init(None, 1, 128, signs.ctypes.data, quats.ctypes.data) == -1
    assert L.isoquant_init(ctypes.byref(h), 1, 64, signs.ctypes.data, quats.ctypes.data) == -2
    assert L.isoquant_init(ctypes.byref(h), 0, 128, signs.ctypes.data, quats.ctypes.data) == -1
    bad = signs.copy()
    bad[0, 3] = 0
    assert L.isoquant_init(ctypes.byref(h), 1, 128, bad.ctypes.data, quats.ctypes.data) == -1
    zq = np.zeros_like(quats)
    assert L.isoquant_init(ctypes.byref(h), 1, 128, signs.ctypes.data, zq.ctypes.data) == -1
    assert L.isoquant_compress_kv(None, None, None, None, 0, 1, None, None) == -1
    assert L.isoquant_attend_decode(None, None, None, 1, 1, 8, None, 1, None, 0, 0.0, None, 0, None, None) == -1


def test_every_entry_rejects_a_null_context(native):
    """Calls given no context (or no output pointer) return INVALID_ARG on
    the host, before any CUDA call; width checks return UNSUPPORTED."""
    L = native.lib()
    sz = ctypes.c_size_t()
    st = ctypes.c_uint32()
    lv = (ctypes.c_float * 16)()
    th = (ctypes.c_float * 16)()
    assert L.isoquant_codebook(None, None) == -1
    assert L.isoquant_codebook_bits(3, None, th) == -1
    assert L.isoquant_codebook_bits(5, lv, th) == -2
    assert L.isoquant_codebook_bits(1, lv, th) == -2
    assert L.isoquant_codebook_bits(2, lv, th) == 0 and L.isoquant_codebook_bits(4, lv, th) == 0
    h = ctypes.c_void_p()
    signs = np.ones((1, 128), np.int8)
    quats = np.zeros((1, 32, 2, 4), np.float32)
    quats[..., 0] = 1
    assert L.isoquant_init_bits(ctypes.byref(h), 1, 128, signs.ctypes.data, quats.ctypes.data, 5) == -2
    assert L.isoquant_init_bits(ctypes.byref(h), 1, 128, signs.ctypes.data, quats.ctypes.data, 1) == -2
    nanq = quats.copy()
    nanq[0, 5, 1, 2] = np.nan
    assert L.isoquant_init_bits(ctypes.byref(h), 1, 128, signs.ctypes.data, nanq.ctypes.data, 3) == -1
    assert L.isoquant_cache_bytes(None, 4, 256, ctypes.byref(sz), ctypes.byref(sz)) == -1
    assert L.isoquant_rotate_q(None, None, 0, 1, 8, None, None) == -1
    assert L.isoquant_decode_prep(None, None, None, None, 1, None, None, 0, 1, 8, None, None) == -1
    assert L.isoquant_workspace_size(None, 1, 1, 8, ctypes.byref(sz)) == -1
    assert L.isoquant_step_workspace_size(None, 1, 1, 8, ctypes.byref(sz)) == -1
    assert L.isoquant_attend_partial(None, None, None, 1, 1, 8, None, 1, None, 0, 0.0, None, 0, None) == -1
    assert L.isoquant_attend_combine(None, 1, 1, 8, None, 256, None, 0, None, None) == -1
    assert L.isoquant_attend_decode_static(None, None, None, 1, 1, 8, None, 1, None, 0, 0.0, None, None) == -1
    assert L.isoquant_decode_step(None, None, None, None, 1, None, None, 0, 1, 1, 8, None, 1, None, 0, 0.0,
                                  None, 0, None, None) == -1
    assert L.isoquant_get_status(None, ctypes.byref(st), None) == -1
    assert L.isoquant_selftest_wait(None, 1000, None, None) == -1
    assert L.isoquant_debug_export_z(None, None, 1, 1, None, None) == -1
    assert L.isoquant_workspace_size_paged(None, 1, 1, 8, 256, ctypes.byref(sz)) == -1
    assert L.isoquant_last_launch_count(None) == 0
    for code in (0, -1, -2, -3, -4, -5, -6):
        assert native.strerror(code)


def test_nvtx_build_compiles(tmp_path):
    """The optional NVTX-traced build (-DISOQUANT_NVTX) of the C-ABI unit
    compiles and pulls in the NVTX ranges."""
    import shutil
    import subprocess
    nvcc = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
    if not os.path.exists(nvcc) and shutil.which("nvcc") is None:
        pytest.skip("no nvcc")
    obj = tmp_path / "api_nvtx.o"
    subprocess.check_call([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", "-Xcompiler",
                           "-fPIC", "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include"), "-DISOQUANT_NVTX",
                           "-c", "-o", str(obj), os.path.join(ROOT, "compressed_space_decode_b200", "csrc", "api.cu")])
    syms = subprocess.run(["nm", str(obj)], capture_output=True, text=True).stdout
    assert "nvtx" in syms.lower()
