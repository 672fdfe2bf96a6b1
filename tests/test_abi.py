"""The C-ABI library loads, exports every function include/sq.h declares, and
rejects bad arguments on the host before any CUDA call (CPU only)."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def sq():
    from w8a8_post_quantization_calibrate_b200 import build
    build.build()
    from w8a8_post_quantization_calibrate_b200 import sq as binding
    return binding


def test_header_symbols_exported(sq):
    names = sq.header_functions()
    assert "sq_w8a8_gemm" in names and "sq_linear" in names and len(names) >= 14
    lib = ctypes.CDLL(sq.LIB_PATH)
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing
    # ...and every exported sq_ function is declared in the header
    out = subprocess.run(["nm", "-D", "--defined-only", sq.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (sq_[a-z0-9_]+)\b", out))
    assert exported == set(names), (exported ^ set(names))


def test_binding_names_match_header(sq):
    for n in sq.header_functions():
        assert hasattr(sq, n), n


def test_version(sq):
    assert sq.sq_version() == 100


def test_host_argument_checks(sq):
    dummy = ctypes.c_void_p(0x1000)  # never dereferenced: every call below fails validation first
    st = ctypes.c_void_p(0)
    assert sq.raw_status("sq_calibrate_absmax", dummy, 7, 4, 16, dummy, st) == sq.SQ_ERR_UNSUPPORTED
    assert sq.raw_status("sq_calibrate_absmax", dummy, sq.SQ_BF16, 4, 17, dummy, st) == sq.SQ_ERR_UNSUPPORTED
    assert sq.raw_status("sq_calibrate_absmax", dummy, sq.SQ_BF16, -1, 16, dummy, st) == sq.SQ_ERR_INVALID_ARG
    assert sq.raw_status("sq_calibrate_absmax", None, sq.SQ_BF16, 4, 16, dummy, st) == sq.SQ_ERR_INVALID_ARG
    assert sq.raw_status("sq_calibrate_absmax", ctypes.c_void_p(0x1008), sq.SQ_BF16, 4, 16, dummy, st) \
        == sq.SQ_ERR_UNSUPPORTED
    assert sq.raw_status("sq_calibrate_absmax", dummy, sq.SQ_F32, 0, 16, dummy, st) == sq.SQ_OK  # no-op
    assert sq.raw_status("sq_smooth_factors", dummy, dummy, 16, ctypes.c_float(1.5), ctypes.c_float(1e-8),
                         dummy, st) == sq.SQ_ERR_INVALID_ARG
    assert sq.raw_status("sq_smooth_factors", dummy, dummy, 16, ctypes.c_float(0.5), ctypes.c_float(-1.0),
                         dummy, st) == sq.SQ_ERR_INVALID_ARG
    assert sq.raw_status("sq_smooth_factors", dummy, dummy, 16, ctypes.c_float(float("nan")),
                         ctypes.c_float(0.0), dummy, st) == sq.SQ_ERR_INVALID_ARG
    assert sq.raw_status("sq_fold_quant_weights", dummy, sq.SQ_I32, 8, 16, dummy, dummy, dummy, st) \
        == sq.SQ_ERR_UNSUPPORTED
    assert sq.raw_status("sq_fold_smooth_quant_pair", dummy, 8, dummy, 4, sq.SQ_I32, 16, dummy, dummy, dummy, dummy,
                         dummy, st) == sq.SQ_ERR_UNSUPPORTED
    assert sq.raw_status("sq_fold_smooth_quant_pair", dummy, 8, dummy, 4, sq.SQ_BF16, 24, dummy, dummy, dummy, dummy,
                         dummy, st) == sq.SQ_ERR_UNSUPPORTED
    assert sq.raw_status("sq_fold_smooth_quant_pair", dummy, 8, dummy, 4, sq.SQ_BF16, 16, None, dummy, dummy, dummy,
                         dummy, st) == sq.SQ_ERR_INVALID_ARG
    assert sq.raw_status("sq_fold_smooth_quant_pair", dummy, 0, dummy, 0, sq.SQ_BF16, 16, dummy, dummy, dummy, dummy,
                         dummy, st) == sq.SQ_OK   # no-op
    assert sq.raw_status("sq_fold_smooth_quant_pair_e4m3", dummy, 8, dummy, 4, sq.SQ_I32, 16, dummy, dummy, dummy,
                         dummy, dummy, st) == sq.SQ_ERR_UNSUPPORTED
    assert sq.raw_status("sq_fold_smooth_quant_pair_e4m3", dummy, 8, dummy, 4, sq.SQ_BF16, 24, dummy, dummy, dummy,
                         dummy, dummy, st) == sq.SQ_ERR_UNSUPPORTED
    assert sq.raw_status("sq_fold_smooth_quant_pair_e4m3", dummy, 8, dummy, 4, sq.SQ_BF16, 16, None, dummy, dummy,
                         dummy, dummy, st) == sq.SQ_ERR_INVALID_ARG
    assert sq.raw_status("sq_smooth_quant_act", dummy, sq.SQ_BF16, 8, 24, dummy, dummy, dummy, st) \
        == sq.SQ_ERR_UNSUPPORTED
    assert sq.raw_status("sq_smooth_quant_act", dummy, sq.SQ_BF16, 8, 16, None, dummy, dummy, st) \
        == sq.SQ_ERR_INVALID_ARG
    gemm = lambda M, N, K, out, ws=None, wsb=0: sq.raw_status(
        "sq_w8a8_gemm", dummy, dummy, dummy, dummy, M, N, K, dummy, out, ws, wsb, st)
    assert gemm(4, 4, 24, sq.SQ_BF16) == sq.SQ_ERR_UNSUPPORTED          # K % 16
    assert gemm(4, 4, 133152, sq.SQ_BF16) == sq.SQ_ERR_UNSUPPORTED      # int32 headroom
    assert gemm(4, 4, 16, 9) == sq.SQ_ERR_UNSUPPORTED                   # dtype
    assert gemm(-1, 4, 16, sq.SQ_F32) == sq.SQ_ERR_INVALID_ARG
    assert gemm(0, 4, 16, sq.SQ_F32) == sq.SQ_OK                        # empty
    assert gemm(4, 64, 16, sq.SQ_F32) == sq.SQ_ERR_INVALID_ARG          # decode path needs workspace
    assert sq.raw_status("sq_set_wait_timeout_ms", 0) == sq.SQ_ERR_INVALID_ARG
    assert sq.raw_status("sq_selftest_wait_timeout", 0, st) == sq.SQ_ERR_INVALID_ARG


def test_workspace_sizes(sq):
    # decode path (M <= 16): M*N int32 partial sums + 4 counters per 128-row tile, 256-aligned
    assert sq.sq_w8a8_gemm_workspace_size(16, 11008, 4096) == 16 * 11008 * 4 + 1536
    assert sq.sq_w8a8_gemm_workspace_size(1, 4096, 11008) == 16384 + 512
    assert sq.sq_w8a8_gemm_workspace_size(4096, 12288, 4096) == 0   # tiled path: none
    assert sq.sq_w8a8_gemm_workspace_size(0, 16, 16) == 0
    need = sq.sq_linear_workspace_size(64, 1024, 1024, sq.torch.float32, sq.torch.float32)
    assert need >= 64 * 1024 + 1024 * 1024 + 3 * 4096


def test_library_links_no_library_gemm(sq):
    """Every step and the alpha search's float product run in libsq's own
    kernels: the library needs no BLAS."""
    out = subprocess.run(["readelf", "-d", sq.LIB_PATH], capture_output=True, text=True).stdout
    needed = re.findall(r"\(NEEDED\)\s+Shared library: \[([^\]]+)\]", out)
    assert needed, out[:500]
    assert not [n for n in needed if "blas" in n.lower()], needed
