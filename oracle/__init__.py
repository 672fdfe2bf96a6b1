"""CPU oracle for the SmoothQuant W8A8 linear layer -- TEST INFRASTRUCTURE.

Only the test suite, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU
baseline / reference arm may import this package. The product path (the CUDA
library ``libsq.so`` and its Python binding) never does, and shares no code with
it.

The arithmetic lives in ``sq_oracle.c`` (plain C, fp32 in the pages' order with
FMA contraction off, fp64 for the identity/error experiments). This module only
builds that file and marshals numpy arrays into it. bf16 tensors are passed as
their raw uint16 bit patterns.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sq_oracle.c")
_LIB = os.path.join(_HERE, "libsq_oracle.so")

F32 = 0
BF16 = 1

# planted-mistake codes of sq_oracle.c (tests only)
MUTATIONS = {
    "round_half_away": 1,
    "recip_scale": 2,
    "no_clamp": 3,
    "alpha_swapped": 4,
    "smooth_multiply": 5,
    "gemm_transposed_w": 6,
    "dequant_drop_sw": 7,
    "no_zero_guard": 8,
    "scale_128": 9,
    "fold_divides": 10,
    "colmax_no_abs": 11,
    "smooth_wrong_index": 12,
}

_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile sq_oracle.c into libsq_oracle.so (gcc, -O2, no FMA contraction)."""
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC):
        return _LIB
    cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
           "-fPIC", "-shared", "-o", _LIB + ".tmp", _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def lib():
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = ctypes.CDLL(_LIB)
            vp, i64, f32, f64 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_float, ctypes.c_double
            L.sqo_set_mutation.argtypes = [ctypes.c_int]
            L.sqo_get_mutation.restype = ctypes.c_int
            L.sqo_bf16_to_f32.argtypes = [ctypes.c_uint16]
            L.sqo_bf16_to_f32.restype = f32
            L.sqo_f32_to_bf16_rne.argtypes = [f32]
            L.sqo_f32_to_bf16_rne.restype = ctypes.c_uint16
            L.sqo_quant_row.argtypes = [vp, i64, vp, vp]
            L.sqo_quant_fixed.argtypes = [vp, i64, f32, vp]
            L.sqo_col_absmax.argtypes = [vp, ctypes.c_int, i64, i64, vp]
            L.sqo_smooth_factors.argtypes = [vp, vp, i64, f32, f32, vp]
            L.sqo_fold_quant_weights.argtypes = [vp, ctypes.c_int, i64, i64, vp, vp, vp]
            L.sqo_smooth_quant_act.argtypes = [vp, ctypes.c_int, i64, i64, vp, vp, vp]
            L.sqo_gemm_i8.argtypes = [vp, vp, i64, i64, i64, vp]
            L.sqo_gemm_i8.restype = i64
            L.sqo_dequant.argtypes = [vp, vp, vp, i64, i64, vp, vp]
            L.sqo_matmul_xwT_f64.argtypes = [vp, vp, i64, i64, i64, vp]
            L.sqo_col_absmax_f64.argtypes = [vp, i64, i64, vp]
            L.sqo_smooth_factors_f64.argtypes = [vp, vp, i64, f64, f64, vp]
            L.sqo_smooth_f64.argtypes = [vp, vp, vp, i64, i64, i64, vp, vp]
            L.sqo_quant_rows_f64.argtypes = [vp, i64, i64, vp, vp]
            L.sqo_w8a8_f64.argtypes = [vp, vp, vp, vp, i64, i64, i64, vp]
            L.sqo_rel_frobenius_f64.argtypes = [vp, vp, i64]
            L.sqo_rel_frobenius_f64.restype = f64
            L.sqo_num_threads.restype = ctypes.c_int
            L.sqo_set_num_threads.argtypes = [ctypes.c_int]
            _lib = L
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _dt(a: np.ndarray) -> int:
    if a.dtype == np.float32:
        return F32
    if a.dtype == np.uint16:
        return BF16
    raise TypeError(f"oracle input must be float32 or uint16 (bf16 bits), got {a.dtype}")


# ---------------------------------------------------------------- controls
def set_mutation(name_or_code) -> None:
    code = MUTATIONS[name_or_code] if isinstance(name_or_code, str) else int(name_or_code)
    lib().sqo_set_mutation(code)


def num_threads() -> int:
    return lib().sqo_num_threads()


def set_num_threads(n: int) -> None:
    lib().sqo_set_num_threads(int(n))


# ---------------------------------------------------------------- scalars
def bf16_to_f32(bits: int) -> float:
    return lib().sqo_bf16_to_f32(bits)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    f = np.vectorize(lambda v: lib().sqo_f32_to_bf16_rne(float(v)), otypes=[np.uint16])
    return f(x)


# ---------------------------------------------------------------- fp32 path
def quant_row(v: np.ndarray):
    """Dynamic symmetric int8 of one row -> (codes int8[K], scale float32)."""
    v = np.ascontiguousarray(v, dtype=np.float32)
    q = np.empty(v.shape[0], np.int8)
    s = np.zeros(1, np.float32)
    lib().sqo_quant_row(_p(v), v.shape[0], _p(q), _p(s))
    return q, s[0]


def quant_fixed(v: np.ndarray, scale: float) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float32)
    q = np.empty(v.size, np.int8)
    lib().sqo_quant_fixed(_p(v), v.size, float(scale), _p(q))
    return q.reshape(v.shape)


def col_absmax(x: np.ndarray, absmax: np.ndarray | None = None) -> np.ndarray:
    """Running per-column max |x| over the rows of a 2-D float32 / bf16-bits array."""
    x = np.ascontiguousarray(x)
    rows, cols = x.shape
    out = np.zeros(cols, np.float32) if absmax is None else absmax
    assert out.dtype == np.float32 and out.shape == (cols,)
    lib().sqo_col_absmax(_p(x), _dt(x), rows, cols, _p(out))
    return out


def smooth_factors(xmax: np.ndarray, wmax: np.ndarray, alpha: float, eps: float = 1e-8) -> np.ndarray:
    xmax = np.ascontiguousarray(xmax, dtype=np.float32)
    wmax = np.ascontiguousarray(wmax, dtype=np.float32)
    s = np.empty_like(xmax)
    lib().sqo_smooth_factors(_p(xmax), _p(wmax), xmax.shape[0], float(alpha), float(eps), _p(s))
    return s


def fold_quant_weights(w: np.ndarray, s: np.ndarray):
    w = np.ascontiguousarray(w)
    s = np.ascontiguousarray(s, dtype=np.float32)
    N, K = w.shape
    wq = np.empty((N, K), np.int8)
    ws = np.empty(N, np.float32)
    lib().sqo_fold_quant_weights(_p(w), _dt(w), N, K, _p(s), _p(wq), _p(ws))
    return wq, ws


def smooth_quant_act(x: np.ndarray, s: np.ndarray):
    x = np.ascontiguousarray(x)
    s = np.ascontiguousarray(s, dtype=np.float32)
    T, K = x.shape
    xq = np.empty((T, K), np.int8)
    xs = np.empty(T, np.float32)
    lib().sqo_smooth_quant_act(_p(x), _dt(x), T, K, _p(s), _p(xq), _p(xs))
    return xq, xs


def gemm_i8(xq: np.ndarray, wq: np.ndarray) -> np.ndarray:
    xq = np.ascontiguousarray(xq, dtype=np.int8)
    wq = np.ascontiguousarray(wq, dtype=np.int8)
    M, K = xq.shape
    N, K2 = wq.shape
    assert K == K2
    acc = np.empty((M, N), np.int32)
    over = lib().sqo_gemm_i8(_p(xq), _p(wq), M, N, K, _p(acc))
    if over:
        raise OverflowError(f"{over} accumulators do not fit in int32")
    return acc


def dequant(acc: np.ndarray, x_scale: np.ndarray, w_scale: np.ndarray):
    """-> (y float32 [M,N], y bf16 bits uint16 [M,N])."""
    acc = np.ascontiguousarray(acc, dtype=np.int32)
    x_scale = np.ascontiguousarray(x_scale, dtype=np.float32)
    w_scale = np.ascontiguousarray(w_scale, dtype=np.float32)
    M, N = acc.shape
    y = np.empty((M, N), np.float32)
    yb = np.empty((M, N), np.uint16)
    lib().sqo_dequant(_p(acc), _p(x_scale), _p(w_scale), M, N, _p(y), _p(yb))
    return y, yb


def linear(x: np.ndarray, w: np.ndarray, alpha: float, eps: float = 1e-8,
           calib: list | None = None):
    """The whole fp32 path on one batch: a1 (on `calib` batches if given, else
    on x) and on w, a2, a3, a4, a5. Returns a dict of every intermediate."""
    xmax = np.zeros(x.shape[1], np.float32)
    for b in (calib if calib is not None else [x]):
        col_absmax(b, xmax)
    wmax = col_absmax(w)
    s = smooth_factors(xmax, wmax, alpha, eps)
    wq, w_scale = fold_quant_weights(w, s)
    xq, x_scale = smooth_quant_act(x, s)
    acc = gemm_i8(xq, wq)
    y, yb = dequant(acc, x_scale, w_scale)
    return dict(xmax=xmax, wmax=wmax, s=s, wq=wq, w_scale=w_scale, xq=xq, x_scale=x_scale,
                acc=acc, y=y, y_bf16=yb)


# ---------------------------------------------------------------- fp64 path
def matmul_xwT_f64(X: np.ndarray, W: np.ndarray) -> np.ndarray:
    X = np.ascontiguousarray(X, dtype=np.float64)
    W = np.ascontiguousarray(W, dtype=np.float64)
    T, K = X.shape
    N = W.shape[0]
    Y = np.empty((T, N), np.float64)
    lib().sqo_matmul_xwT_f64(_p(X), _p(W), T, N, K, _p(Y))
    return Y


def col_absmax_f64(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.zeros(x.shape[1], np.float64)
    lib().sqo_col_absmax_f64(_p(x), x.shape[0], x.shape[1], _p(out))
    return out


def smooth_factors_f64(xmax: np.ndarray, wmax: np.ndarray, alpha: float, eps: float = 0.0):
    xmax = np.ascontiguousarray(xmax, dtype=np.float64)
    wmax = np.ascontiguousarray(wmax, dtype=np.float64)
    s = np.empty_like(xmax)
    lib().sqo_smooth_factors_f64(_p(xmax), _p(wmax), xmax.shape[0], float(alpha), float(eps), _p(s))
    return s


def smooth_f64(X: np.ndarray, W: np.ndarray, s: np.ndarray):
    X = np.ascontiguousarray(X, dtype=np.float64)
    W = np.ascontiguousarray(W, dtype=np.float64)
    s = np.ascontiguousarray(s, dtype=np.float64)
    Xs = np.empty_like(X)
    Ws = np.empty_like(W)
    lib().sqo_smooth_f64(_p(X), _p(W), _p(s), X.shape[0], W.shape[0], X.shape[1], _p(Xs), _p(Ws))
    return Xs, Ws


def quant_rows_f64(v: np.ndarray):
    v = np.ascontiguousarray(v, dtype=np.float64)
    q = np.empty(v.shape, np.int8)
    sc = np.empty(v.shape[0], np.float64)
    lib().sqo_quant_rows_f64(_p(v), v.shape[0], v.shape[1], _p(q), _p(sc))
    return q, sc


def w8a8_f64(X: np.ndarray, W: np.ndarray) -> np.ndarray:
    """Yq = per-token int8(X) x per-output-channel int8(W)^T, dequantized in fp64."""
    xq, sa = quant_rows_f64(X)
    wq, sw = quant_rows_f64(W)
    T, K = xq.shape
    N = wq.shape[0]
    Yq = np.empty((T, N), np.float64)
    lib().sqo_w8a8_f64(_p(xq), _p(sa), _p(wq), _p(sw), T, N, K, _p(Yq))
    return Yq


def rel_frobenius_f64(Yq: np.ndarray, Y: np.ndarray) -> float:
    Yq = np.ascontiguousarray(Yq, dtype=np.float64)
    Y = np.ascontiguousarray(Y, dtype=np.float64)
    return lib().sqo_rel_frobenius_f64(_p(Yq), _p(Y), Y.size)


def w8a8_error_f64(X: np.ndarray, W: np.ndarray, Y: np.ndarray | None = None) -> float:
    """W8A8 relative output error ||Yq - Y||_F / ||Y||_F with Y = X W^T."""
    if Y is None:
        Y = matmul_xwT_f64(X, W)
    return rel_frobenius_f64(w8a8_f64(X, W), Y)
