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
    "tensor_max_unsmoothed": 13,
    "norm_no_eps": 14,
    "norm_mean_abs": 15,
    "split_max_all": 16,
    "split_drop_outliers": 17,
    "e4m3_truncate": 18,
    "pow_exponent": 19,
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
            L.sqo_tensor_absmax.argtypes = [vp, ctypes.c_int, i64, i64, vp, vp]
            L.sqo_quant_act_per_tensor.argtypes = [vp, ctypes.c_int, i64, i64, vp, f32, vp, vp]
            L.sqo_fold_norm_gain.argtypes = [vp, ctypes.c_int, i64, vp, vp]
            L.sqo_rmsnorm_quant_act.argtypes = [vp, ctypes.c_int, i64, i64, vp, f32, vp, vp, vp, vp]
            L.sqo_outlier_split.argtypes = [vp, i64, f32, vp, vp]
            L.sqo_outlier_split.restype = i64
            L.sqo_quant_bulk.argtypes = [vp, ctypes.c_int, i64, i64, vp, vp, vp]
            L.sqo_gather_columns.argtypes = [vp, ctypes.c_int, i64, i64, vp, i64, i64, vp]
            L.sqo_dequant_split.argtypes = [vp, vp, vp, i64, i64, vp, vp, i64, i64, vp, vp, vp]
            L.sqo_e4m3_to_f64.argtypes = [ctypes.c_uint8]
            L.sqo_e4m3_to_f64.restype = f64
            L.sqo_e4m3_from_f64.argtypes = [f64]
            L.sqo_e4m3_from_f64.restype = ctypes.c_uint8
            L.sqo_quant_row_e4m3.argtypes = [vp, i64, vp, vp]
            L.sqo_quant_rows_e4m3_f64.argtypes = [vp, i64, i64, vp, vp]
            L.sqo_w8a8_e4m3_f64.argtypes = [vp, vp, vp, vp, i64, i64, i64, vp]
            L.sqo_fold_quant_weights_e4m3.argtypes = [vp, ctypes.c_int, i64, i64, vp, vp, vp]
            L.sqo_smooth_quant_act_e4m3.argtypes = [vp, ctypes.c_int, i64, i64, vp, vp, vp]
            L.sqo_gemm_dequant_e4m3.argtypes = [vp, vp, vp, vp, i64, i64, i64, vp, vp]
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


# ---------------------------------------------------------------- next steps
def _opt(a):
    return None if a is None else _p(a)


def tensor_absmax(x: np.ndarray, s: np.ndarray | None, amax: float = 0.0) -> np.float32:
    """Running max of |RN(x / s_j)| over a whole batch (s None: of |x|)."""
    x = np.ascontiguousarray(x)
    rows, cols = x.shape
    s = None if s is None else np.ascontiguousarray(s, dtype=np.float32)
    out = np.array([amax], np.float32)
    lib().sqo_tensor_absmax(_p(x), _dt(x), rows, cols, _opt(s), _p(out))
    return out[0]


def quant_act_per_tensor(x: np.ndarray, s: np.ndarray | None, amax: float):
    """Per-tensor int8 of RN(x / s) with range amax -> (codes [T,K], x_scale [T])."""
    x = np.ascontiguousarray(x)
    T, K = x.shape
    s = None if s is None else np.ascontiguousarray(s, dtype=np.float32)
    xq = np.empty((T, K), np.int8)
    xs = np.empty(T, np.float32)
    lib().sqo_quant_act_per_tensor(_p(x), _dt(x), T, K, _opt(s), float(np.float32(amax)), _p(xq), _p(xs))
    return xq, xs


def fold_norm_gain(g: np.ndarray, s: np.ndarray) -> np.ndarray:
    g = np.ascontiguousarray(g)
    s = np.ascontiguousarray(s, dtype=np.float32)
    gf = np.empty(s.shape[0], np.float32)
    lib().sqo_fold_norm_gain(_p(g), _dt(g), s.shape[0], _p(s), _p(gf))
    return gf


def rmsnorm_quant_act(x: np.ndarray, gf: np.ndarray, eps: float, r_in: np.ndarray | None = None):
    """RMSNorm(x; gain gf) then per-token int8 -> (codes, x_scale, r)."""
    x = np.ascontiguousarray(x)
    T, K = x.shape
    gf = np.ascontiguousarray(gf, dtype=np.float32)
    r_in = None if r_in is None else np.ascontiguousarray(r_in, dtype=np.float32)
    xq = np.empty((T, K), np.int8)
    xs = np.empty(T, np.float32)
    r = np.empty(T, np.float32)
    lib().sqo_rmsnorm_quant_act(_p(x), _dt(x), T, K, _p(gf), float(eps), _opt(r_in), _p(xq), _p(xs), _p(r))
    return xq, xs, r


def outlier_split(xmax: np.ndarray, threshold: float):
    """-> (keep float32 [K] of 1/0, outlier indices int32 ascending)."""
    xmax = np.ascontiguousarray(xmax, dtype=np.float32)
    K = xmax.shape[0]
    keep = np.empty(K, np.float32)
    idx = np.empty(K, np.int32)
    n = lib().sqo_outlier_split(_p(xmax), K, float(threshold), _p(keep), _p(idx))
    return keep, idx[:n].copy()


def quant_bulk(x: np.ndarray, keep: np.ndarray):
    x = np.ascontiguousarray(x)
    rows, K = x.shape
    keep = np.ascontiguousarray(keep, dtype=np.float32)
    q = np.empty((rows, K), np.int8)
    sc = np.empty(rows, np.float32)
    lib().sqo_quant_bulk(_p(x), _dt(x), rows, K, _p(keep), _p(q), _p(sc))
    return q, sc


def gather_columns(x: np.ndarray, idx: np.ndarray, ld: int | None = None) -> np.ndarray:
    x = np.ascontiguousarray(x)
    rows, K = x.shape
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    ld = idx.shape[0] if ld is None else ld
    out = np.empty((rows, ld), np.float32)
    lib().sqo_gather_columns(_p(x), _dt(x), rows, K, _p(idx), idx.shape[0], ld, _p(out))
    return out


def dequant_split(acc, x_scale, w_scale, x_out, w_out, n: int | None = None):
    """-> (y float32, y bf16 bits, magnitude |Y_bulk| + sum |x_out w_out| fp64)."""
    acc = np.ascontiguousarray(acc, dtype=np.int32)
    x_scale = np.ascontiguousarray(x_scale, dtype=np.float32)
    w_scale = np.ascontiguousarray(w_scale, dtype=np.float32)
    x_out = np.ascontiguousarray(x_out, dtype=np.float32)
    w_out = np.ascontiguousarray(w_out, dtype=np.float32)
    M, N = acc.shape
    ld = x_out.shape[1]
    assert w_out.shape == (N, ld) and x_out.shape[0] == M
    n = ld if n is None else n
    y = np.empty((M, N), np.float32)
    yb = np.empty((M, N), np.uint16)
    mag = np.empty((M, N), np.float64)
    lib().sqo_dequant_split(_p(acc), _p(x_scale), _p(w_scale), M, N, _p(x_out), _p(w_out), n, ld,
                            _p(y), _p(yb), _p(mag))
    return y, yb, mag


def linear_split(x: np.ndarray, w: np.ndarray, threshold: float, calib: list | None = None):
    """The decomposed layer on one batch: outlier set from the calibration
    maxima of x, bulk int8 of x and w, outlier columns in fp32."""
    xmax = np.zeros(x.shape[1], np.float32)
    for b in (calib if calib is not None else [x]):
        col_absmax(b, xmax)
    keep, idx = outlier_split(xmax, threshold)
    wq, w_scale = quant_bulk(w, keep)
    xq, x_scale = quant_bulk(x, keep)
    x_out = gather_columns(x, idx)
    w_out = gather_columns(w, idx)
    acc = gemm_i8(xq, wq)
    y, yb, mag = dequant_split(acc, x_scale, w_scale, x_out, w_out)
    return dict(xmax=xmax, keep=keep, idx=idx, wq=wq, w_scale=w_scale, xq=xq, x_scale=x_scale,
                x_out=x_out, w_out=w_out, acc=acc, y=y, y_bf16=yb, mag=mag)


def alpha_search(x: np.ndarray, w: np.ndarray, alphas, eps: float = 1e-8, calib: list | None = None):
    """W8A8 relative output error ||Yq - Y||_F / ||Y||_F of the fp32 path for
    each alpha (Y = X W^T in fp64) -> (errors list, best alpha). Ties go to
    the first alpha listed."""
    xf = x.astype(np.float64) if x.dtype != np.uint16 else _bf16_bits_to_f64(x)
    wf = w.astype(np.float64) if w.dtype != np.uint16 else _bf16_bits_to_f64(w)
    Y = matmul_xwT_f64(xf, wf)
    errs = []
    for a in alphas:
        out = linear(x, w, a, eps, calib)
        errs.append(rel_frobenius_f64(out["y"].astype(np.float64), Y))
    best = int(np.argmin(errs))
    return errs, alphas[best]


def _bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def e4m3_to_f64(b: np.ndarray) -> np.ndarray:
    f = np.vectorize(lambda v: lib().sqo_e4m3_to_f64(int(v)), otypes=[np.float64])
    return f(np.asarray(b, dtype=np.uint8))


def e4m3_from_f64(v: np.ndarray) -> np.ndarray:
    f = np.vectorize(lambda x: lib().sqo_e4m3_from_f64(float(x)), otypes=[np.uint8])
    return f(np.asarray(v, dtype=np.float64))


def quant_row_e4m3(v: np.ndarray):
    v = np.ascontiguousarray(v, dtype=np.float32)
    q = np.empty(v.shape[0], np.uint8)
    s = np.zeros(1, np.float32)
    lib().sqo_quant_row_e4m3(_p(v), v.shape[0], _p(q), _p(s))
    return q, s[0]


def quant_rows_e4m3_f64(v: np.ndarray):
    v = np.ascontiguousarray(v, dtype=np.float64)
    q = np.empty(v.shape, np.uint8)
    sc = np.empty(v.shape[0], np.float64)
    lib().sqo_quant_rows_e4m3_f64(_p(v), v.shape[0], v.shape[1], _p(q), _p(sc))
    return q, sc


def w8a8_e4m3_error_f64(X: np.ndarray, W: np.ndarray) -> float:
    """Relative output error with per-token FP8 E4M3 activations and
    per-output-channel FP8 E4M3 weights, fp64."""
    xq, sa = quant_rows_e4m3_f64(X)
    wq, sw = quant_rows_e4m3_f64(W)
    T, K = xq.shape
    N = wq.shape[0]
    Yq = np.empty((T, N), np.float64)
    lib().sqo_w8a8_e4m3_f64(_p(xq), _p(sa), _p(wq), _p(sw), T, N, K, _p(Yq))
    return rel_frobenius_f64(Yq, matmul_xwT_f64(X, W))


def w8a8_per_tensor_error_f64(X: np.ndarray, W: np.ndarray) -> float:
    """Relative output error with ONE activation scale for the whole tensor
    (the per-row quantizer applied to the flattened tensor) and
    per-output-channel weights, fp64."""
    T, K = X.shape
    xq, sa = quant_rows_f64(np.ascontiguousarray(X, dtype=np.float64).reshape(1, T * K))
    wq, sw = quant_rows_f64(W)
    N = wq.shape[0]
    Yq = np.empty((T, N), np.float64)
    lib().sqo_w8a8_f64(_p(xq.reshape(T, K)), _p(np.full(T, sa[0])), _p(wq), _p(sw), T, N, K, _p(Yq))
    return rel_frobenius_f64(Yq, matmul_xwT_f64(X, W))


def fold_quant_weights_e4m3(w: np.ndarray, s: np.ndarray):
    w = np.ascontiguousarray(w)
    s = np.ascontiguousarray(s, dtype=np.float32)
    N, K = w.shape
    wq = np.empty((N, K), np.uint8)
    ws = np.empty(N, np.float32)
    lib().sqo_fold_quant_weights_e4m3(_p(w), _dt(w), N, K, _p(s), _p(wq), _p(ws))
    return wq, ws


def smooth_quant_act_e4m3(x: np.ndarray, s: np.ndarray):
    x = np.ascontiguousarray(x)
    s = np.ascontiguousarray(s, dtype=np.float32)
    T, K = x.shape
    xq = np.empty((T, K), np.uint8)
    xs = np.empty(T, np.float32)
    lib().sqo_smooth_quant_act_e4m3(_p(x), _dt(x), T, K, _p(s), _p(xq), _p(xs))
    return xq, xs


def gemm_dequant_e4m3(xq, x_scale, wq, w_scale):
    """-> (y float32 [M, N], magnitude sum |products| * scales, fp64)."""
    xq = np.ascontiguousarray(xq, dtype=np.uint8)
    wq = np.ascontiguousarray(wq, dtype=np.uint8)
    x_scale = np.ascontiguousarray(x_scale, dtype=np.float32)
    w_scale = np.ascontiguousarray(w_scale, dtype=np.float32)
    M, K = xq.shape
    N = wq.shape[0]
    y = np.empty((M, N), np.float32)
    mag = np.empty((M, N), np.float64)
    lib().sqo_gemm_dequant_e4m3(_p(xq), _p(x_scale), _p(wq), _p(w_scale), M, N, K, _p(y), _p(mag))
    return y, mag
