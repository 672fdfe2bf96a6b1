"""Thin Python binding of libsq (include/sq.h): argument marshalling only.

Every function has the name of the C entry point it calls. Tensors are torch
CUDA tensors (device memory and the current stream come from PyTorch); outputs
not supplied by the caller are allocated with torch. All computation happens in
libsq's kernels: importing this module loads libsq.so and raises if it has not
been built -- there is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# SQ_LIBRARY=debug loads the -DSQ_DEBUG build (index checks in the kernels)
LIB_PATH = os.path.join(_PKG, "libsq_debug.so" if os.environ.get("SQ_LIBRARY") == "debug" else "libsq.so")
HEADER = os.path.join(os.path.dirname(_PKG), "include", "sq.h")

SQ_OK, SQ_ERR_INVALID_ARG, SQ_ERR_UNSUPPORTED, SQ_ERR_CUDA, SQ_ERR_TIMEOUT, SQ_ERR_BOUNDS = 0, 1, 2, 3, 4, 5
SQ_F32, SQ_BF16, SQ_I32 = 0, 1, 2
STATUS_NAMES = {0: "SQ_OK", 1: "SQ_ERR_INVALID_ARG", 2: "SQ_ERR_UNSUPPORTED", 3: "SQ_ERR_CUDA",
                4: "SQ_ERR_TIMEOUT", 5: "SQ_ERR_BOUNDS"}


class SqError(RuntimeError):
    def __init__(self, status: int, where: str, message: str):
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


if not os.path.exists(LIB_PATH):
    raise ImportError(f"{os.path.basename(LIB_PATH)} is not built ({LIB_PATH}); run "
                      "`python -m w8a8_post_quantization_calibrate_b200.build`"
                      + (" --debug" if LIB_PATH.endswith("_debug.so") else ""))

_lib = ctypes.CDLL(LIB_PATH)
_vp, _i64, _f32, _sz, _int = ctypes.c_void_p, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t, ctypes.c_int

_SIGS = {
    "sq_version": ([], _int),
    "sq_calibrate_absmax": ([_vp, _int, _i64, _i64, _vp, _vp], _int),
    "sq_smooth_factors": ([_vp, _vp, _i64, _f32, _f32, _vp, _vp], _int),
    "sq_fold_quant_weights": ([_vp, _int, _i64, _i64, _vp, _vp, _vp, _vp], _int),
    "sq_smooth_quant_act": ([_vp, _int, _i64, _i64, _vp, _vp, _vp, _vp], _int),
    "sq_calibrate_absmax_pair": ([_vp, _i64, _vp, _i64, _int, _i64, _vp, _vp, _vp], _int),
    "sq_fold_smooth_quant_pair": ([_vp, _i64, _vp, _i64, _int, _i64, _vp, _vp, _vp, _vp, _vp, _vp], _int),
    "sq_fold_smooth_quant_pair_e4m3": ([_vp, _i64, _vp, _i64, _int, _i64, _vp, _vp, _vp, _vp, _vp, _vp], _int),
    "sq_fold_quant_weights_e4m3": ([_vp, _int, _i64, _i64, _vp, _vp, _vp, _vp], _int),
    "sq_smooth_quant_act_e4m3": ([_vp, _int, _i64, _i64, _vp, _vp, _vp, _vp], _int),
    "sq_w8a8_gemm_e4m3": ([_vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp, _int, _vp], _int),
    "sq_tensor_absmax": ([_vp, _int, _i64, _i64, _vp, _vp, _vp], _int),
    "sq_quant_act_per_tensor": ([_vp, _int, _i64, _i64, _vp, _vp, _vp, _vp, _vp], _int),
    "sq_fold_norm_gain": ([_vp, _int, _i64, _vp, _vp, _vp], _int),
    "sq_rmsnorm_quant_act": ([_vp, _int, _i64, _i64, _vp, _f32, _vp, _vp, _vp, _vp], _int),
    "sq_outlier_split": ([_vp, _i64, _f32, _vp, _vp, _vp, _vp], _int),
    "sq_quant_bulk": ([_vp, _int, _i64, _i64, _vp, _vp, _vp, _vp], _int),
    "sq_gather_columns": ([_vp, _int, _i64, _i64, _vp, _i64, _i64, _vp, _vp], _int),
    "sq_w8a8_gemm_split": ([_vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp, _vp, _i64, _vp, _int, _vp, _sz, _vp],
                           _int),
    "sq_alpha_search_workspace_size": ([_i64, _i64, _i64, _i64], _sz),
    "sq_alpha_search": ([_vp, _vp, _int, _i64, _i64, _i64, _vp, _i64, _f32, _vp, _vp, _vp, _sz, _vp], _int),
    "sq_w8a8_gemm_workspace_size": ([_i64, _i64, _i64], _sz),
    "sq_w8a8_gemm": ([_vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp, _int, _vp, _sz, _vp], _int),
    "sq_w8a8_gemm_noalloc": ([_vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp, _int, _vp], _int),
    "sq_linear_workspace_size": ([_i64, _i64, _i64, _int, _int], _sz),
    "sq_linear_workspace_offsets": ([_i64, _i64, _i64, _int, _int, _vp], _int),
    "sq_linear": ([_vp, _vp, _int, _i64, _i64, _i64, _f32, _f32, _vp, _int, _vp, _sz, _vp], _int),
    "sq_get_status": ([_vp], _int),
    "sq_last_status_site": ([], ctypes.c_uint),
    "sq_last_error_string": ([], ctypes.c_char_p),
    "sq_set_wait_timeout_ms": ([_i64], _int),
    "sq_selftest_wait_timeout": ([_i64, _vp], _int),
    "sq_selftest_dirty_noalloc_scratch": ([_vp], _int),
    "sq_probe_tensor_int8": ([_i64, _vp, _vp, _vp], _int),
}
for _name, (_args, _res) in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.argtypes = _args
    _fn.restype = _res


def header_functions() -> list[str]:
    """Names of the functions include/sq.h declares."""
    with open(HEADER) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sq_[a-z0-9_]+)\s*\(", text)))


def _check(status: int, where: str) -> None:
    if status != SQ_OK:
        msg = _lib.sq_last_error_string().decode(errors="replace")
        raise SqError(status, where, msg)


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return SQ_F32
    if t.dtype == torch.bfloat16:
        return SQ_BF16
    if t.dtype == torch.int32:
        return SQ_I32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _torch_dtype(code: int):
    return {SQ_F32: torch.float32, SQ_BF16: torch.bfloat16, SQ_I32: torch.int32}[code]


def _dev(t: torch.Tensor, name: str) -> int:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def sq_version() -> int:
    return _lib.sq_version()


def sq_calibrate_absmax(x: torch.Tensor, absmax: torch.Tensor, stream=None) -> torch.Tensor:
    """Running per-column max |x| into `absmax` (float32 [cols], in/out)."""
    rows, cols = x.shape
    _check(_lib.sq_calibrate_absmax(_dev(x, "x"), _dt(x), rows, cols, _dev(absmax, "absmax"),
                                    _stream(stream)), "sq_calibrate_absmax")
    return absmax


def sq_smooth_factors(xmax: torch.Tensor, wmax: torch.Tensor, alpha: float, eps: float = 1e-8,
                      s: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    K = xmax.shape[0]
    if s is None:
        s = torch.empty(K, dtype=torch.float32, device=xmax.device)
    _check(_lib.sq_smooth_factors(_dev(xmax, "xmax"), _dev(wmax, "wmax"), K, float(alpha), float(eps),
                                  _dev(s, "s"), _stream(stream)), "sq_smooth_factors")
    return s


def sq_fold_quant_weights(w: torch.Tensor, s: torch.Tensor, wq: torch.Tensor | None = None,
                          w_scale: torch.Tensor | None = None, stream=None):
    N, K = w.shape
    if wq is None:
        wq = torch.empty((N, K), dtype=torch.int8, device=w.device)
    if w_scale is None:
        w_scale = torch.empty(N, dtype=torch.float32, device=w.device)
    _check(_lib.sq_fold_quant_weights(_dev(w, "w"), _dt(w), N, K, _dev(s, "s"), _dev(wq, "wq"),
                                      _dev(w_scale, "w_scale"), _stream(stream)), "sq_fold_quant_weights")
    return wq, w_scale


def sq_smooth_quant_act(x: torch.Tensor, s: torch.Tensor, xq: torch.Tensor | None = None,
                        x_scale: torch.Tensor | None = None, stream=None):
    T, K = x.shape
    if xq is None:
        xq = torch.empty((T, K), dtype=torch.int8, device=x.device)
    if x_scale is None:
        x_scale = torch.empty(T, dtype=torch.float32, device=x.device)
    _check(_lib.sq_smooth_quant_act(_dev(x, "x"), _dt(x), T, K, _dev(s, "s"), _dev(xq, "xq"),
                                    _dev(x_scale, "x_scale"), _stream(stream)), "sq_smooth_quant_act")
    return xq, x_scale


def sq_calibrate_absmax_pair(x: torch.Tensor, w: torch.Tensor, xmax: torch.Tensor, wmax: torch.Tensor,
                             stream=None):
    """Running column maxima of x into xmax and of w into wmax, one launch."""
    T, K = x.shape
    N = w.shape[0]
    if x.dtype != w.dtype:
        raise TypeError("x and w must have the same dtype")
    _check(_lib.sq_calibrate_absmax_pair(_dev(x, "x"), T, _dev(w, "w"), N, _dt(x), K, _dev(xmax, "xmax"),
                                         _dev(wmax, "wmax"), _stream(stream)), "sq_calibrate_absmax_pair")
    return xmax, wmax


def sq_fold_smooth_quant_pair(w: torch.Tensor, x: torch.Tensor, s: torch.Tensor, wq=None, w_scale=None, xq=None,
                              x_scale=None, stream=None):
    """a3 on w and a4 on x with the same s, in one launch where possible ->
    (wq, w_scale, xq, x_scale)."""
    N, K = w.shape
    T = x.shape[0]
    if x.dtype != w.dtype:
        raise TypeError("x and w must have the same dtype")
    if wq is None:
        wq = torch.empty((N, K), dtype=torch.int8, device=w.device)
    if w_scale is None:
        w_scale = torch.empty(N, dtype=torch.float32, device=w.device)
    if xq is None:
        xq = torch.empty((T, K), dtype=torch.int8, device=x.device)
    if x_scale is None:
        x_scale = torch.empty(T, dtype=torch.float32, device=x.device)
    _check(_lib.sq_fold_smooth_quant_pair(_dev(w, "w"), N, _dev(x, "x"), T, _dt(w), K, _dev(s, "s"), _dev(wq, "wq"),
                                          _dev(w_scale, "w_scale"), _dev(xq, "xq"), _dev(x_scale, "x_scale"),
                                          _stream(stream)), "sq_fold_smooth_quant_pair")
    return wq, w_scale, xq, x_scale


def sq_fold_smooth_quant_pair_e4m3(w: torch.Tensor, x: torch.Tensor, s: torch.Tensor, wq=None, w_scale=None,
                                   xq=None, x_scale=None, stream=None):
    """FP8 E4M3 codes of w (folded) and x (smoothed) in one launch where
    possible -> (wq uint8, w_scale, xq uint8, x_scale)."""
    N, K = w.shape
    T = x.shape[0]
    if x.dtype != w.dtype:
        raise TypeError("x and w must have the same dtype")
    if wq is None:
        wq = torch.empty((N, K), dtype=torch.uint8, device=w.device)
    if w_scale is None:
        w_scale = torch.empty(N, dtype=torch.float32, device=w.device)
    if xq is None:
        xq = torch.empty((T, K), dtype=torch.uint8, device=x.device)
    if x_scale is None:
        x_scale = torch.empty(T, dtype=torch.float32, device=x.device)
    _check(_lib.sq_fold_smooth_quant_pair_e4m3(_dev(w, "w"), N, _dev(x, "x"), T, _dt(w), K, _dev(s, "s"),
                                               _dev(wq, "wq"), _dev(w_scale, "w_scale"), _dev(xq, "xq"),
                                               _dev(x_scale, "x_scale"), _stream(stream)),
           "sq_fold_smooth_quant_pair_e4m3")
    return wq, w_scale, xq, x_scale


def sq_fold_quant_weights_e4m3(w: torch.Tensor, s: torch.Tensor, wq=None, w_scale=None, stream=None):
    """Fold s into W, per-output-channel FP8 E4M3 -> (codes uint8 [N, K], w_scale)."""
    N, K = w.shape
    if wq is None:
        wq = torch.empty((N, K), dtype=torch.uint8, device=w.device)
    if w_scale is None:
        w_scale = torch.empty(N, dtype=torch.float32, device=w.device)
    _check(_lib.sq_fold_quant_weights_e4m3(_dev(w, "w"), _dt(w), N, K, _dev(s, "s"), _dev(wq, "wq"),
                                           _dev(w_scale, "w_scale"), _stream(stream)), "sq_fold_quant_weights_e4m3")
    return wq, w_scale


def sq_smooth_quant_act_e4m3(x: torch.Tensor, s: torch.Tensor, xq=None, x_scale=None, stream=None):
    """Smooth X by s, per-token FP8 E4M3 -> (codes uint8 [T, K], x_scale)."""
    T, K = x.shape
    if xq is None:
        xq = torch.empty((T, K), dtype=torch.uint8, device=x.device)
    if x_scale is None:
        x_scale = torch.empty(T, dtype=torch.float32, device=x.device)
    _check(_lib.sq_smooth_quant_act_e4m3(_dev(x, "x"), _dt(x), T, K, _dev(s, "s"), _dev(xq, "xq"),
                                         _dev(x_scale, "x_scale"), _stream(stream)), "sq_smooth_quant_act_e4m3")
    return xq, x_scale


def sq_w8a8_gemm_e4m3(xq: torch.Tensor, x_scale: torch.Tensor, wq: torch.Tensor, w_scale: torch.Tensor,
                      out_dtype=torch.bfloat16, y: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    M, K = xq.shape
    N = wq.shape[0]
    if y is None:
        y = torch.empty((M, N), dtype=out_dtype, device=xq.device)
    _check(_lib.sq_w8a8_gemm_e4m3(_dev(xq, "xq"), _dev(x_scale, "x_scale"), _dev(wq, "wq"), _dev(w_scale, "w_scale"),
                                  M, N, K, _dev(y, "y"), _dt(y), _stream(stream)), "sq_w8a8_gemm_e4m3")
    return y


def _opt_dev(t: torch.Tensor | None, name: str):
    return None if t is None else _dev(t, name)


def sq_tensor_absmax(x: torch.Tensor, s: torch.Tensor | None, amax: torch.Tensor | None = None,
                     stream=None) -> torch.Tensor:
    """Running per-tensor max |x / s_j| into `amax` (float32 [1], in/out; a
    fresh zero tensor if not given). s None: max |x|."""
    rows, cols = x.shape
    if amax is None:
        amax = torch.zeros(1, dtype=torch.float32, device=x.device)
    _check(_lib.sq_tensor_absmax(_dev(x, "x"), _dt(x), rows, cols, _opt_dev(s, "s"), _dev(amax, "amax"),
                                 _stream(stream)), "sq_tensor_absmax")
    return amax


def sq_quant_act_per_tensor(x: torch.Tensor, s: torch.Tensor | None, amax: torch.Tensor,
                            xq: torch.Tensor | None = None, x_scale: torch.Tensor | None = None,
                            stream=None):
    T, K = x.shape
    if xq is None:
        xq = torch.empty((T, K), dtype=torch.int8, device=x.device)
    if x_scale is None:
        x_scale = torch.empty(T, dtype=torch.float32, device=x.device)
    _check(_lib.sq_quant_act_per_tensor(_dev(x, "x"), _dt(x), T, K, _opt_dev(s, "s"), _dev(amax, "amax"),
                                        _dev(xq, "xq"), _dev(x_scale, "x_scale"), _stream(stream)),
           "sq_quant_act_per_tensor")
    return xq, x_scale


def sq_fold_norm_gain(gain: torch.Tensor, s: torch.Tensor, gain_folded: torch.Tensor | None = None,
                      stream=None) -> torch.Tensor:
    K = gain.shape[0]
    if gain_folded is None:
        gain_folded = torch.empty(K, dtype=torch.float32, device=gain.device)
    _check(_lib.sq_fold_norm_gain(_dev(gain, "gain"), _dt(gain), K, _dev(s, "s"),
                                  _dev(gain_folded, "gain_folded"), _stream(stream)), "sq_fold_norm_gain")
    return gain_folded


def sq_rmsnorm_quant_act(x: torch.Tensor, gain_folded: torch.Tensor, eps: float,
                         xq: torch.Tensor | None = None, x_scale: torch.Tensor | None = None,
                         inv_rms: torch.Tensor | None = None, want_inv_rms: bool = True, stream=None):
    """RMSNorm with the folded gain, then per-token int8 -> (xq, x_scale, inv_rms or None)."""
    T, K = x.shape
    if xq is None:
        xq = torch.empty((T, K), dtype=torch.int8, device=x.device)
    if x_scale is None:
        x_scale = torch.empty(T, dtype=torch.float32, device=x.device)
    if inv_rms is None and want_inv_rms:
        inv_rms = torch.empty(T, dtype=torch.float32, device=x.device)
    _check(_lib.sq_rmsnorm_quant_act(_dev(x, "x"), _dt(x), T, K, _dev(gain_folded, "gain_folded"),
                                     float(eps), _dev(xq, "xq"), _dev(x_scale, "x_scale"),
                                     _opt_dev(inv_rms, "inv_rms"), _stream(stream)), "sq_rmsnorm_quant_act")
    return xq, x_scale, inv_rms


def sq_w8a8_gemm_workspace_size(M: int, N: int, K: int) -> int:
    return int(_lib.sq_w8a8_gemm_workspace_size(M, N, K))


_ws_cache: dict = {}


def gemm_workspace(M: int, N: int, K: int, device) -> torch.Tensor | None:
    """A zero-filled workspace for sq_w8a8_gemm, cached per (device, size);
    calls that complete leave it zero-filled, as the C API requires."""
    need = sq_w8a8_gemm_workspace_size(M, N, K)
    if need == 0:
        return None
    key = (str(device), need)
    ws = _ws_cache.get(key)
    if ws is None:
        ws = torch.zeros(need, dtype=torch.uint8, device=device)
        _ws_cache[key] = ws
    return ws


def sq_w8a8_gemm(xq: torch.Tensor, x_scale: torch.Tensor | None, wq: torch.Tensor,
                 w_scale: torch.Tensor | None, out_dtype=torch.bfloat16, y: torch.Tensor | None = None,
                 workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    M, K = xq.shape
    N = wq.shape[0]
    if y is None:
        y = torch.empty((M, N), dtype=out_dtype, device=xq.device)
    if workspace is None:
        workspace = gemm_workspace(M, N, K, xq.device)
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(_lib.sq_w8a8_gemm(_dev(xq, "xq"), x_scale.data_ptr() if x_scale is not None else None,
                             _dev(wq, "wq"), w_scale.data_ptr() if w_scale is not None else None,
                             M, N, K, _dev(y, "y"), _dt(y), ws_ptr, ws_bytes, _stream(stream)),
           "sq_w8a8_gemm")
    return y


def sq_w8a8_gemm_noalloc(xq: torch.Tensor, x_scale: torch.Tensor | None, wq: torch.Tensor,
                         w_scale: torch.Tensor | None, out_dtype=torch.bfloat16, y: torch.Tensor | None = None,
                         stream=None) -> torch.Tensor:
    """Decode GEMM (1 <= M <= 16) for callers that cannot allocate device
    memory: libsq keeps the scratch in a fixed array of its own. Only `y`, if
    not given, is allocated here (by torch, for the convenience of Python
    callers); the C call itself allocates nothing."""
    M, K = xq.shape
    N = wq.shape[0]
    for name, t in (("wq", wq), ("x_scale", x_scale), ("w_scale", w_scale), ("y", y)):
        if t is not None and t.device != xq.device:
            raise ValueError(f"{name} is on {t.device}, xq on {xq.device}")
    # the C call takes the scratch of the current device: make it xq's
    with torch.cuda.device(xq.device):
        if y is None:
            y = torch.empty((M, N), dtype=out_dtype, device=xq.device)
        _check(_lib.sq_w8a8_gemm_noalloc(_dev(xq, "xq"), x_scale.data_ptr() if x_scale is not None else None,
                                         _dev(wq, "wq"), w_scale.data_ptr() if w_scale is not None else None,
                                         M, N, K, _dev(y, "y"), _dt(y), _stream(stream)),
               "sq_w8a8_gemm_noalloc")
    return y


def sq_selftest_dirty_noalloc_scratch(stream=None) -> None:
    _check(_lib.sq_selftest_dirty_noalloc_scratch(_stream(stream)), "sq_selftest_dirty_noalloc_scratch")


def sq_outlier_split(xmax: torch.Tensor, threshold: float, keep: torch.Tensor | None = None,
                     idx: torch.Tensor | None = None, count: torch.Tensor | None = None, stream=None):
    """-> (keep float32 [K], idx int32 [K] (first `count` valid), count int32 [1]), all on the device."""
    K = xmax.shape[0]
    if keep is None:
        keep = torch.empty(K, dtype=torch.float32, device=xmax.device)
    if idx is None:
        idx = torch.empty(max(K, 1), dtype=torch.int32, device=xmax.device)
    if count is None:
        count = torch.empty(1, dtype=torch.int32, device=xmax.device)
    _check(_lib.sq_outlier_split(_dev(xmax, "xmax"), K, float(threshold), _dev(keep, "keep"), _dev(idx, "idx"),
                                 _dev(count, "count"), _stream(stream)), "sq_outlier_split")
    return keep, idx, count


def sq_quant_bulk(x: torch.Tensor, keep: torch.Tensor, q: torch.Tensor | None = None,
                  scale: torch.Tensor | None = None, stream=None):
    rows, K = x.shape
    if q is None:
        q = torch.empty((rows, K), dtype=torch.int8, device=x.device)
    if scale is None:
        scale = torch.empty(rows, dtype=torch.float32, device=x.device)
    _check(_lib.sq_quant_bulk(_dev(x, "x"), _dt(x), rows, K, _dev(keep, "keep"), _dev(q, "q"),
                              _dev(scale, "scale"), _stream(stream)), "sq_quant_bulk")
    return q, scale


def sq_gather_columns(x: torch.Tensor, idx: torch.Tensor, n: int, ld: int, out: torch.Tensor | None = None,
                      stream=None) -> torch.Tensor:
    rows, K = x.shape
    if out is None:
        out = torch.empty((rows, ld), dtype=torch.float32, device=x.device)
    _check(_lib.sq_gather_columns(_dev(x, "x"), _dt(x), rows, K, _dev(idx, "idx"), int(n), int(ld),
                                  _dev(out, "out"), _stream(stream)), "sq_gather_columns")
    return out


def sq_w8a8_gemm_split(xq: torch.Tensor, x_scale: torch.Tensor, wq: torch.Tensor, w_scale: torch.Tensor,
                       x_out: torch.Tensor, w_out: torch.Tensor, out_dtype=torch.bfloat16,
                       y: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                       stream=None) -> torch.Tensor:
    M, K = xq.shape
    N = wq.shape[0]
    ld = x_out.shape[1]
    if y is None:
        y = torch.empty((M, N), dtype=out_dtype, device=xq.device)
    if workspace is None:
        workspace = gemm_workspace(M, N, K, xq.device)
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(_lib.sq_w8a8_gemm_split(_dev(xq, "xq"), _dev(x_scale, "x_scale"), _dev(wq, "wq"),
                                   _dev(w_scale, "w_scale"), M, N, K, _dev(x_out, "x_out"), _dev(w_out, "w_out"),
                                   ld, _dev(y, "y"), _dt(y), ws_ptr, ws_bytes, _stream(stream)),
           "sq_w8a8_gemm_split")
    return y


def sq_alpha_search_workspace_size(T: int, N: int, K: int, n_alpha: int) -> int:
    return int(_lib.sq_alpha_search_workspace_size(T, N, K, n_alpha))


def sq_alpha_search(x: torch.Tensor, w: torch.Tensor, alphas, eps: float = 1e-8,
                    workspace: torch.Tensor | None = None, stream=None):
    """W8A8 relative output error for each alpha on the calibration batch x
    -> (errors list of float, best alpha). Synchronizes the stream."""
    T, K = x.shape
    N = w.shape[0]
    if x.dtype != w.dtype:
        raise TypeError("x and w must have the same dtype")
    a = (ctypes.c_float * len(alphas))(*[float(v) for v in alphas])
    err = (ctypes.c_double * len(alphas))()
    best = ctypes.c_float(0.0)
    need = sq_alpha_search_workspace_size(T, N, K, len(alphas))
    if workspace is None:
        workspace = torch.zeros(need, dtype=torch.uint8, device=x.device)
    _check(_lib.sq_alpha_search(_dev(x, "x"), _dev(w, "w"), _dt(x), T, N, K, ctypes.cast(a, _vp), len(alphas),
                                float(eps), ctypes.cast(err, _vp), ctypes.cast(ctypes.pointer(best), _vp),
                                workspace.data_ptr(), workspace.numel(), _stream(stream)), "sq_alpha_search")
    return list(err), float(best.value)


def sq_linear_workspace_size(M: int, N: int, K: int, in_dtype=torch.bfloat16, out_dtype=torch.bfloat16) -> int:
    return int(_lib.sq_linear_workspace_size(M, N, K, _dt(torch.empty(0, dtype=in_dtype)),
                                             _dt(torch.empty(0, dtype=out_dtype))))


LINEAR_WORKSPACE_PARTS = ("xmax", "wmax", "s", "xq", "x_scale", "wq", "w_scale")


def sq_linear_workspace_offsets(M: int, N: int, K: int, in_dtype=torch.bfloat16,
                                out_dtype=torch.bfloat16) -> dict:
    """Byte offsets of sq_linear's intermediates inside its workspace."""
    off = (ctypes.c_size_t * len(LINEAR_WORKSPACE_PARTS))()
    _check(_lib.sq_linear_workspace_offsets(M, N, K, _dt(torch.empty(0, dtype=in_dtype)),
                                            _dt(torch.empty(0, dtype=out_dtype)), ctypes.cast(off, _vp)),
           "sq_linear_workspace_offsets")
    return dict(zip(LINEAR_WORKSPACE_PARTS, (int(v) for v in off)))


def sq_linear_workspace_views(workspace: torch.Tensor, M: int, N: int, K: int, in_dtype=torch.bfloat16,
                              out_dtype=torch.bfloat16) -> dict:
    """Tensor views of sq_linear's intermediates (maxima, factors, codes and
    scales) inside a workspace it has used."""
    off = sq_linear_workspace_offsets(M, N, K, in_dtype, out_dtype)
    shapes = {"xmax": ((K,), torch.float32), "wmax": ((K,), torch.float32), "s": ((K,), torch.float32),
              "xq": ((M, K), torch.int8), "x_scale": ((M,), torch.float32),
              "wq": ((N, K), torch.int8), "w_scale": ((N,), torch.float32)}
    views = {}
    for name, (shape, dt) in shapes.items():
        n = 1
        for d in shape:
            n *= d
        nbytes = n * torch.empty(0, dtype=dt).element_size()
        views[name] = workspace[off[name]:off[name] + nbytes].view(dt).view(shape)
    return views


def sq_linear(x: torch.Tensor, w: torch.Tensor, alpha: float, eps: float = 1e-8,
              out_dtype=torch.bfloat16, y: torch.Tensor | None = None,
              workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """The whole path (a1..a5) on one batch. x, w and y may be CUDA tensors or
    (pinned) host tensors; host operands are staged through the workspace."""
    M, K = x.shape
    N = w.shape[0]
    if x.dtype != w.dtype:
        raise TypeError("x and w must have the same dtype")
    if not (x.is_contiguous() and w.is_contiguous()):
        raise ValueError("x and w must be contiguous")
    dev = x.device if x.is_cuda else (w.device if w.is_cuda else torch.device("cuda", torch.cuda.current_device()))
    if y is None:
        y = torch.empty((M, N), dtype=out_dtype, device=dev)
    need = sq_linear_workspace_size(M, N, K, x.dtype, y.dtype)
    if workspace is None:
        workspace = torch.zeros(need, dtype=torch.uint8, device=dev)
    _check(_lib.sq_linear(x.data_ptr(), w.data_ptr(), _dt(x), M, N, K, float(alpha), float(eps),
                          y.data_ptr(), _dt(y), workspace.data_ptr(), workspace.numel(), _stream(stream)),
           "sq_linear")
    return y


def sq_get_status(stream=None) -> int:
    """Synchronize the stream and return (and clear) the device status word."""
    return int(_lib.sq_get_status(_stream(stream)))


def sq_last_status_site() -> int:
    return int(_lib.sq_last_status_site())


def sq_last_error_string() -> str:
    return _lib.sq_last_error_string().decode(errors="replace")


def sq_set_wait_timeout_ms(ms: int) -> None:
    _check(_lib.sq_set_wait_timeout_ms(int(ms)), "sq_set_wait_timeout_ms")


def sq_selftest_wait_timeout(limit_us: int, stream=None) -> None:
    _check(_lib.sq_selftest_wait_timeout(int(limit_us), _stream(stream)), "sq_selftest_wait_timeout")


def sq_probe_tensor_int8(iters: int, clocks: torch.Tensor | None = None, stream=None) -> float:
    """Launch the int8 tensor-core rate probe; returns the int8 operations the
    launch performs (time it with CUDA events on the stream). `clocks`, a
    CUDA int64 tensor of 2 entries if given, receives one SM's cycles and
    nanoseconds over the MMAs."""
    ops = ctypes.c_double(0.0)
    _check(_lib.sq_probe_tensor_int8(int(iters), ctypes.cast(ctypes.pointer(ops), _vp),
                                     None if clocks is None else _dev(clocks, "clocks"), _stream(stream)),
           "sq_probe_tensor_int8")
    return float(ops.value)


def raw_status(fn_name: str, *args) -> int:
    """Call a C entry point with raw ctypes arguments and return its status
    (tests of the host-side argument checks)."""
    return int(getattr(_lib, fn_name)(*args))
