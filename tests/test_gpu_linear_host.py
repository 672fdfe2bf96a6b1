"""sq_linear, the whole layer in one call, on the bench's path: pinned host
bf16 operands at the 7B QKV prefill shape (X [4096 x 4096], W [12288 x 4096],
bf16 Y), so the call stages its inputs on the library's copy stream, runs the
calibration pair launch, the streamed row kernel's pair launch (a3 + a4) and
the paired-SM GEMM, and copies Y back.

Three calls back to back through one workspace, with different inputs each
time and no synchronization in between (each call's input copies overlap the
previous call's GEMM and output copy). Every Y is compared with the oracle on
sampled rows (bf16 within 1 ulp; the kernels do the oracle's fp32 operations,
so the test also expects bit equality) and with the step-by-step device path
in full; the last call's maxima, factors, codes and scales, read from the
workspace, are compared with the oracle's in full, bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import assert_bf16_within_ulp, assert_bitexact_f32, assert_equal, host
from w8a8_post_quantization_calibrate_b200 import synth

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from w8a8_post_quantization_calibrate_b200 import sq  # noqa: E402

DEV = torch.device("cuda", 0)


def _oracle_steps(hx, hw, alpha):
    xmax = oracle.col_absmax(hx)
    wmax = oracle.col_absmax(hw)
    s = oracle.smooth_factors(xmax, wmax, alpha)
    wq, wsc = oracle.fold_quant_weights(hw, s)
    xq, xsc = oracle.smooth_quant_act(hx, s)
    return dict(xmax=xmax, wmax=wmax, s=s, wq=wq, w_scale=wsc, xq=xq, x_scale=xsc)


def test_sq_linear_pinned_host_bf16_qkv_prefill_back_to_back():
    wl = synth.WORKLOADS["qkv_prefill_7b"]
    M, N, K = wl.T, wl.N, wl.K
    x0, w0 = synth.make("qkv_prefill_7b")
    # other inputs of the same recipe: fresh activation draws, another weight draw
    x1 = synth.activations(M, K, wl.outliers, wl.seed, wl.in_dtype, stream=21)
    x2 = synth.activations(M, K, wl.outliers, wl.seed + 7, wl.in_dtype, stream=22)
    w2 = synth.weights(N, K, wl.w_std, wl.seed, wl.in_dtype, stream=23)
    calls = [(x0, w0), (x1, w0), (x2, w2)]
    pinned = [(x.pin_memory(), w.pin_memory(), torch.empty((M, N), dtype=torch.bfloat16).pin_memory())
              for x, w in calls]
    ws = torch.zeros(sq.sq_linear_workspace_size(M, N, K, torch.bfloat16, torch.bfloat16),
                     dtype=torch.uint8, device=DEV)
    stream = torch.cuda.current_stream(DEV)
    for xh, wh, yh in pinned:
        sq.sq_linear(xh, wh, wl.alpha, out_dtype=torch.bfloat16, y=yh, workspace=ws, stream=stream)
    torch.cuda.synchronize(DEV)
    assert sq.sq_get_status() == sq.SQ_OK

    rng = np.random.default_rng(4)
    rows = np.unique(np.concatenate([[0, 1, 127, 128, 255, 256, M - 1], rng.choice(M, 41, replace=False)]))
    last = None
    for i, ((x, w), (_, _, yh)) in enumerate(zip(calls, pinned)):
        hx, hw = synth.host_array(x), synth.host_array(w)
        ref = _oracle_steps(hx, hw, wl.alpha)
        acc = oracle.gemm_i8(np.ascontiguousarray(ref["xq"][rows]), ref["wq"])
        _, y16 = oracle.dequant(acc, ref["x_scale"][rows], ref["w_scale"])
        got = synth.host_array(yh)
        exact = assert_bf16_within_ulp(got[rows], y16, f"call {i}: Y rows vs oracle")
        assert exact == y16.size, f"call {i}: {y16.size - exact} of {y16.size} sampled outputs not bit-equal"
        # the same call's Y in full against the step-by-step device path
        xd, wd = x.to(DEV), w.to(DEV)
        xmax = torch.zeros(K, device=DEV)
        wmax = torch.zeros(K, device=DEV)
        sq.sq_calibrate_absmax(xd, xmax)
        sq.sq_calibrate_absmax(wd, wmax)
        s = sq.sq_smooth_factors(xmax, wmax, wl.alpha)
        wq, wsc = sq.sq_fold_quant_weights(wd, s)
        xq, xsc = sq.sq_smooth_quant_act(xd, s)
        y_steps = host(sq.sq_w8a8_gemm(xq, xsc, wq, wsc, out_dtype=torch.bfloat16))
        assert_equal(got, y_steps, f"call {i}: Y vs the step-by-step path")
        last = ref
    views = sq.sq_linear_workspace_views(ws, M, N, K, torch.bfloat16, torch.bfloat16)
    for name in ("xmax", "wmax", "s", "x_scale", "w_scale"):
        assert_bitexact_f32(host(views[name]), last[name], f"last call: {name}")
    for name in ("xq", "wq"):
        assert_equal(host(views[name]), last[name], f"last call: {name}")
