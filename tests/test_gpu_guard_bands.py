"""No entry point writes outside its output buffers: every output of every
call sits between guard bands of a seeded byte pattern (tests/gpu_helpers.py,
Guarded), on ragged shapes that leave partial tiles, partial chunks and rows
shorter than a lane's share, and the bands are compared after the call. The
values themselves are checked against the oracle by the parity tests; here the
outputs are also compared once with the oracle, so a call that wrote nothing
fails too."""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import Guarded, assert_bitexact_f32, assert_equal, host
from w8a8_post_quantization_calibrate_b200 import synth

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from w8a8_post_quantization_calibrate_b200 import sq  # noqa: E402

DEV = torch.device("cuda", 0)
# (260, 600, 16400): the paired GEMM's 512-column tiles, N and K ragged
SHAPES = [(1, 3, 16), (5, 7, 48), (13, 129, 1040), (130, 257, 2064), (17, 300, 5136), (3, 5, 28672),
          (260, 600, 16400)]


def _xw(T, N, K, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(T, K, generator=g)
    x[:, torch.randperm(K, generator=g)[:3]] *= 40.0
    w = torch.randn(N, K, generator=g) * 0.05
    return x.to(dtype), w.to(dtype)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("T,N,K", SHAPES)
def test_steps_stay_inside_their_outputs(dtype, T, N, K):
    x, w = _xw(T, N, K, dtype, seed=T * 31 + N + K)
    hx, hw = synth.host_array(x), synth.host_array(w)
    xd, wd = x.to(DEV), w.to(DEV)
    xmax, wmax = Guarded((K,), torch.float32, DEV, seed=1), Guarded((K,), torch.float32, DEV, seed=2)
    xmax.t.zero_()
    wmax.t.zero_()
    sq.sq_calibrate_absmax_pair(xd, wd, xmax.t, wmax.t)
    xmax.check("calibrate_absmax_pair xmax")
    wmax.check("calibrate_absmax_pair wmax")
    s = Guarded((K,), torch.float32, DEV, seed=3)
    sq.sq_smooth_factors(xmax.t, wmax.t, 0.5, s=s.t)
    s.check("smooth_factors")
    wq, wsc = Guarded((N, K), torch.int8, DEV, seed=4), Guarded((N,), torch.float32, DEV, seed=5)
    xq, xsc = Guarded((T, K), torch.int8, DEV, seed=6), Guarded((T,), torch.float32, DEV, seed=7)
    sq.sq_fold_smooth_quant_pair(wd, xd, s.t, wq=wq.t, w_scale=wsc.t, xq=xq.t, x_scale=xsc.t)
    for b, n in ((wq, "wq"), (wsc, "w_scale"), (xq, "xq"), (xsc, "x_scale")):
        b.check(f"fold_smooth_quant_pair {n}")
    o_s = oracle.smooth_factors(oracle.col_absmax(hx), oracle.col_absmax(hw), 0.5)
    assert_bitexact_f32(host(s.t), o_s, "s")
    o_wq, _ = oracle.fold_quant_weights(hw, o_s)
    o_xq, _ = oracle.smooth_quant_act(hx, o_s)
    assert_equal(host(wq.t), o_wq, "wq")
    assert_equal(host(xq.t), o_xq, "xq")
    # the separate steps too
    sq.sq_fold_quant_weights(wd, s.t, wq=wq.t, w_scale=wsc.t)
    sq.sq_smooth_quant_act(xd, s.t, xq=xq.t, x_scale=xsc.t)
    for b, n in ((wq, "wq"), (wsc, "w_scale"), (xq, "xq"), (xsc, "x_scale")):
        b.check(f"separate steps {n}")
    for out_dtype in (torch.float32, torch.bfloat16, torch.int32):
        y = Guarded((T, N), out_dtype, DEV, seed=8)
        scales = (xsc.t, wsc.t) if out_dtype != torch.int32 else (None, None)
        sq.sq_w8a8_gemm(xq.t, scales[0], wq.t, scales[1], out_dtype=out_dtype, y=y.t)
        y.check(f"w8a8_gemm {out_dtype}")
        if out_dtype == torch.int32:
            assert_equal(host(y.t), oracle.gemm_i8(o_xq, o_wq), "acc")
    assert sq.sq_get_status() == sq.SQ_OK


@pytest.mark.parametrize("T,N,K", [(1, 3, 16), (5, 7, 48), (16, 300, 1040), (200, 257, 2064), (260, 600, 16384)])
def test_variants_stay_inside_their_outputs(T, N, K):
    x, w = _xw(T, N, K, torch.bfloat16, seed=T + N + K)
    xd, wd = x.to(DEV), w.to(DEV)
    s = torch.rand(K, device=DEV) * 4.0 + 0.25
    amax = Guarded((1,), torch.float32, DEV, seed=9)
    amax.t.zero_()
    sq.sq_tensor_absmax(xd, s, amax.t)
    amax.check("tensor_absmax")
    xq, xsc = Guarded((T, K), torch.int8, DEV, seed=10), Guarded((T,), torch.float32, DEV, seed=11)
    sq.sq_quant_act_per_tensor(xd, s, amax.t, xq=xq.t, x_scale=xsc.t)
    xq.check("quant_act_per_tensor xq")
    xsc.check("quant_act_per_tensor x_scale")
    gain = torch.rand(K, device=DEV) + 0.5
    gf = Guarded((K,), torch.float32, DEV, seed=12)
    sq.sq_fold_norm_gain(gain, s, gain_folded=gf.t)
    gf.check("fold_norm_gain")
    r = Guarded((T,), torch.float32, DEV, seed=13)
    sq.sq_rmsnorm_quant_act(xd, gf.t, 1e-5, xq=xq.t, x_scale=xsc.t, inv_rms=r.t)
    for b, n in ((xq, "xq"), (xsc, "x_scale"), (r, "inv_rms")):
        b.check(f"rmsnorm_quant_act {n}")
    xmax = torch.zeros(K, device=DEV)
    sq.sq_calibrate_absmax(xd, xmax)
    keep, idx, count = (Guarded((K,), torch.float32, DEV, seed=14), Guarded((K,), torch.int32, DEV, seed=15),
                        Guarded((1,), torch.int32, DEV, seed=16))
    sq.sq_outlier_split(xmax, 6.0, keep=keep.t, idx=idx.t, count=count.t)
    for b, n in ((keep, "keep"), (idx, "idx"), (count, "count")):
        b.check(f"outlier_split {n}")
    n_out = int(count.t.item())
    ld = max(4, (n_out + 3) // 4 * 4)
    wq, wsc = Guarded((N, K), torch.int8, DEV, seed=17), Guarded((N,), torch.float32, DEV, seed=18)
    sq.sq_quant_bulk(wd, keep.t, q=wq.t, scale=wsc.t)
    sq.sq_quant_bulk(xd, keep.t, q=xq.t, scale=xsc.t)
    for b, n in ((wq, "bulk wq"), (wsc, "bulk w_scale"), (xq, "bulk xq"), (xsc, "bulk x_scale")):
        b.check(n)
    xo, wo = Guarded((T, ld), torch.float32, DEV, seed=19), Guarded((N, ld), torch.float32, DEV, seed=20)
    sq.sq_gather_columns(xd, idx.t, n_out, ld, out=xo.t)
    sq.sq_gather_columns(wd, idx.t, n_out, ld, out=wo.t)
    xo.check("gather x")
    wo.check("gather w")
    y = Guarded((T, N), torch.bfloat16, DEV, seed=21)
    sq.sq_w8a8_gemm_split(xq.t, xsc.t, wq.t, wsc.t, xo.t, wo.t, out_dtype=torch.bfloat16, y=y.t)
    y.check("w8a8_gemm_split")
    wq8, xq8 = Guarded((N, K), torch.uint8, DEV, seed=22), Guarded((T, K), torch.uint8, DEV, seed=23)
    sq.sq_fold_smooth_quant_pair_e4m3(wd, xd, s, wq=wq8.t, w_scale=wsc.t, xq=xq8.t, x_scale=xsc.t)
    for b, n in ((wq8, "e4m3 wq"), (xq8, "e4m3 xq"), (wsc, "e4m3 w_scale"), (xsc, "e4m3 x_scale")):
        b.check(n)
    y8 = Guarded((T, N), torch.float32, DEV, seed=24)
    sq.sq_w8a8_gemm_e4m3(xq8.t, xsc.t, wq8.t, wsc.t, out_dtype=torch.float32, y=y8.t)
    y8.check("w8a8_gemm_e4m3")
    y2 = Guarded((T, N), torch.bfloat16, DEV, seed=25)
    if T <= 16 and T * N <= 262144:
        sq.sq_w8a8_gemm_noalloc(xq.t, xsc.t, wq.t, wsc.t, out_dtype=torch.bfloat16, y=y2.t)
        y2.check("w8a8_gemm_noalloc")
    assert sq.sq_get_status() == sq.SQ_OK


def test_sq_linear_stays_inside_its_output_and_workspace():
    T, N, K = 37, 300, 4112
    x, w = _xw(T, N, K, torch.bfloat16, seed=5)
    need = sq.sq_linear_workspace_size(T, N, K, torch.bfloat16, torch.bfloat16)
    ws = Guarded((need,), torch.uint8, DEV, seed=26)
    ws.t.zero_()
    y = Guarded((T, N), torch.bfloat16, DEV, seed=27)
    sq.sq_linear(x.pin_memory(), w.pin_memory(), 0.5, out_dtype=torch.bfloat16, y=y.t, workspace=ws.t)
    y.check("sq_linear y")
    ws.check("sq_linear workspace")
    ref = oracle.linear(synth.host_array(x), synth.host_array(w), 0.5)
    assert np.array_equal(host(y.t), ref["y_bf16"])
