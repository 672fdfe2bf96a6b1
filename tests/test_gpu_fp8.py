"""The FP8 E4M3 sibling of the layer: CUDA path vs the CPU oracle through the
C ABI.

Bar: E4M3 codes and scales bit-exact. GEMM output: the tensor cores add the
exact E4M3 products in fp32 in an order of their own, so the output is
compared with the oracle's exact sum under the bound of fp32 summation in any
order, (K - 1) * 2^-24 * sum_k |x_k w_k| * sa * sw, plus the two rounding of
the epilogue (and one bf16 ulp for bf16 output). The largest error seen, in
units of that sum's 2^-24, is reported.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import assert_bitexact_f32, assert_equal, host
from w8a8_post_quantization_calibrate_b200 import synth

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from w8a8_post_quantization_calibrate_b200 import sq  # noqa: E402

DEV = torch.device("cuda", 0)
# (2048, 2064) and (28672, 28688): either side of the streamed kernel's K range
ROW_SHAPES = [(1, 16), (5, 48), (130, 1040), (4, 2048), (4, 2064), (64, 4096), (9, 11008), (3, 28672),
              (3, 28688), (2, 65536)]


def dev(t):
    return t.contiguous().to(DEV)


def outlier_x(T, K, dtype, seed, n_out=3, scale=50.0):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(T, K, generator=g)
    x[:, torch.randperm(K, generator=g)[:n_out]] *= scale
    return x.to(dtype)


def s_for(K, seed):
    return np.random.default_rng(seed).uniform(0.05, 20.0, K).astype(np.float32)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("rows,K", ROW_SHAPES)
def test_e4m3_codes_bitexact(dtype, rows, K):
    x = outlier_x(rows, K, dtype, seed=rows + K)
    if rows > 2:
        x[1] = 0
    s = s_for(K, K)
    sd = dev(torch.from_numpy(s))
    hx = synth.host_array(x)
    q, sc = sq.sq_smooth_quant_act_e4m3(dev(x), sd)
    oq, osc = oracle.smooth_quant_act_e4m3(hx, s)
    assert_equal(host(q), oq, "E4M3 activation codes")
    assert_bitexact_f32(host(sc), osc, "E4M3 activation scales")
    q, sc = sq.sq_fold_quant_weights_e4m3(dev(x), sd)
    oq, osc = oracle.fold_quant_weights_e4m3(hx, s)
    assert_equal(host(q), oq, "E4M3 weight codes")
    assert_bitexact_f32(host(sc), osc, "E4M3 weight scales")


def _codes(M, N, K, seed):
    rng = np.random.default_rng(seed)
    finite = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)
    xq = rng.choice(finite, size=(M, K)).astype(np.uint8)
    wq = rng.choice(finite, size=(N, K)).astype(np.uint8)
    xs = rng.uniform(1e-3, 0.05, M).astype(np.float32)
    ws = rng.uniform(1e-4, 0.01, N).astype(np.float32)
    return xq, wq, xs, ws


def _check_e4m3_gemm(y, xq, xs, wq, ws, out_dtype, what):
    K = xq.shape[1]
    want, mag = oracle.gemm_dequant_e4m3(xq, xs, wq, ws)
    w64 = want.astype(np.float64)
    if out_dtype == torch.float32:
        got = y.astype(np.float64)
        extra = 2.0 ** -22 * np.abs(w64)
    else:
        got = (y.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        extra = 2.0 ** -22 * np.abs(w64) + 2.0 ** (np.floor(np.log2(np.maximum(np.abs(w64), 1e-30))) - 7)
    err = np.abs(got - w64)
    bound = (K - 1) * 2.0 ** -24 * mag + extra
    bad = np.argwhere(err > bound)
    assert bad.size == 0, f"{what}: {len(bad)} outside the fp32 summation bound, first {bad[:3].tolist()}"
    seen = np.max(np.maximum(err - extra, 0.0) / np.maximum(2.0 ** -24 * mag, 1e-300))
    return float(seen)


@pytest.mark.parametrize("M,N,K", [(1, 300, 272), (5, 1024, 4096), (128, 512, 1040), (129, 257, 272),
                                   (300, 1000, 2048), (1024, 768, 4096), (260, 1000, 16400)])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_e4m3_gemm_within_fp32_summation_bound(M, N, K, out_dtype):
    xq, wq, xs, ws = _codes(M, N, K, seed=M + N + K)
    y = sq.sq_w8a8_gemm_e4m3(dev(torch.from_numpy(xq)), dev(torch.from_numpy(xs)), dev(torch.from_numpy(wq)),
                             dev(torch.from_numpy(ws)), out_dtype=out_dtype)
    seen = _check_e4m3_gemm(host(y), xq, xs, wq, ws, out_dtype, f"{M}x{N}x{K}")
    print(f"largest accumulation error {seen:.1f} x 2^-24 sum|p| (bound {K - 1})")
    assert sq.sq_get_status() == sq.SQ_OK


def test_e4m3_experiment_on_gpu():
    """The pages' synthetic data through the FP8 CUDA path (fp32 inputs):
    relative output error 3.3% without smoothing and 2.9% with it."""
    X, W = synth.outlier_experiment_inputs()
    Y = oracle.matmul_xwT_f64(X, W)
    x = dev(torch.from_numpy(X.astype(np.float32)))
    w = dev(torch.from_numpy(W.astype(np.float32)))
    errs = []
    for smooth in (False, True):
        if smooth:
            xmax = torch.zeros(4096, dtype=torch.float32, device=DEV)
            wmax = torch.zeros(4096, dtype=torch.float32, device=DEV)
            sq.sq_calibrate_absmax_pair(x, w, xmax, wmax)
            s = sq.sq_smooth_factors(xmax, wmax, 0.5)
        else:
            s = torch.ones(4096, dtype=torch.float32, device=DEV)
        wq, wsc = sq.sq_fold_quant_weights_e4m3(w, s)
        xq, xs = sq.sq_smooth_quant_act_e4m3(x, s)
        y = host(sq.sq_w8a8_gemm_e4m3(xq, xs, wq, wsc, out_dtype=torch.float32)).astype(np.float64)
        errs.append(100 * oracle.rel_frobenius_f64(y, Y))
    assert round(errs[0], 1) == 3.3 and round(errs[1], 1) == 2.9, errs


def test_e4m3_qkv_prefill_7b_full_size():
    wl = synth.WORKLOADS["qkv_prefill_7b"]
    x, w = synth.make(wl.name)
    hx, hw = synth.host_array(x), synth.host_array(w)
    s = oracle.smooth_factors(oracle.col_absmax(hx), oracle.col_absmax(hw), wl.alpha)
    sd = dev(torch.from_numpy(s))
    xq, xs = sq.sq_smooth_quant_act_e4m3(dev(x), sd)
    wq, wsc = sq.sq_fold_quant_weights_e4m3(dev(w), sd)
    o_xq, o_xs = oracle.smooth_quant_act_e4m3(hx, s)
    o_wq, o_wsc = oracle.fold_quant_weights_e4m3(hw, s)
    assert_equal(host(xq), o_xq, "full-size E4M3 activation codes")
    assert_equal(host(wq), o_wq, "full-size E4M3 weight codes")
    assert_bitexact_f32(host(xs), o_xs, "x_scale")
    assert_bitexact_f32(host(wsc), o_wsc, "w_scale")
    y = host(sq.sq_w8a8_gemm_e4m3(xq, xs, wq, wsc, out_dtype=torch.bfloat16))
    rows = np.array([0, 1, 777, 2048, wl.T - 1])
    _check_e4m3_gemm(y[rows], o_xq[rows], o_xs[rows], o_wq, o_wsc, torch.bfloat16, "full-size FP8 GEMM rows")


def test_e4m3_rejects_int32_output():
    xq = torch.zeros(4, 64, dtype=torch.uint8, device=DEV)
    wq = torch.zeros(8, 64, dtype=torch.uint8, device=DEV)
    sc = torch.ones(8, device=DEV)
    with pytest.raises(sq.SqError) as e:
        sq.sq_w8a8_gemm_e4m3(xq, sc[:4], wq, sc, out_dtype=torch.int32)
    assert e.value.status == sq.SQ_ERR_UNSUPPORTED


def _e4m3_midpoints():
    """Every rounding boundary of E4M3 between its smallest subnormal and 448:
    (k + 1/2) * quantum in each binade (quantum 2^-9 below 2^-6)."""
    mids = [(k + 0.5) * 2.0 ** -9 for k in range(8)]
    for e in range(-6, 9):
        mids += [2.0 ** e * (1 + (k + 0.5) / 8) for k in range(8)]
    return np.array([m for m in mids if m < 448.0])


@pytest.mark.parametrize("K", [4096, 5120, 28672])
def test_e4m3_stream_kernel_midpoints(K):
    """Quotients at, and a few ulps either side of, every E4M3 rounding boundary
    (subnormal band and saturation included), for the streamed kernel's fast
    pass: with a power-of-two scale the quotient is exact, so exact ties occur.
    x = 1 makes the folded value s itself and the smoothed value RN(1/s)."""
    rng = np.random.default_rng(K)
    scale = 0.125                                      # amax = 56 -> scale = 56 / 448
    targets = []
    for m in _e4m3_midpoints():
        v0 = np.float32(m * scale)
        for d in (-3, -1, 0, 1, 3):
            targets.append(np.float32(v0 + d * np.spacing(v0)))
    targets = np.array(targets, np.float32)
    assert len(targets) < K - 1
    s_fold = rng.uniform(0.01, 0.5, K).astype(np.float32)
    s_fold[0] = 56.0
    s_fold[rng.permutation(np.arange(1, K))[: len(targets)]] = targets
    w = torch.ones(4, K, dtype=torch.bfloat16)
    w[1] = -1.0
    w[2, ::2] = 0.75                                   # scale 42 / 448, not a power of two
    w[3] = -0.0                                        # all-zero row of negative zeros: codes 0x80, scale 1
    hw = synth.host_array(w)
    sd = dev(torch.from_numpy(s_fold))
    q, sc = sq.sq_fold_quant_weights_e4m3(dev(w), sd)
    oq, osc = oracle.fold_quant_weights_e4m3(hw, s_fold)
    assert_equal(host(q), oq, "E4M3 fold codes at the boundaries")
    assert_bitexact_f32(host(sc), osc, "E4M3 fold scales")
    s_smooth = (np.float32(1.0) / s_fold).astype(np.float32)
    x = torch.ones(3, K, dtype=torch.bfloat16)
    x[1] = -1.0
    x[2] = 0.0
    q, sc = sq.sq_smooth_quant_act_e4m3(dev(x), dev(torch.from_numpy(s_smooth)))
    oq, osc = oracle.smooth_quant_act_e4m3(synth.host_array(x), s_smooth)
    assert_equal(host(q), oq, "E4M3 smooth codes at the boundaries")
    assert_bitexact_f32(host(sc), osc, "E4M3 smooth scales")


@pytest.mark.parametrize("K", [4096, 5120])
def test_e4m3_stream_kernel_rows(K):
    """Outlier rows, tiny rows (near the exact-path threshold) and many rows per
    group through the streamed kernel's E4M3 pass."""
    x = outlier_x(700, K, torch.bfloat16, seed=K + 11, n_out=4, scale=80.0)
    x[3] *= 1e-30
    x[4] *= 1e-36
    x[5, 7] = 3e4
    s = s_for(K, K + 5)
    sd = dev(torch.from_numpy(s))
    hx = synth.host_array(x)
    q, sc = sq.sq_smooth_quant_act_e4m3(dev(x), sd)
    oq, osc = oracle.smooth_quant_act_e4m3(hx, s)
    assert_equal(host(q), oq, "E4M3 smooth codes")
    assert_bitexact_f32(host(sc), osc, "E4M3 smooth scales")
    q, sc = sq.sq_fold_quant_weights_e4m3(dev(x), sd)
    oq, osc = oracle.fold_quant_weights_e4m3(hx, s)
    assert_equal(host(q), oq, "E4M3 fold codes")
    assert_bitexact_f32(host(sc), osc, "E4M3 fold scales")


@pytest.mark.parametrize("N,T,K", [(300, 37, 4096), (70, 90, 5120), (9, 5, 28672), (20, 12, 11008), (40, 3, 1040)])
def test_e4m3_pair_launch_equals_the_two_calls(N, T, K):
    """FP8 codes of the weights and the activations in one launch (the
    streamed kernel where the rows fill its lanes; K = 28672, 11008 and 1040
    take the two calls): the same bytes and scales as the two calls and the
    oracle."""
    g = torch.Generator().manual_seed(N + 2 * T + K)
    w = (torch.randn(N, K, generator=g) * 0.05).to(torch.bfloat16)
    x = outlier_x(T, K, torch.bfloat16, seed=N + K)
    if T > 2:
        x[1] = 0.0
        x[2] *= 1e-33
    s = s_for(K, K + 9)
    sd, wd, xd = dev(torch.from_numpy(s)), dev(w), dev(x)
    wq, wsc, xq, xsc = sq.sq_fold_smooth_quant_pair_e4m3(wd, xd, sd)
    wq1, wsc1 = sq.sq_fold_quant_weights_e4m3(wd, sd)
    xq1, xsc1 = sq.sq_smooth_quant_act_e4m3(xd, sd)
    assert_equal(host(wq), host(wq1), "pair vs separate: wq")
    assert_equal(host(xq), host(xq1), "pair vs separate: xq")
    assert_bitexact_f32(host(wsc), host(wsc1), "pair vs separate: w_scale")
    assert_bitexact_f32(host(xsc), host(xsc1), "pair vs separate: x_scale")
    oq, osc = oracle.fold_quant_weights_e4m3(synth.host_array(w), s)
    assert_equal(host(wq), oq, "pair wq vs oracle")
    assert_bitexact_f32(host(wsc), osc, "pair w_scale vs oracle")
    oq, osc = oracle.smooth_quant_act_e4m3(synth.host_array(x), s)
    assert_equal(host(xq), oq, "pair xq vs oracle")
    assert_bitexact_f32(host(xsc), osc, "pair x_scale vs oracle")
