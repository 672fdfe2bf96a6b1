"""Per-tensor activation scales (O2 dynamic, O3 static) and the RMSNorm with
the folded gain: CUDA path vs the CPU oracle through the C ABI.

Bar: ranges, codes and scales bit-exact. For the norm, the per-row factor r_t
is an fp64 sum of squares whose rounding order is the kernel's: it must agree
with the oracle's index-order value to 1 fp32 ulp (and does bit for bit on
nearly every row); the codes and scales are then bit-exact given the kernel's
r_t.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import assert_bitexact_f32, assert_equal, bits32, host
from w8a8_post_quantization_calibrate_b200 import synth

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from w8a8_post_quantization_calibrate_b200 import sq  # noqa: E402

DEV = torch.device("cuda", 0)
SHAPES = [(1, 16), (7, 48), (37, 272), (300, 1040), (129, 4096), (9, 11008), (3, 28672), (2, 65536)]


def dev(t):
    return t.contiguous().to(DEV)


def outlier_x(T, K, dtype, seed, n_out=3, scale=50.0):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(T, K, generator=g)
    ch = torch.randperm(K, generator=g)[:n_out]
    x[:, ch] *= scale
    return x.to(dtype)


def s_for(K, seed):
    return np.random.default_rng(seed).uniform(0.05, 20.0, K).astype(np.float32)


# ------------------------------------------------------------------ per-tensor range
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("rows,K", SHAPES)
@pytest.mark.parametrize("smooth", [True, False])
def test_tensor_absmax_bitexact(dtype, rows, K, smooth):
    x = outlier_x(rows, K, dtype, seed=rows + K)
    s = s_for(K, K) if smooth else None
    got = sq.sq_tensor_absmax(dev(x), dev(torch.from_numpy(s)) if smooth else None)
    want = oracle.tensor_absmax(synth.host_array(x), s)
    assert bits32(host(got))[0] == bits32(np.float32(want)), (float(host(got)[0]), float(want))


def test_static_range_equals_range_of_calibration_maxima():
    """Accumulated over calibration batches, and recomputed once from their
    per-channel maxima xmax (a [1 x K] matrix), the static range is the same
    bit for bit: division by s_j > 0 is monotone."""
    K = 4096
    s = dev(torch.from_numpy(s_for(K, 5)))
    batches = [outlier_x(n, K, torch.bfloat16, seed=n) for n in (1, 64, 700)]
    run = torch.zeros(1, dtype=torch.float32, device=DEV)
    xmax = torch.zeros(K, dtype=torch.float32, device=DEV)
    for b in batches:
        sq.sq_tensor_absmax(dev(b), s, run)
        sq.sq_calibrate_absmax(dev(b), xmax)
    from_max = sq.sq_tensor_absmax(xmax.view(1, K), s)
    assert bits32(host(run))[0] == bits32(host(from_max))[0]
    want = np.float32(0.0)
    for b in batches:
        want = oracle.tensor_absmax(synth.host_array(b), host(s), want)
    assert bits32(host(run))[0] == bits32(np.float32(want))


# ------------------------------------------------------------------ per-tensor codes
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("rows,K", SHAPES)
def test_per_tensor_dynamic_bitexact(dtype, rows, K):
    x = outlier_x(rows, K, dtype, seed=3 * rows + K)
    s = s_for(K, K + 2)
    sd = dev(torch.from_numpy(s))
    xd = dev(x)
    amax = sq.sq_tensor_absmax(xd, sd)
    xq, xs = sq.sq_quant_act_per_tensor(xd, sd, amax)
    hx = synth.host_array(x)
    oa = oracle.tensor_absmax(hx, s)
    oq, osc = oracle.quant_act_per_tensor(hx, s, oa)
    assert_equal(host(xq), oq, "per-tensor codes")
    assert_bitexact_f32(host(xs), osc, "per-tensor x_scale")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_per_tensor_static_clips_beyond_range(dtype):
    """A static range calibrated on one batch, applied to a batch up to 4x
    larger: every code equals the oracle's, the excess clamped to +-127."""
    T, K = 300, 1040
    s = s_for(K, 11)
    sd = dev(torch.from_numpy(s))
    calib = outlier_x(T, K, dtype, seed=1)
    amax = sq.sq_tensor_absmax(dev(calib), sd)
    g = torch.Generator().manual_seed(2)
    big = (calib.float() * (1.0 + 3.0 * torch.rand(T, K, generator=g))).to(dtype)
    xq, xs = sq.sq_quant_act_per_tensor(dev(big), sd, amax)
    oq, osc = oracle.quant_act_per_tensor(synth.host_array(big), s, float(host(amax)[0]))
    assert_equal(host(xq), oq, "clipped codes")
    assert_bitexact_f32(host(xs), osc, "static scale")
    assert (np.abs(oq) == 127).sum() > 20


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_per_tensor_extreme_ranges(dtype):
    """Zero range (scale 1, codes 0); a range below 2^-100 and factors whose
    combined multiplier leaves [2^-120, 2^120]: the exact fallbacks give the
    oracle's codes; near-tie values at a range that puts them on half-steps."""
    K = 1040
    g = torch.Generator().manual_seed(4)
    x = torch.randn(6, K, generator=g)
    s = s_for(K, 12)
    cases = []
    cases.append((x * 1e-33, s, None))                              # tiny range
    s2 = s.copy()
    s2[::7] = 1e-35                                                  # a huge range ...
    s2[3::7] = 1e5                                                   # ... and multipliers below 2^-120
    cases.append((x, s2, None))
    cases.append((x, s, 0.0))                                        # zero range
    half = torch.arange(-127, 127, dtype=torch.float32) + 0.5        # exact half-steps at scale 1
    xt = torch.zeros(2, K)
    xt[0, :254] = half
    xt[1, :254] = half + 2.0 ** -10
    cases.append((xt, None, 127.0))
    for xx, ss, fixed in cases:
        xx = xx.to(dtype)
        xd = dev(xx)
        sd = dev(torch.from_numpy(ss)) if ss is not None else None
        if fixed is None:
            amax = sq.sq_tensor_absmax(xd, sd)
        else:
            amax = torch.full((1,), fixed, dtype=torch.float32, device=DEV)
        xq, xs = sq.sq_quant_act_per_tensor(xd, sd, amax)
        hx = synth.host_array(xx)
        oa = oracle.tensor_absmax(hx, ss) if fixed is None else np.float32(fixed)
        assert bits32(host(amax))[0] == bits32(np.float32(oa))
        oq, osc = oracle.quant_act_per_tensor(hx, ss, oa)
        assert_equal(host(xq), oq, "extreme-range codes")
        assert_bitexact_f32(host(xs), osc, "extreme-range scale")


def test_per_tensor_qkv_prefill_7b_full_size():
    wl = synth.WORKLOADS["qkv_prefill_7b"]
    x, w = synth.make(wl.name)
    hx, hw = synth.host_array(x), synth.host_array(w)
    xmax = oracle.col_absmax(hx)
    s = oracle.smooth_factors(xmax, oracle.col_absmax(hw), wl.alpha)
    sd = dev(torch.from_numpy(s))
    xd = dev(x)
    amax = sq.sq_tensor_absmax(xd, sd)
    xq, xs = sq.sq_quant_act_per_tensor(xd, sd, amax)
    oa = oracle.tensor_absmax(hx, s)
    assert bits32(host(amax))[0] == bits32(np.float32(oa))
    oq, osc = oracle.quant_act_per_tensor(hx, s, oa)
    assert_equal(host(xq), oq, "full-size per-tensor codes")
    assert_bitexact_f32(host(xs), osc, "full-size per-tensor scales")


def test_per_tensor_experiment_on_gpu():
    """The pages' synthetic data through the per-tensor CUDA path (fp32 inputs):
    relative output error 21% without smoothing and 2.9% with it."""
    X, W = synth.outlier_experiment_inputs()
    Y = oracle.matmul_xwT_f64(X, W)
    x = dev(torch.from_numpy(X.astype(np.float32)))
    w = dev(torch.from_numpy(W.astype(np.float32)))
    errs = []
    for smooth in (False, True):
        ones = torch.ones(4096, dtype=torch.float32, device=DEV)
        if smooth:
            xmax = torch.zeros(4096, dtype=torch.float32, device=DEV)
            wmax = torch.zeros(4096, dtype=torch.float32, device=DEV)
            sq.sq_calibrate_absmax(x, xmax)
            sq.sq_calibrate_absmax(w, wmax)
            s = sq.sq_smooth_factors(xmax, wmax, 0.5)
        wq, wsc = sq.sq_fold_quant_weights(w, s if smooth else ones)
        amax = sq.sq_tensor_absmax(x, s if smooth else None)
        xq, xs = sq.sq_quant_act_per_tensor(x, s if smooth else None, amax)
        y = host(sq.sq_w8a8_gemm(xq, xs, wq, wsc, out_dtype=torch.float32)).astype(np.float64)
        errs.append(100 * oracle.rel_frobenius_f64(y, Y))
    assert round(errs[0]) == 21 and round(errs[1], 1) == 2.9, errs


# ------------------------------------------------------------------ RMSNorm with the folded gain
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_fold_norm_gain_bitexact(dtype):
    K = 5136
    g = torch.from_numpy(np.random.default_rng(3).uniform(0.2, 2.0, K).astype(np.float32)).to(dtype)
    s = s_for(K, 9)
    got = sq.sq_fold_norm_gain(dev(g), dev(torch.from_numpy(s)))
    assert_bitexact_f32(host(got), oracle.fold_norm_gain(synth.host_array(g), s), "folded gain")


NORM_SHAPES = [(1, 16), (7, 48), (37, 272), (300, 1040), (129, 4096), (33, 5120), (9, 11008), (4, 28672),
               (3, 32768)]


def _check_norm(x, gf, eps, what):
    xq, xs, r = sq.sq_rmsnorm_quant_act(dev(x), dev(torch.from_numpy(gf)), eps)
    hx = synth.host_array(x)
    _, _, o_r = oracle.rmsnorm_quant_act(hx, gf, eps)
    g_r = host(r)
    ulps = np.abs(bits32(g_r).astype(np.int64) - bits32(o_r).astype(np.int64))
    assert ulps.max(initial=0) <= 1, f"{what}: inv_rms {ulps.max()} ulps apart"
    oq, osc, _ = oracle.rmsnorm_quant_act(hx, gf, eps, r_in=g_r)
    assert_equal(host(xq), oq, f"{what} codes")
    assert_bitexact_f32(host(xs), osc, f"{what} scales")
    return int((ulps == 0).sum()), len(ulps)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("rows,K", NORM_SHAPES)
def test_rmsnorm_quant_act(dtype, rows, K):
    if dtype == torch.float32 and K > 16384:
        pytest.skip("fp32 rows above 16384 channels are rejected (covered below)")
    x = outlier_x(rows, K, dtype, seed=rows * 5 + K, scale=30.0)
    if rows > 2:
        x[1] = 0                               # all-zero row: r = 1/sqrt(eps), scale 1, codes 0
    rng = np.random.default_rng(K)
    gain = rng.uniform(0.5, 1.5, K).astype(np.float32)
    gf = oracle.fold_norm_gain(gain, s_for(K, K + 7))
    exact, n = _check_norm(x, gf, 1e-6, f"norm {rows}x{K}")
    assert exact >= n - max(1, n // 100)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_rmsnorm_extreme_rows_and_eps(dtype):
    """Tiny rows (the norm rescales them to O(1)), rows dominated by eps, a
    huge outlier beside tiny values, and a large eps."""
    K = 1040
    g = torch.Generator().manual_seed(8)
    x = torch.randn(6, K, generator=g)
    x[0] *= 1e-30
    x[1] *= 1e-3
    x[2, 9] = 1e30
    x[3, :16] = 0.0
    x = x.to(dtype)
    gf = oracle.fold_norm_gain(np.ones(K, np.float32), s_for(K, 1))
    for eps in (1e-6, 1.0):
        _check_norm(x, gf, eps, f"extreme eps={eps}")


def test_rmsnorm_qkv_prefill_7b_full_size():
    wl = synth.WORKLOADS["qkv_prefill_7b"]
    x, w = synth.make(wl.name)
    hx, hw = synth.host_array(x), synth.host_array(w)
    s = oracle.smooth_factors(oracle.col_absmax(hx), oracle.col_absmax(hw), wl.alpha)
    gain = np.random.default_rng(0).uniform(0.5, 1.5, wl.K).astype(np.float32)
    gf = oracle.fold_norm_gain(gain, s)
    exact, n = _check_norm(x, gf, 1e-5, "full-size norm")
    assert exact >= n - n // 100


def test_rmsnorm_rejects_bad_arguments():
    x = torch.zeros(2, 64, dtype=torch.bfloat16, device=DEV)
    gf = torch.ones(64, dtype=torch.float32, device=DEV)
    with pytest.raises(sq.SqError) as e:
        sq.sq_rmsnorm_quant_act(x, gf, 0.0)
    assert e.value.status == sq.SQ_ERR_INVALID_ARG
    big = torch.zeros(1, 32768 + 16, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(sq.SqError) as e:
        sq.sq_rmsnorm_quant_act(big, torch.ones(32768 + 16, device=DEV), 1e-6)
    assert e.value.status == sq.SQ_ERR_UNSUPPORTED
    f32 = torch.zeros(1, 16384 + 16, dtype=torch.float32, device=DEV)
    with pytest.raises(sq.SqError) as e:
        sq.sq_rmsnorm_quant_act(f32, torch.ones(16384 + 16, device=DEV), 1e-6)
    assert e.value.status == sq.SQ_ERR_UNSUPPORTED
    assert sq.sq_get_status() == sq.SQ_OK
