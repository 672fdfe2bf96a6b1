"""CUDA path vs the CPU oracle, element by element, through the C ABI.

Bar: int8 codes, fp32 scales, maxima, smoothing factors and int32 accumulators
bit-exact; fp32 outputs within 1e-6 relative; bf16 outputs within 1 ulp.
Small shapes span several tiles and ragged tails; the full-size workloads are
checked on sampled rows and, for the int32 product, by Freivalds' check.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import (assert_bf16_within_ulp, assert_bitexact_f32, assert_equal, assert_f32_close,
                         freivalds, host, oracle_rows)
from w8a8_post_quantization_calibrate_b200 import synth

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from w8a8_post_quantization_calibrate_b200 import sq  # noqa: E402  (loads libsq.so; fails loudly if absent)

DEV = torch.device("cuda", 0)


def dev(t: torch.Tensor) -> torch.Tensor:
    return t.contiguous().to(DEV)


def outlier_x(T, K, dtype, seed, n_out=3, scale=50.0):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(T, K, generator=g)
    ch = torch.randperm(K, generator=g)[:n_out]
    x[:, ch] *= scale
    return x.to(dtype)


def rand_w(N, K, dtype, seed, std=0.05):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(N, K, generator=g) * std).to(dtype)


# ------------------------------------------------------------------ a1
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("rows,cols", [(1, 16), (7, 48), (37, 272), (300, 1024), (1000, 4096), (33, 5136)])
def test_calibrate_absmax_bitexact(dtype, rows, cols):
    x = outlier_x(rows, cols, dtype, seed=rows * 7 + cols)
    x[rows // 2, cols - 1] = -77.5
    got = torch.zeros(cols, dtype=torch.float32, device=DEV)
    sq.sq_calibrate_absmax(dev(x), got)
    want = oracle.col_absmax(synth.host_array(x))
    assert_bitexact_f32(host(got), want, "absmax")


def test_calibrate_running_max_over_batches():
    K = 2048
    batches = [outlier_x(n, K, torch.bfloat16, seed=n) for n in (1, 100, 513, 2048)]
    got = torch.zeros(K, dtype=torch.float32, device=DEV)
    want = np.zeros(K, np.float32)
    for b in batches:
        sq.sq_calibrate_absmax(dev(b), got)
        oracle.col_absmax(synth.host_array(b), want)
    assert_bitexact_f32(host(got), want, "running absmax")
    cat = torch.zeros(K, dtype=torch.float32, device=DEV)
    sq.sq_calibrate_absmax(dev(torch.cat(batches)), cat)
    assert_bitexact_f32(host(cat), want, "absmax over concatenation")


# ------------------------------------------------------------------ a2
@pytest.mark.parametrize("alpha", [0.0, 0.25, 0.5, 0.75, 1.0])
def test_smooth_factors_bitexact(alpha):
    rng = np.random.default_rng(1)
    K = 4096 + 16
    xmax = rng.uniform(0.05, 100.0, K).astype(np.float32)
    wmax = rng.uniform(1e-3, 0.5, K).astype(np.float32)
    xmax[3] = 0.0
    wmax[7] = 0.0
    xmax[9] = wmax[9] = 0.0
    s = sq.sq_smooth_factors(dev(torch.from_numpy(xmax)), dev(torch.from_numpy(wmax)), alpha, 1e-8)
    assert_bitexact_f32(host(s), oracle.smooth_factors(xmax, wmax, alpha, 1e-8), f"s (alpha={alpha})")


def test_smooth_factors_generic_alpha_within_ulp():
    rng = np.random.default_rng(2)
    K = 1024
    xmax = rng.uniform(0.05, 100.0, K).astype(np.float32)
    wmax = rng.uniform(1e-3, 0.5, K).astype(np.float32)
    for alpha in (0.3, 0.85):
        got = host(sq.sq_smooth_factors(dev(torch.from_numpy(xmax)), dev(torch.from_numpy(wmax)), alpha))
        want = oracle.smooth_factors(xmax, wmax, alpha)
        d = np.abs(got.view(np.int32).astype(np.int64) - want.view(np.int32).astype(np.int64))
        assert d.max() <= 1, (alpha, d.max())


# ------------------------------------------------------------------ a3 / a4
ROW_SHAPES = [(1, 16), (5, 48), (3, 1024), (130, 1040), (64, 4096), (17, 5120), (9, 11008), (4, 28672),
              (2, 65536)]


def _s_for(K, seed):
    rng = np.random.default_rng(seed)
    s = rng.uniform(0.05, 20.0, K).astype(np.float32)
    return s


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("rows,K", ROW_SHAPES)
def test_smooth_quant_act_bitexact(dtype, rows, K):
    x = outlier_x(rows, K, dtype, seed=K + rows)
    if rows > 2:
        x[1] = 0                               # all-zero row: scale 1, codes 0
        x[2, : K // 2] = 0
    s = _s_for(K, K)
    xq, xs = sq.sq_smooth_quant_act(dev(x), dev(torch.from_numpy(s)))
    wq_, ws_ = oracle.smooth_quant_act(synth.host_array(x), s)
    assert_equal(host(xq), wq_, "xq")
    assert_bitexact_f32(host(xs), ws_, "x_scale")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("rows,K", ROW_SHAPES)
def test_fold_quant_weights_bitexact(dtype, rows, K):
    w = rand_w(rows, K, dtype, seed=K * 3 + rows)
    if rows > 2:
        w[0] = 0
    s = _s_for(K, K + 1)
    wq, wsc = sq.sq_fold_quant_weights(dev(w), dev(torch.from_numpy(s)))
    oq, osc = oracle.fold_quant_weights(synth.host_array(w), s)
    assert_equal(host(wq), oq, "wq")
    assert_bitexact_f32(host(wsc), osc, "w_scale")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_quant_tiny_denormal_and_extreme_rows(dtype):
    """Rows whose maximum is below 2^-100, denormal values and quotients, and a
    huge outlier beside tiny values: the kernels' exact fallbacks must give the
    oracle's codes and scales."""
    K = 1040
    g = torch.Generator().manual_seed(12)
    x = torch.randn(8, K, generator=g)
    x[0] *= 1e-33
    x[1] *= 1e-38
    x[2] = 0.0
    x[2, 5] = 1e-40
    x[3, 7] = 1e30
    x[4] *= 1e-20
    x[5, :16] = 0.0
    x[6] *= 1e30
    x = x.to(dtype)
    s = _s_for(K, 77)
    for fn, ofn in ((sq.sq_smooth_quant_act, oracle.smooth_quant_act),
                    (sq.sq_fold_quant_weights, oracle.fold_quant_weights)):
        gq, gs = fn(dev(x), dev(torch.from_numpy(s)))
        oq, osc = ofn(synth.host_array(x), s)
        assert_equal(host(gq), oq, f"{fn.__name__} codes")
        assert_bitexact_f32(host(gs), osc, f"{fn.__name__} scales")


def test_quant_near_ties_and_worked_example():
    """Rows built so that many quotients sit within a few ulps of k + 1/2 and
    the 30-outlier worked example; s = 1 so x/s is exact."""
    K = 4096
    scale = np.float32(30.0) / np.float32(127.0)
    vals = []
    for k in range(127):
        v0 = np.float32((k + 0.5) * float(scale))
        for d in range(-3, 4):
            vals.append(np.float32(v0 + d * np.spacing(v0)))
    vals = np.array(vals, np.float32)
    row = np.zeros(K, np.float32)
    row[0] = 30.0
    row[1:1 + len(vals)] = vals
    row[1 + len(vals):1 + 2 * len(vals)] = -vals
    row[2000], row[2001] = 0.01, 0.5
    x = torch.from_numpy(np.stack([row, row * 0.5, -row]))
    s = np.ones(K, np.float32)
    xq, xs = sq.sq_smooth_quant_act(dev(x), dev(torch.from_numpy(s)))
    oq, osc = oracle.smooth_quant_act(x.numpy(), s)
    assert_equal(host(xq), oq, "near-tie codes")
    assert_bitexact_f32(host(xs), osc, "scales")
    q0 = host(xq)[0]
    assert q0[2000] == 0 and q0[2001] == 2 and abs(float(host(xs)[0]) - 0.236) < 5e-4


# ------------------------------------------------------------------ a5
def _codes(M, N, K, seed):
    g = torch.Generator().manual_seed(seed)
    xq = torch.randint(-127, 128, (M, K), generator=g, dtype=torch.int8)
    wq = torch.randint(-127, 128, (N, K), generator=g, dtype=torch.int8)
    xs = torch.rand(M, generator=g) * 0.05 + 1e-3
    wsc = torch.rand(N, generator=g) * 0.01 + 1e-4
    return xq, wq, xs, wsc


GEMM_SHAPES = [
    (1, 16, 16), (1, 128, 128), (3, 200, 272), (8, 1000, 512), (16, 1024, 4096), (16, 300, 1040),
    (17, 256, 128), (100, 300, 272), (128, 256, 128), (129, 257, 144), (256, 512, 1024),
    (300, 1000, 2048), (1024, 768, 4096), (129, 4096, 1024), (513, 1000, 1040),
    (1024, 9728, 512), (777, 10000, 272), (2048, 12288, 1024),
    # K >= 16384 and M > 128: the paired kernel's 512-column tiles (ragged N, K
    # not a multiple of the 128-wide k-block, several tiles per pair); just
    # below that K, 256-column tiles
    (300, 1000, 16384), (257, 1536, 16400), (512, 1536, 28672), (300, 1000, 16368),
]


@pytest.mark.parametrize("M,N,K", GEMM_SHAPES)
def test_gemm_int32_exact(M, N, K):
    xq, wq, _, _ = _codes(M, N, K, seed=M * 1000 + N + K)
    acc = sq.sq_w8a8_gemm(dev(xq), None, dev(wq), None, out_dtype=torch.int32)
    assert_equal(host(acc), oracle.gemm_i8(xq.numpy(), wq.numpy()), f"acc {M}x{N}x{K}")
    assert sq.sq_get_status() == sq.SQ_OK


@pytest.mark.parametrize("M,N,K", [(1, 128, 128), (7, 300, 272), (16, 1024, 1024), (100, 300, 272),
                                   (129, 257, 144), (512, 768, 1024), (300, 1000, 16384)])
def test_gemm_dequant_outputs(M, N, K):
    xq, wq, xs, wsc = _codes(M, N, K, seed=M + 7 * N + K)
    acc = oracle.gemm_i8(xq.numpy(), wq.numpy())
    y32, y16 = oracle.dequant(acc, xs.numpy(), wsc.numpy())
    g32 = sq.sq_w8a8_gemm(dev(xq), dev(xs), dev(wq), dev(wsc), out_dtype=torch.float32)
    g16 = sq.sq_w8a8_gemm(dev(xq), dev(xs), dev(wq), dev(wsc), out_dtype=torch.bfloat16)
    exact32 = assert_f32_close(host(g32), y32, "y fp32")
    exact16 = assert_bf16_within_ulp(host(g16), y16, "y bf16")
    assert exact32 == y32.size and exact16 == y16.size  # same op order: bit-exact in fact


def test_gemm_all_127_headroom():
    """Worst-case magnitudes: every code +-127 (|acc| = 127^2 K)."""
    M, N, K = 16, 256, 8192
    xq = torch.full((M, K), 127, dtype=torch.int8)
    wq = torch.full((N, K), -127, dtype=torch.int8)
    wq[::2] = 127
    for m in (M, 256):
        x = xq[:1].expand(m, K).contiguous()
        acc = host(sq.sq_w8a8_gemm(dev(x), None, dev(wq), None, out_dtype=torch.int32))
        assert acc[0, 0] == 127 * 127 * K and acc[0, 1] == -127 * 127 * K
        assert_equal(acc, oracle.gemm_i8(x.numpy(), wq.numpy()), "acc")


def test_gemm_decode_workspace_reuse():
    """The decode path's workspace is left zeroed: repeated calls with the
    same workspace give identical results."""
    M, N, K = 8, 11008, 4096
    xq, wq, xs, wsc = _codes(M, N, K, seed=3)
    ws = torch.zeros(sq.sq_w8a8_gemm_workspace_size(M, N, K), dtype=torch.uint8, device=DEV)
    want = oracle.gemm_i8(xq.numpy(), wq.numpy())
    for _ in range(3):
        acc = sq.sq_w8a8_gemm(dev(xq), None, dev(wq), None, out_dtype=torch.int32, workspace=ws)
        assert_equal(host(acc), want, "decode acc")
    assert int(ws.count_nonzero()) == 0


# ------------------------------------------------------------------ fused launches
PAIR_SHAPES = [(1, 3, 16), (5, 300, 48), (130, 40, 1040), (64, 12288 // 8, 4096), (17, 333, 5120), (4, 9, 28672),
               (3, 2, 65536), (0, 7, 1040), (7, 0, 1040)]


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("T,N,K", PAIR_SHAPES)
def test_fused_calibration_equals_separate_calls(dtype, T, N, K):
    """sq_calibrate_absmax_pair gives the separate calls' results (and the
    oracle's) bit for bit; the quantization steps follow on its maxima."""
    x = outlier_x(max(T, 1), K, dtype, seed=T * 11 + K)[:T]
    w = rand_w(max(N, 1), K, dtype, seed=N * 13 + K)[:N]
    if T > 2:
        x[1] = 0
    xd, wd = dev(x), dev(w)
    xmax = torch.zeros(K, dtype=torch.float32, device=DEV)
    wmax = torch.zeros(K, dtype=torch.float32, device=DEV)
    sq.sq_calibrate_absmax_pair(xd, wd, xmax, wmax)
    hx, hw = synth.host_array(x), synth.host_array(w)
    o_xmax = oracle.col_absmax(hx) if T else np.zeros(K, np.float32)
    o_wmax = oracle.col_absmax(hw) if N else np.zeros(K, np.float32)
    assert_bitexact_f32(host(xmax), o_xmax, "paired xmax")
    assert_bitexact_f32(host(wmax), o_wmax, "paired wmax")
    s = _s_for(K, K + 5)
    sd = dev(torch.from_numpy(s))
    wq, wsc = sq.sq_fold_quant_weights(wd, sd)
    xq, xs = sq.sq_smooth_quant_act(xd, sd)
    if N:
        oq, osc = oracle.fold_quant_weights(hw, s)
        assert_equal(host(wq), oq, "paired wq")
        assert_bitexact_f32(host(wsc), osc, "paired w_scale")
    if T:
        oq, osc = oracle.smooth_quant_act(hx, s)
        assert_equal(host(xq), oq, "paired xq")
        assert_bitexact_f32(host(xs), osc, "paired x_scale")
    assert sq.sq_get_status() == sq.SQ_OK


def test_fused_calibration_full_size_qkv():
    wl = synth.WORKLOADS["qkv_prefill_7b"]
    x, w = synth.make(wl.name)
    xd, wd = dev(x), dev(w)
    K = wl.K
    m1 = torch.zeros(2 * K, dtype=torch.float32, device=DEV)
    m2 = torch.zeros(2 * K, dtype=torch.float32, device=DEV)
    sq.sq_calibrate_absmax_pair(xd, wd, m1[:K], m1[K:])
    sq.sq_calibrate_absmax(xd, m2[:K])
    sq.sq_calibrate_absmax(wd, m2[K:])
    assert torch.equal(m1, m2)


# ------------------------------------------------------------------ whole path
def _check_path(x, w, alpha, out_dtype, rows=None, calib=None):
    """Run every step on the GPU and compare each output with the oracle;
    the GEMM is compared in full, or on `rows` plus Freivalds' check."""
    xd, wd = dev(x), dev(w)
    xmax = torch.zeros(x.shape[1], dtype=torch.float32, device=DEV)
    for b in (calib if calib is not None else [x]):
        sq.sq_calibrate_absmax(dev(b), xmax)
    wmax = torch.zeros(x.shape[1], dtype=torch.float32, device=DEV)
    sq.sq_calibrate_absmax(wd, wmax)
    s = sq.sq_smooth_factors(xmax, wmax, alpha)
    wq, wsc = sq.sq_fold_quant_weights(wd, s)
    xq, xs = sq.sq_smooth_quant_act(xd, s)
    acc = sq.sq_w8a8_gemm(xq, None, wq, None, out_dtype=torch.int32)
    y = sq.sq_w8a8_gemm(xq, xs, wq, wsc, out_dtype=out_dtype)
    assert sq.sq_get_status() == sq.SQ_OK

    hx = synth.host_array(x)
    hw = synth.host_array(w)
    o_xmax = np.zeros(x.shape[1], np.float32)
    for b in (calib if calib is not None else [x]):
        oracle.col_absmax(synth.host_array(b), o_xmax)
    o_wmax = oracle.col_absmax(hw)
    assert_bitexact_f32(host(xmax), o_xmax, "xmax")
    assert_bitexact_f32(host(wmax), o_wmax, "wmax")
    o_s = oracle.smooth_factors(o_xmax, o_wmax, alpha)
    assert_bitexact_f32(host(s), o_s, "s")
    o_wq, o_wsc = oracle.fold_quant_weights(hw, o_s)
    o_xq, o_xs = oracle.smooth_quant_act(hx, o_s)
    g_xq, g_wq = host(xq), host(wq)
    assert_equal(g_wq, o_wq, "wq")
    assert_bitexact_f32(host(wsc), o_wsc, "w_scale")
    assert_equal(g_xq, o_xq, "xq")
    assert_bitexact_f32(host(xs), o_xs, "x_scale")
    g_acc = host(acc)
    if rows is None:
        o_acc = oracle.gemm_i8(o_xq, o_wq)
        assert_equal(g_acc, o_acc, "acc")
        sel = np.arange(x.shape[0])
    else:
        freivalds(g_acc, o_xq, o_wq)
        sel = rows
        o_acc = oracle_rows(o_xq, o_wq, sel)
        assert_equal(g_acc[sel], o_acc, "acc rows")
    y32, y16 = oracle.dequant(o_acc, o_xs[sel], o_wsc)
    gy = host(y)[sel]
    if out_dtype == torch.float32:
        assert_f32_close(gy, y32, "y")
    else:
        assert_bf16_within_ulp(gy, y16, "y")
    return dict(s=o_s, xq=o_xq, xs=o_xs, wq=o_wq, wsc=o_wsc)


def test_tiny_workload_end_to_end():
    wl = synth.WORKLOADS["tiny"]
    x, w = synth.make("tiny")
    _check_path(x, w, wl.alpha, wl.out_dtype)


def test_sq_linear_matches_steps_device_and_host():
    """sq_linear (one call, a1..a5) equals the step-by-step path, with device
    operands and with pinned host operands."""
    x, w = synth.make("tiny", T=100, N=300)
    wl = synth.WORKLOADS["tiny"]
    y_dev = sq.sq_linear(dev(x), dev(w), wl.alpha, out_dtype=torch.float32)
    ref = oracle.linear(synth.host_array(x), synth.host_array(w), wl.alpha)
    assert_f32_close(host(y_dev), ref["y"], "sq_linear device")
    xh, wh = x.pin_memory(), w.pin_memory()
    yh = torch.empty((100, 300), dtype=torch.float32).pin_memory()
    sq.sq_linear(xh, wh, wl.alpha, out_dtype=torch.float32, y=yh)
    torch.cuda.synchronize()
    assert_f32_close(yh.numpy(), ref["y"], "sq_linear host")


def test_sq_linear_back_to_back_host_calls():
    """Host operands through one workspace, three calls without a sync in
    between (each call's input copies overlap the previous call's GEMM and
    output copy): every output equals the oracle's."""
    wl = synth.WORKLOADS["tiny"]
    outs, refs = [], []
    ws = torch.zeros(sq.sq_linear_workspace_size(200, 300, 1024, torch.float32, torch.float32),
                     dtype=torch.uint8, device=DEV)
    for i in range(3):
        x, w = synth.make("tiny", T=200, N=300)
        x = (x * (1.0 + i)).contiguous()
        xh, wh = x.pin_memory(), w.pin_memory()
        yh = torch.empty((200, 300), dtype=torch.float32).pin_memory()
        sq.sq_linear(xh, wh, wl.alpha, out_dtype=torch.float32, y=yh, workspace=ws)
        outs.append((xh, wh, yh))
        refs.append(oracle.linear(synth.host_array(x), synth.host_array(w), wl.alpha)["y"])
    torch.cuda.synchronize()
    for (_, _, yh), ref in zip(outs, refs):
        assert_f32_close(yh.numpy(), ref, "back-to-back sq_linear")


def _rows(T, n=6, seed=0):
    rng = np.random.default_rng(seed)
    return np.unique(np.concatenate([[0, T - 1], rng.choice(T, n, replace=False)]))


def test_qkv_prefill_7b_full_size():
    wl = synth.WORKLOADS["qkv_prefill_7b"]
    x, w = synth.make(wl.name)
    _check_path(x, w, wl.alpha, wl.out_dtype, rows=_rows(wl.T))


@pytest.mark.parametrize("M", synth.DECODE_MS)
@pytest.mark.parametrize("which", ["gate", "down"])
def test_mlp_decode_7b(M, which):
    x, w = synth.make_decode(M, which)
    _check_path(x, w, 0.5, torch.bfloat16)


def test_mlp_prefill_13b_heavy_full_size():
    wl = synth.WORKLOADS["mlp_prefill_13b_heavy"]
    x, w = synth.make(wl.name)
    _check_path(x, w, wl.alpha, wl.out_dtype, rows=_rows(wl.T, seed=1))


def test_down_prefill_70b_full_size_alpha_sweep():
    wl = synth.WORKLOADS["down_prefill_70b"]
    x, w = synth.make(wl.name)
    calib = list(synth.calibration_batches(wl.name))
    for alpha in synth.DOWN_70B_ALPHAS:
        _check_path(x, w, alpha, wl.out_dtype, rows=_rows(wl.T, n=3, seed=int(alpha * 4)), calib=calib)


# ------------------------------------------------------------------ context check
def test_outlier_experiment_on_gpu():
    """The pages' synthetic W8A8 test run through the CUDA path (fp32 inputs):
    relative output error 0.0949 before (s = 1) and 0.0181 after smoothing."""
    X, W = synth.outlier_experiment_inputs()
    Y = oracle.matmul_xwT_f64(X, W)
    x = dev(torch.from_numpy(X.astype(np.float32)))
    w = dev(torch.from_numpy(W.astype(np.float32)))
    errs = []
    for smooth in (False, True):
        if smooth:
            xmax = torch.zeros(4096, dtype=torch.float32, device=DEV)
            wmax = torch.zeros(4096, dtype=torch.float32, device=DEV)
            sq.sq_calibrate_absmax(x, xmax)
            sq.sq_calibrate_absmax(w, wmax)
            s = sq.sq_smooth_factors(xmax, wmax, 0.5)
        else:
            s = torch.ones(4096, dtype=torch.float32, device=DEV)
        wq, wsc = sq.sq_fold_quant_weights(w, s)
        xq, xs = sq.sq_smooth_quant_act(x, s)
        y = host(sq.sq_w8a8_gemm(xq, xs, wq, wsc, out_dtype=torch.float32)).astype(np.float64)
        errs.append(oracle.rel_frobenius_f64(y, Y))
    assert round(errs[0], 4) == 0.0949 and round(errs[1], 4) == 0.0181, errs


# ------------------------------------------------------------------ failure detection
def test_bounded_wait_times_out_with_status():
    """A wait on a barrier nothing arrives at ends with SQ_ERR_TIMEOUT, and the
    context stays usable afterwards."""
    assert sq.sq_get_status() == sq.SQ_OK
    sq.sq_selftest_wait_timeout(20000)
    assert sq.sq_get_status() == sq.SQ_ERR_TIMEOUT
    assert sq.sq_last_status_site() == 1
    assert sq.sq_get_status() == sq.SQ_OK  # cleared
    xq, wq, _, _ = _codes(130, 260, 256, seed=9)
    acc = sq.sq_w8a8_gemm(dev(xq), None, dev(wq), None, out_dtype=torch.int32)
    assert_equal(host(acc), oracle.gemm_i8(xq.numpy(), wq.numpy()), "acc after timeout")
    assert sq.sq_get_status() == sq.SQ_OK


def test_empty_inputs_are_noops():
    z = torch.zeros(0, 64, dtype=torch.bfloat16, device=DEV)
    m = torch.full((64,), 3.0, device=DEV)
    sq.sq_calibrate_absmax(z, m)
    assert float(m.min()) == 3.0
    y = sq.sq_w8a8_gemm(torch.zeros(0, 64, dtype=torch.int8, device=DEV), None,
                        torch.zeros(5, 64, dtype=torch.int8, device=DEV), None, out_dtype=torch.int32)
    assert y.shape == (0, 5)
    assert sq.sq_get_status() == sq.SQ_OK
