"""The CPU oracle pinned to what the pages and mathematics fix (CPU only)."""
import numpy as np
import pytest

import oracle
import pins
from w8a8_post_quantization_calibrate_b200 import synth


@pytest.mark.parametrize("pin", pins.FAST_PINS, ids=lambda f: f.__name__)
def test_fast_pin(pin, oracle_lib):
    pin()


@pytest.mark.parametrize("mutation", sorted(oracle.MUTATIONS))
def test_planted_mistake_fails_a_pin(mutation, oracle_lib):
    """Each plausible mistake, planted in the oracle, fails at least one pin."""
    failed = []
    oracle.set_mutation(mutation)
    try:
        for pin in pins.FAST_PINS:
            try:
                pin()
            except AssertionError:
                failed.append(pin.__name__)
            except (OverflowError, ValueError, FloatingPointError):
                failed.append(pin.__name__)
    finally:
        oracle.set_mutation(0)
    assert failed, f"planted mistake {mutation!r} passed every pin"


@pytest.fixture(scope="module")
def experiment():
    X, W = synth.outlier_experiment_inputs()
    Y = oracle.matmul_xwT_f64(X, W)
    return X, W, Y


def test_outlier_experiment_error_fp64(experiment, oracle_lib):
    """The seeded synthetic W8A8 test: relative output error 0.0949 before and
    0.0181 after smoothing at alpha = 0.5 (printed to 4 decimals)."""
    g = pins.golden("outlier_experiment.json")
    X, W, Y = experiment
    before = oracle.w8a8_error_f64(X, W, Y)
    s = oracle.smooth_factors_f64(oracle.col_absmax_f64(X), oracle.col_absmax_f64(W), 0.5)
    Xs, Ws = oracle.smooth_f64(X, W, s)
    after = oracle.w8a8_error_f64(Xs, Ws, Y)
    d = g["printed_decimals"]
    assert round(before, d) == g["w8a8_rel_error_before"], before
    assert round(after, d) == g["w8a8_rel_error_after"], after


def test_outlier_experiment_channel_ratio(experiment, oracle_lib):
    """Largest channel max / median channel max = 73, leaving 127/73 = 1.7 steps."""
    g = pins.golden("outlier_experiment.json")
    X, _, _ = experiment
    cm = oracle.col_absmax_f64(X)
    ratio = cm.max() / np.median(cm)
    assert round(ratio) == g["largest_over_median_channel_max"], ratio
    assert round(127 / ratio, 1) == g["levels_left_for_typical_channel"]


def test_outlier_experiment_alpha_table(experiment, oracle_lib):
    """The alpha sweep table: act and weight max/median of the smoothed column
    maxima (1 decimal) and the W8A8 error in percent (1 decimal)."""
    g = pins.golden("outlier_experiment.json")
    X, W, Y = experiment
    xmax, wmax = oracle.col_absmax_f64(X), oracle.col_absmax_f64(W)
    for row in g["alpha_table"]:
        s = oracle.smooth_factors_f64(xmax, wmax, row["alpha"])
        Xs, Ws = oracle.smooth_f64(X, W, s)
        cx, cw = oracle.col_absmax_f64(Xs), oracle.col_absmax_f64(Ws)
        assert round(cx.max() / np.median(cx), 1) == row["act_max_over_median"], row
        assert round(cw.max() / np.median(cw), 1) == row["weight_max_over_median"], row
        err = oracle.w8a8_error_f64(Xs, Ws, Y)
        assert round(100 * err, 1) == row["error_percent"], (row, err)


def test_fp32_chain_reproduces_experiment(experiment, oracle_lib):
    """The fp32 path that the GPU kernels must match bit for bit (a1..a5 with
    eps, fp32 arithmetic) gives the same printed errors on the same data, fed
    as fp32: 0.0949 with s = 1 and 0.0181 with smoothing."""
    g = pins.golden("outlier_experiment.json")
    X, W, Y = experiment
    X32, W32 = X.astype(np.float32), W.astype(np.float32)
    ones = np.ones(X.shape[1], np.float32)
    errs = []
    for s in (ones, None):
        if s is None:
            s = oracle.smooth_factors(oracle.col_absmax(X32), oracle.col_absmax(W32), 0.5)
        wq, sw = oracle.fold_quant_weights(W32, s)
        xq, sa = oracle.smooth_quant_act(X32, s)
        y, _ = oracle.dequant(oracle.gemm_i8(xq, wq), sa, sw)
        errs.append(oracle.rel_frobenius_f64(y.astype(np.float64), Y))
    d = g["printed_decimals"]
    assert round(errs[0], d) == g["w8a8_rel_error_before"], errs
    assert round(errs[1], d) == g["w8a8_rel_error_after"], errs


def _smoothed_experiment(X, W):
    s = oracle.smooth_factors_f64(oracle.col_absmax_f64(X), oracle.col_absmax_f64(W), 0.5)
    return oracle.smooth_f64(X, W, s)


def test_per_tensor_and_fp8_errors(experiment, oracle_lib):
    """Same data: per-tensor INT8 activations 21% -> 2.9% with smoothing, per-
    token FP8 E4M3 activations (and FP8 weights) 3.3% -> 2.9%."""
    g = pins.golden("format_and_granularity.json")
    X, W, _ = experiment
    Xs, Ws = _smoothed_experiment(X, W)
    assert round(100 * oracle.w8a8_per_tensor_error_f64(X, W)) == g["per_tensor_int8_percent_before"]
    assert round(100 * oracle.w8a8_per_tensor_error_f64(Xs, Ws), 1) == g["per_tensor_int8_percent_after"]
    assert round(100 * oracle.w8a8_e4m3_error_f64(X, W), 1) == g["per_token_fp8_percent_before"]
    assert round(100 * oracle.w8a8_e4m3_error_f64(Xs, Ws), 1) == g["per_token_fp8_percent_after"]


def test_per_tensor_fp32_chain(experiment, oracle_lib):
    """The fp32 per-tensor path (range of the smoothed batch, one scale, the
    int8 GEMM and epilogue) gives the printed 21% and 2.9% on the same data."""
    g = pins.golden("format_and_granularity.json")
    X, W, Y = experiment
    X32, W32 = X.astype(np.float32), W.astype(np.float32)
    errs = []
    for s in (None, oracle.smooth_factors(oracle.col_absmax(X32), oracle.col_absmax(W32), 0.5)):
        ones = np.ones(X.shape[1], np.float32)
        wq, sw = oracle.fold_quant_weights(W32, ones if s is None else s)
        xq, sa = oracle.quant_act_per_tensor(X32, s, oracle.tensor_absmax(X32, s))
        y, _ = oracle.dequant(oracle.gemm_i8(xq, wq), sa, sw)
        errs.append(100 * oracle.rel_frobenius_f64(y.astype(np.float64), Y))
    assert round(errs[0]) == g["per_tensor_int8_percent_before"], errs
    assert round(errs[1], 1) == g["per_tensor_int8_percent_after"], errs


def test_alpha_search_fp32_path(experiment, oracle_lib):
    """The alpha search over the table's alphas, on the fp32 path fed fp32
    data: the table's error percentages and the minimum at alpha = 0.5."""
    g = pins.golden("outlier_experiment.json")
    X, W, _ = experiment
    alphas = [row["alpha"] for row in g["alpha_table"]]
    errs, best = oracle.alpha_search(X.astype(np.float32), W.astype(np.float32), alphas)
    assert [round(100 * e, 1) for e in errs] == [row["error_percent"] for row in g["alpha_table"]], errs
    assert best == 0.5


def test_fp8_fp32_chain(experiment, oracle_lib):
    """The fp32 FP8 path (folded / smoothed rows, per-row E4M3, exact sum, the
    int8 path's epilogue) gives the printed 3.3% and 2.9% on the same data."""
    g = pins.golden("format_and_granularity.json")
    X, W, Y = experiment
    X32, W32 = X.astype(np.float32), W.astype(np.float32)
    errs = []
    for s in (np.ones(X.shape[1], np.float32),
              oracle.smooth_factors(oracle.col_absmax(X32), oracle.col_absmax(W32), 0.5)):
        wq, sw = oracle.fold_quant_weights_e4m3(W32, s)
        xq, sa = oracle.smooth_quant_act_e4m3(X32, s)
        y, _ = oracle.gemm_dequant_e4m3(xq, sa, wq, sw)
        errs.append(100 * oracle.rel_frobenius_f64(y.astype(np.float64), Y))
    assert round(errs[0], 1) == g["per_token_fp8_percent_before"], errs
    assert round(errs[1], 1) == g["per_token_fp8_percent_after"], errs
