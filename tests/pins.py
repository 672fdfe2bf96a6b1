"""Pins for the CPU oracle: checks against what the pages and mathematics fix,
not against the oracle itself.

Each pin is a function returning None on success and raising AssertionError on
failure. FAST_PINS is the set the planted-mistake test runs under every
mutation; the slow experiment pins live in test_oracle_pins.py.

Independent evaluation. Where a pin needs the exact fp32 result of the
definition it evaluates it in exact rational arithmetic (fractions.Fraction)
and rounds to fp32 with its own nearest-even rule (`rn32`), so no expected value
comes from the code under test or from the same floating-point routine.
"""
from __future__ import annotations

import json
import math
import os
from fractions import Fraction

import numpy as np

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def golden(name: str) -> dict:
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ----------------------------------------------------------- exact helpers
def _bits(v) -> int:
    return int(np.asarray(v, dtype=np.float32).view(np.uint32))


def rn32(fr: Fraction) -> np.float32:
    """Nearest fp32 to an exact rational, ties to even significand."""
    c = np.float32(float(fr))
    cands = [np.nextafter(c, np.float32(-np.inf)), c, np.nextafter(c, np.float32(np.inf))]
    return min(cands, key=lambda v: (abs(Fraction(float(v)) - fr), _bits(v) & 1))


def rne_int(fr: Fraction) -> int:
    """Nearest integer to a rational, ties to even."""
    fl = math.floor(fr)
    d = fr - fl
    if d > Fraction(1, 2):
        return fl + 1
    if d < Fraction(1, 2):
        return fl
    return fl if fl % 2 == 0 else fl + 1


def exact_quant_row(v: np.ndarray):
    """The dynamic symmetric int8 quantizer, each fp32 operation evaluated
    exactly and rounded once: scale = rn32(amax/127), q = clamp(rne(rn32(v/scale)))."""
    amax = max(abs(Fraction(float(x))) for x in v)
    if amax == 0:
        return np.zeros(len(v), np.int8), np.float32(1.0)
    scale = rn32(amax / 127)
    fs = Fraction(float(scale))
    q = [max(-127, min(127, rne_int(Fraction(float(rn32(Fraction(float(x)) / fs)))))) for x in v]
    return np.array(q, np.int8), scale


def ulp32(x: float) -> float:
    x = np.float32(abs(x))
    return float(np.nextafter(x, np.float32(np.inf)) - x)


# ----------------------------------------------------------------- pins
def pin_worked_example():
    """Outlier 30 among 4095 values below 1: scale ~0.236, 0.01 -> 0, 0.5 -> 2."""
    g = golden("worked_example_outlier_30.json")
    rng = np.random.default_rng(7)
    row = rng.uniform(-0.99, 0.99, size=g["K"]).astype(np.float32)
    row[17] = g["outlier"]
    probes = [c[0] for c in g["codes"]]
    row[100:100 + len(probes)] = np.array(probes, np.float32)
    q, scale = oracle.quant_row(row)
    assert round(float(scale), g["scale_printed_decimals"]) == g["scale_approx"], scale
    assert _bits(scale) == _bits(rn32(Fraction(float(np.float32(g["outlier"]))) / 127)), scale
    for i, (_, code) in enumerate(g["codes"]):
        assert int(q[100 + i]) == code, (g["codes"][i], int(q[100 + i]))
    assert int(q[17]) == 127


def pin_ties_half_even():
    """A row whose maximum is 127 has scale exactly 1, so codes are round-half-
    even of the values themselves."""
    vals = np.array([127.0, 2.5, 3.5, -2.5, 126.5, 0.5, 1.5, -0.5, -127.0, 0.0, 64.5, -63.5],
                    np.float32)
    q, scale = oracle.quant_row(vals)
    assert float(scale) == 1.0, scale
    expect = [127, 2, 4, -2, 126, 0, 2, 0, -127, 0, 64, -64]
    assert q.tolist() == expect, q.tolist()


def pin_zero_row():
    """All-zero input gives scale 1 and codes 0 (no 0/0)."""
    q, scale = oracle.quant_row(np.zeros(64, np.float32))
    assert float(scale) == 1.0 and not q.any(), (scale, q)


def pin_clamp_edge():
    """127.6 at scale 1 rounds to 128 and must clamp to 127, not wrap to -128."""
    g = golden("clamp_edge.json")
    v = np.array([g["value"], -g["value"], 128.4, 300.0, -300.0, 126.4], np.float32)
    q = oracle.quant_fixed(v, g["scale"])
    assert int(q[0]) == g["clamped"], q
    assert q.tolist() == [127, -127, 127, 127, -127, 126], q.tolist()
    assert int(q.min()) >= -127


def pin_near_ties_exact():
    """Values within a few ulps of every half-step k+0.5 at the scale set by a
    30 outlier: the oracle's codes equal the exact-rational evaluation of
    clamp(round_half_even(rn32(v / rn32(30/127))))."""
    scale = rn32(Fraction(30) / 127)
    vals = [np.float32(30.0)]
    for k in range(0, 127):
        v0 = rn32((k + Fraction(1, 2)) * Fraction(float(scale)))
        lo, hi = v0, v0
        for _ in range(3):
            lo = np.nextafter(lo, np.float32(-np.inf))
            hi = np.nextafter(hi, np.float32(np.inf))
            vals += [lo, hi]
        vals.append(v0)
    row = np.array(vals + [-v for v in vals[1:]], np.float32)
    row = row[np.abs(row) <= 30.0]
    q, sc = oracle.quant_row(row)
    eq, esc = exact_quant_row(row)
    assert _bits(sc) == _bits(esc), (sc, esc)
    bad = np.nonzero(q != eq)[0]
    assert bad.size == 0, [(float(row[i]), int(q[i]), int(eq[i])) for i in bad[:5]]


def pin_log2k_intervals():
    """One value k times the bulk maximum leaves 254/k grid intervals over the
    bulk: 254.0, 63.5, 15.9, 4.0 and 2, 4, 6 bits lost for k = 4, 16, 64."""
    g = golden("log2k_intervals.json")
    rng = np.random.default_rng(3)
    bulk = (rng.standard_normal(4096) * 0.3).astype(np.float32)
    bmax = float(np.max(np.abs(bulk)))
    base = None
    for row in g["rows"]:
        v = bulk.copy()
        if row["ratio"] is not None:
            v[0] = np.float32(bmax * row["ratio"])
        _, scale = oracle.quant_row(v)
        intervals = 2.0 * bmax / float(scale)
        assert round(intervals, 1) == row["intervals"], (row, intervals)
        if base is None:
            base = intervals
        else:
            assert round(math.log2(base / intervals), 2) == row["bits_lost"], (row, intervals)


def pin_alpha_closed_forms():
    """alpha=0 -> 1/wmax, alpha=1 -> xmax (rounded once to fp32); alpha=1/2 ->
    sqrt(xmax/wmax) within 1 fp32 ulp; eps clamps an all-zero channel."""
    rng = np.random.default_rng(11)
    xmax = (rng.uniform(0.1, 80.0, 512)).astype(np.float32)
    wmax = (rng.uniform(0.01, 0.5, 512)).astype(np.float32)
    xmax[5] = 0.0
    wmax[9] = 0.0
    eps = np.float32(1e-8)
    xm = np.maximum(xmax, eps)
    wm = np.maximum(wmax, eps)
    s0 = oracle.smooth_factors(xmax, wmax, 0.0, float(eps))
    s1 = oracle.smooth_factors(xmax, wmax, 1.0, float(eps))
    sh = oracle.smooth_factors(xmax, wmax, 0.5, float(eps))
    for j in range(512):
        assert _bits(s0[j]) == _bits(rn32(1 / Fraction(float(wm[j])))), (j, s0[j])
        assert _bits(s1[j]) == _bits(xm[j]), (j, s1[j])
        ref = math.sqrt(float(xm[j]) / float(wm[j]))
        assert abs(float(sh[j]) - ref) <= ulp32(ref), (j, sh[j], ref)


def _pow_dec(v: float, a: Fraction):
    """v**a for an fp32 value v and a rational exponent, to 50 significant
    digits (the decimal module's ln and exp are correctly rounded)."""
    import decimal
    ctx = decimal.Context(prec=50)
    dv = ctx.create_decimal_from_float(float(v))
    da = ctx.divide(decimal.Decimal(a.numerator), decimal.Decimal(a.denominator))
    return ctx.exp(ctx.multiply(da, ctx.ln(dv)))


def pin_alpha_generic_pow():
    """alpha outside {0, 1/4, 1/2, 3/4, 1} goes through the general power.
    (1) Dyadic alphas on powers of two give exact powers of two:
    xmax = 2^(8k), wmax = 2^(-8m), alpha = p/8 -> s = 2^(k p + m (8 - p)).
    (2) The alphas the tests use (0.3, 0.4, 0.6, 0.85 as fp32) on random
    maxima: s within 1 fp32 ulp of xmax^alpha / wmax^(1-alpha) evaluated to
    50 digits, with alpha taken exactly as the fp32 value the call receives."""
    for p in (1, 3, 5, 7):
        a = np.float32(p / 8)
        ks = [-3, -1, 0, 1, 2, 4]
        ms = [-2, 0, 1, 3, 5, 7]
        xmax = np.array([2.0 ** (8 * k) for k in ks], np.float32)
        wmax = np.array([2.0 ** (-8 * m) for m in ms], np.float32)
        s = oracle.smooth_factors(xmax, wmax, float(a), 0.0)
        for j, (k, m) in enumerate(zip(ks, ms)):
            want = np.float32(2.0 ** (k * p + m * (8 - p)))
            assert _bits(s[j]) == _bits(want), (p, k, m, s[j], want)
    rng = np.random.default_rng(19)
    xmax = rng.uniform(0.05, 90.0, 48).astype(np.float32)
    wmax = rng.uniform(0.002, 0.6, 48).astype(np.float32)
    for av in (0.3, 0.4, 0.6, 0.85):
        a32 = np.float32(av)
        a = Fraction(float(a32))
        s = oracle.smooth_factors(xmax, wmax, float(a32), 1e-8)
        for j in range(48):
            exact = _pow_dec(xmax[j], a) / _pow_dec(wmax[j], 1 - a)
            ref = float(exact)
            assert abs(float(s[j]) - ref) <= ulp32(ref), (av, j, float(s[j]), ref)


def _outlier_xw(T=96, K=256, N=80, seed=5):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((T, K))
    ch = rng.choice(K, 4, replace=False)
    X[:, ch] *= 40.0
    W = rng.standard_normal((N, K)) * 0.05
    return X, W


def pin_migration_invariants():
    """After smoothing, colmax(Xhat)_j = (xmax_j wmax_j)^(1-alpha) and
    colmax(What)_j = (xmax_j wmax_j)^alpha; so their product is xmax_j wmax_j
    and at alpha=1/2 the two are equal (fp64, rel 1e-12)."""
    X, W = _outlier_xw()
    xmax = oracle.col_absmax_f64(X)
    wmax = oracle.col_absmax_f64(W)
    assert np.all(xmax >= np.abs(X).max(0)) and np.all(xmax <= np.abs(X).max(0))
    for alpha in (0.25, 0.5, 0.75):
        s = oracle.smooth_factors_f64(xmax, wmax, alpha)
        Xs, Ws = oracle.smooth_f64(X, W, s)
        cx = oracle.col_absmax_f64(Xs)
        cw = oracle.col_absmax_f64(Ws)
        p = xmax * wmax
        np.testing.assert_allclose(cx, p ** (1 - alpha), rtol=1e-12)
        np.testing.assert_allclose(cw, p ** alpha, rtol=1e-12)
        if alpha == 0.5:
            np.testing.assert_allclose(cx, cw, rtol=1e-12)


def pin_smoothing_identity():
    """X W^T = (X diag(s)^-1)(W diag(s))^T: unchanged by smoothing in fp64 at
    relative 1e-12."""
    X, W = _outlier_xw()
    s = oracle.smooth_factors_f64(oracle.col_absmax_f64(X), oracle.col_absmax_f64(W), 0.5)
    Xs, Ws = oracle.smooth_f64(X, W, s)
    Y = oracle.matmul_xwT_f64(X, W)
    Y2 = oracle.matmul_xwT_f64(Xs, Ws)
    rel = np.linalg.norm(Y2 - Y) / np.linalg.norm(Y)
    assert rel <= 1e-12, rel
    # and smoothing really moved the outliers (the factor is not trivially 1)
    assert np.abs(Xs).max() < 0.5 * np.abs(X).max()


def pin_calibration_absmax():
    """Per-column max |x|: a planted negative outlier is returned exactly, bf16
    inputs widen exactly, and the running max over batches equals the max over
    their concatenation."""
    rng = np.random.default_rng(2)
    x = rng.standard_normal((37, 48)).astype(np.float32)
    x[11, 3] = -50.25
    x[36, 47] = 9.5
    m = oracle.col_absmax(x)
    assert float(m[3]) == 50.25 and float(m[47]) == 9.5, (m[3], m[47])
    np.testing.assert_array_equal(m, np.abs(x).max(0))
    batches = [rng.standard_normal((n, 48)).astype(np.float32) for n in (1, 5, 17)]
    run = np.zeros(48, np.float32)
    for b in batches:
        oracle.col_absmax(b, run)
    np.testing.assert_array_equal(run, np.abs(np.concatenate(batches)).max(0))
    # bf16: bit pattern 0xC248 is -50.0 exactly
    xb = np.zeros((3, 16), np.uint16)
    xb[1, 2] = 0xC248
    mb = oracle.col_absmax(xb)
    assert float(mb[2]) == 50.0 and float(mb.sum()) == 50.0


def pin_reconstruction_bounds():
    """Round to nearest leaves |v - q*scale| <= scale/2: for activations v =
    X_tj/s_j with the token scale, for weights v = W_nj*s_j with the channel
    scale (v evaluated in fp64 from the inputs; slack for fp32 rounding)."""
    X, W = _outlier_xw(T=40, K=128, N=24, seed=9)
    X = X.astype(np.float32)
    W = W.astype(np.float32)
    xmax = oracle.col_absmax(X)
    wmax = oracle.col_absmax(W)
    s = oracle.smooth_factors(xmax, wmax, 0.5)
    xq, sa = oracle.smooth_quant_act(X, s)
    wq, sw = oracle.fold_quant_weights(W, s)
    s64 = s.astype(np.float64)
    vx = X.astype(np.float64) / s64[None, :]
    vw = W.astype(np.float64) * s64[None, :]
    ex = np.abs(vx - xq.astype(np.float64) * sa[:, None]) / sa[:, None]
    ew = np.abs(vw - wq.astype(np.float64) * sw[:, None]) / sw[:, None]
    assert ex.max() <= 0.5 + 1e-4, ex.max()
    assert ew.max() <= 0.5 + 1e-4, ew.max()
    # every row uses its full grid: the largest magnitude maps to +-127
    assert np.all(np.abs(xq).max(1) == 127) and np.all(np.abs(wq).max(1) == 127)


def pin_gemm_bruteforce():
    """int8 GEMM = exact integer matrix product (numpy int64 matmul), on
    non-square shapes and on the all-127 worst case."""
    rng = np.random.default_rng(4)
    for (M, N, K) in [(3, 5, 7), (17, 9, 64), (1, 33, 130)]:
        xq = rng.integers(-127, 128, (M, K)).astype(np.int8)
        wq = rng.integers(-127, 128, (N, K)).astype(np.int8)
        acc = oracle.gemm_i8(xq, wq)
        ref = xq.astype(np.int64) @ wq.astype(np.int64).T
        np.testing.assert_array_equal(acc.astype(np.int64), ref)
    K = 133144  # largest K whose 127*127*K worst case fits in int32
    ones = np.full((1, K), 127, np.int8)
    acc = oracle.gemm_i8(ones, ones)
    assert int(acc[0, 0]) == 127 * 127 * K == 2147479576
    neg = np.full((1, K), -127, np.int8)
    assert int(oracle.gemm_i8(ones, neg)[0, 0]) == -2147479576


def pin_dequant_epilogue():
    """Y = acc * x_scale[t] * w_scale[n]: exact for power-of-two scales; the
    per-token and per-channel scales factor out (doubling one doubles Y); bf16
    output is round-to-nearest-even of the fp32 value (checked against torch's
    bf16 conversion)."""
    import torch
    acc = np.array([[3, -5, 7], [1 << 20, -(1 << 24) - 1, 0]], np.int32)
    sa = np.array([0.5, 2.0 ** -10], np.float32)
    sw = np.array([0.25, 4.0, 1.0], np.float32)
    y, yb = oracle.dequant(acc, sa, sw)
    ref = acc.astype(np.float64) * sa[:, None].astype(np.float64) * sw[None, :].astype(np.float64)
    ref[1, 1] = float(np.float32(-(1 << 24) - 1)) * 2.0 ** -10 * 4.0  # int->fp32 rounds first
    np.testing.assert_array_equal(y.astype(np.float64), ref)
    y2, _ = oracle.dequant(acc, sa * 2, sw)
    np.testing.assert_array_equal(y2, y * 2)
    rng = np.random.default_rng(8)
    acc = rng.integers(-2 ** 26, 2 ** 26, (16, 64)).astype(np.int32)
    sa = rng.uniform(1e-3, 1.0, 16).astype(np.float32)
    sw = rng.uniform(1e-4, 1e-2, 64).astype(np.float32)
    y, yb = oracle.dequant(acc, sa, sw)
    tb = torch.from_numpy(y).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(yb, tb)
    ties = np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(1.0 + 2.0 ** -8)], np.float32)
    _, tyb = oracle.dequant(np.ones((1, 3), np.int32), np.ones(1, np.float32), ties)
    assert tyb.tolist() == [[0x3F80, 0x3F82, 0xBF80]], [hex(v) for v in tyb[0]]


# ------------------------------------------------- next steps on the layer
def _exact_smoothed(x, s_j):
    return rn32(Fraction(float(x)) / Fraction(float(s_j)))


def pin_per_tensor_scales():
    """Per-tensor range = max over the whole batch of |rn32(x / s_j)| (exact
    rationals); codes = clamp(rne(rn32(rn32(x/s_j) / rn32(amax/127)))), one
    scale for every token; a static range clips a later batch that exceeds it
    to +-127; a zero range gives scale 1 and codes 0."""
    rng = np.random.default_rng(21)
    T, K = 5, 48
    x = rng.normal(size=(T, K)).astype(np.float32)
    x[3, 7] = -9.75
    s = rng.uniform(0.3, 3.0, K).astype(np.float32)
    s[7] = 0.37
    exact = max(abs(Fraction(float(_exact_smoothed(x[t, j], s[j])))) for t in range(T) for j in range(K))
    amax = oracle.tensor_absmax(x, s)
    assert _bits(amax) == _bits(np.float32(float(exact))), (amax, float(exact))
    # running over batches = over their union
    a1 = oracle.tensor_absmax(x[:2], s)
    assert _bits(oracle.tensor_absmax(x[2:], s, a1)) == _bits(amax)
    # no smoothing: plain max |x|
    assert float(oracle.tensor_absmax(x, None)) == float(np.abs(x).max())
    xq, xs = oracle.quant_act_per_tensor(x, s, amax)
    scale = rn32(Fraction(float(amax)) / 127)
    assert all(_bits(v) == _bits(scale) for v in xs), xs
    fs = Fraction(float(scale))
    for t in range(T):
        for j in range(K):
            e = max(-127, min(127, rne_int(Fraction(float(rn32(Fraction(float(_exact_smoothed(x[t, j], s[j]))) / fs))))))
            assert int(xq[t, j]) == e, (t, j, int(xq[t, j]), e)
    # static range from a calibration batch, applied to a larger batch: clipped
    big = (x * 3).astype(np.float32)
    bq, _ = oracle.quant_act_per_tensor(big, s, amax)
    assert int(bq[3, 7]) == -127 and int(bq.max()) <= 127 and int(bq.min()) >= -127
    hot = np.abs(np.array([[float(_exact_smoothed(big[t, j], s[j])) for j in range(K)] for t in range(T)]))
    assert (np.abs(bq[hot > 127.5 * float(scale)]) == 127).all()
    zq, zs = oracle.quant_act_per_tensor(np.zeros((2, 16), np.float32), None, 0.0)
    assert not zq.any() and (zs == 1.0).all()


def pin_norm_fold():
    """Folded gain g'_j = rn32(g_j / s_j) (exact rationals). RMSNorm factor r_t
    = fp32 of torch.nn.functional.rms_norm(x)_j / x_j in fp64 (a library
    routine), to 1 ulp, with eps large enough to matter; codes and scale equal
    the exact-rational evaluation of rn32(rn32(x r_t) g'_j) followed by the
    per-token quantizer; a power-of-two rescaling of the input leaves the codes
    unchanged; an all-zero row gives scale 1 and codes 0."""
    import torch
    rng = np.random.default_rng(22)
    T, K = 4, 64
    x = rng.normal(size=(T, K)).astype(np.float32)
    x[:, 5] *= 40.0
    x[3] = 0.0
    g = rng.uniform(0.5, 1.5, K).astype(np.float32)
    s = rng.uniform(0.2, 4.0, K).astype(np.float32)
    gf = oracle.fold_norm_gain(g, s)
    for j in range(K):
        assert _bits(gf[j]) == _bits(rn32(Fraction(float(g[j])) / Fraction(float(s[j])))), j
    eps = 0.25
    xq, xs, r = oracle.rmsnorm_quant_act(x, gf, eps)
    ref = torch.nn.functional.rms_norm(torch.from_numpy(x.astype(np.float64)), (K,), eps=eps).numpy()
    for t in range(T - 1):
        rt = ref[t, 0] / float(x[t, 0])
        assert abs(float(r[t]) - rt) <= ulp32(rt), (t, float(r[t]), rt)
    assert abs(float(r[T - 1]) - 1.0 / math.sqrt(eps)) <= ulp32(2.0)
    for t in range(T):
        xh = [rn32(Fraction(float(rn32(Fraction(float(x[t, j])) * Fraction(float(r[t]))))) * Fraction(float(gf[j])))
              for j in range(K)]
        eq, esc = exact_quant_row(np.array(xh, np.float32))
        assert _bits(xs[t]) == _bits(esc), (t, xs[t], esc)
        assert np.array_equal(xq[t], eq), (t, np.nonzero(xq[t] != eq))
    assert not xq[T - 1].any() and float(xs[T - 1]) == 1.0
    q4, s4, _ = oracle.rmsnorm_quant_act((x * 4).astype(np.float32), gf, 1e-30)
    q1, s1, _ = oracle.rmsnorm_quant_act(x, gf, 1e-30)
    assert np.array_equal(q4[:T - 1], q1[:T - 1]) and np.array_equal(s4[:T - 1], s1[:T - 1])
    # a given r_t replaces the computed one
    qr, _, rr = oracle.rmsnorm_quant_act(x, gf, eps, r_in=r * 2)
    assert np.array_equal(rr, r * 2)


def pin_decomposition_exact():
    """Bulk channels on the integer grid with a 127 in every row, so the bulk
    quantization is lossless only if its scale ignores the outlier channels;
    outlier channels far off the grid. The decomposed layer then equals the
    exact product X W^T rounded once to fp32 (exact rationals), and the
    outlier set is exactly the channels at or above the threshold."""
    rng = np.random.default_rng(23)
    M, N, K = 4, 6, 32
    out_ch = [3, 17, 30]
    x = rng.integers(-127, 128, (M, K)).astype(np.float32)
    w = rng.integers(-127, 128, (N, K)).astype(np.float32)
    x[:, 0] = 127.0
    w[:, 1] = -127.0
    x[:, out_ch] = rng.uniform(200.0, 1000.0, (M, 3)).astype(np.float32) + np.float32(0.375)
    w[:, out_ch] = rng.normal(size=(N, 3)).astype(np.float32)
    xmax = oracle.col_absmax(x)
    keep, idx = oracle.outlier_split(xmax, 150.0)
    assert idx.tolist() == out_ch and keep.tolist() == [0.0 if j in out_ch else 1.0 for j in range(K)]
    res = oracle.linear_split(x, w, 150.0)
    assert (res["x_scale"] == 1.0).all() and (res["w_scale"] == 1.0).all()
    assert not res["xq"][:, out_ch].any() and not res["wq"][:, out_ch].any()
    for t in range(M):
        for n in range(N):
            exact = sum(Fraction(float(x[t, k])) * Fraction(float(w[n, k])) for k in range(K))
            assert _bits(res["y"][t, n]) == _bits(rn32(exact)), (t, n, res["y"][t, n], float(exact))
    # the worked example with the outlier routed out: the bulk scale covers values below 1
    g = golden("worked_example_outlier_30.json")
    row = np.full(64, 0.9, np.float32)
    row[17] = g["outlier"]
    row[100 % 64] = 0.5
    kp, _ = oracle.outlier_split(np.abs(row), 6.0)
    q, sc = oracle.quant_bulk(row[None, :], kp)
    assert _bits(sc[0]) == _bits(rn32(Fraction(float(np.float32(0.9))) / 127))
    assert int(q[0, 17]) == 0 and int(q[0, 36]) == rne_int(Fraction(float(rn32(Fraction(1, 2) / Fraction(float(sc[0]))))))


def pin_e4m3_codes():
    """FP8 E4M3 (no infinities, largest 448): decoding every byte and encoding
    every representable value, every midpoint between neighbours (ties to the
    even code) and random values agree with torch.float8_e4m3fn (a library
    conversion); values beyond 448 saturate; the per-row FP8 quantizer's
    largest element encodes as 448."""
    import torch
    allb = np.arange(256, dtype=np.uint8)
    dec = oracle.e4m3_to_f64(allb)
    tdec = torch.from_numpy(allb).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    fin = ~np.isnan(tdec)
    assert np.array_equal(np.isnan(dec), ~fin)
    assert np.array_equal(dec[fin], tdec[fin])
    pos = np.unique(dec[fin & (dec >= 0)])
    mids = (pos[1:] + pos[:-1]) / 2
    rng = np.random.default_rng(24)
    vals = np.concatenate([pos, -pos, mids, -mids, rng.uniform(-448, 448, 2000),
                           rng.normal(size=500) * 1e-2, np.array([-0.0, 0.0])])
    ours = oracle.e4m3_from_f64(vals)
    theirs = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    bad = np.nonzero(ours != theirs)[0]
    assert bad.size == 0, [(vals[i], int(ours[i]), int(theirs[i])) for i in bad[:5]]
    assert oracle.e4m3_from_f64(np.array([449.0, 470.0, 1e9, -1e9])).tolist() == [0x7E, 0x7E, 0x7E, 0xFE]
    q, sc = oracle.quant_row_e4m3(np.array([0.5, -3.0, 1.0, 0.0], np.float32))
    assert _bits(sc) == _bits(rn32(Fraction(3) / 448)) and int(q[1]) == 0xFE



def pin_e4m3_gemm_exact():
    """FP8 product: codes decoded by torch.float8_e4m3fn (a library routine),
    summed exactly in fp64 (numpy), rounded once to fp32, then (acc * sa) * sw
    in fp32: equal to the oracle bit for bit."""
    import torch
    rng = np.random.default_rng(25)
    M, N, K = 5, 7, 300
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)
    xq = rng.choice(codes, size=(M, K)).astype(np.uint8)
    wq = rng.choice(codes, size=(N, K)).astype(np.uint8)
    sa = rng.uniform(1e-3, 1.0, M).astype(np.float32)
    sw = rng.uniform(1e-3, 1.0, N).astype(np.float32)
    dx = torch.from_numpy(xq).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    dw = torch.from_numpy(wq).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    acc = dx @ dw.T
    want = (acc.astype(np.float32) * sa[:, None]) * sw[None, :]
    y, _ = oracle.gemm_dequant_e4m3(xq, sa, wq, sw)
    assert np.array_equal(y.view(np.uint32), want.astype(np.float32).view(np.uint32))


FAST_PINS = [
    pin_worked_example,
    pin_ties_half_even,
    pin_zero_row,
    pin_clamp_edge,
    pin_near_ties_exact,
    pin_log2k_intervals,
    pin_alpha_closed_forms,
    pin_alpha_generic_pow,
    pin_migration_invariants,
    pin_smoothing_identity,
    pin_calibration_absmax,
    pin_reconstruction_bounds,
    pin_gemm_bruteforce,
    pin_dequant_epilogue,
    pin_per_tensor_scales,
    pin_norm_fold,
    pin_decomposition_exact,
    pin_e4m3_codes,
    pin_e4m3_gemm_exact,
]
