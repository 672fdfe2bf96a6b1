"""The streamed row kernel (bf16 rows of 2064 to 28672 channels, staged in
shared memory by bulk copies): fold + quantize (a3), smooth + quantize (a4) and
RMSNorm + quantize against the CPU oracle, through the C ABI.

Bar: codes and scales bit-exact. The shapes cover every group width the kernel
uses (2, 4, 8 and 16 warps per row) and every chunk count per lane (5 to 8, and 10), rows
padded to whole lanes and rows that fill them exactly, and many rows per
group (the ring of row slots wraps many times); the
special rows drive its exact paths: near-ties of the fast quotient, many
candidates for the row maximum, tiny, denormal, zero and huge rows.
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
BF16 = torch.bfloat16

# (rows, K) -> warps per row, chunks per lane (padded chunks): 2064 -> 2, 5 (62);
# 4096 -> 2, 8; 4112 -> 2, 10 (126); 5120 -> 2, 10; 6144 -> 4, 6; 6160 -> 4, 7 (126);
# 8192 -> 4, 8; 11008 -> 8, 6 (160); 12304 -> 8, 7 (254); 16384 -> 8, 8;
# 16400 -> 16, 5 (510); 28672 -> 16, 7.
SHAPES = [(1, 2064), (37, 4096), (2500, 4096), (300, 4112), (21, 5120), (17, 6144), (9, 6160), (200, 8192),
          (33, 11008), (5, 12304), (3, 16384), (70, 16384), (6, 16400), (300, 28672)]


def dev(t):
    return t.contiguous().to(DEV)


def s_for(K, seed):
    return np.random.default_rng(seed).uniform(0.05, 20.0, K).astype(np.float32)


def outlier_x(T, K, seed, n_out=3, scale=50.0):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(T, K, generator=g)
    x[:, torch.randperm(K, generator=g)[:n_out]] *= scale
    return x.to(BF16)


def check_fold(w, s, what):
    q, sc = sq.sq_fold_quant_weights(dev(w), dev(torch.from_numpy(s)))
    oq, osc = oracle.fold_quant_weights(synth.host_array(w), s)
    assert_equal(host(q), oq, f"{what} codes")
    assert_bitexact_f32(host(sc), osc, f"{what} scales")


def check_smooth(x, s, what):
    q, sc = sq.sq_smooth_quant_act(dev(x), dev(torch.from_numpy(s)))
    oq, osc = oracle.smooth_quant_act(synth.host_array(x), s)
    assert_equal(host(q), oq, f"{what} codes")
    assert_bitexact_f32(host(sc), osc, f"{what} scales")


def check_norm(x, gf, eps, what):
    xq, xs, r = sq.sq_rmsnorm_quant_act(dev(x), dev(torch.from_numpy(gf)), eps)
    hx = synth.host_array(x)
    _, _, o_r = oracle.rmsnorm_quant_act(hx, gf, eps)
    g_r = host(r)
    ulps = np.abs(bits32(g_r).astype(np.int64) - bits32(o_r).astype(np.int64))
    assert ulps.max(initial=0) <= 1, f"{what}: inv_rms {ulps.max()} ulps apart"
    oq, osc, _ = oracle.rmsnorm_quant_act(hx, gf, eps, r_in=g_r)
    assert_equal(host(xq), oq, f"{what} codes")
    assert_bitexact_f32(host(xs), osc, f"{what} scales")


@pytest.mark.parametrize("rows,K", SHAPES)
def test_fold_stream(rows, K):
    g = torch.Generator().manual_seed(rows + 3 * K)
    w = (torch.randn(rows, K, generator=g) * 0.05).to(BF16)
    if rows > 2:
        w[0] = 0
        w[2, K // 3:] = 0
    check_fold(w, s_for(K, K + 1), f"fold {rows}x{K}")


@pytest.mark.parametrize("rows,K", SHAPES)
def test_smooth_stream(rows, K):
    x = outlier_x(rows, K, seed=K + rows)
    if rows > 2:
        x[1] = 0
        x[2, : K // 2] = 0
    check_smooth(x, s_for(K, K), f"smooth {rows}x{K}")


@pytest.mark.parametrize("rows,K", SHAPES)
def test_norm_stream(rows, K):
    x = outlier_x(rows, K, seed=rows * 5 + K, scale=30.0)
    if rows > 2:
        x[1] = 0
    gain = np.random.default_rng(K).uniform(0.5, 1.5, K).astype(np.float32)
    check_norm(x, oracle.fold_norm_gain(gain, s_for(K, K + 7)), 1e-6, f"norm {rows}x{K}")


# K (a multiple of 16, as the calls require) on either side of the streamed
# kernel's range (2064..28672 channels): the calls pick a kernel by K, and each
# side of each edge must match the oracle
EDGE_K = [2032, 2048, 2064, 2080, 28656, 28672, 28688, 28704]


@pytest.mark.parametrize("K", EDGE_K)
def test_kernel_choice_edges(K):
    rows = 7
    g = torch.Generator().manual_seed(K + 11)
    w = (torch.randn(rows, K, generator=g) * 0.05).to(BF16)
    w[3] = 0
    check_fold(w, s_for(K, K + 2), f"fold {rows}x{K}")
    x = outlier_x(rows, K, seed=K + 13)
    x[4, K // 5:] = 0
    check_smooth(x, s_for(K, K + 3), f"smooth {rows}x{K}")


def _tie_targets(scale):
    """fp32 values a few ulps either side of (k + 1/2) * scale, k = 0..126."""
    out = []
    for k in range(127):
        v0 = np.float32((k + 0.5) * float(scale))
        for d in range(-3, 4):
            out.append(np.float32(v0 + d * np.spacing(v0)))
    return np.array(out, np.float32)


@pytest.mark.parametrize("K", [4096, 8192, 16384, 28672])
def test_near_ties(K):
    """With x = 1 the folded value is s itself and the smoothed value RN(1/s):
    choosing s puts hundreds of quotients within a few ulps of k + 1/2, in
    every lane position of the row."""
    scale = np.float32(30.0) / np.float32(127.0)
    t = _tie_targets(scale)
    rng = np.random.default_rng(K)
    pos = rng.permutation(np.arange(1, K))[: len(t)]
    s_fold = rng.uniform(0.01, 0.2, K).astype(np.float32)
    s_fold[0] = 30.0
    s_fold[pos] = t
    w = torch.ones(3, K, dtype=BF16)
    w[1] = -1.0
    w[2, ::2] = 0.5
    check_fold(w, s_fold, f"fold near ties K={K}")
    s_smooth = (np.float32(1.0) / s_fold).astype(np.float32)
    check_smooth(torch.ones(2, K, dtype=BF16), s_smooth, f"smooth near ties K={K}")


@pytest.mark.parametrize("K", [4096, 28672])
def test_near_ties_in_every_row(K):
    """Hundreds of smoothing near-ties in each of 600 rows (rows 2^k x, which
    keeps every quotient): a lane carries its first tie of a row to the next row
    and repairs the rest at once, across the several rows each CTA works."""
    scale = np.float32(30.0) / np.float32(127.0)
    t = _tie_targets(scale)
    rng = np.random.default_rng(K + 11)
    pos = rng.permutation(np.arange(1, K))[: len(t)]
    s_fold = rng.uniform(0.01, 0.2, K).astype(np.float32)
    s_fold[0] = 30.0
    s_fold[pos] = t
    s_smooth = (np.float32(1.0) / s_fold).astype(np.float32)
    k = torch.from_numpy(rng.integers(-6, 7, 600).astype(np.float32))
    x = (torch.ones(600, K) * torch.pow(2.0, k)[:, None]).to(BF16)
    x[::7] = -x[::7]
    check_smooth(x, s_smooth, f"smooth near ties in every row K={K}")
    check_fold(x, s_fold, f"fold near ties in every row K={K}")


@pytest.mark.parametrize("K", [4096, 5120, 6160, 16384])
def test_many_candidates_for_the_maximum(K):
    """Smoothed rows whose largest values differ by a few ulps, spread over
    all lanes and warps of the group: only exact divisions can tell them
    apart, so the scale is right only if every candidate is resolved."""
    rng = np.random.default_rng(K + 1)
    base = np.float32(3.0)
    s = np.full(K, base, np.float32)
    n = 300
    pos = rng.choice(K, n, replace=False)
    s[pos] = base + (rng.integers(-4, 5, n) * np.spacing(base)).astype(np.float32)
    x = torch.ones(4, K, dtype=BF16)
    x[1] = -1.0
    x[2] = float(np.float32(1.5))
    x[3, ::3] = 7.0
    check_smooth(x, s, f"candidates K={K}")
    check_fold(x, s, f"fold near-equal maxima K={K}")


def test_tiny_denormal_zero_and_huge_rows():
    K = 4096
    g = torch.Generator().manual_seed(12)
    x = torch.randn(9, K, generator=g)
    x[0] *= 1e-33
    x[1] *= 1e-38
    x[2] = 0.0
    x[2, 5] = 1e-39
    x[3, 7] = 1e30
    x[4] *= 1e-20
    x[5, :16] = 0.0
    x[6] *= 1e30
    x[7] = 0.0
    x = x.to(BF16)
    s = s_for(K, 77)
    check_smooth(x, s, "extreme rows, smooth")
    check_fold(x, s, "extreme rows, fold")
    gf = oracle.fold_norm_gain(np.ones(K, np.float32), s_for(K, 1))
    for eps in (1e-6, 1.0):
        check_norm(x, gf, eps, f"extreme rows, norm eps={eps}")


def _half_step_rows(K, seed):
    """Raw bf16 rows whose maximum is 127 * 2^e, so the scale is the power of
    two 2^e and every value (2k + 1) 2^(e - 1) is an exact half-step of the
    grid: round half to even decides its code. Rows at e = -3 (values below
    one), e = -60 and e = +40, and a row of N(0, 1) data (its own ties)."""
    rng = np.random.default_rng(seed)
    odd = (2 * rng.integers(0, 127, K) + 1).astype(np.float64) * rng.choice([-1.0, 1.0], K)
    rows = []
    for e in (-3, -60, 40):
        r = odd * 2.0 ** (e - 1)
        r[rng.integers(0, K)] = 127.0 * 2.0 ** e
        rows.append(r)
    rows.append(rng.standard_normal(K))
    return torch.tensor(np.array(rows), dtype=torch.float64).to(BF16)


@pytest.mark.parametrize("K", [512, 2048, 4096, 28672])
def test_exact_half_steps_of_raw_bf16(K):
    """Raw bf16 values on exact half-steps take the near-tie path of the fold
    (multiplier 1 and a power of two), of the bulk quantizer (0/1 multiplier)
    and of RMSNorm; K = 512 and 2048 run the register kernel, 4096 and 28672
    the streamed one."""
    x = _half_step_rows(K, K + 3)
    hx = synth.host_array(x)
    assert (x.float().abs() == 127.0 * 2.0 ** -3).any(), "the bf16 rows hold the maxima exactly"
    check_fold(x, np.ones(K, np.float32), f"half steps, fold s=1, K={K}")
    check_fold(x, np.full(K, 0.25, np.float32), f"half steps, fold s=1/4, K={K}")
    keep = np.ones(K, np.float32)
    keep[np.random.default_rng(K).choice(K, 5, replace=False)] = 0.0
    q, sc = sq.sq_quant_bulk(dev(x), dev(torch.from_numpy(keep)))
    oq, osc = oracle.quant_bulk(hx, keep)
    assert_equal(host(q), oq, f"half steps, bulk codes K={K}")
    assert_bitexact_f32(host(sc), osc, f"half steps, bulk scales K={K}")


def test_keep_mask_fold_is_the_bulk_quantizer():
    """The decomposition's bulk quantizer (a 0/1 multiplier) on the streamed path."""
    K = 4096
    x = outlier_x(64, K, seed=5, n_out=6, scale=20.0)
    keep = np.ones(K, np.float32)
    keep[np.random.default_rng(5).choice(K, 6, replace=False)] = 0.0
    q, sc = sq.sq_quant_bulk(dev(x), dev(torch.from_numpy(keep)))
    oq, osc = oracle.quant_bulk(synth.host_array(x), keep)
    assert_equal(host(q), oq, "bulk codes")
    assert_bitexact_f32(host(sc), osc, "bulk scales")


# (300, 200, 28672) and (200, 100, 16400): 16-warp rows, enough rows that
# CTAs run from the weights into the activations where the pair is one launch.
PAIR_SHAPES = [(300, 37, 4096), (1000, 7, 4112), (70, 90, 5120), (64, 200, 6160), (5, 900, 4096), (50, 3, 16384),
               (9, 5, 28672), (300, 200, 28672), (200, 100, 16400), (40, 33, 2048)]


@pytest.mark.parametrize("dtype", [BF16, torch.float32])
@pytest.mark.parametrize("N,T,K", PAIR_SHAPES)
def test_pair_launch_equals_the_two_calls(dtype, N, T, K):
    """a3 and a4 in one launch (weights' rows, then activations' rows): the
    same codes and scales as the two calls and as the oracle. K = 28672 (two
    multiplier tables do not fit beside the ring) and K = 2048 or fp32 rows
    (outside the streamed kernel) take the two calls."""
    g = torch.Generator().manual_seed(N + T + K)
    w = (torch.randn(N, K, generator=g) * 0.05).to(dtype)
    x = outlier_x(T, K, seed=N * 7 + K).to(dtype)
    if N > 2:
        w[1] = 0
    if T > 2:
        x[2] = 0
        x[1] *= 1e-35
    s = s_for(K, K + 3)
    sd = dev(torch.from_numpy(s))
    wd, xd = dev(w), dev(x)
    wq, wsc, xq, xsc = sq.sq_fold_smooth_quant_pair(wd, xd, sd)
    wq1, wsc1 = sq.sq_fold_quant_weights(wd, sd)
    xq1, xsc1 = sq.sq_smooth_quant_act(xd, sd)
    assert_equal(host(wq), host(wq1), "pair vs separate: wq")
    assert_equal(host(xq), host(xq1), "pair vs separate: xq")
    assert_bitexact_f32(host(wsc), host(wsc1), "pair vs separate: w_scale")
    assert_bitexact_f32(host(xsc), host(xsc1), "pair vs separate: x_scale")
    oq, osc = oracle.fold_quant_weights(synth.host_array(w), s)
    assert_equal(host(wq), oq, "pair wq vs oracle")
    assert_bitexact_f32(host(wsc), osc, "pair w_scale vs oracle")
    oq, osc = oracle.smooth_quant_act(synth.host_array(x), s)
    assert_equal(host(xq), oq, "pair xq vs oracle")
    assert_bitexact_f32(host(xsc), osc, "pair x_scale vs oracle")
    assert sq.sq_get_status() == sq.SQ_OK


def test_pair_launch_qkv_prefill_7b_full_size():
    wl = synth.WORKLOADS["qkv_prefill_7b"]
    x, w = synth.make(wl.name)
    hx, hw = synth.host_array(x), synth.host_array(w)
    s = oracle.smooth_factors(oracle.col_absmax(hx), oracle.col_absmax(hw), wl.alpha)
    wq, wsc, xq, xsc = sq.sq_fold_smooth_quant_pair(dev(w), dev(x), dev(torch.from_numpy(s)))
    oq, osc = oracle.fold_quant_weights(hw, s)
    assert_equal(host(wq), oq, "full-size pair wq")
    assert_bitexact_f32(host(wsc), osc, "full-size pair w_scale")
    oq, osc = oracle.smooth_quant_act(hx, s)
    assert_equal(host(xq), oq, "full-size pair xq")
    assert_bitexact_f32(host(xsc), osc, "full-size pair x_scale")
