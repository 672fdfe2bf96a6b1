"""The mixed-precision decomposition (static outlier channels in fp32, the
rest in int8): CUDA path vs the CPU oracle through the C ABI.

Bar: outlier set, bulk codes and scales, gathered columns bit-exact. Output:
the oracle adds the outlier term in fp64 and rounds once; the kernel adds it
as an fp32 fused multiply-add chain, so the two differ by at most
(ld + 1) * 2^-24 * (|Y_bulk| + sum |x_out w_out|), written in the test (plus
one bf16 ulp for bf16 output, where the two fp32 values may round to
neighbouring bf16 values).
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import assert_bitexact_f32, assert_equal, host, oracle_rows
from w8a8_post_quantization_calibrate_b200 import synth

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from w8a8_post_quantization_calibrate_b200 import sq  # noqa: E402

DEV = torch.device("cuda", 0)


def dev(t):
    return t.contiguous().to(DEV)


def planted(T, K, dtype, seed, n_out, scale=14.0):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(T, K, generator=g)
    ch = torch.randperm(K, generator=g)[:n_out]
    x[:, ch] *= scale
    return x.to(dtype), sorted(ch.tolist())


def assert_split_close(got, want32, want16, mag, ld, out_dtype, what):
    tol = (ld + 1) * 2.0 ** -24 * mag
    if out_dtype == torch.float32:
        err = np.abs(got.astype(np.float64) - want32.astype(np.float64))
        bad = np.argwhere(err > tol)
    else:
        # the fp32 values may straddle a bf16 rounding boundary: one bf16 ulp more
        g = (got.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        w = (want16.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        err = np.abs(g - w)
        a = np.maximum(np.abs(want32.astype(np.float64)), 1e-30)
        ulp16 = 2.0 ** (np.floor(np.log2(a)) - 7)
        bad = np.argwhere(err > tol + ulp16)
    assert bad.size == 0, f"{what}: {len(bad)} outside tolerance, first {bad[:3].tolist()}"


@pytest.mark.parametrize("K,thr", [(16, 1.5), (1040, 40.0), (4096, 40.0), (5120, 0.0), (11008, 1e9), (28672, 40.0)])
def test_outlier_split_exact(K, thr):
    x, ch = planted(64, K, torch.float32, seed=K, n_out=min(K, 9), scale=60.0)
    xmax = torch.zeros(K, dtype=torch.float32, device=DEV)
    sq.sq_calibrate_absmax(dev(x), xmax)
    keep, idx, count = sq.sq_outlier_split(xmax, thr)
    ok, oi = oracle.outlier_split(host(xmax), thr)
    n = int(host(count)[0])
    assert n == len(oi)
    assert_equal(host(idx)[:n], oi, "outlier indices")
    assert_bitexact_f32(host(keep), ok, "keep mask")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("rows,K", [(1, 16), (37, 272), (300, 1040), (64, 4096), (9, 11008), (3, 28672)])
def test_quant_bulk_and_gather_exact(dtype, rows, K):
    x, ch = planted(rows, K, dtype, seed=rows * 3 + K, n_out=min(5, K // 4))
    keep = np.ones(K, np.float32)
    keep[ch] = 0.0
    q, sc = sq.sq_quant_bulk(dev(x), dev(torch.from_numpy(keep)))
    oq, osc = oracle.quant_bulk(synth.host_array(x), keep)
    assert_equal(host(q), oq, "bulk codes")
    assert_bitexact_f32(host(sc), osc, "bulk scales")
    idx = torch.tensor(ch, dtype=torch.int32)
    ld = (len(ch) + 3) // 4 * 4 + 4
    out = sq.sq_gather_columns(dev(x), dev(idx), len(ch), ld)
    assert_bitexact_f32(host(out), oracle.gather_columns(synth.host_array(x), idx.numpy(), ld), "gathered")


def _split_operands(M, N, K, ld, seed):
    g = torch.Generator().manual_seed(seed)
    xq = torch.randint(-127, 128, (M, K), generator=g, dtype=torch.int8)
    wq = torch.randint(-127, 128, (N, K), generator=g, dtype=torch.int8)
    xs = torch.rand(M, generator=g) * 0.05 + 1e-3
    wsc = torch.rand(N, generator=g) * 0.01 + 1e-4
    xo = torch.randn(M, ld, generator=g) * 20.0
    wo = torch.randn(N, ld, generator=g) * 0.1
    return xq, wq, xs, wsc, xo, wo


@pytest.mark.parametrize("M,N,K,ld", [(1, 300, 272, 4), (8, 4096, 1024, 8), (16, 1100, 4096, 32),
                                      (100, 300, 272, 4), (128, 512, 1024, 16), (300, 1000, 1040, 8),
                                      (1024, 2048, 4096, 4)])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_gemm_split_epilogue(M, N, K, ld, out_dtype):
    xq, wq, xs, wsc, xo, wo = _split_operands(M, N, K, ld, seed=M + N + ld)
    y = sq.sq_w8a8_gemm_split(dev(xq), dev(xs), dev(wq), dev(wsc), dev(xo), dev(wo), out_dtype=out_dtype)
    acc = oracle.gemm_i8(xq.numpy(), wq.numpy())
    y32, y16, mag = oracle.dequant_split(acc, xs.numpy(), wsc.numpy(), xo.numpy(), wo.numpy())
    assert_split_close(host(y), y32, y16, mag, ld, out_dtype, f"split {M}x{N}x{K} ld={ld}")
    assert sq.sq_get_status() == sq.SQ_OK


def test_gemm_split_with_no_outliers_is_the_plain_gemm():
    xq, wq, xs, wsc, _, _ = _split_operands(200, 300, 272, 4, seed=1)
    e = torch.zeros(200, 0, dtype=torch.float32)
    y0 = sq.sq_w8a8_gemm_split(dev(xq), dev(xs), dev(wq), dev(wsc), dev(e), dev(torch.zeros(300, 0)),
                               out_dtype=torch.float32)
    y1 = sq.sq_w8a8_gemm(dev(xq), dev(xs), dev(wq), dev(wsc), out_dtype=torch.float32)
    assert_bitexact_f32(host(y0), host(y1), "ld = 0")
    with pytest.raises(sq.SqError) as err:
        sq.sq_w8a8_gemm_split(dev(xq), dev(xs), dev(wq), dev(wsc), dev(torch.zeros(200, 6)),
                              dev(torch.zeros(300, 6)), out_dtype=torch.float32)
    assert err.value.status == sq.SQ_ERR_UNSUPPORTED
    with pytest.raises(sq.SqError) as err:
        sq.sq_w8a8_gemm_split(dev(xq), dev(xs), dev(wq), dev(wsc), dev(torch.zeros(200, 36)),
                              dev(torch.zeros(300, 36)), out_dtype=torch.float32)
    assert err.value.status == sq.SQ_ERR_UNSUPPORTED


def _check_layer(x, w, thr, out_dtype, rows=None):
    """Every step of the decomposed layer on the GPU against the oracle."""
    K = x.shape[1]
    xd, wd = dev(x), dev(w)
    xmax = torch.zeros(K, dtype=torch.float32, device=DEV)
    sq.sq_calibrate_absmax(xd, xmax)
    keep, idx, count = sq.sq_outlier_split(xmax, thr)
    n = int(host(count)[0])
    ld = max(4, (n + 3) // 4 * 4)
    wq, wsc = sq.sq_quant_bulk(wd, keep)
    xq, xs = sq.sq_quant_bulk(xd, keep)
    xo = sq.sq_gather_columns(xd, idx, n, ld)
    wo = sq.sq_gather_columns(wd, idx, n, ld)
    y = sq.sq_w8a8_gemm_split(xq, xs, wq, wsc, xo, wo, out_dtype=out_dtype)
    assert sq.sq_get_status() == sq.SQ_OK
    hx, hw = synth.host_array(x), synth.host_array(w)
    ok, oi = oracle.outlier_split(oracle.col_absmax(hx), thr)
    assert_equal(host(idx)[:n], oi, "outlier set")
    o_wq, o_wsc = oracle.quant_bulk(hw, ok)
    o_xq, o_xs = oracle.quant_bulk(hx, ok)
    assert_equal(host(wq), o_wq, "bulk wq")
    assert_equal(host(xq), o_xq, "bulk xq")
    assert_bitexact_f32(host(wsc), o_wsc, "bulk w_scale")
    assert_bitexact_f32(host(xs), o_xs, "bulk x_scale")
    o_xo = oracle.gather_columns(hx, oi, ld)
    o_wo = oracle.gather_columns(hw, oi, ld)
    assert_bitexact_f32(host(xo), o_xo, "x_out")
    assert_bitexact_f32(host(wo), o_wo, "w_out")
    sel = np.arange(x.shape[0]) if rows is None else rows
    acc = oracle_rows(o_xq, o_wq, sel)
    y32, y16, mag = oracle.dequant_split(acc, o_xs[sel], o_wsc, o_xo[sel], o_wo)
    assert_split_close(host(y)[sel], y32, y16, mag, ld, out_dtype, "decomposed layer")
    return n


def test_decomposed_layer_planted_outliers():
    """Five dimensions x14 in every token of a [512 x 256] activation, W
    [128 x 256] ~ N(0, 0.1): the recipe of the "Route it, or move it" cell."""
    x, ch = planted(512, 256, torch.float32, seed=0, n_out=5)
    w = torch.randn(128, 256, generator=torch.Generator().manual_seed(1)) * 0.1
    n = _check_layer(x, w, 26.0, torch.float32)
    assert n == 5


def test_decomposed_qkv_prefill_7b_full_size():
    wl = synth.WORKLOADS["qkv_prefill_7b"]
    x, w = synth.make(wl.name)
    rng = np.random.default_rng(2)
    rows = np.unique(np.concatenate([[0, wl.T - 1], rng.choice(wl.T, 6, replace=False)]))
    n = _check_layer(x, w, 12.0, torch.bfloat16, rows=rows)
    assert n >= 1
