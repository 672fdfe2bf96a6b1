"""The decode GEMM (M <= 16 tokens) through the C ABI against the oracle.

sq_w8a8_gemm takes decode-sized M through the cluster kernel: whole 128-row
weight tiles per thread-block cluster, the tiles' k-blocks split between the
cluster's CTAs, partial sums merged in the owning CTA's shared memory. The
shapes below reach its edge cases: one tile and one k-block (CTAs with empty
ranges), tiles cut short by N, tiles whose k-blocks span three or more CTAs,
more tiles than clusters and fewer. The split-K stream kernel (behind
sq_w8a8_gemm_noalloc) computes the same sums through global memory; both must
equal the oracle bit for bit (int32) and give its epilogue's values.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import assert_bf16_within_ulp, assert_equal, assert_f32_close, host

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from w8a8_post_quantization_calibrate_b200 import sq  # noqa: E402

DEV = torch.device("cuda", 0)

SHAPES = [(1, 1, 16), (1, 128, 16), (2, 129, 112), (16, 100, 128), (5, 300, 144), (13, 1000, 1040),
          (16, 2304, 4096), (1, 4096, 11008), (8, 4096, 11008), (16, 11008, 4096), (3, 20000, 272),
          (16, 640, 28672), (7, 257, 65536)]


def _codes(M, N, K, seed):
    g = torch.Generator().manual_seed(seed)
    xq = torch.randint(-127, 128, (M, K), generator=g, dtype=torch.int8)
    wq = torch.randint(-127, 128, (N, K), generator=g, dtype=torch.int8)
    xs = torch.rand(M, generator=g) * 0.05 + 1e-3
    wsc = torch.rand(N, generator=g) * 0.01 + 1e-4
    return xq, wq, xs, wsc


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_decode_gemm_matches_oracle(M, N, K):
    xq, wq, xs, wsc = _codes(M, N, K, seed=M * 7919 + N * 13 + K)
    acc = oracle.gemm_i8(xq.numpy(), wq.numpy())
    y32, y16 = oracle.dequant(acc, xs.numpy(), wsc.numpy())
    xqd, wqd, xsd, wsd = xq.to(DEV), wq.to(DEV), xs.to(DEV), wsc.to(DEV)
    assert_equal(host(sq.sq_w8a8_gemm(xqd, None, wqd, None, out_dtype=torch.int32)), acc, "int32")
    g32 = host(sq.sq_w8a8_gemm(xqd, xsd, wqd, wsd, out_dtype=torch.float32))
    g16 = host(sq.sq_w8a8_gemm(xqd, xsd, wqd, wsd, out_dtype=torch.bfloat16))
    assert assert_f32_close(g32, y32, "fp32") == y32.size
    assert assert_bf16_within_ulp(g16, y16, "bf16") == y16.size
    if M * N <= 262144:
        s16 = host(sq.sq_w8a8_gemm_noalloc(xqd, xsd, wqd, wsd, out_dtype=torch.bfloat16))
        assert_equal(s16, g16, "stream-K kernel vs cluster kernel")
    assert sq.sq_get_status() == sq.SQ_OK


def test_decode_gemm_back_to_back_on_one_stream():
    """Launches that follow one another closely (programmatic dependent launch
    lets the next one start its set-up early) keep their results apart."""
    M, N, K = 16, 11008, 4096
    outs, wants = [], []
    for i in range(4):
        xq, wq, xs, wsc = _codes(M, N, K, seed=100 + i)
        outs.append(sq.sq_w8a8_gemm(xq.to(DEV), None, wq.to(DEV), None, out_dtype=torch.int32))
        wants.append(oracle.gemm_i8(xq.numpy(), wq.numpy()))
    torch.cuda.synchronize()
    for i, (o, w) in enumerate(zip(outs, wants)):
        assert_equal(host(o), w, f"launch {i}")
    assert sq.sq_get_status() == sq.SQ_OK
