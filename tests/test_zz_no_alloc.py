"""sq_w8a8_gemm_noalloc: the decode GEMM for callers that cannot allocate
device memory (a server that has reserved the GPU's memory up front, a decode
loop that cannot afford cudaMalloc's device-wide synchronization, a plug-in
without access to its host's allocator). The library keeps this path's scratch
in a fixed array of its own.

Checked through the C ABI against the oracle's int32 product and epilogue and
against the existing entry point sq_w8a8_gemm, with the tolerances the other
tests use, on two calls in a row (the second call reuses the shared scratch
the first one left behind); after a call that left the scratch dirty; and for
the claim itself, that a call allocates no device memory. This file is
collected last so that a run stopping at the first failure has already run
every other test; it also passes alone in a fresh process.
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


def _operands(M, N, K, seed):
    g = torch.Generator().manual_seed(seed)
    xq = torch.randint(-127, 128, (M, K), generator=g, dtype=torch.int8)
    wq = torch.randint(-127, 128, (N, K), generator=g, dtype=torch.int8)
    xs = torch.rand(M, generator=g) * 0.05 + 1e-3
    wsc = torch.rand(N, generator=g) * 0.01 + 1e-4
    return xq, wq, xs, wsc


def _oracle(xq, wq, xs, wsc):
    acc = oracle.gemm_i8(xq.numpy(), wq.numpy())
    y32, y16 = oracle.dequant(acc, xs.numpy(), wsc.numpy())
    return acc, y32, y16


def _check_three(M, N, xqd, wqd, xsd, wsd, acc, y32, y16, what):
    got_i32 = host(sq.sq_w8a8_gemm_noalloc(xqd, None, wqd, None, out_dtype=torch.int32))
    got_f32 = host(sq.sq_w8a8_gemm_noalloc(xqd, xsd, wqd, wsd, out_dtype=torch.float32))
    got_b16 = host(sq.sq_w8a8_gemm_noalloc(xqd, xsd, wqd, wsd, out_dtype=torch.bfloat16))
    assert_equal(got_i32, acc, f"int32 accumulators vs oracle, {what}")
    assert_f32_close(got_f32, y32, f"fp32 output vs oracle, {what}")
    assert_bf16_within_ulp(got_b16, y16, f"bf16 output vs oracle, {what}")
    return got_i32, got_f32, got_b16


@pytest.mark.parametrize("M,N,K", [(1, 4096, 11008), (8, 11008, 4096), (16, 11008, 4096), (5, 300, 272)])
def test_noalloc_matches_oracle_and_workspace_entry_point_twice(M, N, K):
    xq, wq, xs, wsc = _operands(M, N, K, seed=M * 31 + N)
    acc, y32, y16 = _oracle(xq, wq, xs, wsc)
    xqd, wqd, xsd, wsd = xq.to(DEV), wq.to(DEV), xs.to(DEV), wsc.to(DEV)
    ref_i32 = host(sq.sq_w8a8_gemm(xqd, None, wqd, None, out_dtype=torch.int32))
    ref_f32 = host(sq.sq_w8a8_gemm(xqd, xsd, wqd, wsd, out_dtype=torch.float32))
    ref_b16 = host(sq.sq_w8a8_gemm(xqd, xsd, wqd, wsd, out_dtype=torch.bfloat16))
    for call in range(2):
        got_i32, got_f32, got_b16 = _check_three(M, N, xqd, wqd, xsd, wsd, acc, y32, y16, f"call {call}")
        assert_equal(got_i32, ref_i32, f"int32 accumulators vs sq_w8a8_gemm, call {call}")
        assert_f32_close(got_f32, ref_f32, f"fp32 output vs sq_w8a8_gemm, call {call}")
        assert_bf16_within_ulp(got_b16, ref_b16, f"bf16 output vs sq_w8a8_gemm, call {call}")
    assert sq.sq_get_status() == sq.SQ_OK


def test_noalloc_clears_a_dirty_scratch():
    """A call that stopped early would leave partial sums and completion counts
    behind in the shared array; the next call must not see them."""
    M, N, K = 16, 11008, 4096
    xq, wq, xs, wsc = _operands(M, N, K, seed=77)
    acc, y32, y16 = _oracle(xq, wq, xs, wsc)
    xqd, wqd, xsd, wsd = xq.to(DEV), wq.to(DEV), xs.to(DEV), wsc.to(DEV)
    for call in range(2):
        sq.sq_selftest_dirty_noalloc_scratch()
        _check_three(M, N, xqd, wqd, xsd, wsd, acc, y32, y16, f"after a dirty scratch, call {call}")
    assert sq.sq_get_status() == sq.SQ_OK


def test_noalloc_call_allocates_nothing():
    """With y supplied, a call (after the first one on the device, which looks up
    the array's address and loads the kernel) changes neither torch's allocation
    count nor the device's free memory."""
    M, N, K = 8, 11008, 4096
    xq, wq, xs, wsc = _operands(M, N, K, seed=5)
    acc, _, y16 = _oracle(xq, wq, xs, wsc)
    xqd, wqd, xsd, wsd = xq.to(DEV), wq.to(DEV), xs.to(DEV), wsc.to(DEV)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=DEV)
    sq.sq_w8a8_gemm_noalloc(xqd, xsd, wqd, wsd, y=y)
    torch.cuda.synchronize()
    torch_before = torch.cuda.memory_allocated(DEV)
    free_before, _ = torch.cuda.mem_get_info(DEV)
    for _ in range(3):
        sq.sq_w8a8_gemm_noalloc(xqd, xsd, wqd, wsd, y=y)
    torch.cuda.synchronize()
    free_after, _ = torch.cuda.mem_get_info(DEV)
    assert torch.cuda.memory_allocated(DEV) == torch_before
    assert free_after == free_before, (free_before, free_after)
    assert_bf16_within_ulp(host(y), y16, "bf16 output into a supplied y")


def test_noalloc_rejects_sizes_beyond_its_scratch():
    xq, wq, _, _ = _operands(16, 256, 64, seed=1)
    xq, wq = xq.to(DEV), wq.to(DEV)
    with pytest.raises(sq.SqError) as e:
        sq.sq_w8a8_gemm_noalloc(torch.zeros((17, 64), dtype=torch.int8, device=DEV), None, wq, None,
                                out_dtype=torch.int32)
    assert e.value.status == sq.SQ_ERR_UNSUPPORTED and "maximum" in str(e.value)
    big_w = torch.zeros((20000, 64), dtype=torch.int8, device=DEV)   # 16 * 20000 > 262,144
    with pytest.raises(sq.SqError) as e:
        sq.sq_w8a8_gemm_noalloc(xq, None, big_w, None, out_dtype=torch.int32)
    assert e.value.status == sq.SQ_ERR_UNSUPPORTED and "scratch" in str(e.value)
    # the largest size it accepts still works
    w_max = torch.randint(-127, 128, (16384, 64), dtype=torch.int8)
    a = host(sq.sq_w8a8_gemm_noalloc(xq, None, w_max.to(DEV), None, out_dtype=torch.int32))
    assert np.array_equal(a, oracle.gemm_i8(xq.cpu().numpy(), w_max.numpy()))
