"""sq_w8a8_gemm_noalloc: the decode GEMM for callers that cannot allocate
device memory (a server that has reserved the GPU's memory up front, a decode
loop that cannot afford cudaMalloc's device-wide synchronization, a plug-in
without access to its host's allocator). The library keeps this path's scratch
in a fixed array of its own.

Checked through the C ABI against the existing entry point sq_w8a8_gemm, with
the tolerances the other tests use, on two calls in a row (the second call
reuses the shared scratch the first one left behind). This file is collected
last so that a run stopping at the first failure has already run every other
test; it also passes alone in a fresh process.
"""
import numpy as np
import pytest
import torch

from gpu_helpers import assert_bf16_within_ulp, assert_equal, assert_f32_close, host

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from w8a8_post_quantization_calibrate_b200 import sq  # noqa: E402

DEV = torch.device("cuda", 0)


def _operands(M, N, K, seed):
    g = torch.Generator().manual_seed(seed)
    xq = torch.randint(-127, 128, (M, K), generator=g, dtype=torch.int8).to(DEV)
    wq = torch.randint(-127, 128, (N, K), generator=g, dtype=torch.int8).to(DEV)
    xs = (torch.rand(M, generator=g) * 0.05 + 1e-3).to(DEV)
    wsc = (torch.rand(N, generator=g) * 0.01 + 1e-4).to(DEV)
    return xq, wq, xs, wsc


@pytest.mark.parametrize("M,N,K", [(1, 4096, 11008), (8, 11008, 4096), (16, 11008, 4096), (5, 300, 272)])
def test_noalloc_matches_workspace_entry_point_twice(M, N, K):
    xq, wq, xs, wsc = _operands(M, N, K, seed=M * 31 + N)
    ref_i32 = host(sq.sq_w8a8_gemm(xq, None, wq, None, out_dtype=torch.int32))
    ref_f32 = host(sq.sq_w8a8_gemm(xq, xs, wq, wsc, out_dtype=torch.float32))
    ref_b16 = host(sq.sq_w8a8_gemm(xq, xs, wq, wsc, out_dtype=torch.bfloat16))
    for call in range(2):
        got_i32 = host(sq.sq_w8a8_gemm_noalloc(xq, None, wq, None, out_dtype=torch.int32))
        got_f32 = host(sq.sq_w8a8_gemm_noalloc(xq, xs, wq, wsc, out_dtype=torch.float32))
        got_b16 = host(sq.sq_w8a8_gemm_noalloc(xq, xs, wq, wsc, out_dtype=torch.bfloat16))
        assert_equal(got_i32, ref_i32, f"int32 accumulators, call {call}")
        assert_f32_close(got_f32, ref_f32, f"fp32 output, call {call}")
        assert_bf16_within_ulp(got_b16, ref_b16, f"bf16 output, call {call}")
    assert sq.sq_get_status() == sq.SQ_OK


def test_noalloc_rejects_sizes_beyond_its_scratch():
    xq, wq, xs, wsc = _operands(16, 256, 64, seed=1)
    with pytest.raises(sq.SqError) as e:
        sq.sq_w8a8_gemm_noalloc(torch.zeros((17, 64), dtype=torch.int8, device=DEV), None, wq, None,
                                out_dtype=torch.int32)
    assert e.value.status == sq.SQ_ERR_UNSUPPORTED and "maximum" in str(e.value)
    big_w = torch.zeros((20000, 64), dtype=torch.int8, device=DEV)   # 16 * 20000 > 262,144
    with pytest.raises(sq.SqError) as e:
        sq.sq_w8a8_gemm_noalloc(xq, None, big_w, None, out_dtype=torch.int32)
    assert e.value.status == sq.SQ_ERR_UNSUPPORTED and "scratch" in str(e.value)
    # the largest size it accepts still works
    w_max = torch.randint(-127, 128, (16384, 64), dtype=torch.int8, device=DEV)
    a = host(sq.sq_w8a8_gemm_noalloc(xq, None, w_max, None, out_dtype=torch.int32))
    b = host(sq.sq_w8a8_gemm(xq, None, w_max, None, out_dtype=torch.int32))
    assert np.array_equal(a, b)
