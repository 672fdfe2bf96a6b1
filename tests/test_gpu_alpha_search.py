"""The per-layer alpha search through the C ABI against the oracle's search
(the fp32 path per alpha, error against the fp64 product).

Bar: every quantized output Yq(alpha) is the bit-exact fp32 path (checked by
the other tests), so the errors differ only through the reference product Y
(fp32-accumulated on the GPU, fp64 in the oracle) and the order of the fp64
sums. With fp32 operands the GPU's Y is a chain of fp32 fused multiply-adds in
k order; with bf16 operands every product is exact and the tensor cores add
them in fp32 in their own order. A relative error d in Y moves an error e by at
most about d (1 + e): the differences seen on these cases are <= 7e-7 of e
(fp32) and <= 2e-5 (bf16, K = 16384), and the tests allow 1e-5 and 1e-4, with
the same best alpha.
"""
import numpy as np
import pytest
import torch

import oracle
import pins
from w8a8_post_quantization_calibrate_b200 import synth

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from w8a8_post_quantization_calibrate_b200 import sq  # noqa: E402

DEV = torch.device("cuda", 0)
RTOL = {torch.float32: 1e-5, torch.bfloat16: 1e-4}


def test_alpha_search_reproduces_the_alpha_table():
    """The pages' synthetic data (fp32): the table's errors 3.5 / 1.8 / 3.5 /
    9.8 percent and the minimum at alpha = 0.5."""
    g = pins.golden("outlier_experiment.json")
    X, W = synth.outlier_experiment_inputs()
    alphas = [row["alpha"] for row in g["alpha_table"]]
    x = torch.from_numpy(X.astype(np.float32)).to(DEV)
    w = torch.from_numpy(W.astype(np.float32)).to(DEV)
    errs, best = sq.sq_alpha_search(x, w, alphas)
    assert [round(100 * e, 1) for e in errs] == [row["error_percent"] for row in g["alpha_table"]], errs
    assert best == 0.5
    o_errs, o_best = oracle.alpha_search(X.astype(np.float32), W.astype(np.float32), alphas)
    np.testing.assert_allclose(errs, o_errs, rtol=RTOL[torch.float32])
    assert o_best == best


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("T,N,K", [(8, 300, 272), (100, 520, 1040), (512, 1024, 4096), (256, 512, 16384)])
def test_alpha_search_matches_oracle(dtype, T, N, K):
    g = torch.Generator().manual_seed(T + N)
    x = torch.randn(T, K, generator=g)
    x[:, torch.randperm(K, generator=g)[:4]] *= 40.0
    w = (torch.randn(N, K, generator=g) * 0.05).to(dtype)
    x = x.to(dtype)
    alphas = [0.0, 0.25, 0.4, 0.5, 0.6, 0.75, 0.85, 1.0]
    errs, best = sq.sq_alpha_search(x.to(DEV), w.to(DEV), alphas)
    o_errs, o_best = oracle.alpha_search(synth.host_array(x), synth.host_array(w), alphas)
    np.testing.assert_allclose(errs, o_errs, rtol=RTOL[dtype])
    assert best == o_best or abs(o_errs[alphas.index(best)] - min(o_errs)) <= RTOL[dtype] * min(o_errs)
    assert sq.sq_get_status() == sq.SQ_OK


def test_alpha_search_rejects_bad_alphas():
    x = torch.zeros(4, 64, device=DEV)
    w = torch.zeros(8, 64, device=DEV)
    with pytest.raises(sq.SqError) as e:
        sq.sq_alpha_search(x, w, [0.5, 1.5])
    assert e.value.status == sq.SQ_ERR_INVALID_ARG
