"""The evaluation helpers of compare_rtn (torch, CPU) against the oracle."""
import numpy as np
import pytest

from oracle import gptq_ref as o


def _prep(seed, R, C, act=False, mix=3, rel=0.01):
    g = np.random.default_rng(seed)
    X = g.standard_normal((4 * C, C))
    X += g.standard_normal((4 * C, mix)) @ g.standard_normal((mix, C))
    X *= g.uniform(0.3, 3.0, size=C)
    W = 0.02 * g.standard_normal((R, C))
    H, n = o.hessian(X)
    return W, X, H, n


def test_rtn_comparison_arithmetic_matches_the_oracle():
    """The evaluation helpers of compare_rtn (torch) against the oracle's dequantize and
    reconstruction error: the same Q and, with H given by its upper triangle, the
    same objective tr((W-Q) H (W-Q)^T) = (2/n) ||(W-Q) X^T||^2."""
    import torch
    from post_weight_quantization_20_b200 import compare_rtn as CR
    W, X, H, n = _prep(61, 6, 40)
    out = o.gptq_quantize(W, H, 3, 8, False, True, 0.01, 8)
    Q = CR.dequantize(torch.from_numpy(out["codes"]), torch.from_numpy(out["scales"]),
                      torch.from_numpy(out["zeros"]), torch.from_numpy(out["g_idx"]))
    np.testing.assert_array_equal(Q.numpy(), out["Q"])
    Hup = torch.from_numpy(np.triu(H) + np.tril(np.full_like(H, np.nan), -1))   # lower: garbage
    got = CR.objective(torch.from_numpy(W), Q, Hup)
    assert got == pytest.approx(o.reconstruction_error(W, out["Q"], H, n) * 2 / n, rel=1e-12)
