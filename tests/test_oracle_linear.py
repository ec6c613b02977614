"""Pins for the oracle's fake-quantized linear layer and GELU (CPU).

The linear is Y = X̂ Ŵᵀ + b (Tail-Aware HiFloat4 arXiv abstract: W4A4 fake
quantization of the main linear layers); the oracle's triple loop is checked
against numpy's float64 matmul.  The tanh-form GELU (the FFN activation; not
on the pages) is checked against torch's float64 implementation and its
closed-form symmetry gelu(x) - gelu(-x) = x.
"""
import math

import numpy as np
import torch

import oracle


def test_linear_vs_numpy_matmul():
    rng = np.random.default_rng(4)
    for M, N, K in [(1, 1, 64), (3, 5, 128), (17, 33, 192)]:
        x = rng.standard_normal((M, K))
        w = rng.standard_normal((N, K))
        b = rng.standard_normal(N)
        y = oracle.linear(x, w, b, threads=2)
        want = x @ w.T + b
        assert np.allclose(y, want, rtol=1e-13, atol=1e-12)
        y0 = oracle.linear(x, w, None)
        assert np.allclose(y0, x @ w.T, rtol=1e-13, atol=1e-12)
        # operand order: a transposed operand would fail this non-square case
        assert y.shape == (M, N)


def test_linear_exact_on_dyadic_operands():
    # HiF4-dequantized operands are dyadic with few bits: small sums are exact
    x = np.array([[0.25, -1.75, 3.5, 0.0] * 16])
    w = np.array([[1.0, 0.5, -0.25, 7.0] * 16, [0.75] * 64])
    y = oracle.linear(x, w, None)
    assert y[0, 0] == 16 * (0.25 - 0.875 - 0.875)
    assert y[0, 1] == 0.75 * 16 * (0.25 - 1.75 + 3.5)


def test_gelu_tanh():
    xs = np.linspace(-12, 12, 241)
    want = torch.nn.functional.gelu(torch.tensor(xs, dtype=torch.float64), approximate="tanh").numpy()
    got = np.array([oracle.gelu_tanh(v) for v in xs])
    assert np.allclose(got, want, rtol=1e-14, atol=1e-15)
    assert oracle.gelu_tanh(0.0) == 0.0
    for v in [0.1, 1.0, 3.0]:
        assert math.isclose(oracle.gelu_tanh(v) - oracle.gelu_tanh(-v), v, rel_tol=1e-14)
    y = oracle.linear(np.array([[1.0] * 64]), np.array([[0.5] * 64]), None, gelu=True)
    assert math.isclose(y[0, 0], oracle.gelu_tanh(32.0))
