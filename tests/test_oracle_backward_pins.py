"""Pins of the oracle's backward pass (straight-through estimator) against
things other than itself: central finite differences of the forward it
differentiates, torch autograd in double, and the invariances of LayerNorm.

The straight-through estimator defines the gradient as that of the forward
with the quantizers replaced by the identity (the pages: the non-differentiable
quantization functions are bypassed, the Hadamard matrix's orthogonality
carries the gradient).  For the activation path that surrogate is
y = (H LN(x) / sqrt(K)) (alpha w)^T; for the weight path y = A (alpha w)^T with
A = s q the forward's dequantized activations.  A dropped mean term, a sign
slip, a transposed product or a missing 1/sqrt(K) fails these.  CPU only.
"""
import numpy as np
import pytest
import torch


def _surrogate_t(orc, x):
    """H LN(x) / sqrt(K) per row in double, from the oracle's pinned forward steps."""
    K = x.shape[1]
    return np.stack([orc.fht_unnormalized(orc.layernorm_row(r)) for r in x]) / np.sqrt(K)


def _case(M, K, N, seed, offset=0.0):
    rng = np.random.default_rng(seed)
    x = (rng.standard_normal((M, K)) * rng.uniform(0.5, 3.0) + offset).astype(np.float32)
    w = rng.integers(-1, 2, (N, K)).astype(np.int8)
    alpha = 0.0173
    g_y = rng.standard_normal((M, N))
    return x, w, alpha, g_y


@pytest.mark.parametrize("M,K,N,seed,offset", [(2, 8, 3, 1, 0.0), (3, 16, 5, 2, 4.0), (1, 32, 7, 3, -2.0)])
def test_activation_gradient_matches_finite_differences(orc, M, K, N, seed, offset):
    x, w, alpha, g_y = _case(M, K, N, seed, offset)
    g_x, _, _ = orc.backward_act_rows(x, w, alpha, g_y)
    wd = alpha * w.astype(np.float64)
    x64 = x.astype(np.float64)

    def loss(xx):
        return float(np.sum(g_y * (_surrogate_t(orc, xx) @ wd.T)))

    h = 1e-5
    fd = np.empty_like(x64)
    for m in range(M):
        for j in range(K):
            xp, xm = x64.copy(), x64.copy()
            xp[m, j] += h
            xm[m, j] -= h
            fd[m, j] = (loss(xp) - loss(xm)) / (2 * h)
    np.testing.assert_allclose(g_x, fd, rtol=1e-6, atol=1e-8 * np.abs(fd).max())


def test_activation_gradient_matches_torch_autograd(orc):
    M, K, N = 3, 64, 32
    x, w, alpha, g_y = _case(M, K, N, 7, 1.5)
    g_x, g_u, g_t = orc.backward_act_rows(x, w, alpha, g_y)
    xt = torch.tensor(x, dtype=torch.float64, requires_grad=True)
    H = torch.tensor([[(-1.0) ** bin(i & j).count("1") for j in range(K)] for i in range(K)], dtype=torch.float64)
    u = torch.nn.functional.layer_norm(xt, (K,), eps=1e-5)
    t = u @ H / np.sqrt(K)
    y = t @ (alpha * torch.tensor(w, dtype=torch.float64)).T
    y.backward(torch.tensor(g_y, dtype=torch.float64))
    np.testing.assert_allclose(g_x, xt.grad.numpy(), rtol=1e-10, atol=1e-13)
    # the intermediate gradients: dL/dt and dL/du
    np.testing.assert_allclose(g_t, g_y @ (alpha * w.astype(np.float64)), rtol=1e-10, atol=1e-15)
    tt = t.detach().requires_grad_(True)
    (tt @ (alpha * torch.tensor(w, dtype=torch.float64)).T).backward(torch.tensor(g_y, dtype=torch.float64))
    np.testing.assert_allclose(g_t, tt.grad.numpy(), rtol=1e-10, atol=1e-15)


def test_weight_gradient_matches_autograd_and_is_not_transposed(orc):
    rng = np.random.default_rng(11)
    M, N, K = 3, 5, 8
    codes = rng.integers(-8, 8, (M, K)).astype(np.int8)
    scales = rng.uniform(0.1, 1.0, M).astype(np.float32)
    g_y = rng.standard_normal((M, N))
    g_W = orc.backward_weight(g_y, codes, scales)
    assert g_W.shape == (N, K)
    A = torch.tensor(codes, dtype=torch.float64) * torch.tensor(scales, dtype=torch.float64)[:, None]
    Wd = torch.zeros((N, K), dtype=torch.float64, requires_grad=True)
    (A @ Wd.T).backward(torch.tensor(g_y, dtype=torch.float64))
    np.testing.assert_allclose(g_W, Wd.grad.numpy(), rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("K,offset", [(4096, 0.0), (1024, 100.0)])
def test_layernorm_gradient_invariances(orc, K, offset):
    """LN(x) does not change when x is shifted or (eps aside) scaled, so g_x has
    no component along the ones vector, and (without eps) none along x - mu."""
    rng = np.random.default_rng(K)
    x = rng.standard_normal(K) * 2.0 + offset
    g_u = rng.standard_normal(K)
    g_x = orc.ln_backward_row(x, g_u)
    scale = np.linalg.norm(g_x) * np.sqrt(K)
    assert abs(g_x.sum()) <= 1e-12 * scale
    d = x - x.mean()
    var = d @ d / K
    # with eps the scale invariance is broken by eps / (var + eps) relative
    assert abs(g_x @ d) <= (1e-5 / var + 1e-12) * scale * np.linalg.norm(d)


def test_transform_gradient_is_orthogonal(orc):
    x, w, alpha, g_y = _case(4, 2048, 64, 5)
    _, g_u, g_t = orc.backward_act_rows(x, w, alpha, g_y)
    np.testing.assert_allclose(np.linalg.norm(g_u, axis=1), np.linalg.norm(g_t, axis=1), rtol=1e-12)
