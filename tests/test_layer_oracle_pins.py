"""Pins of the layer oracle (oracle/gdn2_layer_oracle.c: the prologue's short
causal convolution, SiLU, L2 norm and gate activations, and the epilogue's
RMS norm with a SiLU output gate), all on the CPU, against things other than
the oracle itself: an independent fp64 composition of torch CPU operators
(conv1d, silu, normalize, logsigmoid, sigmoid, autograd for the backward),
central finite differences of every backward, and closed forms."""
import numpy as np
import pytest
import torch

import oracle

rng = np.random.default_rng(2024)


def _x(*shape, scale=1.0):
    return scale * rng.standard_normal(shape)


def torch_path(x, W, l2):
    """fp64 torch: depthwise causal conv1d (left zero padding of K-1), SiLU, L2 norm."""
    B, T, H, D = x.shape
    K = W.shape[-1]
    xt = x.permute(0, 2, 3, 1).reshape(B, H * D, T)
    y = torch.nn.functional.conv1d(torch.nn.functional.pad(xt, (K - 1, 0)), W[:, None, :], groups=H * D)
    s = torch.nn.functional.silu(y).reshape(B, H, D, T).permute(0, 3, 1, 2)
    if l2:
        s = s / torch.sqrt((s * s).sum(-1, keepdim=True) + 1e-6)
    return s


def torch_epilogue(o, g, gamma):
    r = torch.rsqrt((o * o).mean(-1, keepdim=True) + 1e-6)
    return o * r * gamma * torch.nn.functional.silu(g)


@pytest.mark.parametrize("l2", [True, False])
@pytest.mark.parametrize("K", [1, 4])
def test_prologue_path_against_torch(l2, K):
    x, W, dout = _x(2, 9, 3, 8), _x(3 * 8, K, scale=0.5), _x(2, 9, 3, 8)
    out = oracle.prologue_path(x, W, l2)
    dx, dW = oracle.prologue_path_bwd(x, W, dout, l2)
    xt = torch.tensor(x, requires_grad=True)
    Wt = torch.tensor(W, requires_grad=True)
    ot = torch_path(xt, Wt, l2)
    (ot * torch.tensor(dout)).sum().backward()
    np.testing.assert_allclose(out, ot.detach().numpy(), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(dx, xt.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dW, Wt.grad.numpy(), rtol=1e-10, atol=1e-12)


def test_prologue_finite_differences():
    x, W, dout = _x(1, 6, 2, 4), _x(2 * 4, 4, scale=0.5), _x(1, 6, 2, 4)
    dx, dW = oracle.prologue_path_bwd(x, W, dout, True)
    h = 1e-6
    L = lambda xx, WW: float(np.sum(oracle.prologue_path(xx, WW, True) * dout))
    for idx in [(0, 0, 0, 0), (0, 3, 1, 2), (0, 5, 1, 3), (0, 2, 0, 1)]:
        e = np.zeros_like(x)
        e[idx] = h
        fd = (L(x + e, W) - L(x - e, W)) / (2 * h)
        assert abs(fd - dx[idx]) <= 1e-6 * max(1.0, abs(fd))
    for idx in [(0, 0), (5, 3), (7, 1)]:
        e = np.zeros_like(W)
        e[idx] = h
        fd = (L(x, W + e) - L(x, W - e)) / (2 * h)
        assert abs(fd - dW[idx]) <= 1e-6 * max(1.0, abs(fd))


def test_prologue_closed_forms():
    x = _x(2, 7, 2, 16)
    K = 4
    # a filter that passes the current token only: out = silu(x) / |silu(x)|
    W = np.zeros((2 * 16, K))
    W[:, K - 1] = 1.0
    out = oracle.prologue_path(x, W, True)
    s = x / (1 + np.exp(-x))
    np.testing.assert_allclose(out, s / np.sqrt((s * s).sum(-1, keepdims=True) + 1e-6), rtol=1e-13)
    # unit norm (up to the eps) per token and head
    W = _x(2 * 16, K)
    n = np.linalg.norm(oracle.prologue_path(x, W, True), axis=-1)
    assert np.all(np.abs(n - 1.0) < 1e-4)
    # causality: changing a late token leaves the earlier outputs alone
    x2 = x.copy()
    x2[:, 5] += 1.0
    a, b = oracle.prologue_path(x, W, False), oracle.prologue_path(x2, W, False)
    np.testing.assert_array_equal(a[:, :5], b[:, :5])
    assert np.any(a[:, 5] != b[:, 5])
    # a filter tap j reads the token K-1-j steps back
    W = np.zeros((2 * 16, K))
    W[:, 0] = 1.0
    out = oracle.prologue_path(x, W, False)
    np.testing.assert_array_equal(out[:, :K - 1], np.zeros_like(out[:, :K - 1]))
    np.testing.assert_allclose(out[:, K - 1:], s[:, :-(K - 1)], rtol=1e-14)


@pytest.mark.parametrize("kind", ["log_alpha", "sigmoid"])
def test_gates(kind):
    x = _x(1000, scale=4.0)
    out = oracle.gate(x, kind)
    xt = torch.tensor(x, requires_grad=True)
    ref = torch.nn.functional.logsigmoid(xt) if kind == "log_alpha" else torch.sigmoid(xt)
    np.testing.assert_allclose(out, ref.detach().numpy(), rtol=1e-13, atol=1e-15)
    dout = _x(1000)
    (ref * torch.tensor(dout)).sum().backward()
    np.testing.assert_allclose(oracle.gate_bwd(x, dout, kind), xt.grad.numpy(), rtol=1e-12, atol=1e-15)
    if kind == "log_alpha":
        assert np.all(out < 0) and np.allclose(np.exp(out), 1 / (1 + np.exp(-x)))


def test_epilogue_against_torch_and_finite_differences():
    o, g, gamma, dz = _x(2, 5, 3, 16), _x(2, 5, 3, 16), _x(16, scale=0.5) + 1.0, _x(2, 5, 3, 16)
    z = oracle.epilogue(o, g, gamma)
    dO, dg, dgamma = oracle.epilogue_bwd(o, g, gamma, dz)
    ot, gt, wt = (torch.tensor(a, requires_grad=True) for a in (o, g, gamma))
    zt = torch_epilogue(ot, gt, wt)
    (zt * torch.tensor(dz)).sum().backward()
    np.testing.assert_allclose(z, zt.detach().numpy(), rtol=1e-12, atol=1e-14)
    for a, b in ((dO, ot.grad), (dg, gt.grad), (dgamma, wt.grad)):
        np.testing.assert_allclose(a, b.numpy(), rtol=1e-10, atol=1e-12)
    h = 1e-6
    L = lambda oo, gg, ww: float(np.sum(oracle.epilogue(oo, gg, ww) * dz))
    for idx in [(0, 0, 0, 0), (1, 4, 2, 15), (0, 2, 1, 7)]:
        e = np.zeros_like(o)
        e[idx] = h
        assert abs((L(o + e, g, gamma) - L(o - e, g, gamma)) / (2 * h) - dO[idx]) < 1e-6
        assert abs((L(o, g + e, gamma) - L(o, g - e, gamma)) / (2 * h) - dg[idx]) < 1e-6
    e = np.zeros_like(gamma)
    e[3] = h
    assert abs((L(o, g, gamma + e) - L(o, g, gamma - e)) / (2 * h) - dgamma[3]) < 1e-6


def test_epilogue_closed_form():
    # a constant row c 1 has rms |c|: z = sign(c) gamma silu(g) (up to the eps)
    o = np.full((1, 1, 1, 16), -3.0)
    g = _x(1, 1, 1, 16)
    gamma = _x(16)
    z = oracle.epilogue(o, g, gamma)
    np.testing.assert_allclose(z[0, 0, 0], -gamma * g[0, 0, 0] / (1 + np.exp(-g[0, 0, 0])), rtol=1e-6)
