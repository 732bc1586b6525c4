"""Pins of the backward oracle (oracle/moe_backward.py), CPU only.

The pages print no backward equations; the backward is the derivative of the
forward layer of the "DeepSeek-V3 technical report" summary, Method §2 (and of
the softmax-over-top-k gate of "DeepSeek model architecture explained"). It is
pinned here against things that do not share its derivation: central finite
differences of the forward oracle, torch.autograd on an independent torch
formulation of the forward, and closed forms (a single selected expert has a
constant gate, so no gradient reaches the router)."""
import numpy as np
import pytest
import torch

from oracle import moe_backward as mb
from oracle import moe_oracle as om


def _rand(rng, *shape, scale=1.0):
    return scale * rng.standard_normal(shape)


def _fd(f, x, eps=1e-6):
    """Central differences of the scalar f() w.r.t. every entry of array x (in place)."""
    g = np.zeros_like(x)
    it = np.nditer(x, flags=["multi_index"])
    for _ in it:
        i = it.multi_index
        old = x[i]
        x[i] = old + eps
        fp = f()
        x[i] = old - eps
        fm = f()
        x[i] = old
        g[i] = (fp - fm) / (2 * eps)
    return g


def _close(a, b, rtol=1e-6, atol=1e-8):
    np.testing.assert_allclose(a, b, rtol=rtol, atol=atol)


def test_ffn_backward_matches_finite_differences():
    rng = np.random.default_rng(0)
    n, d, I = 3, 8, 4
    x, w1, w3, w2 = _rand(rng, n, d), _rand(rng, I, d), _rand(rng, I, d), _rand(rng, d, I)
    dy = _rand(rng, n, d)
    loss = lambda: float((dy * om.ffn(x, w1, w3, w2)).sum())
    dx, dw1, dw3, dw2 = mb.ffn_backward(x, w1, w3, w2, dy)
    _close(dx, _fd(loss, x))
    _close(dw1, _fd(loss, w1))
    _close(dw3, _fd(loss, w3))
    _close(dw2, _fd(loss, w2))


def test_silu_grad_matches_finite_differences():
    a = np.linspace(-8, 8, 33)
    fd = (om.silu(a + 1e-6) - om.silu(a - 1e-6)) / 2e-6
    _close(mb.silu_grad(a), fd, rtol=1e-7, atol=1e-9)


def _tiny_problem(kind, seed=1, T=5, d=8, n_routed=6, K=2, I=4, n_shared=1):
    rng = np.random.default_rng(seed)
    u = _rand(rng, T, d)
    e = _rand(rng, n_routed, d, scale=0.5)
    b = _rand(rng, n_routed, scale=0.05)
    W = [(_rand(rng, I, d, scale=0.5), _rand(rng, I, d, scale=0.5), _rand(rng, d, I, scale=0.5))
         for _ in range(n_routed)]
    shared = [(_rand(rng, I, d, scale=0.5), _rand(rng, I, d, scale=0.5),
               _rand(rng, d, I, scale=0.5)) for _ in range(n_shared)]
    bias = b if kind == "sigmoid" else None
    idx = om.route(u, e, bias, K, 2.5, kind).idx
    dout = _rand(rng, T, d)
    return u, e, W, shared, idx, dout


@pytest.mark.parametrize("kind", ["sigmoid", "softmax"])
def test_layer_backward_matches_finite_differences(kind):
    S = 2.5
    u, e, W, shared, idx, dout = _tiny_problem(kind)

    def loss():
        g = om.gates_for_indices(u, e, idx, S, kind)
        return float((dout * om.layer_output(u, idx, g, lambda i: W[i], shared)).sum())

    gr = mb.layer_backward(u, e, idx, S, lambda i: W[i], shared, dout, kind)
    _close(gr.du, _fd(loss, u))
    _close(gr.de, _fd(loss, e))
    for i in np.unique(idx):
        w1, w3, w2 = W[i]
        _close(gr.dw1[int(i)], _fd(loss, w1))
        _close(gr.dw3[int(i)], _fd(loss, w3))
        _close(gr.dw2[int(i)], _fd(loss, w2))
    for (w1, w3, w2), (g1, g3, g2) in zip(shared, gr.dshared):
        _close(g1, _fd(loss, w1))
        _close(g3, _fd(loss, w3))
        _close(g2, _fd(loss, w2))
    # experts no token chose get no gradient entry; their centroid rows stay 0
    unused = sorted(set(range(len(W))) - set(np.unique(idx).tolist()))
    for i in unused:
        assert i not in gr.dw1
        assert np.all(gr.de[i] == 0)


def _torch_forward(u, e, idx, S, W, shared, kind):
    """The layer forward written with torch ops (gather, softmax, silu), so that
    autograd derives its gradient independently of the hand-written backward."""
    z = u @ e.T
    zs = torch.gather(z, 1, idx)
    if kind == "sigmoid":
        s = torch.sigmoid(zs)
        g = S * s / s.sum(dim=1, keepdim=True)
    else:
        g = S * torch.softmax(zs, dim=1)
    out = u.clone()
    for (w1, w3, w2) in shared:
        out = out + (torch.nn.functional.silu(u @ w1.T) * (u @ w3.T)) @ w2.T
    for k in range(idx.shape[1]):
        for i in torch.unique(idx[:, k]).tolist():
            m = idx[:, k] == i
            w1, w3, w2 = W[i]
            y = (torch.nn.functional.silu(u[m] @ w1.T) * (u[m] @ w3.T)) @ w2.T
            out = out.index_add(0, torch.nonzero(m).flatten(), g[m, k:k + 1] * y)
    return out


@pytest.mark.parametrize("kind", ["sigmoid", "softmax"])
def test_layer_backward_matches_torch_autograd(kind):
    S = 2.5
    u, e, W, shared, idx, dout = _tiny_problem(kind, seed=7, T=9, d=16, n_routed=8, K=3, I=8,
                                               n_shared=2)
    tu = torch.tensor(u, requires_grad=True)
    te = torch.tensor(e, requires_grad=True)
    tW = [tuple(torch.tensor(w, requires_grad=True) for w in ws) for ws in W]
    tS = [tuple(torch.tensor(w, requires_grad=True) for w in ws) for ws in shared]
    out = _torch_forward(tu, te, torch.tensor(idx), S, tW, tS, kind)
    (out * torch.tensor(dout)).sum().backward()
    gr = mb.layer_backward(u, e, idx, S, lambda i: W[i], shared, dout, kind)
    _close(gr.du, tu.grad.numpy(), rtol=1e-10, atol=1e-12)
    _close(gr.de, te.grad.numpy(), rtol=1e-10, atol=1e-12)
    for i in np.unique(idx):
        for got, ref in zip((gr.dw1[int(i)], gr.dw3[int(i)], gr.dw2[int(i)]), tW[int(i)]):
            _close(got, ref.grad.numpy(), rtol=1e-10, atol=1e-12)
    for got3, ref3 in zip(gr.dshared, tS):
        for got, ref in zip(got3, ref3):
            _close(got, ref.grad.numpy(), rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("kind", ["sigmoid", "softmax"])
def test_single_expert_gate_is_constant(kind):
    """K = 1: the gate is S whatever the score, so dz = 0 and de = 0; du is
    the residual plus the FFN paths only."""
    rng = np.random.default_rng(3)
    sel = rng.uniform(0.1, 0.9, size=(6, 1))
    dg = rng.standard_normal((6, 1))
    np.testing.assert_array_equal(mb.gate_backward(sel, dg, 2.5, kind), np.zeros((6, 1)))


def test_sigmoid_gate_backward_two_experts_closed_form():
    """K = 2, g_1 = S s_1 / (s_1 + s_2): dg_1/ds_1 = S s_2 / (s_1+s_2)^2 and
    dg_1/ds_2 = -S s_1 / (s_1+s_2)^2, times s (1 - s) for the logit."""
    S = 2.5
    s1, s2 = 0.3, 0.6
    sel = np.array([[s1, s2]])
    dz = mb.gate_backward(sel, np.array([[1.0, 0.0]]), S, "sigmoid")
    tot = s1 + s2
    _close(dz[0, 0], S * s2 / tot ** 2 * s1 * (1 - s1), rtol=1e-14)
    _close(dz[0, 1], -S * s1 / tot ** 2 * s2 * (1 - s2), rtol=1e-14)
