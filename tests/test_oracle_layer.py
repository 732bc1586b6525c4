"""Pins for the oracle's dispatch order, expert FFN and layer output (CPU only).

The pages never define the expert FFN; the SwiGLU form is pinned against
torch's own silu / matmul, and the layer equation against special cases that
reduce to a dense FFN, closed forms and symmetries.
"""
import numpy as np
import torch
import torch.nn.functional as F

from mixture_experts_layer_58_b200 import synth
from oracle import moe_oracle as om


def _small(T=40, d=32, n=6, k=2, ns=1, inter=16, seed=0):
    g = torch.Generator().manual_seed(seed)
    u = torch.randn(T, d, generator=g, dtype=torch.float64)
    e = 0.3 * torch.randn(n, d, generator=g, dtype=torch.float64)
    ws = [tuple(0.2 * torch.randn(s, generator=g, dtype=torch.float64)
                for s in ((inter, d), (inter, d), (d, inter))) for _ in range(n)]
    sh = [tuple(0.2 * torch.randn(s, generator=g, dtype=torch.float64)
                for s in ((inter, d), (inter, d), (d, inter))) for _ in range(ns)]
    b = 0.05 * torch.randn(n, generator=g, dtype=torch.float64)
    return u, e, b, ws, sh


def _torch_swiglu(x, w1, w3, w2):
    return (F.silu(x @ w1.T) * (x @ w3.T)) @ w2.T


def test_ffn_matches_torch_silu_matmul():
    u, _, _, ws, _ = _small()
    got = om.ffn(u, *ws[0])
    want = _torch_swiglu(u, *ws[0]).numpy()
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)


def test_dense_reduction_one_expert_top1():
    # N_r = 1, K = 1, S = 1, N_s = 0  ->  h' = u + FFN(u), a dense SwiGLU layer
    u, _, _, ws, _ = _small(n=1)
    e = torch.zeros(1, u.shape[1], dtype=torch.float64)
    out, r = om.layer(u, e, None, lambda i: ws[i], [], top_k=1, routed_scale=1.0)
    assert np.all(r.idx == 0)
    np.testing.assert_allclose(r.gate, 1.0, rtol=0, atol=0)
    want = (u + _torch_swiglu(u, *ws[0])).numpy()
    np.testing.assert_allclose(out, want, rtol=1e-12, atol=1e-12)


def test_dense_reduction_with_shared_expert():
    u, _, _, ws, sh = _small(n=1, ns=1)
    e = torch.zeros(1, u.shape[1], dtype=torch.float64)
    out, _ = om.layer(u, e, None, lambda i: ws[i], sh, top_k=1, routed_scale=1.0)
    want = (u + _torch_swiglu(u, *ws[0]) + _torch_swiglu(u, *sh[0])).numpy()
    np.testing.assert_allclose(out, want, rtol=1e-12, atol=1e-12)


def test_no_residual_matches_listing_form():
    # the deepseekmodel.com listing returns routed + shared with no residual
    u, e, b, ws, sh = _small()
    with_res, r = om.layer(u, e, b, lambda i: ws[i], sh, 2, 1.0)
    without, _ = om.layer(u, e, b, lambda i: ws[i], sh, 2, 1.0, residual=False)
    np.testing.assert_allclose(with_res - without, u.numpy(), rtol=0, atol=1e-13)


def test_shared_experts_sum_equals_concatenated_ffn():
    # two shared FFNs summed == one FFN with concatenated hidden units
    u, _, _, _, sh = _small(ns=2)
    w1 = torch.cat([sh[0][0], sh[1][0]], 0)
    w3 = torch.cat([sh[0][1], sh[1][1]], 0)
    w2 = torch.cat([sh[0][2], sh[1][2]], 1)
    np.testing.assert_allclose(om.shared_output(u, sh), _torch_swiglu(u, w1, w3, w2).numpy(),
                               rtol=1e-12, atol=1e-12)


def test_all_experts_selected_closed_form():
    # K = N_r: every expert is selected whatever the bias; the output is
    # u + shared + S * sum_i (s_i / sum_j s_j) FFN_i(u)
    u, e, b, ws, sh = _small(n=5)
    out, _ = om.layer(u, e, b, lambda i: ws[i], sh, top_k=5, routed_scale=2.5)
    s = torch.sigmoid(u @ e.T)
    g = 2.5 * s / s.sum(1, keepdim=True)
    want = u + _torch_swiglu(u, *sh[0])
    for i in range(5):
        want = want + g[:, i:i + 1] * _torch_swiglu(u, *ws[i])
    np.testing.assert_allclose(out, want.numpy(), rtol=1e-12, atol=1e-12)


def test_token_permutation_equivariance():
    u, e, b, ws, sh = _small()
    perm = torch.randperm(u.shape[0], generator=torch.Generator().manual_seed(1))
    out, _ = om.layer(u, e, b, lambda i: ws[i], sh, 2, 1.0)
    out_p, _ = om.layer(u[perm], e, b, lambda i: ws[i], sh, 2, 1.0)
    np.testing.assert_allclose(out_p, out[perm.numpy()], rtol=1e-13, atol=1e-13)


def test_expert_relabelling_invariance():
    u, e, b, ws, sh = _small()
    perm = torch.randperm(e.shape[0], generator=torch.Generator().manual_seed(2))
    out, _ = om.layer(u, e, b, lambda i: ws[i], sh, 2, 1.0)
    out_p, _ = om.layer(u, e[perm], b[perm], lambda i: ws[int(perm[i])], sh, 2, 1.0)
    np.testing.assert_allclose(out_p, out, rtol=1e-13, atol=1e-13)


def test_routed_part_linear_in_w2_and_scale():
    u, e, b, ws, sh = _small()
    base, _ = om.layer(u, e, b, lambda i: ws[i], [], 2, 1.0, residual=False)
    scaled, _ = om.layer(u, e, b, lambda i: ws[i], [], 2, 3.0, residual=False)
    np.testing.assert_allclose(scaled, 3.0 * base, rtol=1e-12, atol=1e-13)
    ws2 = [(a, c, 2.0 * w2) for (a, c, w2) in ws]
    doubled, _ = om.layer(u, e, b, lambda i: ws2[i], [], 2, 1.0, residual=False)
    np.testing.assert_allclose(doubled, 2.0 * base, rtol=1e-12, atol=1e-13)


def test_routed_output_equals_per_token_loop():
    # the per-expert grouping equals the plain per-token sum of the equation
    u, e, b, ws, sh = _small(T=12)
    r = om.route(u, e, b, 2, 1.7)
    grouped = om.routed_output(u, r.idx, r.gate, lambda i: ws[i])
    for t in range(u.shape[0]):
        acc = torch.zeros(u.shape[1], dtype=torch.float64)
        for k in range(2):
            acc += r.gate[t, k] * _torch_swiglu(u[t:t + 1], *ws[r.idx[t, k]])[0]
        np.testing.assert_allclose(grouped[t], acc.numpy(), rtol=1e-12, atol=1e-13)


def test_gates_for_indices_reproduces_route():
    cfg = synth.CONFIGS["tiny"]
    u, e, b = synth.tokens(cfg), synth.centroids(cfg), synth.bias(cfg)
    r = om.route(u, e, b, cfg.top_k, 1.3)
    np.testing.assert_array_equal(om.gates_for_indices(u, e, r.idx, 1.3), r.gate)


# ---------------- dispatch order ----------------

def test_dispatch_handworked():
    # 3 tokens, K = 2, 3 experts: rows grouped by expert, ascending token inside
    idx = np.array([[2, 0], [0, 1], [2, 1]])
    d = om.dispatch(idx, 3)
    assert d.offsets.tolist() == [0, 2, 4, 6]
    # expert 0: tokens 0, 1 -> rows 0, 1; expert 1: tokens 1, 2 -> rows 2, 3;
    # expert 2: tokens 0, 2 -> rows 4, 5
    assert d.src.tolist() == [0, 1, 1, 2, 0, 2]
    assert d.pos.tolist() == [[4, 0], [1, 2], [5, 3]]


def test_dispatch_bijection_and_stability():
    cfg = synth.CONFIGS["tiny"]
    u, e, b = synth.tokens(cfg), synth.centroids(cfg), synth.bias(cfg)
    r = om.route(u, e, b, cfg.top_k, cfg.routed_scale)
    d = om.dispatch(r.idx, cfg.n_routed)
    n = cfg.T * cfg.top_k
    assert sorted(d.pos.ravel().tolist()) == list(range(n))
    assert np.array_equal(d.offsets, np.concatenate([[0], np.cumsum(r.counts)]))
    for t in range(cfg.T):
        for k in range(cfg.top_k):
            p = d.pos[t, k]
            assert d.src[p] == t
            ex = r.idx[t, k]
            assert d.offsets[ex] <= p < d.offsets[ex + 1]
    for ex in range(cfg.n_routed):
        rows = d.src[d.offsets[ex]:d.offsets[ex + 1]]
        assert np.all(np.diff(rows) > 0)
