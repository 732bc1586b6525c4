"""fp64 backward of the DeepSeekMoE layer, for the oracle.

TEST INFRASTRUCTURE: only the tests, the smoke check and the benchmark's
CPU-baseline leg may import this module.

Sources:
  [V3]   "DeepSeek-V3 technical report" summary (xyznot.com), "Method" §2:
         the layer output h'_t = u_t + sum_i FFN_i^(s)(u_t)
         + sum_i g_{i,t} FFN_i^(r)(u_t), the gates g_{i,t} = s_{i,t} / sum of
         the selected s (times the routed scale), s_{i,t} = Sigmoid(u_t . e_i),
         and the biased top-K that decides only WHICH experts are used.
  [ARCH] "DeepSeek model architecture explained" (deepseekmodel.com): the
         softmax-over-top-k gate variant, and, in the block-quantisation
         pseudocode, that gradients are computed in BF16.

The pages print no backward equations. What this module computes is the exact
derivative of the forward oracle (moe_oracle.layer_output with the gates of
moe_oracle.gates_from_selection), written out by the chain rule:

  * the selection idx is piecewise constant in u and e: no gradient flows
    through which experts are chosen, only through the gate values of the
    selected ones; the bias b (selection only) gets none;
  * FFN(x) = W2 (silu(W1 x) * (W3 x)); with a = W1 x, c = W3 x,
    h = silu(a) * c:  dh = W2^T dy,  dW2 = dy h^T,  dc = dh * silu(a),
    da = dh * c * silu'(a) with silu'(a) = sig(a) (1 + a (1 - sig(a))),
    dx = W1^T da + W3^T dc,  dW1 = da x^T,  dW3 = dc x^T;
  * routed term g_k y_k: dy_k = g_k dout, dg_k = dout . y_k;
  * sigmoid gate g_k = S s_k / sum_j s_j (sum over the selected):
    ds_k = (S / sum) (dg_k - sum_j dg_j s_j / sum), then dz_k = ds_k s_k (1 - s_k);
  * softmax gate g_k = S p_k, p = softmax of the selected logits z:
    dz_k = g_k (dg_k - sum_j p_j dg_j);
  * z_{t,i} = u_t . e_i: du_t += sum_k dz_k e_{idx_k}, de_{idx_k} += dz_k u_t;
  * the residual passes dout to du unchanged.

Pinned in tests/test_oracle_backward.py by central finite differences of the
forward oracle (every output, both gate kinds) and by torch.autograd on an
independent torch formulation of the forward.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

from .moe_oracle import _f64, affinity_logits, gates_from_selection, sigmoid


def silu_grad(a: np.ndarray) -> np.ndarray:
    """d silu(a) / da = sig(a) (1 + a (1 - sig(a)))."""
    s = sigmoid(a)
    return s * (1.0 + a * (1.0 - s))


def ffn_backward(x, w1, w3, w2, dy):
    """Gradients of y = W2 (silu(W1 x) * (W3 x)) for rows x [n,d] given dy [n,d].

    Returns (dx [n,d], dw1 [I,d], dw3 [I,d], dw2 [d,I]), fp64."""
    x, w1, w3, w2, dy = (_f64(v) for v in (x, w1, w3, w2, dy))
    a = x @ w1.T
    c = x @ w3.T
    sa = a * sigmoid(a)
    h = sa * c
    dh = dy @ w2
    dw2 = dy.T @ h
    dc = dh * sa
    da = dh * c * silu_grad(a)
    dx = da @ w1 + dc @ w3
    return dx, da.T @ x, dc.T @ x, dw2


def gate_backward(score_sel, dgate, routed_scale: float, kind: str = "sigmoid"):
    """dL/dz of the selected logits [T,K] from dL/dg [T,K].

    score_sel: the selected scores, s = Sigmoid(z) (kind 'sigmoid') or the raw
    logits z (kind 'softmax'), [T,K]."""
    sc = _f64(score_sel)
    dg = _f64(dgate)
    S = float(routed_scale)
    if kind == "sigmoid":
        tot = sc.sum(axis=1, keepdims=True)
        ds = (S / tot) * (dg - (dg * sc).sum(axis=1, keepdims=True) / tot)
        return ds * sc * (1.0 - sc)
    if kind == "softmax":
        m = sc.max(axis=1, keepdims=True)
        p = np.exp(sc - m)
        p /= p.sum(axis=1, keepdims=True)
        return S * p * (dg - (p * dg).sum(axis=1, keepdims=True))
    raise ValueError(f"unknown gate kind {kind!r}")


@dataclass
class LayerGrads:
    du: np.ndarray                    # [T,d]
    de: np.ndarray                    # [N_r,d] centroids
    dgate: np.ndarray                 # [T,K] dL/dg of each selected slot
    dz: np.ndarray                    # [T,K] dL/dz of each selected logit
    dw1: dict = field(default_factory=dict)   # expert -> [I,d]
    dw3: dict = field(default_factory=dict)   # expert -> [I,d]
    dw2: dict = field(default_factory=dict)   # expert -> [d,I]
    dshared: list = field(default_factory=list)   # [(dw1, dw3, dw2)] per shared expert


def layer_backward(u, e, idx, routed_scale: float, expert, shared, dout,
                   kind: str = "sigmoid", residual: bool = True) -> LayerGrads:
    """Backward of h' = layer_output(u, idx, gates(u, e, idx), expert, shared)
    with the selection idx [T,K] held fixed.

    expert(i) -> (w1, w3, w2) of routed expert i; shared: list of (w1, w3, w2)."""
    u64 = _f64(u)
    e64 = _f64(e)
    idx = np.asarray(idx, dtype=np.int64)
    dout = _f64(dout)
    T, K = idx.shape
    z = affinity_logits(u64, e64)
    score = sigmoid(z) if kind == "sigmoid" else z
    sel = np.take_along_axis(score, idx, axis=1)        # [T,K]
    gate = gates_from_selection(score, idx, routed_scale, kind)

    du = dout.copy() if residual else np.zeros_like(u64)
    out = LayerGrads(du=du, de=np.zeros_like(e64), dgate=np.zeros((T, K)), dz=np.zeros((T, K)))
    for (w1, w3, w2) in (shared or []):
        dx, dw1, dw3, dw2 = ffn_backward(u64, w1, w3, w2, dout)
        du += dx
        out.dshared.append((dw1, dw3, dw2))
    for i in np.unique(idx):
        t, k = np.nonzero(idx == i)
        w1, w3, w2 = (_f64(w) for w in expert(int(i)))
        x = u64[t]
        a = x @ w1.T
        y = ((a * sigmoid(a)) * (x @ w3.T)) @ w2.T
        out.dgate[t, k] = np.einsum("nd,nd->n", dout[t], y)
        dx, dw1, dw3, dw2 = ffn_backward(x, w1, w3, w2, gate[t, k][:, None] * dout[t])
        np.add.at(du, t, dx)
        out.dw1[int(i)], out.dw3[int(i)], out.dw2[int(i)] = dw1, dw3, dw2
    out.dz = gate_backward(sel, out.dgate, routed_scale, kind)
    for k in range(K):
        du += out.dz[:, k:k + 1] * e64[idx[:, k]]
        np.add.at(out.de, idx[:, k], out.dz[:, k:k + 1] * u64)
    return out
