"""fp64 CPU oracle of the DeepSeekMoE layer forward and its bias update.

TEST INFRASTRUCTURE. Only the tests, the package's smoke check and the
benchmark's CPU-baseline leg may import this module. The product path never
calls it, and it shares no code with the CUDA kernels or their binding.

Sources (web pages; the page title and the section they fall in):
  [V3]  "DeepSeek-V3 technical report" summary (xyznot.com, arXiv 2412.19437),
        Method §2 "DeepSeekMoE with auxiliary-loss-free balancing":
        the output equation h'_t, the affinity s_{i,t}, the selection equation
        g'_{i,t}, the normalisation of g', and the end-of-step bias update.
        "Main ideas": 1 shared + 256 routed experts, 8 active.
  [ARCH] "DeepSeek model architecture explained" (deepseekmodel.com),
        DeepSeekMoE forward listing: top-k over the raw gate logits, softmax
        over the k selected logits in fp32, routed sum + shared expert.

Every input float array is converted to fp64 (the exact value of the bf16 or
fp32 number it holds) and all arithmetic below is fp64, with no intermediate
rounding. The only rounding is the bias vector, which is state stored in fp32.

Readings where the pages are silent:
  * the expert FFN is SwiGLU without biases, W2 (silu(W1 x) * (W3 x));
    the pages never define ExpertFFN  -> parity of the FFN itself is pinned
    only by the dense special case and library identities (tests);
  * N_s shared experts are N_s independent FFNs summed ([V3] h'_t);
  * the routed scale S multiplies the normalised gates;
  * top-k ties: the lower expert index wins; selected experts are listed in
    descending key order, ties in ascending index;
  * "overloaded" / "underloaded" is relative to the mean load T*K/N_r,
    compared exactly in integers (N_r*c_i vs T*K); equal load = no change;
  * the softmax gate form of [ARCH] has no bias and no sigmoid.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np


def _f64(x) -> np.ndarray:
    """Exact fp64 copy of a numpy array or a torch tensor (bf16 included)."""
    if hasattr(x, "detach"):                       # torch tensor, never imported here
        x = x.detach()
        if str(x.dtype) == "torch.bfloat16":
            x = x.float()
        x = x.cpu().numpy()
    return np.asarray(x, dtype=np.float64)


# --------------------------------------------------------------------------
# Routing: affinity, bias-adjusted top-K, gates, load counts  ([V3] Method §2)
# --------------------------------------------------------------------------

def affinity_logits(u, e) -> np.ndarray:
    """z_{t,i} = u_t . e_i for every token t and routed expert i ([V3] s_{i,t}
    argument). u [T,d], e [N_r,d] -> z [T,N_r] fp64."""
    return _f64(u) @ _f64(e).T


def sigmoid(z: np.ndarray) -> np.ndarray:
    """Sigmoid(z) = 1 / (1 + exp(-z)) ([V3] s_{i,t} = Sigmoid(u_t^T e_i))."""
    return 1.0 / (1.0 + np.exp(-z))


@dataclass
class Routing:
    idx: np.ndarray       # [T,K] int64, selected experts, descending key
    gate: np.ndarray      # [T,K] fp64, g_{i,t} of each selected expert
    counts: np.ndarray    # [N_r] int64, tokens routed to each expert
    keys: np.ndarray      # [T,N_r] fp64, selection key of every expert
    score: np.ndarray     # [T,N_r] fp64, s_{i,t} (sigmoid) or z_{t,i} (softmax)
    sorted_keys: np.ndarray   # [T,K+1] fp64, the K+1 largest keys, descending

    def boundary_gap(self) -> np.ndarray:
        """Key gap between the K-th and (K+1)-th expert of each token."""
        k = self.idx.shape[1]
        if self.sorted_keys.shape[1] <= k:
            return np.full(self.idx.shape[0], np.inf)
        return self.sorted_keys[:, k - 1] - self.sorted_keys[:, k]

    def min_adjacent_gap(self) -> np.ndarray:
        """Smallest gap between neighbours among the K+1 largest keys: below a
        threshold, either the selected set or its order is a near-tie."""
        return np.min(self.sorted_keys[:, :-1] - self.sorted_keys[:, 1:], axis=1)


def select_topk(keys: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k largest keys per row, in descending key order; equal
    keys keep ascending expert index (stable sort on -key). This is the Topk
    set of [V3]'s g'_{i,t} equation with the tie reading stated above."""
    order = np.argsort(-keys, axis=1, kind="stable")
    return order[:, :k]


def gates_from_selection(score: np.ndarray, idx: np.ndarray, routed_scale: float,
                         kind: str = "sigmoid") -> np.ndarray:
    """Gate value of each selected expert.

    sigmoid ([V3]): g'_{i,t} = s_{i,t} for selected i (the UNBIASED affinity;
    the bias only chooses), g_{i,t} = g'_{i,t} / sum_j g'_{j,t}, times S.
    softmax ([ARCH]): softmax over the k selected raw logits, times S.
    """
    sel = np.take_along_axis(score, idx, axis=1)
    if kind == "sigmoid":
        g = sel / sel.sum(axis=1, keepdims=True)
    elif kind == "softmax":
        m = sel.max(axis=1, keepdims=True)
        ex = np.exp(sel - m)
        g = ex / ex.sum(axis=1, keepdims=True)
    else:
        raise ValueError(kind)
    return routed_scale * g


def expert_counts(idx: np.ndarray, n_routed: int) -> np.ndarray:
    """c_i = number of (token, slot) pairs routed to expert i."""
    c = np.zeros(n_routed, dtype=np.int64)
    for i in idx.reshape(-1):
        c[i] += 1
    return c


def route(u, e, b, top_k: int, routed_scale: float, kind: str = "sigmoid") -> Routing:
    """Full routing of a batch ([V3] Method §2; [ARCH] for kind='softmax').

    sigmoid: s = Sigmoid(u e^T); key = s + b; Topk of the keys; gates from s.
    softmax: z = u e^T; key = z (no bias); Topk; softmax over selected z.
    """
    z = affinity_logits(u, e)
    if kind == "sigmoid":
        score = sigmoid(z)
        keys = score + _f64(b)[None, :] if b is not None else score.copy()
    elif kind == "softmax":
        score = z
        keys = z.copy()
    else:
        raise ValueError(kind)
    n_routed = keys.shape[1]
    kk = min(top_k + 1, n_routed)
    top = select_topk(keys, kk)
    idx = top[:, :top_k]
    sorted_keys = np.take_along_axis(keys, top, axis=1)
    gate = gates_from_selection(score, idx, routed_scale, kind)
    return Routing(idx=idx, gate=gate, counts=expert_counts(idx, n_routed), keys=keys,
                   score=score, sorted_keys=sorted_keys)


def gates_for_indices(u, e, idx, routed_scale: float, kind: str = "sigmoid") -> np.ndarray:
    """The oracle's fp64 gates for a GIVEN selection idx [T,K] (used to check the
    layer output on the GPU's own routing when a near-tie flipped an expert)."""
    z = affinity_logits(u, e)
    score = sigmoid(z) if kind == "sigmoid" else z
    return gates_from_selection(score, np.asarray(idx, dtype=np.int64), routed_scale, kind)


# --------------------------------------------------------------------------
# Dispatch order (expert-contiguous rows)
# --------------------------------------------------------------------------

@dataclass
class Dispatch:
    offsets: np.ndarray   # [N_r+1] int64, exclusive scan of counts
    pos: np.ndarray       # [T,K] int64, row of (t, slot k) in the permuted buffer
    src: np.ndarray       # [T*K] int64, token of each permuted row


def dispatch(idx, n_routed: int) -> Dispatch:
    """Expert-contiguous order of the (token, slot) pairs: expert 0's tokens
    first, then expert 1's, ...; inside an expert, ascending token index. This
    is the grouping the [ARCH] listing does with its per-expert mask
    (hidden_states[expert_mask]), written out as explicit row numbers."""
    idx = np.asarray(idx, dtype=np.int64)
    T, K = idx.shape
    counts = expert_counts(idx, n_routed)
    offsets = np.zeros(n_routed + 1, dtype=np.int64)
    for i in range(n_routed):
        offsets[i + 1] = offsets[i] + counts[i]
    nxt = offsets[:-1].copy()
    pos = np.full((T, K), -1, dtype=np.int64)
    src = np.full(T * K, -1, dtype=np.int64)
    for i in range(n_routed):
        for t in range(T):
            for k in range(K):
                if idx[t, k] == i:
                    pos[t, k] = nxt[i]
                    src[nxt[i]] = t
                    nxt[i] += 1
    return Dispatch(offsets=offsets, pos=pos, src=src)


# --------------------------------------------------------------------------
# Expert FFN and the layer output ([V3] output equation h'_t)
# --------------------------------------------------------------------------

def silu(a: np.ndarray) -> np.ndarray:
    """silu(a) = a * Sigmoid(a)."""
    return a * sigmoid(a)


def ffn(x, w1, w3, w2) -> np.ndarray:
    """SwiGLU expert: FFN(x) = W2 (silu(W1 x) * (W3 x)), row-wise for x [n,d];
    w1, w3 [I,d], w2 [d,I]."""
    x = _f64(x)
    a = x @ _f64(w1).T
    g = x @ _f64(w3).T
    return (silu(a) * g) @ _f64(w2).T


def shared_output(u, shared) -> np.ndarray:
    """sum_{i<=N_s} FFN_i^(s)(u_t). `shared` is a list of (w1,w3,w2) triples, one
    per shared expert (or None / empty for N_s = 0)."""
    u64 = _f64(u)
    out = np.zeros_like(u64)
    for (w1, w3, w2) in (shared or []):
        out += ffn(u64, w1, w3, w2)
    return out


def routed_output(u, idx, gate, expert) -> np.ndarray:
    """sum_i g_{i,t} FFN_i^(r)(u_t) over the experts with non-zero g.

    `expert(i)` returns the (w1,w3,w2) of routed expert i. The FFN of expert i
    is evaluated on all tokens that selected it at once (a matrix product over
    those tokens), then each token adds g times its row."""
    u64 = _f64(u)
    idx = np.asarray(idx, dtype=np.int64)
    gate = _f64(gate)
    out = np.zeros_like(u64)
    for i in np.unique(idx):
        t, k = np.nonzero(idx == i)
        w1, w3, w2 = expert(int(i))
        y = ffn(u64[t], w1, w3, w2)
        out[t] += gate[t, k][:, None] * y
    return out


def layer_output(u, idx, gate, expert, shared, residual: bool = True) -> np.ndarray:
    """h'_t = u_t + sum_s FFN^(s)(u_t) + sum_i g_{i,t} FFN_i^(r)(u_t)  ([V3])."""
    out = routed_output(u, idx, gate, expert) + shared_output(u, shared)
    if residual:
        out += _f64(u)
    return out


def layer(u, e, b, expert, shared, top_k: int, routed_scale: float,
          kind: str = "sigmoid", residual: bool = True):
    """Route then combine: returns (h' [T,d] fp64, Routing)."""
    r = route(u, e, b, top_k, routed_scale, kind)
    return layer_output(u, r.idx, r.gate, expert, shared, residual), r


# --------------------------------------------------------------------------
# Auxiliary-loss-free bias update ([V3] Method §2, end of each step)
# --------------------------------------------------------------------------

def bias_update(counts, b, T: int, top_k: int, gamma: float) -> np.ndarray:
    """b_i <- b_i - gamma if expert i is overloaded, + gamma if underloaded.

    Load is compared with the mean T*K/N_r exactly, as N_r*c_i vs T*K. gamma is
    the fp32 value the kernels receive; the sum is formed in fp64 (exact for
    fp32 operands of these magnitudes) and the result stored as fp32."""
    c = np.asarray(counts, dtype=np.int64)
    n = c.shape[0]
    g = float(np.float32(gamma))
    b64 = np.asarray(b, dtype=np.float32).astype(np.float64)
    out = b64.copy()
    for i in range(n):
        if n * c[i] > T * top_k:
            out[i] = b64[i] - g
        elif n * c[i] < T * top_k:
            out[i] = b64[i] + g
    return out.astype(np.float32)
