"""Shared helpers of the GPU parity tests: build a layer from the seeded
inputs, hand the same values to the oracle, and compare."""
from __future__ import annotations

import numpy as np
import torch

from mixture_experts_layer_58_b200 import synth
from oracle import moe_oracle as om

NEAR_TIE = 1e-5          # key gap below which a selection is a near-tie
OUT_MAX_TOL = 1e-2       # max|diff| <= 1e-2 * max|ref|     (bf16 outputs)
OUT_MEAN_TOL = 5e-3      # mean|diff| / mean|ref| <= 5e-3   (bf16 outputs)
GATE_RTOL = {"sigmoid": 5e-5, "softmax": 2e-4}


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


class Inputs:
    """Seeded inputs of a workload, the device layer built from them, and an
    accessor for the oracle's copy of any expert's weights."""

    def __init__(self, cfg: synth.MoEConfig, T: int | None = None, fused_gather: bool = False,
                 fused_scatter: bool = False, fused_combine: bool = False):
        from mixture_experts_layer_58_b200.layer import MoELayer
        self.cfg = cfg
        self.u = synth.tokens(cfg, T)
        self.T = self.u.shape[0]
        self.e = synth.centroids(cfg)
        self.b = synth.bias(cfg)
        wdev = "cuda" if cfg.weights_on_gpu else "cpu"
        self.wdev = wdev
        W1, W3, W2 = synth.all_expert_weights(cfg, wdev)
        self.shared = synth.shared_weights(cfg, wdev)
        if not cfg.weights_on_gpu:
            self.W = (W1, W3, W2)
        self.layer = MoELayer(self.e, self.b, W1, W3, W2, self.shared, top_k=cfg.top_k,
                              routed_scale=cfg.routed_scale, gate_kind=cfg.gate_kind,
                              gamma=cfg.gamma, fused_gather=fused_gather,
                              fused_scatter=fused_scatter, fused_combine=fused_combine)
        del W1, W3, W2
        self.u_dev = self.u.cuda()
        self._cache = {}

    def expert(self, i: int):
        """(w1, w3, w2) of routed expert i as host fp32 arrays (exact bf16 values)."""
        if i not in self._cache:
            if self.cfg.weights_on_gpu:
                ws = synth.expert_weights(self.cfg, i, "cuda")
            else:
                ws = (self.W[0][i], self.W[1][i], self.W[2][i])
            self._cache[i] = tuple(w.float().cpu().numpy() for w in ws)
            if len(self._cache) > 8:
                self._cache.pop(next(iter(self._cache)))
        return self._cache[i]

    def shared_list(self):
        if self.shared is None:
            return []
        return [tuple(w.float().cpu().numpy() for w in self.shared)]

    def oracle_route(self, bias=None):
        b = self.b if bias is None else bias
        return om.route(self.u, self.e, b if self.cfg.gate_kind == "sigmoid" else None,
                        self.cfg.top_k, self.cfg.routed_scale, self.cfg.gate_kind)


def check_route(gpu_idx, gpu_gate, gpu_counts, r: om.Routing, routed_scale, u, e, kind,
                rows=None):
    """Indices bit-exact except near-ties (any adjacent pair of the K+1 largest
    oracle keys closer than NEAR_TIE); near-tie selections must still be a
    valid top-K within that margin; counts exact once the near-tie tokens'
    own contributions are set aside; gates close to the oracle's fp64 gates
    for the GPU's own selection. Returns the number of near-tie tokens."""
    gpu_idx = np.asarray(gpu_idx, dtype=np.int64)
    T, K = gpu_idx.shape
    n = r.keys.shape[1]
    sel = slice(None) if rows is None else rows
    keys = r.keys[sel] if rows is not None else r.keys
    near = r.min_adjacent_gap() < NEAR_TIE
    ok = ~near
    bad = np.nonzero(np.any(gpu_idx[ok] != r.idx[ok], axis=1))[0]
    assert bad.size == 0, f"{bad.size} non-near-tie tokens differ, first {np.nonzero(ok)[0][bad[:5]]}"
    for t in np.nonzero(near)[0]:
        chosen = gpu_idx[t]
        assert len(set(chosen.tolist())) == K
        rest = np.setdiff1d(np.arange(n), chosen)
        kc = keys[t][chosen]
        if rest.size:
            assert kc.min() >= keys[t][rest].max() - NEAR_TIE
        assert np.all(np.diff(kc) <= NEAR_TIE)
    gc = np.asarray(gpu_counts, dtype=np.int64)
    assert gc.sum() == T * K
    assert np.array_equal(gc, np.bincount(gpu_idx.ravel(), minlength=n))
    oc = r.counts - np.bincount(r.idx[near].ravel(), minlength=n)
    assert np.array_equal(gc - np.bincount(gpu_idx[near].ravel(), minlength=n), oc)
    g_ref = om.gates_for_indices(u, e, gpu_idx, routed_scale, kind)
    # fp32 logits carry an absolute error of ~1e-5 at d = 7168; a softmax gate's
    # relative error equals its logit's absolute error, a sigmoid gate's is
    # damped by s'(z)/s(z) <= 1
    rtol = GATE_RTOL[kind]
    np.testing.assert_allclose(np.asarray(gpu_gate, dtype=np.float64), g_ref, rtol=rtol,
                               atol=1e-6)
    np.testing.assert_allclose(np.asarray(gpu_gate, dtype=np.float64).sum(1), routed_scale,
                               rtol=1e-5)
    return int(near.sum())


def check_close(got, ref, max_tol=OUT_MAX_TOL, mean_tol=OUT_MEAN_TOL, what="output"):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    diff = np.abs(got - ref)
    mx = diff.max() / max(np.abs(ref).max(), 1e-30)
    mean = diff.mean() / max(np.abs(ref).mean(), 1e-30)
    assert mx <= max_tol, f"{what}: max|diff| = {mx:.3e} * max|ref| > {max_tol}"
    assert mean <= mean_tol, f"{what}: mean rel err {mean:.3e} > {mean_tol}"
    return mx, mean
