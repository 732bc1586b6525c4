"""Pins for the oracle's routing and bias update (CPU only).

Each check comes from something other than the oracle's own formulas: hand
worked fractions (tests/golden), brute force over all subsets, library
routines (torch.topk / torch.softmax), and invariants of the equations.
"""
import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from mixture_experts_layer_58_b200 import synth
from oracle import moe_oracle as om

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _logit(sym: str) -> float:
    table = {"ln3": math.log(3.0), "-ln3": -math.log(3.0), "ln7": math.log(7.0), "0": 0.0}
    return table[sym]


def test_route_handworked_golden():
    spec = json.load(open(os.path.join(GOLDEN, "route_handworked.json")))
    for case in spec["cases"]:
        z = np.array([_logit(s) for s in case["logits"]])
        u = np.ones((1, 1))
        e = z[:, None]
        r = om.route(u, e, np.array(case["bias"], dtype=np.float64), case["top_k"],
                     case["scale"], case["kind"])
        assert r.idx[0].tolist() == case["idx"], case["name"]
        want = np.array([float(Fraction(g)) for g in case["gate"]])
        np.testing.assert_allclose(r.gate[0], want, rtol=1e-13, err_msg=case["name"])


def test_topk_matches_brute_force_over_all_subsets():
    cfg = synth.CONFIGS["tiny"]
    u, e, b = synth.tokens(cfg), synth.centroids(cfg), synth.bias(cfg)
    r = om.route(u, e, b, cfg.top_k, cfg.routed_scale)
    n = cfg.n_routed
    subsets = np.array(list(itertools.combinations(range(n), cfg.top_k)))   # C(16,4) = 1820
    for t in range(cfg.T):
        sums = r.keys[t][subsets].sum(axis=1)
        best = subsets[np.argmax(sums)]
        assert sorted(r.idx[t].tolist()) == sorted(best.tolist())
        # descending key order inside the selection
        assert np.all(np.diff(r.keys[t][r.idx[t]]) <= 0)
        # every selected key beats every unselected key
        rest = np.setdiff1d(np.arange(n), r.idx[t])
        assert r.keys[t][r.idx[t]].min() >= r.keys[t][rest].max()


def test_selection_equals_torch_topk():
    cfg = synth.CONFIGS["tiny"]
    u, e, b = synth.tokens(cfg), synth.centroids(cfg), synth.bias(cfg)
    r = om.route(u, e, b, cfg.top_k, cfg.routed_scale)
    z = torch.tensor(u.double().numpy() @ e.double().numpy().T)
    keys = torch.sigmoid(z) + b.double()[None, :]
    _, ti = torch.topk(keys, cfg.top_k, dim=1, sorted=True)
    assert np.array_equal(r.idx, ti.numpy())


def test_gates_sum_to_scale_and_follow_unbiased_affinity():
    cfg = synth.CONFIGS["tiny"].replace(routed_scale=2.5, bias_lo=-0.2, bias_hi=0.2)
    u, e, b = synth.tokens(cfg), synth.centroids(cfg), synth.bias(cfg)
    r = om.route(u, e, b, cfg.top_k, cfg.routed_scale)
    np.testing.assert_allclose(r.gate.sum(axis=1), 2.5, rtol=1e-14)
    assert np.all(r.gate > 0)
    s = 1.0 / (1.0 + np.exp(-(u.double().numpy() @ e.double().numpy().T)))
    s_sel = np.take_along_axis(s, r.idx, axis=1)
    # g_k / g_0 == s_k / s_0 (the bias only selects)
    np.testing.assert_allclose(r.gate / r.gate[:, :1], s_sel / s_sel[:, :1], rtol=1e-13)


def test_bias_changes_selection_not_gate_formula():
    # a large bias on one expert forces it into every token's selection
    cfg = synth.CONFIGS["tiny"]
    u, e = synth.tokens(cfg), synth.centroids(cfg)
    b = np.zeros(cfg.n_routed)
    b[5] = 10.0
    r = om.route(u, e, b, cfg.top_k, 1.0)
    assert np.all(r.idx[:, 0] == 5)
    assert r.counts[5] == cfg.T


def test_softmax_gate_matches_torch_listing_form():
    cfg = synth.CONFIGS["tiny"]
    u, e = synth.tokens(cfg), synth.centroids(cfg)
    r = om.route(u, e, None, cfg.top_k, 1.0, kind="softmax")
    logits = torch.tensor(u.double().numpy() @ e.double().numpy().T)
    w, ti = torch.topk(logits, cfg.top_k, dim=-1)
    w = torch.softmax(w, dim=-1)
    assert np.array_equal(r.idx, ti.numpy())
    np.testing.assert_allclose(r.gate, w.numpy(), rtol=1e-13)


def test_counts_histogram_and_total():
    for name in ("tiny", "mid"):
        cfg = synth.CONFIGS[name]
        u, e, b = synth.tokens(cfg), synth.centroids(cfg), synth.bias(cfg)
        r = om.route(u, e, b, cfg.top_k, cfg.routed_scale)
        assert r.counts.sum() == cfg.T * cfg.top_k
        assert np.array_equal(r.counts, np.bincount(r.idx.ravel(), minlength=cfg.n_routed))
        # each token selects K distinct experts
        assert all(len(set(row)) == cfg.top_k for row in r.idx.tolist())


def test_near_tie_measures():
    keys = np.array([[0.9, 0.5, 0.5 + 5e-6, 0.1]])
    r = om.Routing(idx=np.array([[0, 2]]), gate=None, counts=None, keys=keys, score=keys,
                   sorted_keys=np.array([[0.9, 0.5 + 5e-6, 0.5]]))
    assert r.boundary_gap()[0] == pytest.approx(5e-6)
    assert r.min_adjacent_gap()[0] == pytest.approx(5e-6)


def test_bias_update_handworked_golden():
    spec = json.load(open(os.path.join(GOLDEN, "bias_update_handworked.json")))
    out = om.bias_update(spec["counts"], np.array(spec["bias_in"], dtype=np.float32),
                         spec["T"], spec["top_k"], spec["gamma"])
    assert out.dtype == np.float32
    assert out.tolist() == spec["bias_out"]


def test_bias_update_sign_invariant_and_fp32_storage():
    rng = np.random.default_rng(3)
    n, T, K = 64, 4096, 6
    counts = rng.multinomial(T * K, np.ones(n) / n)
    b = rng.uniform(-0.05, 0.05, n).astype(np.float32)
    gamma = 0.001
    out = om.bias_update(counts, b, T, K, gamma)
    mean = T * K / n
    for i in range(n):
        if counts[i] > mean:
            assert out[i] < b[i]
        elif counts[i] < mean:
            assert out[i] > b[i]
        else:
            assert out[i] == b[i]
        # equals the correctly rounded fp32 sum of b and -+gamma (fp32 state)
        step = np.float32(gamma) * np.float32(np.sign(mean - counts[i]))
        assert out[i] == np.float32(b[i] + step)


def test_bias_update_mean_exact_in_integers():
    # T*K/N_r = 24576/64 = 384 exactly: an expert with 384 is unchanged
    counts = np.full(64, 384)
    counts[0], counts[1] = 385, 383
    out = om.bias_update(counts, np.zeros(64, np.float32), 4096, 6, 0.001)
    assert out[0] < 0 and out[1] > 0 and np.all(out[2:] == 0)
