"""Parity at the full V3 layer shape (d=7168, 256 routed experts top-8, 1 shared,
I=2048) in the launch configuration the benchmark times: routing and dispatch
are checked over every token, the expert FFN and the layer output on sampled
tokens / rows the fp64 oracle computes one by one. Needs a B200."""
import numpy as np
import pytest
import torch

from mixture_experts_layer_58_b200 import _lib as L
from mixture_experts_layer_58_b200 import synth
from oracle import moe_oracle as om

from gpu_support import Inputs, check_close, check_route, f64

pytestmark = pytest.mark.gpu


def _dispatch_invariants(lay, T, K, n_routed):
    idx = lay.topk_idx.cpu().numpy().astype(np.int64)
    counts = lay.counts.cpu().numpy().astype(np.int64)
    off = lay.offsets.cpu().numpy().astype(np.int64)
    pos = lay.pos.cpu().numpy().astype(np.int64)
    src = lay.src.cpu().numpy().astype(np.int64)
    if off.size == n_routed + 2:
        # the shared expert as group n_routed: its rows follow the routed ones
        assert off[-1] == T * K + T
        off = off[:-1]
    assert np.array_equal(off, np.concatenate([[0], np.cumsum(counts)]))
    assert np.array_equal(np.sort(pos.ravel()), np.arange(T * K))
    t_of = np.repeat(np.arange(T), K)
    assert np.array_equal(src[pos.ravel()], t_of)
    # each row lies in its expert's range, rows of an expert in ascending token order
    e_of = idx.ravel()
    assert np.all((off[e_of] <= pos.ravel()) & (pos.ravel() < off[e_of + 1]))
    order = np.lexsort((t_of, e_of))
    assert np.array_equal(pos.ravel()[order], np.arange(T * K))
    return idx, off, pos, src


def _sample_tokens(idx, counts, rng, n_random=8):
    hot = int(np.argmax(counts))
    nz = np.nonzero(counts)[0]
    cold = int(nz[np.argmin(counts[nz])])
    t_hot = np.nonzero((idx == hot).any(1))[0][:4]
    t_cold = np.nonzero((idx == cold).any(1))[0][:4]
    t_rand = rng.choice(idx.shape[0], size=min(n_random, idx.shape[0]), replace=False)
    return np.unique(np.concatenate([t_hot, t_cold, t_rand])), hot


def _check_sampled_output(inp, lay, tokens):
    cfg = inp.cfg
    idx = lay.topk_idx.cpu().numpy()[tokens]
    u_s = inp.u[torch.from_numpy(tokens)]
    g = om.gates_for_indices(u_s, inp.e, idx, cfg.routed_scale, cfg.gate_kind)
    ref = om.layer_output(u_s, idx, g, inp.expert, inp.shared_list())
    got = f64(lay.out)[tokens]
    return check_close(got, ref, what=f"{cfg.name} sampled output")


@pytest.fixture(scope="module")
def v3p(cuda_ok):
    from mixture_experts_layer_58_b200 import build
    build.build()
    inp = Inputs(synth.CONFIGS["v3p"])
    inp.layer.forward(inp.u_dev)
    torch.cuda.synchronize()
    assert L.moe_get_device_status() == 0
    yield inp
    del inp
    torch.cuda.empty_cache()


def test_v3p_routing_all_tokens(v3p):
    cfg, lay = v3p.cfg, v3p.layer
    r = v3p.oracle_route()
    near = check_route(lay.topk_idx.cpu().numpy(), lay.topk_gate.cpu().numpy(),
                       lay.counts.cpu().numpy(), r, cfg.routed_scale, v3p.u, v3p.e, cfg.gate_kind)
    assert near < 0.02 * cfg.T
    # the workload is skewed as specified: hottest expert ~10x the mean load
    assert lay.counts.max().item() > 8 * cfg.T * cfg.top_k / cfg.n_routed


def test_v3p_dispatch_all_rows(v3p):
    cfg, lay = v3p.cfg, v3p.layer
    idx, off, pos, src = _dispatch_invariants(lay, cfg.T, cfg.top_k, cfg.n_routed)
    rng = np.random.default_rng(0)
    rows = rng.choice(cfg.T * cfg.top_k, size=2048, replace=False)
    xp = lay.x_perm[torch.from_numpy(rows).cuda()].cpu()
    assert torch.equal(xp, v3p.u[torch.from_numpy(src[rows])])


def test_v3p_hottest_expert_rows_incl_ragged_tail(v3p):
    """Rows of the most loaded expert (40 M-tiles, ragged last tile) through the
    expert FFN against the fp64 FFN of the same rows."""
    cfg, lay = v3p.cfg, v3p.layer
    counts = lay.counts.cpu().numpy()
    off = lay.offsets.cpu().numpy()
    hot = int(np.argmax(counts))
    a, b = int(off[hot]), int(off[hot + 1])
    rows = np.unique(np.concatenate([np.arange(a, a + 64), np.arange(max(a, b - 96), b),
                                     np.random.default_rng(1).integers(a, b, 128)]))
    x = lay.x_perm[torch.from_numpy(rows).cuda()].float().cpu().numpy()
    ref = om.ffn(x, *v3p.expert(hot))
    got = f64(lay.y_perm[torch.from_numpy(rows).cuda()])
    check_close(got, ref, what="hottest expert FFN")


def test_v3p_sampled_layer_output(v3p):
    lay = v3p.layer
    idx = lay.topk_idx.cpu().numpy()
    tokens, _ = _sample_tokens(idx, lay.counts.cpu().numpy(), np.random.default_rng(2))
    _check_sampled_output(v3p, lay, tokens)


@pytest.mark.parametrize("name", ["v3d", "v3d_softmax"])
def test_v3_decode_layer(name, cuda_ok):
    from mixture_experts_layer_58_b200 import build
    build.build()
    inp = Inputs(synth.CONFIGS[name])
    cfg, lay = inp.cfg, inp.layer
    lay.forward(inp.u_dev)
    torch.cuda.synchronize()
    assert L.moe_get_device_status() == 0
    r = inp.oracle_route()
    check_route(lay.topk_idx.cpu().numpy(), lay.topk_gate.cpu().numpy(),
                lay.counts.cpu().numpy(), r, cfg.routed_scale, inp.u, inp.e, cfg.gate_kind)
    _dispatch_invariants(lay, cfg.T, cfg.top_k, cfg.n_routed)
    tokens, _ = _sample_tokens(lay.topk_idx.cpu().numpy(), lay.counts.cpu().numpy(),
                               np.random.default_rng(3), n_random=4)
    _check_sampled_output(inp, lay, tokens)
    del inp
    torch.cuda.empty_cache()


def test_v3p_fused_gather_sampled(cuda_ok):
    """V3 prefill in the fused mode (no x_perm copy): routing of every token and
    sampled outputs against the oracle."""
    from mixture_experts_layer_58_b200 import build
    build.build()
    inp = Inputs(synth.CONFIGS["v3p"], fused_gather=True)
    cfg, lay = inp.cfg, inp.layer
    lay.forward(inp.u_dev)
    torch.cuda.synchronize()
    assert L.moe_get_device_status() == 0
    r = inp.oracle_route()
    check_route(lay.topk_idx.cpu().numpy(), lay.topk_gate.cpu().numpy(),
                lay.counts.cpu().numpy(), r, cfg.routed_scale, inp.u, inp.e, cfg.gate_kind)
    tokens, _ = _sample_tokens(lay.topk_idx.cpu().numpy(), lay.counts.cpu().numpy(),
                               np.random.default_rng(5), n_random=4)
    _check_sampled_output(inp, lay, tokens)
    del inp
    torch.cuda.empty_cache()


def test_v3p_shared_expert_grouped_bit_identical(v3p):
    """CTA-pair tiles: the shared expert as group N_r of the routed GEMMs (its
    rows appended by moe_permute_shared) against the benchmark's layer, where
    it runs in its own launches: the same bits."""
    cfg, lay = v3p.cfg, v3p.layer
    assert not lay.shared_in_grouped
    want = lay.out.clone()
    lay.shared_grouped = True
    lay._T = -1                                   # re-allocate with the extra group
    got = lay.forward(v3p.u_dev)
    torch.cuda.synchronize()
    assert L.moe_get_device_status() == 0
    assert lay.shared_in_grouped
    assert torch.equal(got, want)
    rk = cfg.T * cfg.top_k
    assert torch.equal(lay.x_perm[rk:].cpu(), v3p.u)
    _dispatch_invariants(lay, cfg.T, cfg.top_k, cfg.n_routed)
    lay.shared_grouped = False
    lay._T = -1
