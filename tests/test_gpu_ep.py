"""Expert-parallel layer on one B200.

- moe_gather_rows bit-exact against indexing (out-of-range rows -> zeros).
- W ranks emulated in one process: one ExpertParallelMoELayer per rank (its
  slice of the experts), the all-to-all exchanges done by the test as plain
  copies between the stage methods (no kernel waits on another). Each rank's
  output must match the oracle on that rank's tokens and the single-GPU layer
  on the ranks' batches laid end to end.
- The forward with its NCCL collectives in a one-rank process group.
"""
import os
import socket
from datetime import timedelta

import numpy as np
import pytest
import torch
import torch.distributed as dist

from mixture_experts_layer_58_b200 import _lib as L
from mixture_experts_layer_58_b200 import synth
from mixture_experts_layer_58_b200.ep import ExpertParallelMoELayer
from mixture_experts_layer_58_b200.layer import MoELayer
from oracle import moe_oracle as om

from gpu_support import check_close, check_route, f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built(cuda_ok):
    from mixture_experts_layer_58_b200 import build
    build.build()
    L.load()


@pytest.mark.parametrize("n_src,n,d", [(1000, 1500, 7168), (37, 300, 256), (5, 9, 8)])
def test_gather_rows_bit_exact(n_src, n, d):
    g = torch.Generator().manual_seed(n + d)
    src = torch.randn(n_src, d, generator=g).bfloat16()
    idx = torch.randint(0, n_src, (n,), generator=g, dtype=torch.int32)
    idx[::7] = -1
    idx[3::11] = n_src                      # out of range: zero rows
    want = torch.zeros(n, d, dtype=torch.bfloat16)
    ok = (idx >= 0) & (idx < n_src)
    want[ok] = src[idx[ok].long()]
    dst = torch.full((n, d), 7.0, dtype=torch.bfloat16, device="cuda")
    L.moe_gather_rows(src.cuda(), n_src, idx.cuda(), n, d, dst)
    torch.cuda.synchronize()
    assert torch.equal(dst.cpu(), want)


def _weights(cfg):
    W1, W3, W2 = synth.all_expert_weights(cfg, "cpu")
    return W1, W3, W2, synth.shared_weights(cfg, "cpu")


def _emulated_forward(cfg, Ts, world):
    """One layer per rank in this process; the exchanges are copies."""
    e, b = synth.centroids(cfg), synth.bias(cfg)
    W1, W3, W2, shared = _weights(cfg)
    lays = [ExpertParallelMoELayer(e, b, W1, W3, W2, shared, top_k=cfg.top_k,
                                   routed_scale=cfg.routed_scale, gate_kind=cfg.gate_kind,
                                   gamma=cfg.gamma, world=world, rank=r) for r in range(world)]
    us = [synth.tokens(cfg.replace(seed=r), T) for r, T in enumerate(Ts)]
    ud = [u.cuda() for u in us]
    for lay, u in zip(lays, ud):
        lay.begin(u)
    counts = [lay.counts.cpu() for lay in lays]
    # expert-contiguous row offsets from the loads (an empty batch runs no
    # permute, so its offsets buffer is not written)
    offs = [torch.cat([torch.zeros(1, dtype=torch.int64), c.long().cumsum(0)]) for c in counts]
    nl = lays[0].n_local
    plans = []
    for p, lay in enumerate(lays):
        recv = torch.stack([counts[q][p * nl:(p + 1) * nl] for q in range(world)])
        plans.append(lay.plan(counts[p], recv))
    for p, lay in enumerate(lays):              # dispatch exchange
        parts = [lays[q].x_perm[int(offs[q][p * nl]):int(offs[q][(p + 1) * nl])]
                 for q in range(world)]
        if plans[p].n_recv:
            lay.x_recv[:plans[p].n_recv].copy_(torch.cat(parts))
    ys = [lay.experts(plans[p]) for p, lay in enumerate(lays)]
    for q, lay in enumerate(lays):              # return exchange
        parts = []
        for p in range(world):
            s = sum(plans[p].recv_splits[:q])
            parts.append(ys[p][s:s + plans[p].recv_splits[q]])
        if Ts[q]:
            lay.y_perm[:Ts[q] * cfg.top_k].copy_(torch.cat(parts))
    outs = [lay.finish(u).clone() for lay, u in zip(lays, ud)]
    torch.cuda.synchronize()
    assert L.moe_get_device_status() == 0
    return lays, us, outs, (e, b, W1, W3, W2, shared)


@pytest.mark.parametrize("name,Ts,world", [("tiny", [64, 40], 2), ("tiny", [64, 0, 17, 64], 4),
                                           ("mid", [4096, 1000], 2)])
def test_emulated_ranks_match_oracle_and_single_gpu(name, Ts, world):
    cfg = synth.CONFIGS[name]
    lays, us, outs, (e, b, W1, W3, W2, shared) = _emulated_forward(cfg, Ts, world)
    expert = lambda i: (W1[i].float().numpy(), W3[i].float().numpy(), W2[i].float().numpy())
    sh = [tuple(w.float().numpy() for w in shared)]
    for lay, u, out in zip(lays, us, outs):
        if u.shape[0] == 0:
            continue
        r = om.route(u, e, b, cfg.top_k, cfg.routed_scale, cfg.gate_kind)
        gidx = lay.topk_idx.cpu().numpy()
        check_route(gidx, lay.topk_gate.cpu().numpy(), lay.counts.cpu().numpy(), r,
                    cfg.routed_scale, u, e, cfg.gate_kind)
        g = om.gates_for_indices(u, e, gidx, cfg.routed_scale, cfg.gate_kind)
        check_close(f64(out), om.layer_output(u, gidx, g, expert, sh))
    # the single-GPU layer on the ranks' batches end to end
    single = MoELayer(e, b, W1, W3, W2, shared, top_k=cfg.top_k, routed_scale=cfg.routed_scale,
                      gate_kind=cfg.gate_kind, gamma=cfg.gamma)
    ref = single.forward(torch.cat(us).cuda()).float().cpu()
    got = torch.cat(outs).float().cpu()
    check_close(got.numpy(), ref.numpy(), max_tol=4e-3, mean_tol=1e-3, what="vs single GPU")


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def test_forward_through_nccl_one_rank():
    """forward() with its NCCL all-to-alls in a one-rank group equals the
    single-GPU layer, and step()'s bias update matches the oracle's."""
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(_free_port())
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=timedelta(seconds=120))
    try:
        cfg = synth.CONFIGS["tiny"]
        e, b = synth.centroids(cfg), synth.bias(cfg)
        W1, W3, W2, shared = _weights(cfg)
        lay = ExpertParallelMoELayer(e, b, W1, W3, W2, shared, top_k=cfg.top_k,
                                     routed_scale=cfg.routed_scale, gamma=cfg.gamma)
        assert lay.world == 1 and lay.n_local == cfg.n_routed
        u = synth.tokens(cfg)
        out = lay.step(u.cuda()).float().cpu()
        torch.cuda.synchronize()
        single = MoELayer(e, b, W1, W3, W2, shared, top_k=cfg.top_k,
                          routed_scale=cfg.routed_scale, gamma=cfg.gamma)
        ref = single.forward(u.cuda()).float().cpu()
        check_close(out.numpy(), ref.numpy(), max_tol=4e-3, mean_tol=1e-3, what="vs single GPU")
        want_b = om.bias_update(lay.counts.cpu().numpy(), b.numpy(), cfg.T, cfg.top_k, cfg.gamma)
        assert np.array_equal(lay.bias.cpu().numpy(), want_b)
        assert lay.last_plan.n_recv == cfg.T * cfg.top_k
        assert L.moe_get_device_status() == 0
    finally:
        dist.destroy_process_group()
