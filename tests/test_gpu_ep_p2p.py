"""Expert parallelism over peer memory on one B200.

- moe_ep_plan_device against the host plan (moe_ep_plan) and a brute-force
  construction of every row's destination.
- W ranks emulated in one process: one PeerExpertParallelMoELayer per rank,
  linked so that each one's peer tables point at the others' buffers on this
  GPU; the stages run rank by rank (each kernel only stores or loads, none
  waits on another). Each rank's output must match the oracle and the
  single-GPU layer on the ranks' batches laid end to end.
- forward() with its NCCL all-gather and barriers in a one-rank group, and the
  bias update from the device plan's summed loads.
- A receive capacity too small for a step: the status word reports it and no
  row is stored past the buffer.
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
from mixture_experts_layer_58_b200.ep import PeerExpertParallelMoELayer, link_emulated_ranks
from mixture_experts_layer_58_b200.layer import MoELayer
from oracle import moe_oracle as om

from gpu_support import check_close, check_route, f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built(cuda_ok):
    from mixture_experts_layer_58_b200 import build
    build.build()
    L.load()


@pytest.mark.parametrize("world,n_local", [(1, 16), (2, 8), (4, 64), (8, 32)])
def test_device_plan_matches_host_plan(world, n_local):
    n = world * n_local
    g = torch.Generator().manual_seed(world * 100 + n_local)
    allc = torch.randint(0, 50, (world, n), generator=g, dtype=torch.int32)
    allc[:, ::5] = 0                                   # empty experts
    dev = allc.cuda()
    for rank in range(world):
        dest = torch.empty(n, dtype=torch.int32, device="cuda")
        goff = torch.empty(n_local + 1, dtype=torch.int32, device="cuda")
        gc = torch.empty(n, dtype=torch.int32, device="cuda")
        L.moe_ep_plan_device(dev, world, n_local, rank, 1 << 30, dest, goff, gc)
        torch.cuda.synchronize()
        assert torch.equal(gc.cpu(), allc.sum(0).to(torch.int32))
        # the host plan of the same exchange gives the same group offsets
        recv = allc[:, rank * n_local:(rank + 1) * n_local].contiguous()
        ss = torch.empty(world, dtype=torch.int64)
        rs = torch.empty(world, dtype=torch.int64)
        go = torch.empty(n_local + 1, dtype=torch.int32)
        L.moe_ep_plan(allc[rank].contiguous(), recv, world, n_local, 0, ss, rs, go)
        assert torch.equal(goff.cpu(), go)
        # brute force: the owner's buffer is expert-major, sources in rank order
        want = []
        for E in range(n):
            q, e = divmod(E, n_local)
            base = int(allc[:, q * n_local:q * n_local + e].sum())
            want.append(base + int(allc[:rank, E].sum()))
        assert dest.cpu().tolist() == want
    assert L.moe_get_device_status() == 0


def _weights(cfg):
    W1, W3, W2 = synth.all_expert_weights(cfg, "cpu")
    return W1, W3, W2, synth.shared_weights(cfg, "cpu")


def _emulated_forward(cfg, Ts, world, capacity=None):
    e, b = synth.centroids(cfg), synth.bias(cfg)
    W1, W3, W2, shared = _weights(cfg)
    cap = sum(Ts) * cfg.top_k if capacity is None else capacity
    lays = [PeerExpertParallelMoELayer(e, b, W1, W3, W2, shared, top_k=cfg.top_k,
                                       routed_scale=cfg.routed_scale, gate_kind=cfg.gate_kind,
                                       gamma=cfg.gamma, world=world, rank=r,
                                       recv_capacity=max(cap, 1)) for r in range(world)]
    us = [synth.tokens(cfg.replace(seed=r), T) for r, T in enumerate(Ts)]
    ud = [u.cuda() for u in us]
    for lay, u in zip(lays, ud):
        lay.begin(u)
    link_emulated_ranks(lays)
    allc = torch.stack([lay.counts for lay in lays])         # the all-gather
    for lay in lays:
        lay.all_counts.copy_(allc)
        lay.plan()
    for lay, u in zip(lays, ud):
        lay.dispatch(u)
    for lay in lays:
        lay.experts()
    outs = [lay.finish(u).clone() for lay, u in zip(lays, ud)]
    torch.cuda.synchronize()
    return lays, us, outs, (e, b, W1, W3, W2, shared)


@pytest.mark.parametrize("name,Ts,world", [("tiny", [64, 40], 2), ("tiny", [64, 0, 17, 64], 4),
                                           ("mid", [4096, 1000], 2)])
def test_emulated_p2p_ranks_match_oracle_and_single_gpu(name, Ts, world):
    cfg = synth.CONFIGS[name]
    lays, us, outs, (e, b, W1, W3, W2, shared) = _emulated_forward(cfg, Ts, world)
    assert L.moe_get_device_status() == 0
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
    single = MoELayer(e, b, W1, W3, W2, shared, top_k=cfg.top_k, routed_scale=cfg.routed_scale,
                      gate_kind=cfg.gate_kind, gamma=cfg.gamma)
    ref = single.forward(torch.cat(us).cuda()).float().cpu()
    got = torch.cat(outs).float().cpu()
    check_close(got.numpy(), ref.numpy(), max_tol=4e-3, mean_tol=1e-3, what="vs single GPU")
    # every rank's receive buffer holds its experts' rows of all ranks
    single_counts = single.counts.cpu()
    for lay in lays:
        lo = lay.expert_lo
        assert int(lay.goff[-1]) == int(single_counts[lo:lo + lay.n_local].sum())
        assert torch.equal(lay.global_counts.cpu(), single_counts)


def test_receive_capacity_overflow_is_reported_not_written():
    cfg = synth.CONFIGS["tiny"]
    Ts = [64, 64]
    cap = 100                                   # < the 256 rows each rank receives on average
    lays, us, outs, _ = _emulated_forward(cfg, Ts, 2, capacity=cap)
    st = L.moe_get_device_status()             # reads and clears the status word
    assert st == 16, st
    for lay, out in zip(lays, outs):
        assert int(lay.goff[-1]) > cap
        assert bool(torch.isfinite(out.float()).all())
    assert L.moe_get_device_status() == 0


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


@pytest.mark.parametrize("name,mb", [("tiny", 1), ("mid", 1), ("tiny", 2), ("mid", 2)])
def test_p2p_forward_through_nccl_one_rank(name, mb):
    """forward() with its NCCL all-gather and barriers in a one-rank group
    (mb = 2: two micro-batches, the second's exchange on its own stream beside
    the first's GEMMs) equals the single-GPU layer; step()'s bias update
    matches the oracle's on the loads of the whole step."""
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(_free_port())
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=timedelta(seconds=120))
    try:
        cfg = synth.CONFIGS[name]
        e, b = synth.centroids(cfg), synth.bias(cfg)
        W1, W3, W2, shared = _weights(cfg)
        lay = PeerExpertParallelMoELayer(e, b, W1, W3, W2, shared, top_k=cfg.top_k,
                                         routed_scale=cfg.routed_scale, gamma=cfg.gamma,
                                         micro_batches=mb)
        assert lay.world == 1 and lay.n_local == cfg.n_routed
        u = synth.tokens(cfg)
        out = lay.step(u.cuda()).float().cpu()
        torch.cuda.synchronize()
        single = MoELayer(e, b, W1, W3, W2, shared, top_k=cfg.top_k,
                          routed_scale=cfg.routed_scale, gamma=cfg.gamma)
        ref = single.forward(u.cuda()).float().cpu()
        check_close(out.numpy(), ref.numpy(), max_tol=4e-3, mean_tol=1e-3, what="vs single GPU")
        counts = single.counts.cpu().numpy()
        want_b = om.bias_update(counts, b.numpy(), cfg.T, cfg.top_k, cfg.gamma)
        assert np.array_equal(lay.bias.cpu().numpy(), want_b)
        assert L.moe_get_device_status() == 0
        lay.close()
    finally:
        dist.destroy_process_group()
