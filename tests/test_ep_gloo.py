"""Expert-parallel exchanges on CPU: W gloo ranks, each holding N_r/W routed
experts, route their own (ragged, possibly empty) batches with the oracle and
move the rows with the product's exchange functions (ep.exchange_counts,
ep.plan_exchange, ep.dispatch_rows, ep.return_rows). Each rank evaluates only
its own experts (oracle FFN, fp64 rows) and combines its own tokens; the
result must equal the single-process oracle layer on that rank's tokens."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from mixture_experts_layer_58_b200 import ep, synth
from oracle import moe_oracle as om

BATCHES = {2: [64, 40], 4: [64, 40, 1, 0]}


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cfg = synth.CONFIGS["tiny"]
        T, K, n_routed = BATCHES[world][rank], cfg.top_k, cfg.n_routed
        nl = n_routed // world
        u = synth.tokens(cfg.replace(seed=rank), T)
        e, b = synth.centroids(cfg), synth.bias(cfg)
        W1, W3, W2 = synth.all_expert_weights(cfg, "cpu")
        shared = [tuple(w.float().numpy() for w in synth.shared_weights(cfg, "cpu"))]
        r = om.route(u, e, b, K, cfg.routed_scale)
        disp = om.dispatch(r.idx, n_routed)
        x_perm = torch.from_numpy(u.double().numpy()[disp.src].copy())
        counts = torch.from_numpy(r.counts.astype(np.int32))
        recv = ep.exchange_counts(counts)
        plan = ep.plan_exchange(counts, recv.view(world, nl), world, nl)
        x_recv = torch.full((max(plan.n_recv, 1), cfg.d), float("nan"), dtype=torch.float64)
        xr = ep.dispatch_rows(x_perm, plan, x_recv).numpy()
        x_exp = xr[plan.regroup.numpy()]
        y_exp = np.zeros_like(x_exp)
        go = plan.group_offsets.numpy()
        for el in range(nl):
            g = rank * nl + el
            if go[el + 1] > go[el]:
                y_exp[go[el]:go[el + 1]] = om.ffn(x_exp[go[el]:go[el + 1]], W1[g].float().numpy(),
                                                  W3[g].float().numpy(), W2[g].float().numpy())
        y_src = torch.from_numpy(y_exp[plan.ungroup.numpy()].copy())
        y_perm = torch.full((T * K, cfg.d), float("nan"), dtype=torch.float64)
        yp = ep.return_rows(y_src, plan, y_perm).numpy()
        out = u.double().numpy() + om.shared_output(u, shared)
        for k in range(K):
            out += r.gate[:, k:k + 1] * yp[disp.pos[:, k]]
        q.put((rank, plan.send_splits, plan.recv_splits, out))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_expert_parallel_exchange_reproduces_the_layer(world):
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=180) for _ in range(world)), key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    cfg = synth.CONFIGS["tiny"]
    e, b = synth.centroids(cfg), synth.bias(cfg)
    W1, W3, W2 = synth.all_expert_weights(cfg, "cpu")
    shared = [tuple(w.float().numpy() for w in synth.shared_weights(cfg, "cpu"))]
    expert = lambda i: (W1[i].float().numpy(), W3[i].float().numpy(), W2[i].float().numpy())
    sent = np.array([s for _, s, _, _ in res])          # sent[q, p]: rows q -> p
    received = np.array([rs for _, _, rs, _ in res])    # received[p, q]: rows p <- q
    assert np.array_equal(sent, received.T)
    for rank, _, _, out in res:
        u = synth.tokens(cfg.replace(seed=rank), BATCHES[world][rank])
        ref, _ = om.layer(u, e, b, expert, shared, cfg.top_k, cfg.routed_scale)
        assert np.all(np.isfinite(out))
        np.testing.assert_allclose(out, ref, rtol=1e-9, atol=1e-9)
