"""Data-parallel path on CPU: two gloo ranks each route their own batch with the
oracle, sum their loads through dp.sync_load, and must end with the same bias
as one process updating from the concatenated batch."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from mixture_experts_layer_58_b200 import dp, synth
from oracle import moe_oracle as om


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
        u = synth.tokens(cfg.replace(seed=rank))
        e, b = synth.centroids(cfg), synth.bias(cfg)
        r = om.route(u, e, b, cfg.top_k, cfg.routed_scale)
        counts = torch.from_numpy(r.counts.astype(np.int32))
        T_global = dp.sync_load(counts, cfg.T)
        new_b = om.bias_update(counts.numpy(), b.numpy(), T_global, cfg.top_k, cfg.gamma)
        q.put((rank, T_global, counts.numpy().tolist(), new_b.tolist()))
    finally:
        dist.destroy_process_group()


def test_two_ranks_share_the_global_bias_update():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    cfg = synth.CONFIGS["tiny"]
    # single process over the concatenated batch
    u = torch.cat([synth.tokens(cfg.replace(seed=r)) for r in range(world)])
    e, b = synth.centroids(cfg), synth.bias(cfg)
    r_all = om.route(u, e, b, cfg.top_k, cfg.routed_scale)
    want_b = om.bias_update(r_all.counts, b.numpy(), world * cfg.T, cfg.top_k, cfg.gamma)
    for rank, T_global, counts, new_b in res:
        assert T_global == world * cfg.T
        assert counts == r_all.counts.tolist()
        assert np.array_equal(np.array(new_b, dtype=np.float32), want_b)


def _grad_rank(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from oracle import moe_backward as mb
        u, e, W, shared, idx, dout = _grad_case(rank)
        gr = mb.layer_backward(u, e, idx, 1.0, lambda i: W[i], shared, dout)
        grads = [torch.from_numpy(gr.de.copy()), torch.from_numpy(gr.dshared[0][0].copy()),
                 torch.from_numpy(gr.dshared[0][2].copy())]
        dp.allreduce_grads(grads)
        q.put((rank, [g.numpy().tolist() for g in grads]))
    finally:
        dist.destroy_process_group()


def _grad_case(rank):
    """A Tiny-shaped training batch per rank (fp64 host arrays)."""
    rng = np.random.default_rng(100 + rank)
    T, d, n_r, K, I = 12, 16, 6, 2, 8
    wr = np.random.default_rng(7)            # the replicated parameters
    e = wr.standard_normal((n_r, d)) * 0.5
    W = [(wr.standard_normal((I, d)) * 0.5, wr.standard_normal((I, d)) * 0.5,
          wr.standard_normal((d, I)) * 0.5) for _ in range(n_r)]
    shared = [(wr.standard_normal((I, d)) * 0.5, wr.standard_normal((I, d)) * 0.5,
               wr.standard_normal((d, I)) * 0.5)]
    u = rng.standard_normal((T, d))
    idx = om.route(u, e, None, K, 1.0).idx
    dout = rng.standard_normal((T, d))
    return u, e, W, shared, idx, dout


def test_two_ranks_average_their_gradients():
    """dp.allreduce_grads: the averaged gradients of two ranks equal the
    gradient of the mean of their losses, i.e. the oracle backward over the
    concatenated batch with dL/dh' halved."""
    from oracle import moe_backward as mb
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_grad_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    cases = [_grad_case(r) for r in range(world)]
    u = np.concatenate([c[0] for c in cases])
    idx = np.concatenate([c[4] for c in cases])
    dout = np.concatenate([c[5] for c in cases]) / world
    e, W, shared = cases[0][1], cases[0][2], cases[0][3]
    ref = mb.layer_backward(u, e, idx, 1.0, lambda i: W[i], shared, dout)
    want = [ref.de, ref.dshared[0][0], ref.dshared[0][2]]
    for rank, grads in res:
        for got, w in zip(grads, want):
            np.testing.assert_allclose(np.asarray(got), w, rtol=1e-10, atol=1e-12)
