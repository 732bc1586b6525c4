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
