"""Expert-parallel host logic, no GPU: the exchange plan (moe_ep_plan in the
C library) against a brute-force construction, and W ranks emulated in one
process -- the product's plan moving the rows, the oracle computing each
rank's experts -- against the single-process oracle layer."""
import numpy as np
import pytest
import torch

from mixture_experts_layer_58_b200 import _lib as L
from mixture_experts_layer_58_b200 import ep, synth
from oracle import moe_oracle as om


@pytest.fixture(scope="module", autouse=True)
def _built():
    from mixture_experts_layer_58_b200 import build
    build.build()
    L.load()


def brute_force_plan(local_counts, recv_counts):
    """Label every received row (source q, expert e, r-th of them) in the
    order it arrives (source-major), then sort the labels expert-major."""
    world, n_local = recv_counts.shape
    arrived = [(q, e, r) for q in range(world) for e in range(n_local)
               for r in range(recv_counts[q, e])]
    expert_major = sorted(arrived, key=lambda x: (x[1], x[0], x[2]))
    where = {lab: i for i, lab in enumerate(arrived)}
    regroup = np.array([where[lab] for lab in expert_major], dtype=np.int64)
    offs = np.zeros(n_local + 1, dtype=np.int64)
    for e in range(n_local):
        offs[e + 1] = offs[e] + recv_counts[:, e].sum()
    send = local_counts.reshape(world, n_local).sum(1)
    return send, recv_counts.sum(1), offs, regroup


@pytest.mark.parametrize("world,n_local", [(1, 1), (1, 16), (2, 8), (3, 5), (4, 4), (8, 32)])
def test_plan_matches_brute_force(world, n_local):
    rng = np.random.default_rng(world * 100 + n_local)
    for trial in range(4):
        hi = [0, 1, 5, 40][trial]
        local = rng.integers(0, hi + 1, size=world * n_local).astype(np.int32)
        recv = rng.integers(0, hi + 1, size=(world, n_local)).astype(np.int32)
        if trial == 3:
            recv[:, 1 % n_local] = 0          # an expert nobody routes to
            recv[world - 1, :] = 0            # a rank that sends nothing here
        p = ep.plan_exchange(torch.from_numpy(local), torch.from_numpy(recv), world, n_local)
        send, rsplit, offs, regroup = brute_force_plan(local, recv)
        assert p.send_splits == send.tolist()
        assert p.recv_splits == rsplit.tolist()
        assert p.n_recv == int(recv.sum())
        assert p.group_offsets.tolist() == offs.tolist()
        assert p.regroup.tolist() == regroup.tolist()
        # ungroup is the inverse permutation
        ug = p.ungroup.numpy()
        assert np.array_equal(np.sort(ug), np.arange(p.n_recv))
        assert np.array_equal(ug[p.regroup.numpy()], np.arange(p.n_recv))


def test_plan_rejects_bad_counts():
    ss = torch.empty(2, dtype=torch.int64)
    rs = torch.empty(2, dtype=torch.int64)
    go = torch.empty(3, dtype=torch.int32)
    rg = torch.empty(8, dtype=torch.int32)
    ug = torch.empty(8, dtype=torch.int32)
    good = torch.tensor([1, 2, 3, 0], dtype=torch.int32)
    neg = torch.tensor([1, -2, 3, 0], dtype=torch.int32)
    recv = torch.tensor([[1, 2], [3, 0]], dtype=torch.int32)
    with pytest.raises(L.MoEError) as ex:
        L.moe_ep_plan(neg, recv, 2, 2, 8, ss, rs, go, rg, ug)
    assert ex.value.status == L.MOE_ERR_INVALID_ARG
    with pytest.raises(L.MoEError) as ex:                # capacity 5 < 6 rows
        L.moe_ep_plan(good, recv, 2, 2, 5, ss, rs, go, rg, ug)
    assert ex.value.status == L.MOE_ERR_INVALID_ARG
    with pytest.raises(L.MoEError):
        L.moe_ep_plan(good, recv, 0, 2, 8, ss, rs, go, rg, ug)
    with pytest.raises(ValueError):                      # wrong dtype for the splits
        L.moe_ep_plan(good, recv, 2, 2, 8, go, rs, go, rg, ug)
    # sizes only (no regroup/ungroup): capacity is not needed
    assert L.moe_ep_plan(good, recv, 2, 2, 0, ss, rs, go) == 6
    assert ss.tolist() == [3, 3] and rs.tolist() == [3, 3] and go.tolist() == [0, 4, 6]


def emulate_ranks(cfg, Ts, world):
    """Each rank routes its own tokens with the oracle and lays its rows out
    expert-contiguously (the oracle's dispatch order); the product's plans
    move the rows between ranks (by slicing, as the all-to-all would); each
    rank runs only its own experts (oracle FFN on the regrouped rows); the
    results come back and each rank combines its tokens."""
    e, b = synth.centroids(cfg), synth.bias(cfg)
    W1, W3, W2 = synth.all_expert_weights(cfg, "cpu")
    shared = [tuple(w.float().numpy() for w in synth.shared_weights(cfg, "cpu"))]
    n_routed, K = cfg.n_routed, cfg.top_k
    nl = n_routed // world
    us = [synth.tokens(cfg.replace(seed=r), T) for r, T in enumerate(Ts)]
    routes = [om.route(u, e, b, K, cfg.routed_scale) for u in us]
    disp = [om.dispatch(r.idx, n_routed) for r in routes]
    x_perm = [u.double().numpy()[d.src] for u, d in zip(us, disp)]
    counts = [r.counts.astype(np.int32) for r in routes]
    plans = []
    for p in range(world):
        recv = np.stack([counts[q][p * nl:(p + 1) * nl] for q in range(world)])
        plans.append(ep.plan_exchange(torch.from_numpy(counts[p]), torch.from_numpy(recv),
                                      world, nl))
    # dispatch: rank q's x_perm rows of rank p's experts, sources in rank order
    x_recv = []
    for p in range(world):
        parts = [x_perm[q][disp[q].offsets[p * nl]:disp[q].offsets[(p + 1) * nl]]
                 for q in range(world)]
        assert [len(x) for x in parts] == plans[p].recv_splits
        x_recv.append(np.concatenate(parts))
    y_src = []
    for p in range(world):
        pl = plans[p]
        x_exp = x_recv[p][pl.regroup.numpy()]
        y_exp = np.zeros_like(x_exp)
        go = pl.group_offsets.numpy()
        for el in range(nl):
            g = p * nl + el
            rows = slice(go[el], go[el + 1])
            if go[el + 1] > go[el]:
                y_exp[rows] = om.ffn(x_exp[rows], W1[g].float().numpy(), W3[g].float().numpy(),
                                     W2[g].float().numpy())
        y_src.append(y_exp[pl.ungroup.numpy()])
    outs = []
    for q in range(world):
        parts = []
        for p in range(world):
            start = sum(plans[p].recv_splits[:q])
            parts.append(y_src[p][start:start + plans[p].recv_splits[q]])
        y_perm = np.concatenate(parts)
        assert len(y_perm) == Ts[q] * K == sum(plans[q].send_splits)
        out = us[q].double().numpy() + om.shared_output(us[q], shared)
        pos = disp[q].pos
        for k in range(K):
            out += routes[q].gate[:, k:k + 1] * y_perm[pos[:, k]]
        outs.append(out)
    return us, routes, outs, (W1, W3, W2), shared


@pytest.mark.parametrize("world,Ts", [(1, [64]), (2, [64, 40]), (4, [64, 1, 0, 33]),
                                      (16, [8] * 16)])
def test_emulated_ranks_reproduce_the_single_process_layer(world, Ts):
    cfg = synth.CONFIGS["tiny"]
    us, routes, outs, (W1, W3, W2), shared = emulate_ranks(cfg, Ts, world)
    expert = lambda i: (W1[i].float().numpy(), W3[i].float().numpy(), W2[i].float().numpy())
    for u, r, out in zip(us, routes, outs):
        ref = om.layer_output(u, r.idx, r.gate, expert, shared)
        np.testing.assert_allclose(out, ref, rtol=1e-9, atol=1e-9)


def test_layer_rejects_an_uneven_split_and_a_wrong_expert_count():
    """Raised on the host before any device memory is touched."""
    from mixture_experts_layer_58_b200.ep import ExpertParallelMoELayer
    cfg = synth.CONFIGS["tiny"]                 # 16 routed experts
    e, b = synth.centroids(cfg), synth.bias(cfg)
    W1, W3, W2 = synth.all_expert_weights(cfg, "cpu")
    with pytest.raises(ValueError, match="do not split"):
        ExpertParallelMoELayer(e, b, W1, W3, W2, top_k=4, routed_scale=1.0, world=3, rank=0)
    with pytest.raises(ValueError, match="expected 8 or 16 experts"):
        ExpertParallelMoELayer(e, b, W1[:5], W3[:5], W2[:5], top_k=4, routed_scale=1.0,
                               world=2, rank=1)

