"""Parity of the training path (forward with saved pre-activations, then the
backward calls) on a B200: the expert dgrad / wgrad GEMMs against fp32 torch
products of the same bf16 operands, and the whole layer backward against the
fp64 backward oracle (oracle/moe_backward.py) on the GPU's own routing.

Tolerances: every gradient passes through a few bf16 roundings (y, dy, the
saved pre-activations a and c, da/dc, dx, and the bf16 result itself), each
<= 2^-9 relative; with fp32 accumulation the worst element stays within
3e-2 of max|ref| and the mean error within 1e-2 of mean|ref|. The centroid
gradient sums dz-weighted rows whose dz comes from a difference of gate
terms; it gets 5e-2 / 2e-2."""
import numpy as np
import pytest
import torch

from mixture_experts_layer_58_b200 import _lib as L
from mixture_experts_layer_58_b200 import synth
from oracle import moe_backward as mb

from gpu_support import Inputs, check_close, f64

pytestmark = pytest.mark.gpu

GRAD_MAX, GRAD_MEAN = 3e-2, 1e-2
DE_MAX, DE_MEAN = 5e-2, 2e-2


def _silu_grad(a):
    s = torch.sigmoid(a)
    return s * (1 + a * (1 - s))


def _interleave16(a, c):
    """[n, I] x2 -> [n, 2I] in the packed W13 column order."""
    n, I = a.shape
    return torch.stack([a.view(n, I // 16, 16), c.view(n, I // 16, 16)], dim=2).reshape(n, 2 * I)


def _deinterleave16(x):
    n, I2 = x.shape
    v = x.view(n, I2 // 32, 2, 16)
    return v[:, :, 0].reshape(n, I2 // 2), v[:, :, 1].reshape(n, I2 // 2)


def test_dgrad_kernels_match_torch(cuda_ok):
    """moe_expert_up_swiglu_train (h and the saved ac), moe_expert_down_backward
    (dh = dy W2 and the SwiGLU backward) and moe_expert_up_backward
    (dx = dac W13) over ragged groups; inter = 384 leaves a half 256-column
    block in the down backward."""
    from mixture_experts_layer_58_b200 import build
    build.build()
    sizes = [0, 1, 63, 64, 65, 127, 128, 129, 200, 300]
    G, d, inter = len(sizes), 256, 384
    rows = sum(sizes)
    gen = torch.Generator(device="cuda").manual_seed(21)
    x = torch.randn(rows, d, generator=gen, device="cuda").bfloat16()
    dy = torch.randn(rows, d, generator=gen, device="cuda").bfloat16()
    w1 = (0.05 * torch.randn(G, inter, d, generator=gen, device="cuda")).bfloat16()
    w3 = (0.05 * torch.randn(G, inter, d, generator=gen, device="cuda")).bfloat16()
    w2 = (0.05 * torch.randn(G, d, inter, generator=gen, device="cuda")).bfloat16()
    w13 = torch.empty(G, 2 * inter, d, dtype=torch.bfloat16, device="cuda")
    L.moe_pack_w13(w1, w3, G, inter, d, w13)
    off = torch.tensor(np.concatenate([[0], np.cumsum(sizes)]), dtype=torch.int32, device="cuda")
    h = torch.empty(rows, inter, dtype=torch.bfloat16, device="cuda")
    ac = torch.empty(rows, 2 * inter, dtype=torch.bfloat16, device="cuda")
    dac = torch.empty_like(ac)
    dx = torch.empty(rows, d, dtype=torch.bfloat16, device="cuda")
    L.moe_expert_up_swiglu_train(x, off, G, rows, d, inter, w13, h, ac)
    L.moe_expert_down_backward(dy, ac, off, G, rows, d, inter, w2, dac)
    L.moe_expert_up_backward(dac, off, G, rows, d, inter, w13, dx)
    torch.cuda.synchronize()
    assert L.moe_get_device_status() == 0
    o = off.cpu().tolist()
    for g in range(G):
        a0, b0 = o[g], o[g + 1]
        if a0 == b0:
            continue
        xg = x[a0:b0].float()
        a_ref = xg @ w1[g].float().T
        c_ref = xg @ w3[g].float().T
        ag, cg = _deinterleave16(ac[a0:b0].float())
        check_close(f64(ag), f64(a_ref), max_tol=1e-2, mean_tol=3e-3, what=f"a, group {g}")
        check_close(f64(cg), f64(c_ref), max_tol=1e-2, mean_tol=3e-3, what=f"c, group {g}")
        check_close(f64(h[a0:b0]), f64(torch.nn.functional.silu(a_ref) * c_ref), max_tol=1e-2,
                    mean_tol=3e-3, what=f"h, group {g}")
        # backward from the GPU's own bf16 ac (the values the kernel used)
        a, c = ag, cg
        dh = dy[a0:b0].float() @ w2[g].float()
        da = dh * c * _silu_grad(a)
        dc = dh * torch.nn.functional.silu(a)
        check_close(f64(dac[a0:b0]), f64(_interleave16(da, dc)), max_tol=1e-2, mean_tol=3e-3,
                    what=f"dac, group {g} ({b0 - a0} rows)")
        dx_ref = dac[a0:b0].float() @ w13[g].float()
        check_close(f64(dx[a0:b0]), f64(dx_ref), max_tol=1e-2, mean_tol=3e-3,
                    what=f"dx, group {g} ({b0 - a0} rows)")


@pytest.mark.parametrize("m,n", [(256, 384), (128, 256)])
def test_wgrad_matches_torch(m, n, cuda_ok):
    """dW_g = a_g^T b_g over ragged groups (K blocks of 64 rows that run into
    the next group are masked); an empty group gives zeros; rows past the
    last group are not summed."""
    from mixture_experts_layer_58_b200 import build
    build.build()
    sizes = [65, 0, 1, 63, 64, 130, 7, 256, 0, 100]
    G = len(sizes)
    rows = sum(sizes)
    pad = 40
    gen = torch.Generator(device="cuda").manual_seed(5)
    a = torch.randn(rows + pad, m, generator=gen, device="cuda").bfloat16()
    b = torch.randn(rows + pad, n, generator=gen, device="cuda").bfloat16()
    off = torch.tensor(np.concatenate([[0], np.cumsum(sizes)]), dtype=torch.int32, device="cuda")
    dw = torch.full((G, m, n), 7.0, dtype=torch.bfloat16, device="cuda")
    L.moe_expert_wgrad(a, b, off, G, rows + pad, m, n, dw)
    torch.cuda.synchronize()
    assert L.moe_get_device_status() == 0
    o = off.cpu().tolist()
    for g in range(G):
        a0, b0 = o[g], o[g + 1]
        if a0 == b0:
            assert bool((dw[g] == 0).all()), f"group {g} is empty: expected zeros"
            continue
        ref = a[a0:b0].float().T @ b[a0:b0].float()
        check_close(f64(dw[g]), f64(ref), max_tol=1e-2, mean_tol=3e-3,
                    what=f"dW group {g} ({b0 - a0} rows)")


def _unpack_w13(g13):
    """[G, 2I, d] packed -> (dW1 [G, I, d], dW3 [G, I, d])."""
    G, I2, d = g13.shape
    v = g13.view(G, I2 // 32, 2, 16, d)
    return v[:, :, 0].reshape(G, I2 // 2, d), v[:, :, 1].reshape(G, I2 // 2, d)


def _layer_case(name):
    if name == "tiny_softmax":
        return synth.CONFIGS["tiny"].replace(gate_kind="softmax", routed_scale=1.0)
    return synth.CONFIGS[name]


@pytest.mark.parametrize("name,T", [("tiny", None), ("tiny", 200), ("tiny_softmax", None),
                                    ("mid", None)])
def test_layer_backward_matches_oracle(name, T, cuda_ok):
    from mixture_experts_layer_58_b200 import build
    build.build()
    cfg = _layer_case(name)
    inp = Inputs(cfg, T=T)
    lay = inp.layer
    lay.forward(inp.u_dev, train=True)
    g = torch.Generator().manual_seed(99)
    dout = torch.randn(inp.T, cfg.d, generator=g).bfloat16()
    du = lay.backward(dout.cuda())
    torch.cuda.synchronize()
    assert L.moe_get_device_status() == 0

    idx = lay.topk_idx.cpu().numpy().astype(np.int64)
    ref = mb.layer_backward(inp.u, inp.e, idx, cfg.routed_scale, inp.expert, inp.shared_list(),
                            dout, cfg.gate_kind)
    check_close(f64(du), ref.du, max_tol=GRAD_MAX, mean_tol=GRAD_MEAN, what="du")
    check_close(f64(lay.dgate), ref.dgate, max_tol=GRAD_MAX, mean_tol=GRAD_MEAN, what="dgate")
    check_close(f64(lay.grad_centroids), ref.de, max_tol=DE_MAX, mean_tol=DE_MEAN, what="de")
    dw1, dw3 = _unpack_w13(lay.grad_w13)
    for i in np.unique(idx):
        i = int(i)
        check_close(f64(dw1[i]), ref.dw1[i], max_tol=GRAD_MAX, mean_tol=GRAD_MEAN,
                    what=f"dW1 expert {i}")
        check_close(f64(dw3[i]), ref.dw3[i], max_tol=GRAD_MAX, mean_tol=GRAD_MEAN,
                    what=f"dW3 expert {i}")
        check_close(f64(lay.grad_w2[i]), ref.dw2[i], max_tol=GRAD_MAX, mean_tol=GRAD_MEAN,
                    what=f"dW2 expert {i}")
    unused = sorted(set(range(cfg.n_routed)) - set(np.unique(idx).tolist()))
    for i in unused:
        assert bool((lay.grad_w2[i] == 0).all()) and bool((lay.grad_w13[i] == 0).all())
    if ref.dshared:
        s1, s3, s2 = ref.dshared[0]
        g1, g3 = _unpack_w13(lay.grad_ws13)
        check_close(f64(g1[0]), s1, max_tol=GRAD_MAX, mean_tol=GRAD_MEAN, what="shared dW1")
        check_close(f64(g3[0]), s3, max_tol=GRAD_MAX, mean_tol=GRAD_MEAN, what="shared dW3")
        check_close(f64(lay.grad_ws2), s2, max_tol=GRAD_MAX, mean_tol=GRAD_MEAN,
                    what="shared dW2")


def test_v3p_backward_sampled(cuda_ok):
    """The training step at the full V3 prefill shape, in the launch
    configuration `bench.py --mode train` times: du on sampled tokens (those
    of the hottest and the least-loaded expert and random ones), the complete
    weight gradients of the least-loaded expert, and sampled columns of the
    centroid gradient, each against the fp64 backward oracle computed for
    exactly those entries."""
    from mixture_experts_layer_58_b200 import build
    from oracle import moe_oracle as om
    build.build()
    cfg = synth.CONFIGS["v3p"]
    inp = Inputs(cfg)
    lay = inp.layer
    lay.forward(inp.u_dev, train=True)
    g = torch.Generator().manual_seed(99)
    dout = (0.05 * torch.randn(cfg.T, cfg.d, generator=g)).bfloat16()
    du = lay.backward(dout.cuda())
    torch.cuda.synchronize()
    assert L.moe_get_device_status() == 0

    idx = lay.topk_idx.cpu().numpy().astype(np.int64)
    counts = np.bincount(idx.ravel(), minlength=cfg.n_routed)
    hot = int(np.argmax(counts))
    cold = int(np.argmin(np.where(counts > 0, counts, counts.max() + 1)))
    rng = np.random.default_rng(4)
    t_hot = np.nonzero((idx == hot).any(1))[0][:3]
    t_cold = np.nonzero((idx == cold).any(1))[0]
    tokens = np.unique(np.concatenate([t_hot, t_cold, rng.choice(cfg.T, 4, replace=False)]))
    S = cfg.routed_scale
    shared = inp.shared_list()

    # du and dgate of the sampled tokens: the oracle backward of those tokens
    # alone is exact (tokens are independent given the selection)
    ref = mb.layer_backward(inp.u[torch.from_numpy(tokens)], inp.e, idx[tokens], S, inp.expert,
                            shared, dout[torch.from_numpy(tokens)], cfg.gate_kind)
    check_close(f64(du)[tokens], ref.du, max_tol=GRAD_MAX, mean_tol=GRAD_MEAN, what="du (sampled)")
    check_close(f64(lay.dgate)[tokens], ref.dgate, max_tol=GRAD_MAX, mean_tol=GRAD_MEAN,
                what="dgate (sampled)")

    # complete dW1/dW3/dW2 of the least-loaded expert: its rows are all of t_cold
    k_cold = np.nonzero(idx[t_cold] == cold)[1]
    gate = om.gates_for_indices(inp.u[torch.from_numpy(t_cold)], inp.e, idx[t_cold], S,
                                cfg.gate_kind)
    w1, w3, w2 = inp.expert(cold)
    dy = gate[np.arange(len(t_cold)), k_cold][:, None] * f64(dout)[t_cold]
    _, rw1, rw3, rw2 = mb.ffn_backward(f64(inp.u)[t_cold], w1, w3, w2, dy)
    dw1, dw3 = _unpack_w13(lay.grad_w13[cold:cold + 1])
    check_close(f64(dw1[0]), rw1, max_tol=GRAD_MAX, mean_tol=GRAD_MEAN, what=f"dW1 expert {cold}")
    check_close(f64(dw3[0]), rw3, max_tol=GRAD_MAX, mean_tol=GRAD_MEAN, what=f"dW3 expert {cold}")
    check_close(f64(lay.grad_w2[cold]), rw2, max_tol=GRAD_MAX, mean_tol=GRAD_MEAN,
                what=f"dW2 expert {cold}")

    # centroid gradient of the least-loaded expert: sum over its tokens of dz u
    full_cold = mb.layer_backward(inp.u[torch.from_numpy(t_cold)], inp.e, idx[t_cold], S,
                                  inp.expert, shared, dout[torch.from_numpy(t_cold)],
                                  cfg.gate_kind)
    check_close(f64(lay.grad_centroids[cold]), full_cold.de[cold], max_tol=DE_MAX,
                mean_tol=DE_MEAN, what=f"de expert {cold}")
    del inp
    torch.cuda.empty_cache()
