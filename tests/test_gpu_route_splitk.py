"""The split-K gate GEMM (moe_route_splitk) against the fp64 oracle and
against the one-pass moe_route (one CTA per 128 tokens below 256 tokens,
CTA pairs from 256) on the same inputs: selection bit-exact away
from near-ties, gates and loads as the oracle's, ragged and degenerate
shapes, the workspace contract. Needs a B200."""
import numpy as np
import pytest
import torch

from mixture_experts_layer_58_b200 import _lib as L
from mixture_experts_layer_58_b200 import synth
from oracle import moe_oracle as om

from gpu_support import NEAR_TIE, check_route

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built(cuda_ok):
    from mixture_experts_layer_58_b200 import build
    build.build()
    L.load()


def _route_both(cfg, T, bias=None):
    """(split-K result, one-pass result, oracle routing) on the workload's first T tokens."""
    cfg = cfg.replace(T=max(cfg.T, T))          # the draw must hold T rows
    u = synth.tokens(cfg, T)
    assert u.shape == (T, cfg.d)
    e = synth.centroids(cfg)
    b = synth.bias(cfg) if bias is None else bias
    use_b = b if cfg.gate_kind == "sigmoid" else None
    ud, ed = u.cuda(), e.cuda()
    bd = use_b.cuda() if use_b is not None else None
    K, n = cfg.top_k, cfg.n_routed
    res = []
    for split in (True, False):
        idx = torch.full((T, K), -7, dtype=torch.int32, device="cuda")
        gate = torch.full((T, K), -7.0, dtype=torch.float32, device="cuda")
        counts = torch.full((n,), 99, dtype=torch.int32, device="cuda")
        if split:
            ws_bytes = L.moe_route_splitk_workspace_size(T, cfg.d, n)
            ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
            L.moe_route_splitk(ud, ed, bd, T, cfg.d, n, K, cfg.gate_kind, cfg.routed_scale, idx,
                               gate, counts, ws, ws_bytes)
        else:
            L.moe_route(ud, ed, bd, T, cfg.d, n, K, cfg.gate_kind, cfg.routed_scale, idx, gate,
                        counts)
        torch.cuda.synchronize()
        res.append((idx.cpu().numpy(), gate.cpu().numpy(), counts.cpu().numpy()))
    assert L.moe_get_device_status() == 0
    r = om.route(u, e, use_b, K, cfg.routed_scale, cfg.gate_kind)
    return res[0], res[1], r, u, e


CASES = [
    ("tiny", 64, {}),
    ("tiny", 1, {}),
    ("tiny", 129, {}),
    ("tiny", 383, {}),
    ("tiny", 64, {"n_routed": 20, "top_k": 2}),          # 20 experts: padded MMA columns
    ("tiny", 64, {"gate_kind": "softmax", "bias_lo": 0.0, "bias_hi": 0.0}),
    ("tiny", 64, {"n_routed": 8, "top_k": 8}),           # every expert selected
    # T >= 256: moe_route takes the CTA-pair kernel (N = N_r padded to 32)
    ("tiny", 300, {"n_routed": 20, "top_k": 2}),
    ("tiny", 300, {"n_routed": 8, "top_k": 8}),
    ("tiny", 513, {"gate_kind": "softmax", "bias_lo": 0.0, "bias_hi": 0.0}),
    ("mid", 1000, {}),
    ("v3d", 128, {}),                                    # V3 decode: d 7168, 256 experts, top-8
    ("v3d", 2048, {}),
    ("v3d_softmax", 128, {}),
]


@pytest.mark.parametrize("name,T,kw", CASES)
def test_splitk_route_matches_oracle_and_one_pass(name, T, kw):
    cfg = synth.CONFIGS[name].replace(**kw) if kw else synth.CONFIGS[name]
    (si, sg, sc), (oi, og, oc), r, u, e = _route_both(cfg, T)
    check_route(si, sg, sc, r, cfg.routed_scale, u, e, cfg.gate_kind)
    check_route(oi, og, oc, r, cfg.routed_scale, u, e, cfg.gate_kind)
    # the two forms add the same fp32 products in another order: indices agree
    # wherever the oracle's keys are not near-tied
    near = r.min_adjacent_gap() < NEAR_TIE
    assert np.array_equal(si[~near], oi[~near])


def test_splitk_route_every_token_on_one_expert():
    cfg = synth.CONFIGS["tiny"].replace(T=300)
    b = synth.bias(cfg).clone()
    b[7] = 5.0
    (si, sg, sc), _, r, u, e = _route_both(cfg, 300, bias=b)
    check_route(si, sg, sc, r, cfg.routed_scale, u, e, cfg.gate_kind)
    assert sc[7] == 300 and np.all(si[:, 0] == 7)


def test_splitk_route_workspace_contract_and_empty_batch():
    cfg = synth.CONFIGS["v3d"]
    T, n, K = 128, cfg.n_routed, cfg.top_k
    need = L.moe_route_splitk_workspace_size(T, cfg.d, n)
    assert need % 256 == 0 and need >= T * n * 4
    u = synth.tokens(cfg, T).cuda()
    e = synth.centroids(cfg).cuda()
    idx = torch.empty((T, K), dtype=torch.int32, device="cuda")
    gate = torch.empty((T, K), dtype=torch.float32, device="cuda")
    counts = torch.full((n,), 5, dtype=torch.int32, device="cuda")
    small = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(L.MoEError) as ex:
        L.moe_route_splitk(u, e, None, T, cfg.d, n, K, "sigmoid", 1.0, idx, gate, counts, small,
                           small.numel())
    assert ex.value.status == L.MOE_ERR_WORKSPACE
    with pytest.raises(L.MoEError) as ex:
        L.moe_route_splitk(u, e, None, T, cfg.d, n, K, "sigmoid", 1.0, idx, gate, counts, None, 0)
    assert ex.value.status == L.MOE_ERR_WORKSPACE
    # T = 0: loads zeroed, no workspace needed, nothing else written
    L.moe_route_splitk(u, e, None, 0, cfg.d, n, K, "sigmoid", 1.0, idx, gate, counts, None, 0)
    torch.cuda.synchronize()
    assert int(counts.abs().sum()) == 0
    assert L.moe_get_device_status() == 0
