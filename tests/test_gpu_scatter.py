"""The fused-scatter mode: the down-projection multiplies every routed row by
its gate in its epilogue and writes it to the row of its (token, slot) pair;
the combine adds K adjacent rows. Against the oracle, and call by call against
the plain five-call path on the same inputs. Needs a B200."""
import numpy as np
import pytest
import torch

from mixture_experts_layer_58_b200 import _lib as L
from mixture_experts_layer_58_b200 import synth
from oracle import moe_oracle as om

from gpu_support import Inputs, check_close, check_route, f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built(cuda_ok):
    from mixture_experts_layer_58_b200 import build
    build.build()
    L.load()


def _forward(inp, residual=True):
    out = inp.layer.forward(inp.u_dev, residual=residual)
    torch.cuda.synchronize()
    assert L.moe_get_device_status() == 0
    return out


# tiny: groups of < 256 rows on average -> 1-CTA tiles; mid: CTA-pair tiles;
# T = 383 leaves a ragged last chunk of tokens and ragged group tails
@pytest.mark.parametrize("name,T,gather", [("tiny", None, False), ("tiny", 383, False),
                                           ("mid", None, False), ("mid", None, True)])
def test_fused_scatter_layer_matches_oracle(name, T, gather):
    cfg = synth.CONFIGS[name] if T is None else synth.CONFIGS[name].replace(T=512)
    inp = Inputs(cfg, T=T, fused_scatter=True, fused_gather=gather)
    out = _forward(inp)
    lay = inp.layer
    r = inp.oracle_route()
    gidx = lay.topk_idx.cpu().numpy()
    check_route(gidx, lay.topk_gate.cpu().numpy(), lay.counts.cpu().numpy(), r,
                cfg.routed_scale, inp.u, inp.e, cfg.gate_kind)
    g = om.gates_for_indices(inp.u, inp.e, gidx, cfg.routed_scale, cfg.gate_kind)
    ref = om.layer_output(inp.u, gidx, g, inp.expert, inp.shared_list())
    check_close(f64(out), ref)


def test_slot_index_inverts_pos():
    cfg = synth.CONFIGS["mid"]
    inp = Inputs(cfg, fused_scatter=True)
    _forward(inp)
    lay = inp.layer
    pos = lay.pos.cpu().numpy().reshape(-1)
    slot = lay.dst_slot.cpu().numpy()
    assert np.array_equal(slot[pos], np.arange(pos.size))
    assert sorted(slot.tolist()) == list(range(pos.size))


def test_scattered_rows_are_gate_times_plain_rows_and_combine_sums_them():
    """Row s of the slot buffer equals g[s] * y_perm[pos[s]] of the plain path
    up to the one extra bf16 rounding the plain path makes (y before the
    gate), and moe_combine_slots equals the fp64 sum of its operands up to
    its one bf16 rounding."""
    cfg = synth.CONFIGS["mid"]
    plain = Inputs(cfg)
    _forward(plain)
    y_plain = f64(plain.layer.y_perm)
    pos = plain.layer.pos.cpu().numpy().reshape(-1)
    gate = plain.layer.topk_gate.cpu().numpy().astype(np.float64).reshape(-1)
    fused = Inputs(cfg, fused_scatter=True)
    out = _forward(fused)
    lay = fused.layer
    assert np.array_equal(lay.pos.cpu().numpy().reshape(-1), pos)
    y_slots = f64(lay.y_perm)
    want = gate[:, None] * y_plain[pos]
    # the same fp32 accumulator a on both sides (same kernel, same tiles):
    # |round(g a) - g round(a)| <= 2 half-ulps of bf16 = 2^-7 |g a|
    err = np.abs(y_slots - want)
    assert np.all(err <= 1.01 * 2.0 ** -7 * np.abs(want)), err.max()
    T, K, d = cfg.T, cfg.top_k, cfg.d
    u, sh = f64(fused.u_dev), f64(lay.shared_out)
    ys = y_slots.reshape(T, K, d)
    ref = u + sh + ys.sum(1)
    mag = np.abs(u) + np.abs(sh) + np.abs(ys).sum(1)
    got = f64(out)
    # one bf16 rounding of an fp32 sum
    assert np.all(np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-6 * mag)


def test_fused_scatter_without_residual_matches_oracle():
    cfg = synth.CONFIGS["tiny"]
    inp = Inputs(cfg, fused_scatter=True)
    out = _forward(inp, residual=False)
    gidx = inp.layer.topk_idx.cpu().numpy()
    g = om.gates_for_indices(inp.u, inp.e, gidx, cfg.routed_scale, cfg.gate_kind)
    ref = om.layer_output(inp.u, gidx, g, inp.expert, inp.shared_list(), residual=False)
    check_close(f64(out), ref)


# tiny: 1-CTA tiles (one thread stores a row's 256 features and counts them);
# mid: CTA-pair tiles (a half-warp stores and counts 128 features); T = 383:
# ragged token chunks and group tails; no shared expert; no residual
@pytest.mark.parametrize("name,T,residual,kw", [("tiny", None, True, {}),
                                                ("tiny", 383, True, {}),
                                                ("tiny", None, True, {"n_shared": 0}),
                                                ("mid", None, True, {}),
                                                ("mid", None, False, {})])
def test_fused_combine_bit_identical_to_scatter_then_combine(name, T, residual, kw):
    """The combine in the down-projection's epilogue (the store that completes
    a token's slot rows over a 128-feature block adds them) gives the same
    bits as moe_combine_slots after the scattering down-projection, and the
    oracle's layer output."""
    cfg = synth.CONFIGS[name].replace(**kw)
    if T is not None:
        cfg = cfg.replace(T=512)
    a = Inputs(cfg, T=T, fused_scatter=True)
    want = _forward(a, residual).clone()
    b = Inputs(cfg, T=T, fused_combine=True)
    assert b.layer.fused_combine
    got = _forward(b, residual)
    assert torch.equal(got, want)
    lay = b.layer
    gidx = lay.topk_idx.cpu().numpy()
    g = om.gates_for_indices(b.u, b.e, gidx, cfg.routed_scale, cfg.gate_kind)
    ref = om.layer_output(b.u, gidx, g, b.expert, b.shared_list(), residual=residual)
    check_close(f64(got), ref)
    # a second forward on the same buffers (counts re-zeroed by the call)
    again = _forward(b, residual)
    assert torch.equal(again, want)


def test_fused_combine_v3p_bit_identical():
    """V3 prefill (CTA-pair tiles, 256 experts, Zipf-skewed groups): the fused
    combine against the scatter + combine pair on the same inputs."""
    cfg = synth.CONFIGS["v3p"]
    a = Inputs(cfg, fused_scatter=True)
    want = _forward(a).clone()
    del a
    torch.cuda.empty_cache()
    b = Inputs(cfg, fused_combine=True)
    got = _forward(b)
    assert torch.equal(got, want)


def test_fused_combine_workspace_contract():
    cfg = synth.CONFIGS["tiny"]
    inp = Inputs(cfg, fused_combine=True)
    _forward(inp)
    lay = inp.layer
    T, K, d = cfg.T, cfg.top_k, cfg.d
    need = L.moe_expert_down_scatter_combine_workspace_size(T, d)
    assert need >= T * (d // 128) * 4 and need % 256 == 0
    small = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
    args = (lay.ffn_ws, lay.offsets, cfg.n_routed, T * K, cfg.inter, d, lay.w2, lay.dst_slot,
            lay.topk_gate, T, K, lay.y_perm, lay.shared_out, inp.u_dev, lay.out)
    with pytest.raises(L.MoEError) as ex:
        L.moe_expert_down_scatter_combine(*args, small, small.numel())
    assert ex.value.status == L.MOE_ERR_WORKSPACE
    with pytest.raises(L.MoEError) as ex:
        L.moe_expert_down_scatter_combine(*args, None, 0)
    assert ex.value.status == L.MOE_ERR_WORKSPACE
    assert L.moe_get_device_status() == 0
