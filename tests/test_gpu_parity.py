"""Parity of every C-ABI call with the fp64 oracle on the Tiny and Mid
workloads and on edge cases (ragged, empty, degenerate). Needs a B200."""
import numpy as np
import pytest
import torch

from mixture_experts_layer_58_b200 import _lib as L
from mixture_experts_layer_58_b200 import synth
from mixture_experts_layer_58_b200.layer import MoELayer
from oracle import moe_oracle as om

from gpu_support import Inputs, check_close, check_route, f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built(cuda_ok):
    from mixture_experts_layer_58_b200 import build
    build.build()
    L.load()


def _run_forward(inp: Inputs, residual=True):
    out = inp.layer.forward(inp.u_dev, residual=residual)
    torch.cuda.synchronize()
    assert L.moe_get_device_status() == 0
    return out


def _full_check(inp: Inputs, residual=True):
    cfg = inp.cfg
    out = _run_forward(inp, residual)
    lay = inp.layer
    r = inp.oracle_route()
    gidx = lay.topk_idx.cpu().numpy()
    near = check_route(gidx, lay.topk_gate.cpu().numpy(), lay.counts.cpu().numpy(), r,
                       cfg.routed_scale, inp.u, inp.e, cfg.gate_kind)
    # output on the GPU's own selection (gates recomputed by the oracle in fp64)
    g = om.gates_for_indices(inp.u, inp.e, gidx, cfg.routed_scale, cfg.gate_kind)
    ref = om.layer_output(inp.u, gidx, g, inp.expert, inp.shared_list(), residual=residual)
    mx, mean = check_close(f64(out), ref)
    return near, mx, mean


def test_tiny_layer_forward_matches_oracle():
    inp = Inputs(synth.CONFIGS["tiny"])
    _full_check(inp)


def test_tiny_every_call_matches_oracle():
    cfg = synth.CONFIGS["tiny"]
    inp = Inputs(cfg)
    lay = inp.layer
    _run_forward(inp)
    T, K, d = cfg.T, cfg.top_k, cfg.d
    gidx = lay.topk_idx.cpu().numpy()
    # permute: bit-exact against the oracle's dispatch order of the same indices
    disp = om.dispatch(gidx, cfg.n_routed)
    assert np.array_equal(lay.offsets.cpu().numpy(), disp.offsets)
    assert np.array_equal(lay.pos.cpu().numpy(), disp.pos)
    assert np.array_equal(lay.src.cpu().numpy(), disp.src)
    xp = lay.x_perm.cpu()
    assert torch.equal(xp, inp.u[torch.from_numpy(disp.src)])
    # routed FFN: each expert's rows against the fp64 FFN of the same rows
    y = f64(lay.y_perm)
    ref = np.zeros_like(y)
    for i in range(cfg.n_routed):
        a, b = disp.offsets[i], disp.offsets[i + 1]
        if b > a:
            ref[a:b] = om.ffn(xp[a:b].float().numpy(), *inp.expert(i))
    check_close(y, ref, what="routed FFN")
    # shared FFN
    sh = om.shared_output(inp.u, inp.shared_list())
    check_close(f64(lay.shared_out), sh, what="shared FFN")
    # combine: fp64 sum of the GPU's own operands -> only the bf16 rounding differs
    g = lay.topk_gate.cpu().numpy().astype(np.float64)
    want = f64(inp.u) + f64(lay.shared_out)
    for k in range(K):
        want += g[:, k:k + 1] * y[disp.pos[:, k]]
    got = f64(lay.out)
    assert np.all(np.abs(got - want) <= np.abs(want) * 2.0 ** -8 + 1e-6)


def test_tiny_bias_update_bit_exact():
    cfg = synth.CONFIGS["tiny"]
    inp = Inputs(cfg)
    lay = inp.layer
    b0 = lay.bias.cpu().numpy().copy()
    lay.step(inp.u_dev)
    torch.cuda.synchronize()
    want = om.bias_update(lay.counts.cpu().numpy(), b0, cfg.T, cfg.top_k, cfg.gamma)
    assert np.array_equal(lay.bias.cpu().numpy(), want)


def test_mid_layer_forward_matches_oracle():
    inp = Inputs(synth.CONFIGS["mid"])
    near, mx, mean = _full_check(inp)
    assert near < 0.05 * inp.T


def test_mid_sixteen_bias_steps():
    """16 route -> update steps on the same batch (b starts at 0). Each step's
    routing is checked against the oracle under the GPU's current bias, and
    each update is bit-exact against the oracle's update of the GPU's counts."""
    cfg = synth.CONFIGS["mid"]
    inp = Inputs(cfg)
    lay = inp.layer
    lay.allocate(cfg.T)
    first_max = None
    for step in range(cfg.bias_steps):
        b_before = lay.bias.cpu().numpy().copy()
        lay.route(inp.u_dev)
        lay.update_bias()
        torch.cuda.synchronize()
        counts = lay.counts.cpu().numpy()
        r = inp.oracle_route(bias=torch.from_numpy(b_before))
        check_route(lay.topk_idx.cpu().numpy(), lay.topk_gate.cpu().numpy(), counts, r,
                    cfg.routed_scale, inp.u, inp.e, cfg.gate_kind)
        want = om.bias_update(counts, b_before, cfg.T, cfg.top_k, cfg.gamma)
        assert np.array_equal(lay.bias.cpu().numpy(), want), f"step {step}"
        if first_max is None:
            first_max = counts.max()
    assert L.moe_get_device_status() == 0


@pytest.mark.parametrize("T", [1, 127, 129, 200, 383])
def test_ragged_token_counts(T):
    inp = Inputs(synth.CONFIGS["tiny"].replace(T=512), T=T)
    _full_check(inp)


def test_softmax_gate_variant():
    inp = Inputs(synth.CONFIGS["tiny"].replace(gate_kind="softmax", bias_lo=0.0, bias_hi=0.0))
    _full_check(inp)


def test_no_residual_listing_form():
    inp = Inputs(synth.CONFIGS["tiny"])
    _full_check(inp, residual=False)


def test_experts_not_multiple_of_16_and_empty_experts():
    # 20 experts (padded to 32 MMA columns), top-2: several experts get no token
    cfg = synth.CONFIGS["tiny"].replace(n_routed=20, top_k=2, T=48)
    inp = Inputs(cfg)
    _full_check(inp)


def test_all_tokens_on_one_expert():
    cfg = synth.CONFIGS["tiny"].replace(T=300)
    inp = Inputs(cfg)
    inp.layer.bias[7] = 5.0
    b = inp.b.clone()
    b[7] = 5.0
    inp.b = b
    near, _, _ = _full_check(inp)
    assert int(inp.layer.counts[7]) == cfg.T


def test_dense_reduction_one_expert_top1():
    # N_r = 1, K = 1, S = 1, no shared expert: h' = u + FFN(u)
    cfg = synth.CONFIGS["tiny"].replace(n_routed=1, top_k=1, n_shared=0, T=130)
    inp = Inputs(cfg)
    out = _run_forward(inp)
    w1, w3, w2 = inp.expert(0)
    ref = f64(inp.u) + om.ffn(inp.u.float().numpy(), w1, w3, w2)
    check_close(f64(out), ref)
    assert np.all(inp.layer.topk_gate.cpu().numpy() == 1.0)


def test_all_experts_selected():
    # K = N_r = 8: selection covers every expert whatever the bias
    cfg = synth.CONFIGS["tiny"].replace(n_routed=8, top_k=8)
    inp = Inputs(cfg)
    _full_check(inp)
    assert np.all(inp.layer.counts.cpu().numpy() == cfg.T)


def test_empty_batch():
    cfg = synth.CONFIGS["tiny"]
    inp = Inputs(cfg, T=64)
    lay = inp.layer
    u0 = torch.empty((0, cfg.d), dtype=torch.bfloat16, device="cuda")
    lay.allocate(0)
    lay.counts.fill_(7)
    out = lay.forward(u0)
    lay.update_bias()
    torch.cuda.synchronize()
    assert out.shape == (0, cfg.d)
    assert int(lay.counts.abs().sum()) == 0
    assert np.array_equal(lay.bias.cpu().numpy(), inp.b.numpy())   # mean 0, loads 0: no change


def test_run_to_run_bit_identical():
    inp = Inputs(synth.CONFIGS["mid"])
    a = _run_forward(inp).clone()
    b = _run_forward(inp).clone()
    assert torch.equal(a, b)


def test_grouped_ffn_single_group_vs_torch_matmul():
    """moe_grouped_ffn with G = 1 against fp32 torch matmuls of the same bf16
    operands (h rounded to bf16 between the two GEMMs as the kernel does)."""
    g = torch.Generator(device="cuda").manual_seed(11)
    rows, d, inter = 333, 512, 384
    x = torch.randn(rows, d, generator=g, device="cuda").bfloat16()
    w1 = (0.05 * torch.randn(inter, d, generator=g, device="cuda")).bfloat16()
    w3 = (0.05 * torch.randn(inter, d, generator=g, device="cuda")).bfloat16()
    w2 = (0.05 * torch.randn(d, inter, generator=g, device="cuda")).bfloat16()
    w13 = torch.empty(1, 2 * inter, d, dtype=torch.bfloat16, device="cuda")
    L.moe_pack_w13(w1[None].contiguous(), w3[None].contiguous(), 1, inter, d, w13)
    off = torch.tensor([0, rows], dtype=torch.int32, device="cuda")
    y = torch.empty(rows, d, dtype=torch.bfloat16, device="cuda")
    wsb = L.moe_grouped_ffn_workspace_size(rows, inter)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    L.moe_grouped_ffn(x, None, off, 1, rows, d, inter, w13, None, w2, None, L.MOE_BF16, y, ws, wsb)
    torch.cuda.synchronize()
    a = x.float() @ w1.float().T
    b = x.float() @ w3.float().T
    h = (torch.nn.functional.silu(a) * b).bfloat16()
    ref = h.float() @ w2.float().T
    check_close(y.float().cpu().numpy(), ref.cpu().numpy(), max_tol=1e-2, mean_tol=3e-3)
    hk = ws[: rows * inter * 2].view(torch.bfloat16).view(rows, inter)
    check_close(hk.float().cpu().numpy(), h.float().cpu().numpy(), max_tol=1e-2, mean_tol=3e-3,
                what="h")


@pytest.mark.parametrize("extra", [0, 256, 600])
def test_grouped_ffn_tile_paths_by_group_size(extra):
    """Group sizes that hit every tile path of both grouped-GEMM forms: empty
    groups, ragged last tiles of every size, full tiles. Each group against fp32
    torch matmuls of the same bf16 operands, h rounded to bf16 as the kernel
    does; rows past the last group stay untouched."""
    # extra = 0: groups average < 256 rows -> single-CTA 128-row tiles;
    # extra = 256, 600: larger groups -> CTA-pair tiles of 256 rows, the last
    # one an MMA of N = its rows rounded up to 32 (1..256 valid rows: 257,
    # 271, ... leave 1, 15, 16, 17, 31, 32, 33, ... rows in the last tile).
    sizes = [1, 15, 0, 16, 17, 31, 32, 33, 100, 127, 128, 129, 255, 256, 0, 300, 384, 385, 513]
    sizes = [s + extra if s else 0 for s in sizes]
    G, d, inter = len(sizes), 256, 256
    rows = sum(sizes)
    pad = 64                                   # rows after the last group
    g = torch.Generator(device="cuda").manual_seed(12)
    x = torch.randn(rows + pad, d, generator=g, device="cuda").bfloat16()
    w1 = (0.05 * torch.randn(G, inter, d, generator=g, device="cuda")).bfloat16()
    w3 = (0.05 * torch.randn(G, inter, d, generator=g, device="cuda")).bfloat16()
    w2 = (0.05 * torch.randn(G, d, inter, generator=g, device="cuda")).bfloat16()
    w13 = torch.empty(G, 2 * inter, d, dtype=torch.bfloat16, device="cuda")
    L.moe_pack_w13(w1, w3, G, inter, d, w13)
    off = torch.tensor(np.concatenate([[0], np.cumsum(sizes)]), dtype=torch.int32, device="cuda")
    y = torch.full((rows + pad, d), 3.0, dtype=torch.bfloat16, device="cuda")
    wsb = L.moe_grouped_ffn_workspace_size(rows + pad, inter)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    L.moe_grouped_ffn(x, None, off, G, rows + pad, d, inter, w13, None, w2, None, L.MOE_BF16, y,
                      ws, wsb)
    torch.cuda.synchronize()
    assert L.moe_get_device_status() == 0
    assert bool((y[rows:] == 3.0).all())
    o = off.cpu().tolist()
    for i in range(G):
        a, b = o[i], o[i + 1]
        if a == b:
            continue
        xa = x[a:b].float()
        h = (torch.nn.functional.silu(xa @ w1[i].float().T) * (xa @ w3[i].float().T)).bfloat16()
        ref = h.float() @ w2[i].float().T
        check_close(y[a:b].float().cpu().numpy(), ref.cpu().numpy(), max_tol=1e-2,
                    mean_tol=3e-3, what=f"group {i} ({b - a} rows)")


def test_grouped_ffn_most_groups_pair_tiles():
    """The largest group count (1024) on CTA-pair tiles: the group table in
    shared memory at its biggest; sizes from 0 to 700 rows, with empty groups,
    single-row groups and ragged tails. Every group against fp32 torch matmuls
    of the same bf16 operands."""
    G, d, inter = 1024, 256, 128
    rng = np.random.default_rng(13)
    sizes = rng.choice([0, 1, 33, 256, 257, 300, 511, 700], size=G,
                       p=[0.05, 0.1, 0.1, 0.2, 0.1, 0.2, 0.15, 0.1])
    rows = int(sizes.sum())
    assert rows >= 256 * G                     # groups average >= 256 rows: pair tiles
    g = torch.Generator(device="cuda").manual_seed(14)
    x = torch.randn(rows, d, generator=g, device="cuda").bfloat16()
    w1 = (0.05 * torch.randn(G, inter, d, generator=g, device="cuda")).bfloat16()
    w3 = (0.05 * torch.randn(G, inter, d, generator=g, device="cuda")).bfloat16()
    w2 = (0.05 * torch.randn(G, d, inter, generator=g, device="cuda")).bfloat16()
    w13 = torch.empty(G, 2 * inter, d, dtype=torch.bfloat16, device="cuda")
    L.moe_pack_w13(w1, w3, G, inter, d, w13)
    off = torch.tensor(np.concatenate([[0], np.cumsum(sizes)]), dtype=torch.int32, device="cuda")
    y = torch.full((rows, d), 3.0, dtype=torch.bfloat16, device="cuda")
    wsb = L.moe_grouped_ffn_workspace_size(rows, inter)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    L.moe_grouped_ffn(x, None, off, G, rows, d, inter, w13, None, w2, None, L.MOE_BF16, y, ws, wsb)
    torch.cuda.synchronize()
    assert L.moe_get_device_status() == 0
    o = off.cpu().tolist()
    for i in range(G):
        a, b = o[i], o[i + 1]
        if a == b:
            continue
        xa = x[a:b].float()
        h = (torch.nn.functional.silu(xa @ w1[i].float().T) * (xa @ w3[i].float().T)).bfloat16()
        ref = h.float() @ w2[i].float().T
        check_close(y[a:b].float().cpu().numpy(), ref.cpu().numpy(), max_tol=1e-2,
                    mean_tol=3e-3, what=f"group {i} ({b - a} rows)")


@pytest.mark.parametrize("name,T", [("tiny", None), ("tiny", 383), ("mid", None)])
def test_fused_gather_layer_matches_oracle(name, T):
    """The fused mode: dispatch computes only row indices and the up-projection
    gathers the token rows of u itself (TMA gather, four rows per load)."""
    cfg = synth.CONFIGS[name] if T is None else synth.CONFIGS[name].replace(T=512)
    inp = Inputs(cfg, T=T, fused_gather=True)
    _full_check(inp)
    assert inp.layer.x_perm is None           # no expert-contiguous copy was made


def test_gather_up_projection_bit_identical_to_copy():
    """moe_expert_up_swiglu_gather on u + src_token equals moe_expert_up_swiglu
    on the copied x_perm bit for bit (same tiles, same MMA order)."""
    cfg = synth.CONFIGS["mid"]
    inp = Inputs(cfg)
    lay = inp.layer
    _run_forward(inp)
    T, K = cfg.T, cfg.top_k
    rows = T * K
    h_copy = torch.empty((rows, cfg.inter), dtype=torch.bfloat16, device="cuda")
    h_gath = torch.full((rows, cfg.inter), 9.0, dtype=torch.bfloat16, device="cuda")
    L.moe_expert_up_swiglu(lay.x_perm, lay.offsets, cfg.n_routed, rows, cfg.d, cfg.inter, lay.w13,
                           h_copy)
    L.moe_expert_up_swiglu_gather(inp.u_dev, T, lay.src, lay.offsets, cfg.n_routed, rows, cfg.d,
                                  cfg.inter, lay.w13, h_gath)
    torch.cuda.synchronize()
    assert L.moe_get_device_status() == 0
    assert torch.equal(h_copy, h_gath)


def test_bounded_wait_reports_timeout_and_context_survives():
    """A wait that nothing completes gives up after its limit (50 ms here),
    the host reads MOE_ERR_DEVICE_TIMEOUT with the self-test bit, the status is
    cleared, and the layer still runs correctly afterwards."""
    assert L.moe_get_device_status() == 0
    L.moe_selftest_wait_timeout(50)
    torch.cuda.synchronize()
    st = L.moe_get_device_status(clear=True)
    assert st & 8
    assert L.moe_get_device_status() == 0
    inp = Inputs(synth.CONFIGS["tiny"])
    _full_check(inp)


@pytest.mark.parametrize("name", ["tiny", "mid"])
def test_shared_expert_in_line_matches_overlapped(name):
    """The shared expert on its side stream (default) and run in line after
    the routed experts give the same layer output bit for bit, and both match
    the oracle (Mid joins the side stream before the routed GEMMs, Tiny
    before the combine)."""
    cfg = synth.CONFIGS[name]
    inp = Inputs(cfg)
    lay = inp.layer
    assert lay.overlap_shared
    _full_check(inp)
    overlapped = lay.out.clone()
    lay.overlap_shared = False
    _full_check(inp)
    assert torch.equal(lay.out, overlapped)


@pytest.mark.parametrize("name,T", [("tiny", None), ("tiny", 383)])
def test_shared_expert_as_a_routed_group_bit_identical(name, T):
    """The shared expert as group N_r of the routed grouped GEMMs (its rows
    appended by moe_permute_shared) gives the same layer output bit for bit
    as its own G = 1 launches, and matches the oracle. Tiny runs the 1-CTA
    tiles; the V3 prefill test covers the CTA-pair tiles."""
    cfg = synth.CONFIGS[name] if T is None else synth.CONFIGS[name].replace(T=512)
    a = Inputs(cfg, T=T)
    a.layer.shared_grouped = False
    want = _run_forward(a).clone()
    b = Inputs(cfg, T=T)
    b.layer.shared_grouped = True
    assert b.layer.mergeable
    got = _run_forward(b)
    assert b.layer.shared_in_grouped
    assert torch.equal(got, want)
    _full_check(b)


@pytest.mark.parametrize("name", ["tiny", "mid", "v3d"])
def test_cuda_graph_replay_matches_eager_steps(name):
    """capture(T) records a step (forward + bias update) as one CUDA graph,
    side stream included: three replays give the same outputs and biases bit
    for bit as three eager steps on the same inputs (Tiny: 1-CTA tiles and
    the shared expert joined late; Mid: pair tiles, joined early; V3 decode:
    the split-K route)."""
    cfg = synth.CONFIGS[name]
    a = Inputs(cfg)
    want = []
    for _ in range(3):
        want.append(a.layer.step(a.u_dev).clone())
    torch.cuda.synchronize()
    bias_a = a.layer.bias.clone()
    del a
    torch.cuda.empty_cache()
    b = Inputs(cfg)
    b.layer.capture(cfg.T)
    torch.cuda.synchronize()
    assert torch.equal(b.layer.bias, b.b.to(b.layer.bias.device))   # capture changes nothing
    for k in range(3):
        got = b.layer.replay(b.u_dev)
        torch.cuda.synchronize()
        assert torch.equal(got, want[k]), f"replay {k}"
    assert torch.equal(b.layer.bias, bias_a)
    assert L.moe_get_device_status() == 0
