"""FP8 E4M3 variant against the oracle's FP8 emulation: the quantisers
bit-exact (both sides decide every code in fp32), the promoted FP8 expert GEMMs
and the layer within the FP8 tolerance (max|diff| <= 3e-2 * max|ref|).
Needs a B200."""
import numpy as np
import pytest
import torch

from mixture_experts_layer_58_b200 import _lib as L
from mixture_experts_layer_58_b200 import synth
from oracle import fp8 as of
from oracle import moe_oracle as om

from gpu_support import Inputs, check_close, check_route, f64

pytestmark = pytest.mark.gpu

FP8_MAX_TOL = 3e-2      # spec FP8 tolerance
FP8_MEAN_TOL = 1e-2


@pytest.fixture(scope="module", autouse=True)
def _built(cuda_ok):
    from mixture_experts_layer_58_b200 import build
    build.build()
    L.load()


def _rand_bf16(shape, seed, scale=1.0):
    g = torch.Generator(device="cuda").manual_seed(seed)
    return (scale * torch.randn(shape, generator=g, device="cuda")).bfloat16()


def test_activation_quant_bit_exact():
    rows, cols = 300, 384                       # odd number of 128-wide tiles
    x = _rand_bf16((rows, cols), 1)
    x[5, 128:256] = 0                           # all-zero tile -> scale 1
    x[7] *= 1000.0                              # large values
    x[9] *= 1e-4                                # values that land in the subnormal codes
    q = torch.empty((rows, cols), dtype=torch.uint8, device="cuda")
    s = torch.empty((rows, cols // 128), dtype=torch.float32, device="cuda")
    L.moe_quant_act_fp8(x, rows, cols, q, s)
    torch.cuda.synchronize()
    want_q, want_s = of.quant_act_1x128(x.float().cpu().numpy())
    assert np.array_equal(s.cpu().numpy(), want_s)
    assert np.array_equal(q.cpu().numpy(), want_q)


def test_weight_quant_bit_exact():
    G, R, C = 3, 256, 384
    w = _rand_bf16((G, R, C), 2, 0.02)
    w[1, :128, 128:256] = 0
    q = torch.empty((G, R, C), dtype=torch.uint8, device="cuda")
    s = torch.empty((G, R // 128, C // 128), dtype=torch.float32, device="cuda")
    L.moe_quant_weights_fp8(w, G, R, C, q, s)
    torch.cuda.synchronize()
    for g in range(G):
        want_q, want_s = of.quant_weight_128x128(w[g].float().cpu().numpy())
        assert np.array_equal(s[g].cpu().numpy(), want_s)
        assert np.array_equal(q[g].cpu().numpy(), want_q)


def test_fp8_dispatch_quantises_each_token_once_bit_exact():
    """moe_permute_fp8 on bf16 rows: every copied row's codes and scales equal
    the oracle's 1x128 quantisation of its token, and u8 / u_scales hold the
    token's own codes."""
    cfg = synth.CONFIGS["tiny"].replace(T=383, d=512)
    u = _rand_bf16((cfg.T, cfg.d), 11)
    u[5, :128] = 0                                # an all-zero tile: scale 1
    u[9] *= 1e-4
    g = torch.Generator().manual_seed(3)
    idx = torch.argsort(torch.rand(cfg.T, cfg.n_routed, generator=g), 1)[:, :cfg.top_k]
    idx = idx.to(torch.int32).cuda()
    counts = torch.bincount(idx.flatten().long(), minlength=cfg.n_routed).to(torch.int32)
    T, d, K, n = cfg.T, cfg.d, cfg.top_k, cfg.n_routed
    x8 = torch.empty((T * K, d), dtype=torch.uint8, device="cuda")
    xs = torch.empty((T * K, d // 128), dtype=torch.float32, device="cuda")
    u8 = torch.empty((T, d), dtype=torch.uint8, device="cuda")
    us = torch.empty((T, d // 128), dtype=torch.float32, device="cuda")
    off = torch.empty(n + 1, dtype=torch.int32, device="cuda")
    pos = torch.empty((T, K), dtype=torch.int32, device="cuda")
    src = torch.empty(T * K, dtype=torch.int32, device="cuda")
    wsb = L.moe_permute_workspace_size(T, n)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    L.moe_permute_fp8(u, idx, counts.cuda(), T, d, n, K, x8, xs, u8, us, off, pos, src, ws, wsb)
    torch.cuda.synchronize()
    want_q, want_s = of.quant_act_1x128(u.float().cpu().numpy())
    assert np.array_equal(u8.cpu().numpy(), want_q)
    assert np.array_equal(us.cpu().numpy(), want_s)
    srct = src.cpu().numpy().astype(np.int64)
    assert np.array_equal(x8.cpu().numpy(), want_q[srct])
    assert np.array_equal(xs.cpu().numpy(), want_s[srct])
    disp = om.dispatch(idx.cpu().numpy(), n)
    assert np.array_equal(pos.cpu().numpy(), disp.pos)


def test_fp8_up_projection_quantises_h_in_place():
    """moe_expert_up_swiglu_fp8 writes h as E4M3 codes + 1x128 scales decided
    from its fp32 value. Against the oracle's quantisation of the exact h of
    the same FP8 operands: scales within fp32 accumulation error, and a code
    may differ only where h sits at a rounding boundary (by one step)."""
    sizes = [1, 0, 17, 128, 129, 300]
    G, d, inter = len(sizes), 512, 256
    rows = sum(sizes)
    x = _rand_bf16((rows, d), 13)
    w1 = _rand_bf16((G, inter, d), 14, 0.05)
    w3 = _rand_bf16((G, inter, d), 15, 0.05)
    x8 = torch.empty((rows, d), dtype=torch.uint8, device="cuda")
    xs = torch.empty((rows, d // 128), dtype=torch.float32, device="cuda")
    L.moe_quant_act_fp8(x, rows, d, x8, xs)
    stacked = torch.stack([w1, w3], dim=1).contiguous()
    sq = torch.empty((G, 2, inter, d), dtype=torch.uint8, device="cuda")
    w13s = torch.empty((G, 2, inter // 128, d // 128), dtype=torch.float32, device="cuda")
    L.moe_quant_weights_fp8(stacked, 2 * G, inter, d, sq, w13s)
    w13q = torch.empty((G, 2 * inter, d), dtype=torch.uint8, device="cuda")
    L.moe_pack_w13_fp8(sq, G, inter, d, w13q)
    off = torch.tensor(np.concatenate([[0], np.cumsum(sizes)]), dtype=torch.int32, device="cuda")
    h8 = torch.full((rows + 8, inter), 0x55, dtype=torch.uint8, device="cuda")
    hs = torch.full((rows + 8, inter // 128), -1.0, dtype=torch.float32, device="cuda")
    L.moe_expert_up_swiglu_fp8(x8, xs, off, G, rows, d, inter, w13q, w13s, h8, hs)
    torch.cuda.synchronize()
    assert L.moe_get_device_status() == 0
    assert bool((h8[rows:] == 0x55).all()) and bool((hs[rows:] == -1.0).all())
    xq, xsc = x8.cpu().numpy(), xs.cpu().numpy()
    o = off.cpu().tolist()
    got_q, got_s = h8[:rows].cpu().numpy(), hs[:rows].cpu().numpy()
    n_codes = n_diff = 0
    for i in range(G):
        a, b = o[i], o[i + 1]
        if a == b:
            continue
        w1q, w1sc = of.quant_weight_128x128(w1[i].float().cpu().numpy())
        w3q, w3sc = of.quant_weight_128x128(w3[i].float().cpu().numpy())
        ga = of.fp8_gemm(xq[a:b], xsc[a:b], w1q, w1sc)
        gb = of.fp8_gemm(xq[a:b], xsc[a:b], w3q, w3sc)
        h = ga / (1.0 + np.exp(-ga)) * gb
        want_q, want_s = of.quant_act_1x128(h)
        np.testing.assert_allclose(got_s[a:b], want_s, rtol=1e-5)
        dq = got_q[a:b] != want_q
        n_codes += dq.size
        n_diff += int(dq.sum())
        if dq.any():
            # a differing code is the neighbouring E4M3 value
            gv = of.e4m3_decode(got_q[a:b][dq])
            wv = of.e4m3_decode(want_q[dq])
            assert np.all(np.abs(gv - wv) <= 0.126 * np.maximum(np.abs(wv), 2.0 ** -6))
    assert n_diff <= 1e-3 * n_codes, (n_diff, n_codes)


def test_fp8_grouped_ffn_vs_oracle_emulation():
    """Group sizes over every tile path, E4M3 operands from the library's own
    quantisers (bit-exact to the oracle's, checked above); the oracle runs the
    promoted FP8 FFN of the same codes and scales."""
    sizes = [1, 0, 17, 128, 129, 300]
    G, d, inter = len(sizes), 512, 256
    rows = sum(sizes)
    x = _rand_bf16((rows, d), 3)
    w1 = _rand_bf16((G, inter, d), 4, 0.05)
    w3 = _rand_bf16((G, inter, d), 5, 0.05)
    w2 = _rand_bf16((G, d, inter), 6, 0.05)
    x8 = torch.empty((rows, d), dtype=torch.uint8, device="cuda")
    xs = torch.empty((rows, d // 128), dtype=torch.float32, device="cuda")
    L.moe_quant_act_fp8(x, rows, d, x8, xs)
    stacked = torch.stack([w1, w3], dim=1).contiguous()            # [G, 2, inter, d]
    sq = torch.empty((G, 2, inter, d), dtype=torch.uint8, device="cuda")
    w13s = torch.empty((G, 2, inter // 128, d // 128), dtype=torch.float32, device="cuda")
    L.moe_quant_weights_fp8(stacked, 2 * G, inter, d, sq, w13s)
    w13q = torch.empty((G, 2 * inter, d), dtype=torch.uint8, device="cuda")
    L.moe_pack_w13_fp8(sq, G, inter, d, w13q)
    # 64-row interleave: rows [128c, 128c+64) of w13 are W1 rows [64c, 64c+64)
    assert torch.equal(w13q[:, 64:128], sq[:, 1, 0:64]) and torch.equal(w13q[:, 128:192], sq[:, 0, 64:128])
    w2q = torch.empty_like(w2, dtype=torch.uint8)
    w2s = torch.empty((G, d // 128, inter // 128), dtype=torch.float32, device="cuda")
    L.moe_quant_weights_fp8(w2, G, d, inter, w2q, w2s)
    off = torch.tensor(np.concatenate([[0], np.cumsum(sizes)]), dtype=torch.int32, device="cuda")
    y = torch.full((rows, d), 5.0, dtype=torch.bfloat16, device="cuda")
    wsb = L.moe_grouped_ffn_workspace_size(rows, inter, L.MOE_FP8_E4M3)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    L.moe_grouped_ffn(x8, xs, off, G, rows, d, inter, w13q, w13s, w2q, w2s, L.MOE_FP8_E4M3, y, ws,
                      wsb)
    torch.cuda.synchronize()
    assert L.moe_get_device_status() == 0
    o = off.cpu().tolist()
    xq, xsc = x8.cpu().numpy(), xs.cpu().numpy()
    for i in range(G):
        a, b = o[i], o[i + 1]
        if a == b:
            continue
        qexp = of.quant_expert(w1[i], w3[i], w2[i])
        ref = of.ffn_fp8(xq[a:b], xsc[a:b], qexp)
        check_close(f64(y[a:b]), ref, max_tol=FP8_MAX_TOL, mean_tol=FP8_MEAN_TOL,
                    what=f"FP8 group {i} ({b - a} rows)")
        exact = om.ffn(x[a:b].float().cpu().numpy(), *(t.float().cpu().numpy()
                                                       for t in (w1[i], w3[i], w2[i])))
        # against the exact FFN: four E4M3 roundings, each <= 2^-4 relative
        check_close(f64(y[a:b]), exact, max_tol=0.25, mean_tol=0.1, what="FP8 vs exact")


def _fp8_layer_check(cfg, T=None):
    inp = Inputs(cfg.replace(fp8=True), T=T)
    # rebuild the layer in FP8 mode from the same draw
    from mixture_experts_layer_58_b200.layer import MoELayer
    wdev = "cuda" if cfg.weights_on_gpu else "cpu"
    W = synth.all_expert_weights(cfg, wdev)
    lay = MoELayer(inp.e, inp.b, *W, inp.shared, top_k=cfg.top_k, routed_scale=cfg.routed_scale,
                   gate_kind=cfg.gate_kind, gamma=cfg.gamma, fp8=True)
    del W
    out = lay.forward(inp.u_dev)
    torch.cuda.synchronize()
    assert L.moe_get_device_status() == 0
    r = inp.oracle_route()
    gidx = lay.topk_idx.cpu().numpy()
    check_route(gidx, lay.topk_gate.cpu().numpy(), lay.counts.cpu().numpy(), r, cfg.routed_scale,
                inp.u, inp.e, cfg.gate_kind)
    return inp, lay, out, gidx


def test_fp8_tiny_layer_vs_oracle():
    cfg = synth.CONFIGS["tiny"]
    inp, lay, out, gidx = _fp8_layer_check(cfg)
    g = om.gates_for_indices(inp.u, inp.e, gidx, cfg.routed_scale)
    qexp = lambda i: of.quant_expert(*inp.expert(i))          # noqa: E731
    qsh = [of.quant_expert(*inp.shared_list()[0])]
    ref = of.layer_output_fp8(inp.u, gidx, g, qexp, qsh)
    check_close(f64(out), ref, max_tol=FP8_MAX_TOL, mean_tol=FP8_MEAN_TOL, what="FP8 tiny layer")


def test_fp8_mid_layer_vs_oracle():
    cfg = synth.CONFIGS["mid"]
    inp, lay, out, gidx = _fp8_layer_check(cfg)
    rng = np.random.default_rng(0)
    tokens = np.sort(rng.choice(cfg.T, size=256, replace=False))
    u_s = inp.u[torch.from_numpy(tokens)]
    g = om.gates_for_indices(u_s, inp.e, gidx[tokens], cfg.routed_scale)
    cache = {}

    def qexp(i):
        if i not in cache:
            cache[i] = of.quant_expert(*inp.expert(i))
        return cache[i]
    qsh = [of.quant_expert(*inp.shared_list()[0])]
    ref = of.layer_output_fp8(u_s, gidx[tokens], g, qexp, qsh)
    check_close(f64(out)[tokens], ref, max_tol=FP8_MAX_TOL, mean_tol=FP8_MEAN_TOL,
                what="FP8 mid layer (256 sampled tokens)")


def test_fp8_v3p_sampled_tokens():
    """The full V3 prefill shape in FP8 (the benchmark's v3p_fp8 workload):
    routing of every token, the layer output of sampled tokens against the
    oracle's FP8 emulation of the same weights."""
    cfg = synth.CONFIGS["v3p"]
    inp, lay, out, gidx = _fp8_layer_check(cfg)
    counts = lay.counts.cpu().numpy()
    hot = int(np.argmax(counts))
    t_hot = np.nonzero((gidx == hot).any(1))[0][:2]
    rng = np.random.default_rng(4)
    tokens = np.unique(np.concatenate([t_hot, rng.choice(cfg.T, size=4, replace=False)]))
    u_s = inp.u[torch.from_numpy(tokens)]
    g = om.gates_for_indices(u_s, inp.e, gidx[tokens], cfg.routed_scale)
    qexp = lambda i: of.quant_expert(*inp.expert(i))          # noqa: E731
    qsh = [of.quant_expert(*inp.shared_list()[0])]
    ref = of.layer_output_fp8(u_s, gidx[tokens], g, qexp, qsh)
    check_close(f64(out)[tokens], ref, max_tol=FP8_MAX_TOL, mean_tol=FP8_MEAN_TOL,
                what="FP8 V3 prefill (sampled tokens)")


@pytest.mark.parametrize("name", ["tiny", "mid"])
def test_fp8_shared_expert_overlapped_matches_in_line(name):
    """FP8: the shared expert on its side stream, with its own quantisation of
    u (default), and in line on the codes the dispatch wrote give the same
    layer output bit for bit: both quantise u by the same 1x128 rule."""
    cfg = synth.CONFIGS[name]
    inp, lay, out, gidx = _fp8_layer_check(cfg)
    assert lay.overlap_shared
    overlapped = out.clone()
    lay.overlap_shared = False
    out2 = lay.forward(inp.u_dev)
    torch.cuda.synchronize()
    assert L.moe_get_device_status() == 0
    assert torch.equal(out2, overlapped)
