"""Grouped calls given malformed device offsets: negative, decreasing and
past-the-end entries. Every kernel clamps the array into [0, rows] and raises
each entry to the largest one before it, so the groups it runs are disjoint,
in order and inside the operands. The outputs must equal fp32 torch products
over those effective groups, and guard rows around every output (and bytes
past the workspace) must stay untouched. Needs a B200."""
import numpy as np
import pytest
import torch

from mixture_experts_layer_58_b200 import _lib as L
from oracle import fp8 as of

from gpu_support import check_close

pytestmark = pytest.mark.gpu

GUARD = 64          # guard rows on each side of an output
SENTINEL = 3.0


@pytest.fixture(scope="module", autouse=True)
def _built(cuda_ok):
    from mixture_experts_layer_58_b200 import build
    build.build()
    L.load()


def effective(off, rows):
    """The groups a kernel runs for the device array `off`: each entry
    clamped into [0, rows], then the running maximum."""
    o = np.clip(np.asarray(off, dtype=np.int64), 0, rows)
    return np.maximum.accumulate(o)


def guarded(rows, cols, dtype=torch.bfloat16):
    """(whole buffer filled with SENTINEL, view of its `rows` middle rows)."""
    big = torch.full((rows + 2 * GUARD, cols), SENTINEL, dtype=dtype, device="cuda")
    return big, big[GUARD:GUARD + rows]


def assert_guards(big, rows, what):
    assert bool((big[:GUARD] == SENTINEL).all()), f"{what}: write before the output"
    assert bool((big[GUARD + rows:] == SENTINEL).all()), f"{what}: write after the output"


def rand(shape, g, scale=1.0):
    return (scale * torch.randn(shape, generator=g, device="cuda")).bfloat16()


# (rows, device offsets): 300 rows over 5 groups -> single-CTA tiles;
# 1024 rows over 3 groups (>= 256 rows per group on average) -> CTA-pair tiles
CASES = [
    (300, [-77, 130, 60, 250, 2 ** 31 - 1, -5]),
    (1024, [-1000, 700, 300, 5000]),
]


@pytest.mark.parametrize("rows,off", CASES)
@pytest.mark.parametrize("dtype", ["bf16", "fp8"])
def test_grouped_ffn_with_malformed_offsets(rows, off, dtype):
    G, d, inter = len(off) - 1, 256, 256
    g = torch.Generator(device="cuda").manual_seed(31)
    x = rand((rows, d), g)
    w1, w3 = rand((G, inter, d), g, 0.05), rand((G, inter, d), g, 0.05)
    w2 = rand((G, d, inter), g, 0.05)
    off_dev = torch.tensor(off, dtype=torch.int32, device="cuda")
    ybig, y = guarded(rows, d)
    dt = L.MOE_FP8_E4M3 if dtype == "fp8" else L.MOE_BF16
    wsb = L.moe_grouped_ffn_workspace_size(rows, inter, dt)
    ws = torch.full((wsb + 4096,), 0xAB, dtype=torch.uint8, device="cuda")
    if dtype == "bf16":
        w13 = torch.empty(G, 2 * inter, d, dtype=torch.bfloat16, device="cuda")
        L.moe_pack_w13(w1, w3, G, inter, d, w13)
        L.moe_grouped_ffn(x, None, off_dev, G, rows, d, inter, w13, None, w2, None, dt, y, ws, wsb)
    else:
        x8 = torch.empty((rows, d), dtype=torch.uint8, device="cuda")
        xs = torch.empty((rows, d // 128), dtype=torch.float32, device="cuda")
        L.moe_quant_act_fp8(x, rows, d, x8, xs)
        stacked = torch.stack([w1, w3], dim=1).contiguous()
        sq = torch.empty((G, 2, inter, d), dtype=torch.uint8, device="cuda")
        w13s = torch.empty((G, 2, inter // 128, d // 128), dtype=torch.float32, device="cuda")
        L.moe_quant_weights_fp8(stacked, 2 * G, inter, d, sq, w13s)
        w13 = torch.empty((G, 2 * inter, d), dtype=torch.uint8, device="cuda")
        L.moe_pack_w13_fp8(sq, G, inter, d, w13)
        w2q = torch.empty((G, d, inter), dtype=torch.uint8, device="cuda")
        w2s = torch.empty((G, d // 128, inter // 128), dtype=torch.float32, device="cuda")
        L.moe_quant_weights_fp8(w2, G, d, inter, w2q, w2s)
        L.moe_grouped_ffn(x8, xs, off_dev, G, rows, d, inter, w13, w13s, w2q, w2s, dt, y, ws, wsb)
    torch.cuda.synchronize()
    assert L.moe_get_device_status() == 0
    assert_guards(ybig, rows, "y")
    assert bool((ws[wsb:] == 0xAB).all()), "write past the workspace"
    eff = effective(off, rows).tolist()
    for i in range(G):
        a, b = eff[i], eff[i + 1]
        if a == b:
            continue
        if dtype == "bf16":
            xa = x[a:b].float()
            h = torch.nn.functional.silu(xa @ w1[i].float().T) * (xa @ w3[i].float().T)
            ref = (h.bfloat16().float() @ w2[i].float().T).cpu().numpy()
            tol = (1e-2, 3e-3)
        else:
            # the oracle's FP8 emulation of the same group (its quantisers
            # give the kernels' codes bit for bit)
            xq, xs_ = of.quant_act_1x128(x[a:b].float().cpu().numpy())
            qe = of.quant_expert(w1[i].float().cpu(), w3[i].float().cpu(), w2[i].float().cpu())
            ref = of.ffn_fp8(xq, xs_, qe)
            tol = (3e-2, 1e-2)
        check_close(y[a:b].float().cpu().numpy(), ref, max_tol=tol[0], mean_tol=tol[1],
                    what=f"{dtype} group {i} rows [{a}, {b})")


@pytest.mark.parametrize("rows,off", CASES[:1])
def test_backward_gemms_with_malformed_offsets(rows, off):
    """Expert dgrad (down with the SwiGLU backward, up), the grouped weight
    gradient and the centroid gradient on the same malformed offsets."""
    G, d, inter = len(off) - 1, 256, 256
    g = torch.Generator(device="cuda").manual_seed(32)
    off_dev = torch.tensor(off, dtype=torch.int32, device="cuda")
    eff = effective(off, rows).tolist()
    dy = rand((rows, d), g)
    ac = rand((rows, 2 * inter), g)
    w2 = rand((G, d, inter), g, 0.05)
    w13 = rand((G, 2 * inter, d), g, 0.05)
    dacbig, dac = guarded(rows, 2 * inter)
    L.moe_expert_down_backward(dy, ac, off_dev, G, rows, d, inter, w2, dac)
    dxbig, dx = guarded(rows, d)
    dac_in = rand((rows, 2 * inter), g)
    L.moe_expert_up_backward(dac_in, off_dev, G, rows, d, inter, w13, dx)
    m, n = d, inter
    a_in, b_in = rand((rows, m), g), rand((rows, n), g)
    dw = torch.full((G + 1, m, n), SENTINEL, dtype=torch.bfloat16, device="cuda")
    L.moe_expert_wgrad(a_in, b_in, off_dev, G, rows, m, n, dw[:G])
    xp = rand((rows, d), g)
    dz = torch.randn(rows, generator=g, device="cuda")
    de = torch.full((G + 1, d), SENTINEL, dtype=torch.bfloat16, device="cuda")
    cws = L.moe_centroid_grad_workspace_size(rows, G, d)
    cg_ws = torch.empty(cws, dtype=torch.uint8, device="cuda")
    L.moe_centroid_grad(xp, dz, off_dev, G, rows, d, de[:G], cg_ws, cws)
    torch.cuda.synchronize()
    assert L.moe_get_device_status() == 0
    assert_guards(dacbig, rows, "dac")
    assert_guards(dxbig, rows, "dx")
    assert bool((dw[G] == SENTINEL).all()), "write past dw"
    assert bool((de[G] == SENTINEL).all()), "write past de"
    for i in range(G):
        a, b = eff[i], eff[i + 1]
        ref_dw = a_in[a:b].float().T @ b_in[a:b].float()
        ref_de = (dz[a:b, None] * xp[a:b].float()).sum(0)
        if a == b:
            assert bool((dw[i] == 0).all()) and bool((de[i] == 0).all())
            continue
        check_close(dw[i].float().cpu().numpy(), ref_dw.cpu().numpy(), max_tol=1e-2,
                    mean_tol=3e-3, what=f"dw group {i}")
        check_close(de[i].float().cpu().numpy(), ref_de.cpu().numpy(), max_tol=1e-2,
                    mean_tol=3e-3, what=f"de group {i}")
        ref_dx = dac_in[a:b].float() @ w13[i].float()
        check_close(dx[a:b].float().cpu().numpy(), ref_dx.cpu().numpy(), max_tol=1e-2,
                    mean_tol=3e-3, what=f"dx group {i}")
