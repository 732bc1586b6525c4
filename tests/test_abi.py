"""C-ABI library checks that need no GPU: it loads, exports every symbol the
header declares, and rejects bad arguments on the host before any launch.

Every call below fails validation before the library touches CUDA, so the
fake (never dereferenced) pointers are safe on a machine with or without a GPU.
"""
import ctypes
import os
import re

import pytest

from mixture_experts_layer_58_b200 import _lib as L

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")

A = 0x10000      # fake 16-byte aligned address (never dereferenced)
MIS = 0x10002    # fake misaligned address


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from mixture_experts_layer_58_b200 import build
    build.build()
    return L.load()


def test_header_declares_the_five_calls():
    names = declared_symbols()
    for n in ("moe_route", "moe_permute", "moe_grouped_ffn", "moe_combine", "moe_bias_update"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    raw = ctypes.CDLL(L.LIB_PATH)
    missing = [n for n in declared_symbols() if not hasattr(raw, n)]
    assert not missing, missing


def test_binding_covers_every_symbol():
    assert set(declared_symbols()) <= set(L._SIGS)


def test_version_and_strerror(lib):
    assert L.moe_version() >= 100
    for code in (0, -1, -2, -3, -4, -5):
        assert L.moe_strerror(code) and L.moe_strerror(code) != "unknown status"
    assert L.moe_strerror(-99) == "unknown status"


def test_workspace_sizes(lib):
    assert L.moe_permute_workspace_size(16384, 256) == 128 * 256 * 4
    assert L.moe_permute_workspace_size(200, 16) == 256          # 2 chunks * 16 * 4 = 128 -> 256
    assert L.moe_grouped_ffn_workspace_size(131072, 2048) == 131072 * 2048 * 2
    assert L.moe_grouped_ffn_workspace_size(0, 2048) == 256
    # one workspace for the five calls of a V3 prefill forward: the h of the
    # routed rows dominates
    assert L.moe_workspace_size(16384, 7168, 256, 8, 2048, 2048) == 131072 * 2048 * 2
    assert L.moe_workspace_size(64, 256, 16, 4, 128, 4096) == 64 * 4096 * 2


def rc_route(lib, **kw):
    a = dict(u=A, c=A, b=None, T=64, d=256, n=16, k=4, kind=0, s=1.0, idx=A, gate=A, cnt=A)
    a.update(kw)
    return lib.moe_route(a["u"], a["c"], a["b"], a["T"], a["d"], a["n"], a["k"], a["kind"],
                         a["s"], a["idx"], a["gate"], a["cnt"], None)


def test_route_rejects_bad_arguments(lib):
    assert rc_route(lib, T=-1) == L.MOE_ERR_INVALID_ARG
    assert rc_route(lib, d=0) == L.MOE_ERR_INVALID_ARG
    assert rc_route(lib, k=0) == L.MOE_ERR_INVALID_ARG
    assert rc_route(lib, kind=7) == L.MOE_ERR_INVALID_ARG
    assert rc_route(lib, u=None) == L.MOE_ERR_INVALID_ARG
    assert rc_route(lib, u=MIS) == L.MOE_ERR_INVALID_ARG
    assert rc_route(lib, c=MIS) == L.MOE_ERR_INVALID_ARG
    assert rc_route(lib, cnt=None) == L.MOE_ERR_INVALID_ARG
    assert rc_route(lib, idx=None) == L.MOE_ERR_INVALID_ARG
    assert rc_route(lib, s=float("nan")) == L.MOE_ERR_INVALID_ARG
    assert rc_route(lib, k=9, n=16) == L.MOE_ERR_UNSUPPORTED_SHAPE
    assert rc_route(lib, k=8, n=4) == L.MOE_ERR_UNSUPPORTED_SHAPE
    assert rc_route(lib, n=300) == L.MOE_ERR_UNSUPPORTED_SHAPE
    assert rc_route(lib, d=200) == L.MOE_ERR_UNSUPPORTED_SHAPE


def rc_permute(lib, **kw):
    a = dict(u=A, idx=A, cnt=A, T=64, d=256, n=16, k=4, x=A, off=A, pos=A, src=A, ws=A, wsb=4096)
    a.update(kw)
    return lib.moe_permute(a["u"], a["idx"], a["cnt"], a["T"], a["d"], a["n"], a["k"], a["x"],
                           a["off"], a["pos"], a["src"], a["ws"], a["wsb"], None)


def test_permute_rejects_bad_arguments(lib):
    assert rc_permute(lib, T=-5) == L.MOE_ERR_INVALID_ARG
    assert rc_permute(lib, off=None) == L.MOE_ERR_INVALID_ARG
    assert rc_permute(lib, x=MIS) == L.MOE_ERR_INVALID_ARG
    assert rc_permute(lib, pos=None) == L.MOE_ERR_INVALID_ARG
    assert rc_permute(lib, k=9) == L.MOE_ERR_UNSUPPORTED_SHAPE
    assert rc_permute(lib, ws=None) == L.MOE_ERR_WORKSPACE
    assert rc_permute(lib, wsb=16) == L.MOE_ERR_WORKSPACE
    assert rc_permute(lib, ws=MIS) == L.MOE_ERR_WORKSPACE


def rc_ffn(lib, **kw):
    a = dict(x=A, off=A, G=16, rows=256, d=256, inter=128, w13=A, w2=A, dt=0, y=A, ws=A,
             wsb=1 << 20)
    a.update(kw)
    return lib.moe_grouped_ffn(a["x"], None, a["off"], a["G"], a["rows"], a["d"], a["inter"],
                               a["w13"], None, a["w2"], None, a["dt"], a["y"], a["ws"], a["wsb"],
                               None)


def test_grouped_ffn_rejects_bad_arguments(lib):
    assert rc_ffn(lib, G=0) == L.MOE_ERR_INVALID_ARG
    assert rc_ffn(lib, rows=-1) == L.MOE_ERR_INVALID_ARG
    assert rc_ffn(lib, dt=5) == L.MOE_ERR_INVALID_ARG
    # FP8 without its scale tensors
    assert rc_ffn(lib, dt=L.MOE_FP8_E4M3) == L.MOE_ERR_INVALID_ARG
    assert rc_ffn(lib, inter=100) == L.MOE_ERR_UNSUPPORTED_SHAPE
    assert rc_ffn(lib, d=384) == L.MOE_ERR_UNSUPPORTED_SHAPE
    assert rc_ffn(lib, G=5000) == L.MOE_ERR_UNSUPPORTED_SHAPE
    assert rc_ffn(lib, ws=None) == L.MOE_ERR_WORKSPACE
    assert rc_ffn(lib, wsb=1024) == L.MOE_ERR_WORKSPACE
    # the halves: misaligned / null operands
    assert lib.moe_expert_up_swiglu(MIS, A, 16, 256, 256, 128, A, A, None) == L.MOE_ERR_INVALID_ARG
    assert lib.moe_expert_down(A, None, 16, 256, 128, 256, A, A, None) == L.MOE_ERR_INVALID_ARG


def test_combine_bias_pack_reject_bad_arguments(lib):
    assert lib.moe_combine(A, A, A, None, None, 4, 256, 9, A, None) == L.MOE_ERR_UNSUPPORTED_SHAPE
    assert lib.moe_combine(None, A, A, None, None, 4, 256, 4, A, None) == L.MOE_ERR_INVALID_ARG
    assert lib.moe_combine(A, A, A, MIS, None, 4, 256, 4, A, None) == L.MOE_ERR_INVALID_ARG
    assert lib.moe_combine(A, A, A, None, None, -1, 256, 4, A, None) == L.MOE_ERR_INVALID_ARG
    assert lib.moe_bias_update(None, A, 16, 64, 4, 0.001, None) == L.MOE_ERR_INVALID_ARG
    assert lib.moe_bias_update(A, A, 0, 64, 4, 0.001, None) == L.MOE_ERR_INVALID_ARG
    assert lib.moe_bias_update(A, A, 16, 64, 4, float("nan"), None) == L.MOE_ERR_INVALID_ARG
    assert lib.moe_pack_w13(A, A, 2, 100, 256, A, None) == L.MOE_ERR_UNSUPPORTED_SHAPE
    assert lib.moe_pack_w13(A, None, 2, 128, 256, A, None) == L.MOE_ERR_INVALID_ARG
    assert lib.moe_get_device_status(None, 0) == L.MOE_ERR_INVALID_ARG


def test_binding_raises_moe_error(lib):
    with pytest.raises(L.MoEError) as ei:
        L.moe_combine(A, A, A, None, None, 4, 256, 9, A, stream=0)
    assert ei.value.status == L.MOE_ERR_UNSUPPORTED_SHAPE


def test_fp8_entry_points_reject_bad_arguments(lib):
    assert lib.moe_quant_act_fp8(A, 4, 200, A, A, None) == L.MOE_ERR_UNSUPPORTED_SHAPE
    assert lib.moe_quant_act_fp8(A, -1, 256, A, A, None) == L.MOE_ERR_INVALID_ARG
    assert lib.moe_quant_act_fp8(MIS, 4, 256, A, A, None) == L.MOE_ERR_INVALID_ARG
    assert lib.moe_quant_act_fp8(A, 4, 256, A, None, None) == L.MOE_ERR_INVALID_ARG
    assert lib.moe_quant_weights_fp8(A, 2, 100, 256, A, A, None) == L.MOE_ERR_UNSUPPORTED_SHAPE
    assert lib.moe_quant_weights_fp8(A, 0, 128, 256, A, A, None) == L.MOE_ERR_INVALID_ARG
    assert lib.moe_quant_weights_fp8(A, 2, 128, 256, MIS, A, None) == L.MOE_ERR_INVALID_ARG
    # moe_permute_fp8(u, idx, counts, T, d, n, K, x8, xs, u8, us, off, pos, src, ws, wsb)
    assert lib.moe_permute_fp8(A, A, A, 64, 256, 16, 4, A, None, None, None, A, A, A, A, 4096,
                               None) == L.MOE_ERR_INVALID_ARG
    assert lib.moe_permute_fp8(A, A, A, 64, 256, 16, 4, A, A, A, None, A, A, A, A, 4096,
                               None) == L.MOE_ERR_INVALID_ARG          # u8 without u_scales
    assert lib.moe_permute_fp8(MIS, A, A, 64, 256, 16, 4, A, A, None, None, A, A, A, A, 4096,
                               None) == L.MOE_ERR_INVALID_ARG
    assert lib.moe_permute_fp8(A, A, A, 64, 256, 16, 4, A, A, None, None, A, A, A, None, 4096,
                               None) == L.MOE_ERR_WORKSPACE
    # moe_expert_up_swiglu_fp8(x8, xs, off, G, rows, d, inter, w13, w13s, h8, hs)
    assert lib.moe_expert_up_swiglu_fp8(A, None, A, 4, 256, 256, 128, A, A, A, A,
                                        None) == L.MOE_ERR_INVALID_ARG
    assert lib.moe_expert_up_swiglu_fp8(A, A, A, 4, 256, 256, 128, A, A, MIS, A,
                                        None) == L.MOE_ERR_INVALID_ARG
    assert lib.moe_expert_up_swiglu_fp8(A, A, A, 4, 256, 256, 128, A, A, A, None,
                                        None) == L.MOE_ERR_INVALID_ARG
    assert lib.moe_pack_w13_fp8(A, 2, 100, 256, A, None) == L.MOE_ERR_UNSUPPORTED_SHAPE
    assert lib.moe_pack_w13_fp8(None, 2, 128, 256, A, None) == L.MOE_ERR_INVALID_ARG
    assert lib.moe_expert_down_fp8(A, A, A, 4, 256, 128, 256, A, A, MIS,
                                   None) == L.MOE_ERR_INVALID_ARG
    assert L.moe_grouped_ffn_workspace_size(1024, 2048, L.MOE_FP8_E4M3) == \
        1024 * 2048 + 1024 * 16 * 4


def test_fused_gather_entry_points_reject_bad_arguments(lib):
    assert lib.moe_permute_index(A, A, -1, 16, 4, A, A, A, A, 4096, None) == L.MOE_ERR_INVALID_ARG
    assert lib.moe_permute_index(A, A, 64, 16, 9, A, A, A, A, 4096, None) == \
        L.MOE_ERR_UNSUPPORTED_SHAPE
    assert lib.moe_permute_index(A, A, 64, 16, 4, A, A, A, None, 4096, None) == L.MOE_ERR_WORKSPACE
    assert lib.moe_expert_up_swiglu_gather(MIS, 64, A, A, 16, 256, 256, 128, A, A, None) == \
        L.MOE_ERR_INVALID_ARG
    assert lib.moe_expert_up_swiglu_gather(A, 64, None, A, 16, 256, 256, 128, A, A, None) == \
        L.MOE_ERR_INVALID_ARG
    assert lib.moe_expert_up_swiglu_gather(A, 0, A, A, 16, 256, 256, 128, A, A, None) == \
        L.MOE_ERR_INVALID_ARG


def test_gather_rows_rejects_bad_arguments(lib):
    assert lib.moe_gather_rows(A, 10, A, -1, 256, A, None) == L.MOE_ERR_INVALID_ARG
    assert lib.moe_gather_rows(A, -1, A, 4, 256, A, None) == L.MOE_ERR_INVALID_ARG
    assert lib.moe_gather_rows(A, 10, A, 4, 0, A, None) == L.MOE_ERR_INVALID_ARG
    assert lib.moe_gather_rows(A, 10, A, 4, 12, A, None) == L.MOE_ERR_UNSUPPORTED_SHAPE
    assert lib.moe_gather_rows(MIS, 10, A, 4, 256, A, None) == L.MOE_ERR_INVALID_ARG
    assert lib.moe_gather_rows(A, 10, A, 4, 256, MIS, None) == L.MOE_ERR_INVALID_ARG
    assert lib.moe_gather_rows(A, 10, None, 4, 256, A, None) == L.MOE_ERR_INVALID_ARG
    assert lib.moe_gather_rows(A, 10, A, 0, 256, A, None) == L.MOE_OK     # nothing to do


def test_selftest_rejects_bad_limit(lib):
    assert lib.moe_selftest_wait_timeout(0, None) == L.MOE_ERR_INVALID_ARG
    assert lib.moe_selftest_wait_timeout(20000, None) == L.MOE_ERR_INVALID_ARG


def test_backward_entry_points_reject_bad_arguments(lib):
    E = L.MOE_ERR_INVALID_ARG
    U = L.MOE_ERR_UNSUPPORTED_SHAPE
    # training forward: ac is required and aligned
    assert lib.moe_expert_up_swiglu_train(A, A, 4, 256, 256, 128, A, A, None, None) == E
    assert lib.moe_expert_up_swiglu_train(A, A, 4, 256, 256, 128, A, A, MIS, None) == E
    assert lib.moe_expert_up_swiglu_train(A, A, 4, 256, 256, 100, A, A, A, None) == U
    # combine backward
    assert lib.moe_combine_backward(A, A, A, A, -1, 256, 4, A, A, None) == E
    assert lib.moe_combine_backward(A, A, A, A, 64, 256, 9, A, A, None) == U
    assert lib.moe_combine_backward(A, A, A, A, 64, 256, 4, MIS, A, None) == E
    assert lib.moe_combine_backward(A, A, A, A, 64, 256, 4, A, None, None) == E
    # expert dgrad
    assert lib.moe_expert_down_backward(A, None, A, 4, 256, 256, 128, A, A, None) == E
    assert lib.moe_expert_down_backward(A, A, A, 4, 256, 200, 128, A, A, None) == U
    assert lib.moe_expert_up_backward(A, A, 4, 256, 256, 128, A, MIS, None) == E
    assert lib.moe_expert_up_backward(A, A, 0, 256, 256, 128, A, A, None) == E
    # expert wgrad
    assert lib.moe_expert_wgrad(A, A, A, 4, 256, 100, 256, A, None) == U
    assert lib.moe_expert_wgrad(A, A, A, 4, 256, 128, 200, A, None) == U
    assert lib.moe_expert_wgrad(A, None, A, 4, 256, 128, 256, A, None) == E
    assert lib.moe_expert_wgrad(A, A, None, 4, 256, 128, 256, A, None) == E
    # gate backward
    assert lib.moe_gate_backward(A, A, A, A, A, A, 64, 256, 16, 4, 2, ctypes.c_float(1.0), A, A,
                                 None) == E
    assert lib.moe_gate_backward(A, A, A, A, A, A, 64, 256, 16, 17, 0, ctypes.c_float(1.0), A, A,
                                 None) == U
    assert lib.moe_gate_backward(A, A, A, A, A, A, 64, 256, 16, 4, 0, ctypes.c_float(0.0), A, A,
                                 None) == E
    assert lib.moe_gate_backward(A, A, A, A, None, A, 64, 256, 16, 4, 0, ctypes.c_float(1.0), A,
                                 A, None) == E
    # du combine, centroid gradient
    assert lib.moe_combine_dx(A, A, A, A, A, A, A, 64, 256, 9, A, None) == U
    assert lib.moe_combine_dx(MIS, A, A, A, A, A, A, 64, 256, 4, A, None) == E
    assert lib.moe_combine_dx(A, A, A, A, None, A, A, 64, 256, 4, A, None) == E
    assert lib.moe_centroid_grad(A, A, A, 16, 256, 250, A, A, 1 << 20, None) == U
    assert lib.moe_centroid_grad(A, None, A, 16, 256, 256, A, A, 1 << 20, None) == E
    assert lib.moe_centroid_grad(A, A, A, 1024, 256, 256, A, A, 1 << 30, None) == U
    assert lib.moe_centroid_grad(A, A, A, 16, 256, 256, A, None, 1 << 20, None) == \
        L.MOE_ERR_WORKSPACE
    assert lib.moe_centroid_grad(A, A, A, 16, 256, 256, A, A, 16, None) == L.MOE_ERR_WORKSPACE
    # chunk starts (17 ints -> 80 B), row ranges (2 + 16 chunks -> 144 B), fp32 partials
    assert L.moe_centroid_grad_workspace_size(256, 16, 256) == 80 + 144 + 18 * 256 * 4


def test_header_is_c99_and_the_library_links_from_c(lib, tmp_path):
    """A plain C program includes moe.h, links libmoe.so and calls the entry
    points that need no GPU (tests/c_abi_check.c)."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    exe = tmp_path / "c_abi_check"
    pkg = os.path.dirname(L.LIB_PATH)
    subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c_abi_check.c"), "-o", str(exe),
                    "-L", pkg, "-l:libmoe.so", "-Wl,-rpath," + pkg], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, out.stderr
    assert out.stdout.strip() == "ok"



def test_fused_scatter_entry_points_reject_bad_arguments(lib):
    # moe_slot_index(pos, T, top_k, rows, dst_slot)
    assert lib.moe_slot_index(A, -1, 4, 8, A, None) == L.MOE_ERR_INVALID_ARG
    assert lib.moe_slot_index(A, 2, 9, 8, A, None) == L.MOE_ERR_UNSUPPORTED_SHAPE
    assert lib.moe_slot_index(A, 2, 4, 8, None, None) == L.MOE_ERR_INVALID_ARG
    assert lib.moe_slot_index(None, 2, 4, 8, A, None) == L.MOE_ERR_INVALID_ARG
    # moe_expert_down_scatter(h, off, G, rows, inter, d, w2, slot, gate, T, K, y)
    ok = dict(h=A, off=A, G=4, rows=64, inter=128, d=256, w2=A, slot=A, gate=A, T=16, K=4, y=A)

    def ds(**kw):
        a = dict(ok)
        a.update(kw)
        return lib.moe_expert_down_scatter(a["h"], a["off"], a["G"], a["rows"], a["inter"],
                                           a["d"], a["w2"], a["slot"], a["gate"], a["T"],
                                           a["K"], a["y"], None)
    assert ds(d=100) == L.MOE_ERR_UNSUPPORTED_SHAPE
    assert ds(T=-1) == L.MOE_ERR_INVALID_ARG
    assert ds(slot=None) == L.MOE_ERR_INVALID_ARG
    assert ds(gate=None) == L.MOE_ERR_INVALID_ARG
    assert ds(y=MIS) == L.MOE_ERR_INVALID_ARG
    # moe_combine_slots(y, pos, shared, residual, T, d, K, out)
    assert lib.moe_combine_slots(A, A, None, None, 4, 256, 9, A, None) == \
        L.MOE_ERR_UNSUPPORTED_SHAPE
    assert lib.moe_combine_slots(MIS, A, None, None, 4, 256, 4, A, None) == L.MOE_ERR_INVALID_ARG
    assert lib.moe_combine_slots(A, None, None, None, 4, 256, 4, A, None) == L.MOE_ERR_INVALID_ARG
    assert lib.moe_combine_slots(A, A, MIS, None, 4, 256, 4, A, None) == L.MOE_ERR_INVALID_ARG


def test_peer_memory_ep_entry_points_reject_bad_arguments(lib):
    # moe_ep_plan_device(all_counts, world, n_local, rank, cap, dest, goff, gcounts)
    assert lib.moe_ep_plan_device(A, 0, 8, 0, 10, None, A, A, A, None) == L.MOE_ERR_INVALID_ARG
    assert lib.moe_ep_plan_device(A, 2, 8, 2, 10, None, A, A, A, None) == L.MOE_ERR_INVALID_ARG
    assert lib.moe_ep_plan_device(A, 2, 8, 0, -1, None, A, A, A, None) == L.MOE_ERR_INVALID_ARG
    assert lib.moe_ep_plan_device(A, 4, 65, 0, 10, None, A, A, A, None) == \
        L.MOE_ERR_UNSUPPORTED_SHAPE
    assert lib.moe_ep_plan_device(A, 2, 8, 0, 10, None, None, A, A, None) == L.MOE_ERR_INVALID_ARG
    # moe_ep_dispatch_p2p(u, idx, pos, off, dest, T, d, n_routed, K, world, peer_x, cap)
    assert lib.moe_ep_dispatch_p2p(A, A, A, A, A, 4, 256, 16, 4, 3, A, 10, None) == \
        L.MOE_ERR_UNSUPPORTED_SHAPE                                  # 16 experts over 3 ranks
    assert lib.moe_ep_dispatch_p2p(MIS, A, A, A, A, 4, 256, 16, 4, 2, A, 10, None) == \
        L.MOE_ERR_INVALID_ARG
    assert lib.moe_ep_dispatch_p2p(A, A, A, A, A, 4, 256, 16, 4, 2, None, 10, None) == \
        L.MOE_ERR_INVALID_ARG
    # moe_ep_combine_p2p(peer_y, idx, pos, off, dest, gate, shared, res, T, d, n, K, W, cap, out)
    assert lib.moe_ep_combine_p2p(A, A, A, A, A, A, None, None, 4, 256, 16, 9, 2, 10, A,
                                  None) == L.MOE_ERR_UNSUPPORTED_SHAPE
    assert lib.moe_ep_combine_p2p(A, A, A, A, A, None, None, None, 4, 256, 16, 4, 2, 10, A,
                                  None) == L.MOE_ERR_INVALID_ARG
    assert lib.moe_ep_combine_p2p(A, A, A, A, A, A, None, None, 4, 256, 16, 4, 2, 10, MIS,
                                  None) == L.MOE_ERR_INVALID_ARG
    # IPC helpers: null arguments
    assert lib.moe_ipc_get_handle(None, A, None) == L.MOE_ERR_INVALID_ARG
    assert lib.moe_ipc_open_handle(None, None) == L.MOE_ERR_INVALID_ARG
    assert lib.moe_ipc_close_handle(None) == L.MOE_ERR_INVALID_ARG


def test_fused_combine_entry_point_rejects_bad_arguments(lib):
    # moe_expert_down_scatter_combine(h, off, G, rows, inter, d, w2, slot, gate, T, K, y,
    #                                 shared, residual, out, ws, ws_bytes)
    need = L.moe_expert_down_scatter_combine_workspace_size(16, 256)
    assert need == 256 and L.moe_expert_down_scatter_combine_workspace_size(16384, 7168) == \
        16384 * 56 * 4
    ok = dict(h=A, off=A, G=4, rows=64, inter=128, d=256, w2=A, slot=A, gate=A, T=16, K=4, y=A,
              sh=None, res=None, out=A, ws=A, wsb=need)

    def dsc(**kw):
        a = dict(ok)
        a.update(kw)
        return lib.moe_expert_down_scatter_combine(
            a["h"], a["off"], a["G"], a["rows"], a["inter"], a["d"], a["w2"], a["slot"],
            a["gate"], a["T"], a["K"], a["y"], a["sh"], a["res"], a["out"], a["ws"], a["wsb"],
            None)
    assert dsc(d=100) == L.MOE_ERR_UNSUPPORTED_SHAPE
    assert dsc(K=9) == L.MOE_ERR_UNSUPPORTED_SHAPE
    assert dsc(T=-1) == L.MOE_ERR_INVALID_ARG
    assert dsc(out=None) == L.MOE_ERR_INVALID_ARG
    assert dsc(out=MIS) == L.MOE_ERR_INVALID_ARG
    assert dsc(sh=MIS) == L.MOE_ERR_INVALID_ARG
    assert dsc(res=MIS) == L.MOE_ERR_INVALID_ARG
    assert dsc(ws=None) == L.MOE_ERR_WORKSPACE
    assert dsc(wsb=need - 1) == L.MOE_ERR_WORKSPACE
    assert dsc(ws=MIS) == L.MOE_ERR_WORKSPACE


def test_split_route_entry_point_rejects_bad_arguments(lib):
    need = L.moe_route_splitk_workspace_size(128, 7168, 256)
    # 28 slices of K (4 K blocks of 64 each) x 128 tokens x 256 experts, fp32
    assert need == 28 * 128 * 256 * 4
    assert L.moe_route_splitk_workspace_size(16384, 7168, 256) == 16384 * 256 * 4   # one slice

    def rs(**kw):
        a = dict(u=A, c=A, b=None, T=64, d=256, n=16, k=4, kind=0, s=1.0, idx=A, gate=A, cnt=A,
                 ws=A, wsb=L.moe_route_splitk_workspace_size(64, 256, 16))
        a.update(kw)
        return lib.moe_route_splitk(a["u"], a["c"], a["b"], a["T"], a["d"], a["n"], a["k"],
                                    a["kind"], a["s"], a["idx"], a["gate"], a["cnt"], a["ws"],
                                    a["wsb"], None)
    assert rs(T=-1) == L.MOE_ERR_INVALID_ARG
    assert rs(kind=7) == L.MOE_ERR_INVALID_ARG
    assert rs(u=MIS) == L.MOE_ERR_INVALID_ARG
    assert rs(d=200) == L.MOE_ERR_UNSUPPORTED_SHAPE
    assert rs(n=300) == L.MOE_ERR_UNSUPPORTED_SHAPE
    assert rs(k=9) == L.MOE_ERR_UNSUPPORTED_SHAPE
    assert rs(ws=None) == L.MOE_ERR_WORKSPACE
    assert rs(wsb=16) == L.MOE_ERR_WORKSPACE
    assert rs(ws=MIS) == L.MOE_ERR_WORKSPACE


def test_permute_shared_rejects_bad_arguments(lib):
    def ps(**kw):
        a = dict(u=A, idx=A, cnt=A, T=64, d=256, n=16, k=4, x=A, off=A, pos=A, src=A, ws=A,
                 wsb=L.moe_permute_workspace_size(64, 16))
        a.update(kw)
        return lib.moe_permute_shared(a["u"], a["idx"], a["cnt"], a["T"], a["d"], a["n"], a["k"],
                                      a["x"], a["off"], a["pos"], a["src"], a["ws"], a["wsb"],
                                      None)
    assert ps(T=-1) == L.MOE_ERR_INVALID_ARG
    assert ps(off=None) == L.MOE_ERR_INVALID_ARG
    assert ps(d=100) == L.MOE_ERR_UNSUPPORTED_SHAPE
    assert ps(k=9) == L.MOE_ERR_UNSUPPORTED_SHAPE
    assert ps(x=MIS) == L.MOE_ERR_INVALID_ARG
    assert ps(ws=None) == L.MOE_ERR_WORKSPACE
