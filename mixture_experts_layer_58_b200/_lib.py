"""ctypes binding of libmoe.so: the C-ABI entry points under the same names.

Argument marshalling only: tensors become device pointers (data_ptr()),
None becomes NULL, the stream defaults to torch's current CUDA stream. Every
non-zero status raises MoEError. There is no fallback: if the library is
missing, loading it raises.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = -1
MOE_ERR_UNSUPPORTED_SHAPE = -2
MOE_ERR_CUDA = -3
MOE_ERR_DEVICE_TIMEOUT = -4
MOE_ERR_WORKSPACE = -5

MOE_GATE_SIGMOID_BIAS = 0
MOE_GATE_SOFTMAX_TOPK = 1
MOE_BF16 = 0
MOE_FP8_E4M3 = 1

GATE_KINDS = {"sigmoid": MOE_GATE_SIGMOID_BIAS, "softmax": MOE_GATE_SOFTMAX_TOPK}


class MoEError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = f"{where}: status {status}"
        try:
            msg += f" ({_L().moe_strerror(status).decode()})"
            if status == MOE_ERR_CUDA:
                msg += f", cuda error {_L().moe_last_cuda_error()}"
        except Exception:  # noqa: BLE001 - the message is best effort
            pass
        super().__init__(msg)


_vp, _i, _ll, _f, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong, ctypes.c_float, ctypes.c_size_t

_SIGS = {
    "moe_route": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _i, _f, _vp, _vp, _vp, _vp]),
    "moe_route_splitk": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _i, _f, _vp, _vp, _vp, _vp, _sz,
                              _vp]),
    "moe_route_splitk_workspace_size": (_sz, [_i, _i, _i]),
    "moe_permute": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "moe_permute_workspace_size": (_sz, [_i, _i]),
    "moe_permute_shared": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "moe_permute_noalloc": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp]),
    "moe_permute_index": (_i, [_vp, _vp, _i, _i, _i, _vp, _vp, _vp, _vp, _sz, _vp]),
    "moe_expert_up_swiglu_gather": (_i, [_vp, _i, _vp, _vp, _i, _i, _i, _i, _vp, _vp, _vp]),
    "moe_grouped_ffn": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _i, _vp, _vp,
                             _sz, _vp]),
    "moe_grouped_ffn_workspace_size": (_sz, [_i, _i, _i]),
    "moe_workspace_size": (_sz, [_i, _i, _i, _i, _i, _i, _i]),
    "moe_expert_up_swiglu": (_i, [_vp, _vp, _i, _i, _i, _i, _vp, _vp, _vp]),
    "moe_expert_down": (_i, [_vp, _vp, _i, _i, _i, _i, _vp, _vp, _vp]),
    "moe_quant_act_fp8": (_i, [_vp, _i, _i, _vp, _vp, _vp]),
    "moe_quant_weights_fp8": (_i, [_vp, _i, _i, _i, _vp, _vp, _vp]),
    "moe_permute_fp8": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                             _vp, _sz, _vp]),
    "moe_expert_up_swiglu_fp8": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp]),
    "moe_pack_w13_fp8": (_i, [_vp, _i, _i, _i, _vp, _vp]),
    "moe_expert_down_fp8": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _vp, _vp, _vp, _vp]),
    "moe_combine": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _vp, _vp]),
    "moe_bias_update": (_i, [_vp, _vp, _i, _ll, _i, _f, _vp]),
    "moe_slot_index": (_i, [_vp, _i, _i, _i, _vp, _vp]),
    "moe_expert_down_scatter": (_i, [_vp, _vp, _i, _i, _i, _i, _vp, _vp, _vp, _i, _i, _vp,
                                     _vp]),
    "moe_combine_slots": (_i, [_vp, _vp, _vp, _vp, _i, _i, _i, _vp, _vp]),
    "moe_expert_down_scatter_combine": (_i, [_vp, _vp, _i, _i, _i, _i, _vp, _vp, _vp, _i, _i,
                                             _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "moe_expert_down_scatter_combine_workspace_size": (_sz, [_i, _i]),
    "moe_pack_w13": (_i, [_vp, _vp, _i, _i, _i, _vp, _vp]),
    "moe_strerror": (ctypes.c_char_p, [_i]),
    "moe_last_cuda_error": (_i, []),
    "moe_get_device_status": (_i, [ctypes.POINTER(ctypes.c_uint), _i]),
    "moe_version": (_i, []),
    "moe_selftest_wait_timeout": (_i, [_i, _vp]),
    "moe_expert_up_swiglu_train": (_i, [_vp, _vp, _i, _i, _i, _i, _vp, _vp, _vp, _vp]),
    "moe_combine_backward": (_i, [_vp, _vp, _vp, _vp, _i, _i, _i, _vp, _vp, _vp]),
    "moe_expert_down_backward": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _vp, _vp, _vp]),
    "moe_expert_up_backward": (_i, [_vp, _vp, _i, _i, _i, _i, _vp, _vp, _vp]),
    "moe_expert_wgrad": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _vp, _vp]),
    "moe_gate_backward": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _f, _vp, _vp,
                               _vp]),
    "moe_combine_dx": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _vp, _vp]),
    "moe_centroid_grad": (_i, [_vp, _vp, _vp, _i, _i, _i, _vp, _vp, _sz, _vp]),
    "moe_centroid_grad_workspace_size": (_sz, [_i, _i, _i]),
    "moe_ep_plan": (_i, [_vp, _vp, _i, _i, _ll, _vp, _vp, _vp, _vp, _vp,
                         ctypes.POINTER(ctypes.c_longlong)]),
    "moe_gather_rows": (_i, [_vp, _i, _vp, _i, _i, _vp, _vp]),
    "moe_ep_plan_device": (_i, [_vp, _i, _i, _i, _ll, _vp, _vp, _vp, _vp, _vp]),
    "moe_ep_dispatch_p2p": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp, _ll, _vp]),
    "moe_ep_combine_p2p": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i,
                                _ll, _vp, _vp]),
    "moe_ipc_get_handle": (_i, [_vp, _vp, ctypes.POINTER(ctypes.c_longlong)]),
    "moe_ipc_open_handle": (_i, [_vp, ctypes.POINTER(ctypes.c_void_p)]),
    "moe_ipc_close_handle": (_i, [_vp]),
}

_LIB = None


def _L():
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is not built: run "
                              "`python -m mixture_experts_layer_58_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = lib
    return _LIB


def load():
    """Load libmoe.so (raises if absent) and return the ctypes handle."""
    return _L()


def _p(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(s):
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(rc: int, where: str) -> None:
    if rc != MOE_OK:
        raise MoEError(rc, where)


def moe_route(u, centroids, bias, T, d, n_routed, top_k, kind, routed_scale, topk_idx,
              topk_gate, expert_counts, stream=None):
    k = GATE_KINDS.get(kind, kind)
    _check(_L().moe_route(_p(u), _p(centroids), _p(bias), T, d, n_routed, top_k, k,
                          float(routed_scale), _p(topk_idx), _p(topk_gate), _p(expert_counts),
                          _stream(stream)), "moe_route")


def moe_route_splitk_workspace_size(T, d, n_routed):
    return _L().moe_route_splitk_workspace_size(T, d, n_routed)


def moe_route_splitk(u, centroids, bias, T, d, n_routed, top_k, kind, routed_scale, topk_idx,
                     topk_gate, expert_counts, workspace, ws_bytes, stream=None):
    k = GATE_KINDS.get(kind, kind)
    _check(_L().moe_route_splitk(_p(u), _p(centroids), _p(bias), T, d, n_routed, top_k, k,
                                 float(routed_scale), _p(topk_idx), _p(topk_gate),
                                 _p(expert_counts), _p(workspace), ws_bytes, _stream(stream)),
           "moe_route_splitk")


def moe_permute(u, topk_idx, expert_counts, T, d, n_routed, top_k, x_perm, expert_offsets, pos,
                src_token, workspace, ws_bytes, stream=None):
    _check(_L().moe_permute(_p(u), _p(topk_idx), _p(expert_counts), T, d, n_routed, top_k,
                            _p(x_perm), _p(expert_offsets), _p(pos), _p(src_token),
                            _p(workspace), ws_bytes, _stream(stream)), "moe_permute")


def moe_permute_shared(u, topk_idx, expert_counts, T, d, n_routed, top_k, x_perm, expert_offsets,
                       pos, src_token, workspace, ws_bytes, stream=None):
    _check(_L().moe_permute_shared(_p(u), _p(topk_idx), _p(expert_counts), T, d, n_routed, top_k,
                                   _p(x_perm), _p(expert_offsets), _p(pos), _p(src_token),
                                   _p(workspace), ws_bytes, _stream(stream)), "moe_permute_shared")


def moe_permute_noalloc(u, topk_idx, expert_counts, T, d, n_routed, top_k, x_perm,
                        expert_offsets, pos, src_token, stream=None):
    """moe_permute for callers that cannot allocate device memory: no workspace
    argument; the library's own 256 KiB device array serves as scratch (shared
    by every call on the device, so calls must not overlap on the GPU)."""
    _check(_L().moe_permute_noalloc(_p(u), _p(topk_idx), _p(expert_counts), T, d, n_routed,
                                    top_k, _p(x_perm), _p(expert_offsets), _p(pos),
                                    _p(src_token), _stream(stream)), "moe_permute_noalloc")


def moe_permute_index(topk_idx, expert_counts, T, n_routed, top_k, expert_offsets, pos, src_token,
                      workspace, ws_bytes, stream=None):
    _check(_L().moe_permute_index(_p(topk_idx), _p(expert_counts), T, n_routed, top_k,
                                  _p(expert_offsets), _p(pos), _p(src_token), _p(workspace),
                                  ws_bytes, _stream(stream)), "moe_permute_index")


def moe_expert_up_swiglu_gather(u, T, src_token, group_offsets, G, rows, d, inter, w13, h,
                                stream=None):
    _check(_L().moe_expert_up_swiglu_gather(_p(u), T, _p(src_token), _p(group_offsets), G, rows, d,
                                            inter, _p(w13), _p(h), _stream(stream)),
           "moe_expert_up_swiglu_gather")


def moe_permute_workspace_size(T, n_routed) -> int:
    return _L().moe_permute_workspace_size(T, n_routed)


def moe_grouped_ffn(x, x_scales, group_offsets, G, rows, d, inter, w13, w13_scales, w2,
                    w2_scales, dtype, y, workspace, ws_bytes, stream=None):
    _check(_L().moe_grouped_ffn(_p(x), _p(x_scales), _p(group_offsets), G, rows, d, inter,
                                _p(w13), _p(w13_scales), _p(w2), _p(w2_scales), dtype, _p(y),
                                _p(workspace), ws_bytes, _stream(stream)), "moe_grouped_ffn")


def moe_workspace_size(T, d, n_routed, top_k, inter, shared_inter=0, dtype=MOE_BF16) -> int:
    return int(_L().moe_workspace_size(T, d, n_routed, top_k, inter, shared_inter, dtype))


def moe_grouped_ffn_workspace_size(rows, inter, dtype=MOE_BF16) -> int:
    return _L().moe_grouped_ffn_workspace_size(rows, inter, dtype)


def moe_expert_up_swiglu(x, group_offsets, G, rows, d, inter, w13, h, stream=None):
    _check(_L().moe_expert_up_swiglu(_p(x), _p(group_offsets), G, rows, d, inter, _p(w13), _p(h),
                                     _stream(stream)), "moe_expert_up_swiglu")


def moe_expert_down(h, group_offsets, G, rows, inter, d, w2, y, stream=None):
    _check(_L().moe_expert_down(_p(h), _p(group_offsets), G, rows, inter, d, _p(w2), _p(y),
                                _stream(stream)), "moe_expert_down")


def moe_quant_act_fp8(x, rows, cols, q, scales, stream=None):
    _check(_L().moe_quant_act_fp8(_p(x), rows, cols, _p(q), _p(scales), _stream(stream)),
           "moe_quant_act_fp8")


def moe_quant_weights_fp8(w, G, R, C, q, scales, stream=None):
    _check(_L().moe_quant_weights_fp8(_p(w), G, R, C, _p(q), _p(scales), _stream(stream)),
           "moe_quant_weights_fp8")


def moe_permute_fp8(u, topk_idx, expert_counts, T, d, n_routed, top_k, x8, x_scales, u8,
                    u_scales, expert_offsets, pos, src_token, workspace, ws_bytes, stream=None):
    _check(_L().moe_permute_fp8(_p(u), _p(topk_idx), _p(expert_counts), T, d, n_routed, top_k,
                                _p(x8), _p(x_scales), _p(u8), _p(u_scales), _p(expert_offsets),
                                _p(pos), _p(src_token), _p(workspace), ws_bytes, _stream(stream)),
           "moe_permute_fp8")


def moe_expert_up_swiglu_fp8(x8, x_scales, group_offsets, G, rows, d, inter, w13, w13_scales, h8,
                             h_scales, stream=None):
    _check(_L().moe_expert_up_swiglu_fp8(_p(x8), _p(x_scales), _p(group_offsets), G, rows, d,
                                         inter, _p(w13), _p(w13_scales), _p(h8), _p(h_scales),
                                         _stream(stream)), "moe_expert_up_swiglu_fp8")


def moe_pack_w13_fp8(w13_stacked, G, inter, d, w13, stream=None):
    _check(_L().moe_pack_w13_fp8(_p(w13_stacked), G, inter, d, _p(w13), _stream(stream)),
           "moe_pack_w13_fp8")


def moe_expert_down_fp8(h8, h_scales, group_offsets, G, rows, inter, d, w2, w2_scales, y,
                        stream=None):
    _check(_L().moe_expert_down_fp8(_p(h8), _p(h_scales), _p(group_offsets), G, rows, inter, d,
                                    _p(w2), _p(w2_scales), _p(y), _stream(stream)),
           "moe_expert_down_fp8")


def moe_combine(y_perm, pos, topk_gate, shared_out, residual, T, d, top_k, out, stream=None):
    _check(_L().moe_combine(_p(y_perm), _p(pos), _p(topk_gate), _p(shared_out), _p(residual), T,
                            d, top_k, _p(out), _stream(stream)), "moe_combine")


def moe_slot_index(pos, T, top_k, rows, dst_slot, stream=None):
    _check(_L().moe_slot_index(_p(pos), T, top_k, rows, _p(dst_slot), _stream(stream)),
           "moe_slot_index")


def moe_expert_down_scatter(h, group_offsets, G, rows, inter, d, w2, dst_slot, topk_gate, T,
                            top_k, y_slots, stream=None):
    _check(_L().moe_expert_down_scatter(_p(h), _p(group_offsets), G, rows, inter, d, _p(w2),
                                        _p(dst_slot), _p(topk_gate), T, top_k, _p(y_slots),
                                        _stream(stream)), "moe_expert_down_scatter")


def moe_combine_slots(y_slots, pos, shared_out, residual, T, d, top_k, out, stream=None):
    _check(_L().moe_combine_slots(_p(y_slots), _p(pos), _p(shared_out), _p(residual), T, d,
                                  top_k, _p(out), _stream(stream)), "moe_combine_slots")


def moe_expert_down_scatter_combine_workspace_size(T, d):
    return _L().moe_expert_down_scatter_combine_workspace_size(T, d)


def moe_expert_down_scatter_combine(h, group_offsets, G, rows, inter, d, w2, dst_slot, topk_gate,
                                    T, top_k, y_slots, shared_out, residual, out, workspace,
                                    ws_bytes, stream=None):
    _check(_L().moe_expert_down_scatter_combine(
        _p(h), _p(group_offsets), G, rows, inter, d, _p(w2), _p(dst_slot), _p(topk_gate), T,
        top_k, _p(y_slots), _p(shared_out), _p(residual), _p(out), _p(workspace), ws_bytes,
        _stream(stream)), "moe_expert_down_scatter_combine")


def moe_bias_update(expert_counts, bias, n_routed, T, top_k, gamma, stream=None):
    _check(_L().moe_bias_update(_p(expert_counts), _p(bias), n_routed, int(T), top_k,
                                float(gamma), _stream(stream)), "moe_bias_update")


def moe_pack_w13(w1, w3, G, inter, d, w13, stream=None):
    _check(_L().moe_pack_w13(_p(w1), _p(w3), G, inter, d, _p(w13), _stream(stream)),
           "moe_pack_w13")


def _host(t, dtype_name, where):
    """Host pointer of a CPU tensor (None -> NULL); moe_ep_plan reads and
    writes host memory, so a device tensor here is a caller error."""
    if t is None:
        return None
    if t.device.type != "cpu" or not t.is_contiguous() or str(t.dtype) != dtype_name:
        raise ValueError(f"{where}: expected a contiguous CPU {dtype_name} tensor, got "
                         f"{t.dtype} on {t.device}")
    return t.data_ptr()


def moe_ep_plan(local_counts, recv_counts, world, n_local, recv_capacity, send_splits,
                recv_splits, group_offsets, regroup=None, ungroup=None) -> int:
    """Host plan of one expert-parallel exchange (all arguments CPU tensors:
    counts int32, splits int64, offsets/regroup/ungroup int32). Returns the
    number of received rows."""
    w = "moe_ep_plan"
    n = ctypes.c_longlong(0)
    _check(_L().moe_ep_plan(_host(local_counts, "torch.int32", w),
                            _host(recv_counts, "torch.int32", w), int(world), int(n_local),
                            int(recv_capacity), _host(send_splits, "torch.int64", w),
                            _host(recv_splits, "torch.int64", w),
                            _host(group_offsets, "torch.int32", w),
                            _host(regroup, "torch.int32", w), _host(ungroup, "torch.int32", w),
                            ctypes.byref(n)), w)
    return int(n.value)


def moe_gather_rows(src, n_src, index, n, d, dst, stream=None):
    _check(_L().moe_gather_rows(_p(src), n_src, _p(index), n, d, _p(dst), _stream(stream)),
           "moe_gather_rows")


def moe_ep_plan_device(all_counts, world, n_local, rank, recv_capacity, dest_row,
                       group_offsets, global_counts, add_counts=None, stream=None):
    _check(_L().moe_ep_plan_device(_p(all_counts), world, n_local, rank, int(recv_capacity),
                                   _p(add_counts), _p(dest_row), _p(group_offsets),
                                   _p(global_counts), _stream(stream)), "moe_ep_plan_device")


def moe_ep_dispatch_p2p(u, topk_idx, pos, expert_offsets, dest_row, T, d, n_routed, top_k,
                        world, peer_x, recv_capacity, stream=None):
    _check(_L().moe_ep_dispatch_p2p(_p(u), _p(topk_idx), _p(pos), _p(expert_offsets),
                                    _p(dest_row), T, d, n_routed, top_k, world, _p(peer_x),
                                    int(recv_capacity), _stream(stream)), "moe_ep_dispatch_p2p")


def moe_ep_combine_p2p(peer_y, topk_idx, pos, expert_offsets, dest_row, topk_gate, shared_out,
                       residual, T, d, n_routed, top_k, world, recv_capacity, out, stream=None):
    _check(_L().moe_ep_combine_p2p(_p(peer_y), _p(topk_idx), _p(pos), _p(expert_offsets),
                                   _p(dest_row), _p(topk_gate), _p(shared_out), _p(residual), T,
                                   d, n_routed, top_k, world, int(recv_capacity), _p(out),
                                   _stream(stream)), "moe_ep_combine_p2p")


def moe_ipc_get_handle(tensor) -> tuple:
    """(64-byte IPC handle of the allocation holding tensor's data, byte offset)."""
    h = ctypes.create_string_buffer(64)
    off = ctypes.c_longlong(0)
    _check(_L().moe_ipc_get_handle(_p(tensor), h, ctypes.byref(off)), "moe_ipc_get_handle")
    return h.raw, off.value


def moe_ipc_open_handle(handle: bytes) -> int:
    """Map another process's allocation on this GPU; returns its base address."""
    base = ctypes.c_void_p(0)
    _check(_L().moe_ipc_open_handle(ctypes.create_string_buffer(handle, 64), ctypes.byref(base)),
           "moe_ipc_open_handle")
    return base.value


def moe_ipc_close_handle(base: int) -> None:
    _check(_L().moe_ipc_close_handle(base), "moe_ipc_close_handle")


def moe_get_device_status(clear: bool = True) -> int:
    v = ctypes.c_uint(0)
    rc = _L().moe_get_device_status(ctypes.byref(v), 1 if clear else 0)
    if rc not in (MOE_OK, MOE_ERR_DEVICE_TIMEOUT):
        raise MoEError(rc, "moe_get_device_status")
    return int(v.value)


def moe_selftest_wait_timeout(limit_ms: int, stream=None):
    _check(_L().moe_selftest_wait_timeout(limit_ms, _stream(stream)), "moe_selftest_wait_timeout")


def moe_expert_up_swiglu_train(x, group_offsets, G, rows, d, inter, w13, h, ac, stream=None):
    _check(_L().moe_expert_up_swiglu_train(_p(x), _p(group_offsets), G, rows, d, inter, _p(w13),
                                           _p(h), _p(ac), _stream(stream)),
           "moe_expert_up_swiglu_train")


def moe_combine_backward(dout, y_perm, pos, topk_gate, T, d, top_k, dy_perm, dgate, stream=None):
    _check(_L().moe_combine_backward(_p(dout), _p(y_perm), _p(pos), _p(topk_gate), T, d, top_k,
                                     _p(dy_perm), _p(dgate), _stream(stream)),
           "moe_combine_backward")


def moe_expert_down_backward(dy, ac, group_offsets, G, rows, d, inter, w2, dac, stream=None):
    _check(_L().moe_expert_down_backward(_p(dy), _p(ac), _p(group_offsets), G, rows, d, inter,
                                         _p(w2), _p(dac), _stream(stream)),
           "moe_expert_down_backward")


def moe_expert_up_backward(dac, group_offsets, G, rows, d, inter, w13, dx, stream=None):
    _check(_L().moe_expert_up_backward(_p(dac), _p(group_offsets), G, rows, d, inter, _p(w13),
                                       _p(dx), _stream(stream)), "moe_expert_up_backward")


def moe_expert_wgrad(a, b, group_offsets, G, rows, m, n, dw, stream=None):
    _check(_L().moe_expert_wgrad(_p(a), _p(b), _p(group_offsets), G, rows, m, n, _p(dw),
                                 _stream(stream)), "moe_expert_wgrad")


def moe_gate_backward(u, centroids, topk_idx, topk_gate, dgate, pos, T, d, n_routed, top_k, kind,
                      routed_scale, dz, dz_perm, stream=None):
    k = GATE_KINDS.get(kind, kind)
    _check(_L().moe_gate_backward(_p(u), _p(centroids), _p(topk_idx), _p(topk_gate), _p(dgate),
                                  _p(pos), T, d, n_routed, top_k, k, float(routed_scale), _p(dz),
                                  _p(dz_perm), _stream(stream)), "moe_gate_backward")


def moe_combine_dx(dout, dx_perm, pos, dx_shared, dz, topk_idx, centroids, T, d, top_k, du,
                   stream=None):
    _check(_L().moe_combine_dx(_p(dout), _p(dx_perm), _p(pos), _p(dx_shared), _p(dz),
                               _p(topk_idx), _p(centroids), T, d, top_k, _p(du), _stream(stream)),
           "moe_combine_dx")


def moe_centroid_grad(x_perm, dz_perm, expert_offsets, n_routed, rows, d, de, workspace,
                      ws_bytes, stream=None):
    _check(_L().moe_centroid_grad(_p(x_perm), _p(dz_perm), _p(expert_offsets), n_routed, rows, d,
                                  _p(de), _p(workspace), ws_bytes, _stream(stream)),
           "moe_centroid_grad")


def moe_centroid_grad_workspace_size(rows, n_routed, d) -> int:
    return int(_L().moe_centroid_grad_workspace_size(rows, n_routed, d))


def moe_strerror(status: int) -> str:
    return _L().moe_strerror(status).decode()


def moe_version() -> int:
    return _L().moe_version()
