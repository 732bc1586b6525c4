"""MoELayer: device buffers plus the sequence of C-ABI calls of one forward.

PyTorch supplies device memory and the stream; every step of the layer runs
in libmoe.so's kernels:

    moe_route        gate GEMM + sigmoid + biased top-K + gates + counts
    moe_permute      expert-contiguous copy of the token rows
    moe_expert_up_swiglu, moe_expert_down
                     the routed experts' grouped FFN (G = N_r)
    moe_grouped_ffn  the shared expert (G = 1), on a side stream
    moe_combine      h' = u + shared + sum_k g * y
    moe_bias_update  b -= / += gamma from the loads (end of the step)

Training (bf16): forward(u, train=True) also keeps the SwiGLU pre-activations;
backward(dout) then runs the backward calls (combine, expert dgrad and
wgrad, gate, du, centroid gradient) and leaves the weight gradients on the
layer (grad_w13 in the packed W13 layout, grad_w2, grad_ws13, grad_ws2,
grad_centroids).
"""
from __future__ import annotations

import torch

from . import _lib as L


class _Timed:
    """Context manager factory: CUDA events around a call when timers is a dict."""

    def __init__(self, timers):
        self.timers = timers

    def __call__(self, name):
        return _TimedCall(self.timers, name)


class _TimedCall:
    def __init__(self, timers, name):
        self.timers, self.name = timers, name

    def __enter__(self):
        if self.timers is not None:
            self.e0 = torch.cuda.Event(enable_timing=True)
            self.e0.record()

    def __exit__(self, *exc):
        if self.timers is not None:
            e1 = torch.cuda.Event(enable_timing=True)
            e1.record()
            self.timers.setdefault(self.name, []).append((self.e0, e1))
        return False


class MoELayer:
    """One DeepSeekMoE layer resident on a CUDA device.

    Weights are given in the natural layout: w1, w3 [N_r, I, d], w2 [N_r, d, I]
    (bf16) for the routed experts; ws1, ws3 [N_s*I, d], ws2 [d, N_s*I] for the
    shared experts concatenated along I (or None); centroids [N_r, d] bf16;
    bias [N_r] fp32 (the layer keeps its own device copy, updated in place).
    """

    # whether the shared expert may run as a group of the routed GEMMs
    # (subclasses with their own exchange of routed rows keep it apart)
    _merge_shared = True

    def __init__(self, centroids, bias, w1, w3, w2, shared=None, *, top_k: int,
                 routed_scale: float, gate_kind: str = "sigmoid", gamma: float = 0.001,
                 fp8: bool = False, fused_gather: bool = False, fused_scatter: bool = False,
                 fused_combine: bool = False,
                 overlap_shared: bool = True, shared_join: str = "auto",
                 split_route: str = "auto", shared_grouped: bool = False, device="cuda"):
        L.load()
        dev = torch.device(device)
        self.device = dev
        self.n_routed, self.d = centroids.shape
        self.inter = w1.shape[1]
        self.top_k = int(top_k)
        self.routed_scale = float(routed_scale)
        self.gate_kind = gate_kind
        self.gamma = float(gamma)
        bf = torch.bfloat16
        self.fp8 = bool(fp8)
        # fused gather (bf16): the up-projection reads the token rows of u
        # itself, so the dispatch only computes row indices (no x_perm copy)
        self.fused_gather = bool(fused_gather) and not self.fp8
        # fused scatter (bf16): the down-projection multiplies each routed row
        # by its gate and writes it to its (token, slot) row; the combine then
        # adds K adjacent rows per token
        self.fused_scatter = (bool(fused_scatter) or bool(fused_combine)) and not self.fp8
        # fused combine (bf16, implies the fused scatter): the down-projection's
        # epilogue also adds each token's K slot rows to the residual and the
        # shared expert once the last of them is stored; no combine launch
        self.fused_combine = bool(fused_combine) and not self.fp8
        # run the shared expert on a side stream next to the routed path (FP8:
        # with its own quantisation of u, so it does not wait for the dispatch);
        # shared_join: where the current stream waits for it -- "early" (before
        # the routed GEMMs), "late" (before the combine) or "auto" (early when
        # the routed groups average >= 256 rows, else late)
        self.overlap_shared = bool(overlap_shared)
        if shared_join not in ("auto", "early", "late"):
            raise ValueError("shared_join must be 'auto', 'early' or 'late'")
        self.shared_join = shared_join
        self.shared_after_route = False
        # split_route: the gate GEMM split over K (moe_route_splitk) -- "on",
        # "off" or "auto" (on for batches of at most 2048 tokens, where
        # moe_route's 128-token CTAs would leave most SMs idle)
        if split_route not in ("auto", "on", "off"):
            raise ValueError("split_route must be 'auto', 'on' or 'off'")
        self.split_route = split_route
        # shared_grouped: the shared expert as the last group of the routed
        # grouped GEMMs (bf16 five-call form, one shared expert of the routed
        # experts' inter) instead of its own launches beside the route and
        # dispatch; measured slower at V3 prefill (the overlap is worth more
        # than the extra launches cost), so off by default
        self.shared_grouped = bool(shared_grouped)
        self.centroids = centroids.to(dev, bf).contiguous()
        self.bias = (bias.to(dev, torch.float32).contiguous() if bias is not None
                     else torch.zeros(self.n_routed, dtype=torch.float32, device=dev))
        pack = self.pack_w13_fp8 if self.fp8 else self.pack_w13
        # the shared expert can join the routed grouped GEMMs as group N_r when
        # it has the routed experts' shape: then both live in one weight array
        # (routed experts first), and self.w13 / self.ws13 are views of it
        self.mergeable = (self._merge_shared and shared is not None and not self.fp8 and
                          not self.fused_gather and not self.fused_scatter and
                          shared[0].shape[0] == self.inter)
        if self.mergeable:
            ws1, ws3, ws2 = shared
            G, I = self.n_routed, self.inter
            self.w13_all = torch.empty((G + 1, 2 * I, self.d), dtype=bf, device=dev)
            L.moe_pack_w13(w1.to(dev, bf).contiguous(), w3.to(dev, bf).contiguous(), G, I, self.d,
                           self.w13_all)
            L.moe_pack_w13(ws1.to(dev, bf).contiguous()[None], ws3.to(dev, bf).contiguous()[None],
                           1, I, self.d, self.w13_all[G:])
            self.w2_all = torch.empty((G + 1, self.d, I), dtype=bf, device=dev)
            self.w2_all[:G].copy_(w2)
            self.w2_all[G].copy_(ws2)
            self.w13, self.ws13 = self.w13_all[:G], self.w13_all[G:]
            self.w2, self.ws2 = self.w2_all[:G], self.w2_all[G]
            self.shared_inter = I
            shared = None                               # weights placed
        else:
            self.w13 = pack(w1.to(dev, bf).contiguous(), w3.to(dev, bf).contiguous())
            self.w2 = w2.to(dev, bf).contiguous()
        if shared is not None:
            ws1, ws3, ws2 = shared
            self.shared_inter = ws1.shape[0]
            self.ws13 = pack(ws1.to(dev, bf).contiguous()[None], ws3.to(dev, bf).contiguous()[None])
            self.ws2 = ws2.to(dev, bf).contiguous()
        elif not self.mergeable:
            self.shared_inter = 0
            self.ws13 = self.ws2 = None
        if self.fp8:
            # E4M3 weights with one fp32 scale per 128x128 block (the bf16
            # copies are dropped)
            self.w13, self.w13_s = self.w13
            self.w2, self.w2_s = self.quant_weights(self.w2)
            if self.ws13 is not None:
                self.ws13, self.ws13_s = self.ws13
                self.ws2, self.ws2_s = self.quant_weights(self.ws2[None])
        self._T = -1
        self.route_split = False
        self.shared_in_grouped = False
        self._grouped = False

    # ------------------------------------------------------------------ setup
    def pack_w13(self, w1, w3):
        G, inter, d = w1.shape
        w13 = torch.empty((G, 2 * inter, d), dtype=torch.bfloat16, device=self.device)
        L.moe_pack_w13(w1, w3, G, inter, d, w13)
        return w13

    def pack_w13_fp8(self, w1, w3):
        """(E4M3 w13 [G, 2I, d] with W1/W3 interleaved in 64-row chunks,
        scales [G, 2, I/128, d/128]) from bf16 w1, w3 [G, I, d]."""
        G, inter, d = w1.shape
        stacked = torch.stack([w1, w3], dim=1).view(2 * G, inter, d)
        q, s = self.quant_weights(stacked)
        del stacked
        w13 = torch.empty((G, 2 * inter, d), dtype=torch.uint8, device=self.device)
        L.moe_pack_w13_fp8(q, G, inter, d, w13)
        return w13, s.view(G, 2, inter // 128, d // 128)

    def quant_weights(self, w):
        """E4M3 codes [G, R, C] and fp32 scales [G, R/128, C/128] of bf16 w."""
        if w.dim() == 2:
            w = w[None]
        G, R, C = w.shape
        q = torch.empty((G, R, C), dtype=torch.uint8, device=self.device)
        s = torch.empty((G, R // 128, C // 128), dtype=torch.float32, device=self.device)
        L.moe_quant_weights_fp8(w.contiguous(), G, R, C, q, s)
        return q, s

    def allocate(self, T: int) -> None:
        """(Re)allocate the activation buffers for a batch of T tokens."""
        if T == self._T:
            return
        dev, K, d = self.device, self.top_k, self.d
        rows = T * K
        i32 = torch.int32
        # the shared expert as group N_r of the routed GEMMs: T more rows
        self.shared_in_grouped = self.mergeable and self.shared_grouped
        rows_all = rows + (T if self.shared_in_grouped else 0)
        self.topk_idx = torch.empty((T, K), dtype=i32, device=dev)
        self.topk_gate = torch.empty((T, K), dtype=torch.float32, device=dev)
        self.counts = torch.empty(self.n_routed, dtype=i32, device=dev)
        self.offsets = torch.empty(self.n_routed + (2 if self.shared_in_grouped else 1), dtype=i32,
                                   device=dev)
        self.pos = torch.empty((T, K), dtype=i32, device=dev)
        self.src = torch.empty(rows, dtype=i32, device=dev)
        self.dst_slot = (torch.empty(rows, dtype=i32, device=dev) if self.fused_scatter
                         else None)
        self.comb_ws_bytes = (L.moe_expert_down_scatter_combine_workspace_size(T, d)
                              if self.fused_combine else 0)
        self.comb_ws = (torch.empty(self.comb_ws_bytes, dtype=torch.uint8, device=dev)
                        if self.fused_combine else None)
        self.x_perm = (None if (self.fp8 or self.fused_gather) else
                       torch.empty((rows_all, d), dtype=torch.bfloat16, device=dev))
        self.y_perm = torch.empty((rows_all, d), dtype=torch.bfloat16, device=dev)
        self.route_split = (self.split_route == "on" or
                            (self.split_route == "auto" and T <= 2048))
        self.route_ws_bytes = (L.moe_route_splitk_workspace_size(T, d, self.n_routed)
                               if self.route_split else 0)
        self.route_ws = (torch.empty(self.route_ws_bytes, dtype=torch.uint8, device=dev)
                         if self.route_split else None)
        self.perm_ws_bytes = L.moe_permute_workspace_size(T, self.n_routed)
        self.perm_ws = torch.empty(self.perm_ws_bytes, dtype=torch.uint8, device=dev)
        dt = L.MOE_FP8_E4M3 if self.fp8 else L.MOE_BF16
        ffn_ws = max(L.moe_grouped_ffn_workspace_size(rows_all, self.inter, dt),
                     L.moe_grouped_ffn_workspace_size(T, max(self.shared_inter, 128), dt))
        if self.fp8:
            u8 = torch.uint8
            self.u8 = torch.empty((T, d), dtype=u8, device=dev)
            self.u_s = torch.empty((T, d // 128), dtype=torch.float32, device=dev)
            self.x8 = torch.empty((rows, d), dtype=u8, device=dev)
            self.x_s = torch.empty((rows, d // 128), dtype=torch.float32, device=dev)
        self.ffn_ws_bytes = ffn_ws
        self.ffn_ws = torch.empty(ffn_ws, dtype=torch.uint8, device=dev)
        if self.shared_in_grouped:
            self.shared_out = self.y_perm[rows:]        # rows of group N_r
        else:
            self.shared_out = (torch.empty((T, d), dtype=torch.bfloat16, device=dev)
                               if self.ws13 is not None else None)
        # the shared expert runs on a side stream next to the routed path
        # (bf16), so it gets its own workspace
        self.shared_ws_bytes = L.moe_grouped_ffn_workspace_size(T, max(self.shared_inter, 128), dt)
        self.shared_ws = (torch.empty(self.shared_ws_bytes, dtype=torch.uint8, device=dev)
                          if self.ws13 is not None else None)
        self.shared_offsets = torch.tensor([0, T], dtype=i32, device=dev)
        self.out = torch.empty((T, d), dtype=torch.bfloat16, device=dev)
        self._T = T

    # ------------------------------------------------------------------ steps
    def route(self, u):
        T = u.shape[0]
        bias = self.bias if self.gate_kind == "sigmoid" else None
        if self.route_split:
            L.moe_route_splitk(u, self.centroids, bias, T, self.d, self.n_routed, self.top_k,
                               self.gate_kind, self.routed_scale, self.topk_idx, self.topk_gate,
                               self.counts, self.route_ws, self.route_ws_bytes)
        else:
            L.moe_route(u, self.centroids, bias, T, self.d, self.n_routed, self.top_k,
                        self.gate_kind, self.routed_scale, self.topk_idx, self.topk_gate,
                        self.counts)

    def permute(self, u):
        T = u.shape[0]
        if self.fused_gather:
            L.moe_permute_index(self.topk_idx, self.counts, T, self.n_routed, self.top_k,
                                self.offsets, self.pos, self.src, self.perm_ws, self.perm_ws_bytes)
            if self.fused_scatter:
                L.moe_slot_index(self.pos, T, self.top_k, T * self.top_k, self.dst_slot)
            return
        if self.fp8:
            # each token quantised once (1x128 tiles) inside the dispatch, its
            # codes written to its K rows and, for an in-line shared expert, to u8
            own_u8 = self.ws13 is not None and not self.overlap_shared
            L.moe_permute_fp8(u, self.topk_idx, self.counts, T, self.d, self.n_routed, self.top_k,
                              self.x8, self.x_s, self.u8 if own_u8 else None,
                              self.u_s if own_u8 else None, self.offsets,
                              self.pos, self.src, self.perm_ws, self.perm_ws_bytes)
            return
        if self._grouped:
            # u's rows once more after the routed rows: the shared expert's group
            L.moe_permute_shared(u, self.topk_idx, self.counts, T, self.d, self.n_routed,
                                 self.top_k, self.x_perm, self.offsets, self.pos, self.src,
                                 self.perm_ws, self.perm_ws_bytes)
            return
        L.moe_permute(u, self.topk_idx, self.counts, T, self.d, self.n_routed, self.top_k,
                      self.x_perm, self.offsets, self.pos, self.src, self.perm_ws,
                      self.perm_ws_bytes)
        if self.fused_scatter:
            L.moe_slot_index(self.pos, T, self.top_k, T * self.top_k, self.dst_slot)

    def _routed_up(self, T, u):
        rows = T * self.top_k
        if self.fused_gather:
            L.moe_expert_up_swiglu_gather(u, T, self.src, self.offsets, self.n_routed, rows, self.d,
                                          self.inter, self.w13, self.ffn_ws)
        elif self.fp8:
            h8, hs = self._fp8_h()
            L.moe_expert_up_swiglu_fp8(self.x8, self.x_s, self.offsets, self.n_routed, rows,
                                       self.d, self.inter, self.w13, self.w13_s, h8, hs)
        elif self._grouped:
            # routed experts and the shared expert (group N_r) in one launch
            L.moe_expert_up_swiglu(self.x_perm, self.offsets, self.n_routed + 1, rows + T, self.d,
                                   self.inter, self.w13_all, self.ffn_ws)
        else:
            L.moe_expert_up_swiglu(self.x_perm, self.offsets, self.n_routed, rows, self.d,
                                   self.inter, self.w13, self.ffn_ws)

    def _routed_down(self, T, u=None, residual=True, dst=None):
        rows = T * self.top_k
        if self.fused_combine:
            # the shared expert's output must be complete (the caller joins first)
            L.moe_expert_down_scatter_combine(
                self.ffn_ws, self.offsets, self.n_routed, rows, self.inter, self.d, self.w2,
                self.dst_slot, self.topk_gate, T, self.top_k, self.y_perm, self.shared_out,
                u if residual else None, self.out if dst is None else dst, self.comb_ws,
                self.comb_ws_bytes)
        elif self.fp8:
            h8, hs = self._fp8_h()
            L.moe_expert_down_fp8(h8, hs, self.offsets, self.n_routed, rows, self.inter, self.d,
                                  self.w2, self.w2_s, self.y_perm)
        elif self.fused_scatter:
            # y_perm holds the gate-weighted rows in (token, slot) order
            L.moe_expert_down_scatter(self.ffn_ws, self.offsets, self.n_routed, rows, self.inter,
                                      self.d, self.w2, self.dst_slot, self.topk_gate, T,
                                      self.top_k, self.y_perm)
        elif self._grouped:
            # the shared expert's output lands in rows [T*K, T*K + T) = shared_out
            L.moe_expert_down(self.ffn_ws, self.offsets, self.n_routed + 1, rows + T, self.inter,
                              self.d, self.w2_all, self.y_perm)
        else:
            L.moe_expert_down(self.ffn_ws, self.offsets, self.n_routed, rows, self.inter, self.d,
                              self.w2, self.y_perm)

    def _fp8_h(self):
        """Views of the FP8 FFN workspace: h's E4M3 codes and their 1x128
        scales (the layout moe_grouped_ffn uses)."""
        rows = self._T * self.top_k
        h8 = self.ffn_ws
        hs = h8[(rows * self.inter + 255) // 256 * 256:]
        return h8, hs

    def shared_ffn(self, u):
        if self.ws13 is None:
            return
        T = u.shape[0]
        if self.fp8:
            if self.overlap_shared:
                # on the side stream: u's codes of its own (the same 1x128
                # rule as the dispatch's), not waiting for the dispatch
                L.moe_quant_act_fp8(u, T, self.d, self.u8, self.u_s)
            L.moe_grouped_ffn(self.u8, self.u_s, self.shared_offsets, 1, T, self.d,
                              self.shared_inter, self.ws13, self.ws13_s, self.ws2, self.ws2_s,
                              L.MOE_FP8_E4M3, self.shared_out, self.shared_ws,
                              self.shared_ws_bytes)
            return
        L.moe_grouped_ffn(u, None, self.shared_offsets, 1, T, self.d, self.shared_inter, self.ws13,
                          None, self.ws2, None, L.MOE_BF16, self.shared_out, self.shared_ws,
                          self.shared_ws_bytes)

    def combine(self, u, residual: bool = True, out=None):
        T = u.shape[0]
        if self.fused_scatter:
            L.moe_combine_slots(self.y_perm, self.pos, self.shared_out, u if residual else None,
                                T, self.d, self.top_k, self.out if out is None else out)
            return
        L.moe_combine(self.y_perm, self.pos, self.topk_gate, self.shared_out,
                      u if residual else None, T, self.d, self.top_k,
                      self.out if out is None else out)

    def forward(self, u, residual: bool = True, out=None, train: bool = False, timers=None):
        """h' for the bf16 batch u [T, d] (device), written to `out` ([T, d]
        bf16, device) or to the layer's own output buffer, which is returned.
        train=True (bf16, copy-based dispatch) keeps what backward() needs.
        The shared expert depends on u alone: it runs on a side stream
        while the current stream routes and dispatches (and, for decode-sized
        groups, runs the routed experts); the current stream waits for it
        before the routed GEMMs (large groups) or before the combine.
        timers: optional dict; each stage ("route", "permute", "up", "down",
        "shared", "combine") gets a (start, end) CUDA event pair, recorded on
        the stream the stage runs on."""
        assert u.dtype == torch.bfloat16 and u.is_contiguous() and u.device.type == "cuda"
        T = u.shape[0]
        self.allocate(T)
        dst = self.out if out is None else out
        assert dst.shape == (T, self.d) and dst.dtype == torch.bfloat16 and dst.is_contiguous()
        if train:
            if self.fp8 or self.fused_gather or self.fused_scatter:
                raise ValueError("training runs on the bf16 layer with the copy-based dispatch "
                                 "and the plain combine")
            self._allocate_train(T)
        self._train_state = (u, residual) if train else None
        # the shared expert as group N_r of the routed GEMMs (not in training)
        self._grouped = self.shared_in_grouped and not train
        ev = _Timed(timers)
        side = None

        def fork_shared():
            s = self._fork()
            if not torch.cuda.is_current_stream_capturing():
                u.record_stream(s)
            with torch.cuda.stream(s):
                with ev("shared"):
                    if train:
                        self._shared_ffn_train(u)
                    else:
                        self.shared_ffn(u)
            self._join_event.record(s)
            return s

        overlap = T > 0 and self.ws13 is not None and self.overlap_shared and not self._grouped
        # The route kernel needs about as much shared memory per SM as a GEMM
        # CTA, so it cannot share SMs with the shared expert's persistent GEMM;
        # the dispatch's kernels can. shared_after_route: start the shared
        # expert once the route is done, beside the dispatch only.
        if overlap and not self.shared_after_route:
            side = fork_shared()
        with ev("route"):
            self.route(u)
        if overlap and self.shared_after_route:
            side = fork_shared()
        # Where the shared expert rejoins: the routed GEMMs of large groups
        # (CTA-pair form) are compute-bound like the shared expert itself, so
        # the shared expert overlaps only the HBM-bound route and dispatch and
        # the routed GEMMs run alone; decode-sized groups stream their weights
        # from HBM, and the shared expert runs next to them too.
        join_early = side is not None and (
            self.shared_join == "early" or
            (self.shared_join == "auto" and T * self.top_k >= 256 * self.n_routed))
        if T > 0:
            with ev("permute"):
                self.permute(u)
            if join_early:
                torch.cuda.current_stream().wait_event(self._join_event)
            with ev("up"):
                if train:
                    self._routed_up_train(T)
                else:
                    self._routed_up(T, u)
            if self.fused_combine:
                # the down-projection's epilogue reads the shared expert's output
                if side is None:
                    with ev("shared"):
                        self.shared_ffn(u)
                elif not join_early:
                    torch.cuda.current_stream().wait_event(self._join_event)
                with ev("down"):
                    self._routed_down(T, u, residual, dst)
                return dst
            with ev("down"):
                if train:
                    self._routed_down_train(T)
                else:
                    self._routed_down(T)
            if side is None:
                if not self._grouped:                   # (grouped: already in y_perm)
                    with ev("shared"):
                        self.shared_ffn(u)
            elif not join_early:
                torch.cuda.current_stream().wait_event(self._join_event)
            with ev("combine"):
                self.combine(u, residual, dst)
        return dst

    def _fork(self):
        """Side stream for the shared expert, ordered after everything already
        on the current stream (the previous step's combine included)."""
        cur = torch.cuda.current_stream()
        if getattr(self, "_side", None) is None:
            self._side = torch.cuda.Stream(device=self.device)
            self._fork_event = torch.cuda.Event()
            self._join_event = torch.cuda.Event()
        self._fork_event.record(cur)
        self._side.wait_event(self._fork_event)
        return self._side

    # ------------------------------------------------------------------ training
    def _allocate_train(self, T: int) -> None:
        if getattr(self, "_train_T", -1) == T:
            return
        dev, K, d, I = self.device, self.top_k, self.d, self.inter
        rows = T * K
        bf, f32 = torch.bfloat16, torch.float32
        self.h = torch.empty((rows, I), dtype=bf, device=dev)
        self.ac = torch.empty((rows, 2 * I), dtype=bf, device=dev)
        self.dy_perm = torch.empty((rows, d), dtype=bf, device=dev)
        self.dac = torch.empty((rows, 2 * I), dtype=bf, device=dev)
        self.dx_perm = torch.empty((rows, d), dtype=bf, device=dev)
        self.dgate = torch.empty((T, K), dtype=f32, device=dev)
        self.dz = torch.empty((T, K), dtype=f32, device=dev)
        self.dz_perm = torch.empty(rows, dtype=f32, device=dev)
        self.du = torch.empty((T, d), dtype=bf, device=dev)
        self.cg_ws = torch.empty(L.moe_centroid_grad_workspace_size(rows, self.n_routed, d),
                                 dtype=torch.uint8, device=dev)
        if self.ws13 is not None:
            Is = self.shared_inter
            self.h_s = torch.empty((T, Is), dtype=bf, device=dev)
            self.ac_s = torch.empty((T, 2 * Is), dtype=bf, device=dev)
            self.dac_s = torch.empty((T, 2 * Is), dtype=bf, device=dev)
            self.dx_s = torch.empty((T, d), dtype=bf, device=dev)
        if getattr(self, "grad_w13", None) is None:
            self.grad_w13 = torch.empty_like(self.w13)
            self.grad_w2 = torch.empty_like(self.w2)
            self.grad_centroids = torch.empty_like(self.centroids)
            if self.ws13 is not None:
                self.grad_ws13 = torch.empty_like(self.ws13)
                self.grad_ws2 = torch.empty_like(self.ws2)
        self._train_T = T

    def _routed_up_train(self, T):
        rows = T * self.top_k
        L.moe_expert_up_swiglu_train(self.x_perm, self.offsets, self.n_routed, rows, self.d,
                                     self.inter, self.w13, self.h, self.ac)

    def _routed_down_train(self, T):
        rows = T * self.top_k
        L.moe_expert_down(self.h, self.offsets, self.n_routed, rows, self.inter, self.d, self.w2,
                          self.y_perm)

    def _shared_ffn_train(self, u):
        if self.ws13 is None:
            return
        T = u.shape[0]
        L.moe_expert_up_swiglu_train(u, self.shared_offsets, 1, T, self.d, self.shared_inter,
                                     self.ws13, self.h_s, self.ac_s)
        L.moe_expert_down(self.h_s, self.shared_offsets, 1, T, self.shared_inter, self.d, self.ws2,
                          self.shared_out)

    def backward(self, dout, timers=None):
        """Gradients of the last forward(..., train=True) for dL/dh' = dout
        ([T, d] bf16, device). Returns du [T, d] bf16 (the layer's buffer);
        the weight gradients are left in grad_w13 (packed like w13), grad_w2,
        grad_ws13, grad_ws2 and grad_centroids. The bias gets none.
        timers: optional dict; the routed up-projection dgrad ("dx") and the
        routed W13 weight gradient ("dw13") each get a (start, end) pair of
        CUDA events appended to timers[name] on the current stream."""
        if getattr(self, "_train_state", None) is None:
            raise RuntimeError("backward() needs a preceding forward(..., train=True)")
        u, residual = self._train_state
        T, K, d, I, G = u.shape[0], self.top_k, self.d, self.inter, self.n_routed
        assert dout.shape == (T, d) and dout.dtype == torch.bfloat16 and dout.is_contiguous()
        rows = T * K
        if T == 0:
            return self.du
        L.moe_combine_backward(dout, self.y_perm, self.pos, self.topk_gate, T, d, K,
                               self.dy_perm, self.dgate)
        L.moe_expert_down_backward(self.dy_perm, self.ac, self.offsets, G, rows, d, I, self.w2,
                                   self.dac)
        ev = _Timed(timers)
        with ev("dx"):
            L.moe_expert_up_backward(self.dac, self.offsets, G, rows, d, I, self.w13,
                                     self.dx_perm)
        L.moe_expert_wgrad(self.dy_perm, self.h, self.offsets, G, rows, d, I, self.grad_w2)
        with ev("dw13"):
            L.moe_expert_wgrad(self.dac, self.x_perm, self.offsets, G, rows, 2 * I, d,
                               self.grad_w13)
        dx_s = None
        if self.ws13 is not None:
            Is = self.shared_inter
            so = self.shared_offsets
            L.moe_expert_down_backward(dout, self.ac_s, so, 1, T, d, Is, self.ws2, self.dac_s)
            L.moe_expert_up_backward(self.dac_s, so, 1, T, d, Is, self.ws13, self.dx_s)
            L.moe_expert_wgrad(dout, self.h_s, so, 1, T, d, Is, self.grad_ws2)
            L.moe_expert_wgrad(self.dac_s, u, so, 1, T, 2 * Is, d, self.grad_ws13)
            dx_s = self.dx_s
        L.moe_gate_backward(u, self.centroids, self.topk_idx, self.topk_gate, self.dgate, self.pos,
                            T, d, G, K, self.gate_kind, self.routed_scale, self.dz, self.dz_perm)
        L.moe_combine_dx(dout if residual else None, self.dx_perm, self.pos, dx_s, self.dz,
                         self.topk_idx, self.centroids, T, d, K, self.du)
        L.moe_centroid_grad(self.x_perm, self.dz_perm, self.offsets, G, rows, d,
                            self.grad_centroids, self.cg_ws, self.cg_ws.numel())
        return self.du

    def launches_per_backward(self) -> int:
        # combine bwd, down dgrad, up dgrad, 2 wgrad; shared: 4 more; gate bwd,
        # du, centroid grad (chunk table, partial sums, reduction)
        return 5 + (4 if self.ws13 is not None else 0) + 5

    def update_bias(self, counts=None, T=None):
        """End-of-step bias update from this batch's loads (or from counts
        summed over data-parallel ranks with the global T)."""
        c = self.counts if counts is None else counts
        L.moe_bias_update(c, self.bias, self.n_routed, self._T if T is None else T, self.top_k,
                          self.gamma)

    def step(self, u):
        out = self.forward(u)
        if self.gate_kind == "sigmoid":
            self.update_bias()
        return out

    # ------------------------------------------------------------------ CUDA graph
    def capture(self, T: int, residual: bool = True, bias_update: bool = True, u=None):
        """Record one step for batches of T tokens (the forward and, for the
        sigmoid gate with bias_update, the end-of-step bias update) into a CUDA
        graph, so that replay(u) runs all of it with one launch from the host.
        The recorded launches keep this layer's buffers, workspaces and the
        library's tile-counter slots: replays must follow one another on one
        stream and not overlap eager calls of this layer. The shared expert's
        side stream is part of the graph (forked and joined by events).
        u: optional [T, d] bf16 device tensor the graph reads its input from
        (the caller writes each batch into it; replay(u) then copies nothing);
        by default the layer keeps its own input buffer."""
        self.allocate(T)
        dev = self.device
        if u is not None:
            assert u.shape == (T, self.d) and u.dtype == torch.bfloat16 and u.is_contiguous()
            self._gu = u
        else:
            self._gu = torch.zeros((T, self.d), dtype=torch.bfloat16, device=dev)
        self._gout = torch.empty((T, self.d), dtype=torch.bfloat16, device=dev)
        self._g_bias = bias_update and self.gate_kind == "sigmoid"
        # one eager pass first: library initialisation and kernel attributes
        # happen outside the capture
        s = torch.cuda.Stream(device=dev)
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            self.forward(self._gu, residual=residual, out=self._gout)
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize(dev)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self.forward(self._gu, residual=residual, out=self._gout)
            if self._g_bias:
                self.update_bias()
        self._graph = g
        return self._gout

    def replay(self, u):
        """One recorded step on the bf16 batch u [T, d] (device): u is copied
        into the graph's input buffer first. Returns the graph's output buffer
        (overwritten by the next replay)."""
        g = getattr(self, "_graph", None)
        if g is None:
            raise RuntimeError("capture(T) first")
        assert u.shape == self._gu.shape and u.dtype == torch.bfloat16
        if u.data_ptr() != self._gu.data_ptr():
            self._gu.copy_(u)
        g.replay()
        return self._gout

    # kernels launched by one step(): route (1, split over K 2; + a memset), permute (3; FP8:
    # + the activation quantisation), routed and shared FFN, combine (1),
    # bias update (1)
    def launches_per_step(self) -> int:
        # up and down one launch each (FP8: h is quantised in the
        # up-projection's epilogue, u in the dispatch)
        ffn = 2
        perm = 2 if self.fused_gather else 3
        if self.fused_scatter:
            perm += 1                       # the slot index
        n = (2 if self.route_split else 1) + perm + ffn + (0 if self.fused_combine else 1)
        if self.ws13 is not None and not getattr(self, "shared_in_grouped", False):
            n += ffn
            if self.fp8 and self.overlap_shared:
                n += 1                      # the shared expert's own quantisation of u
        if self.gate_kind == "sigmoid":
            n += 1
        return n
