"""Expert parallelism of the DeepSeekMoE layer: W ranks, one per GPU.

Rank p holds the routed experts [p*n_local, (p+1)*n_local) (n_routed =
W*n_local); the centroids, the bias and the shared expert are replicated.
Fine-grained routing sends each token to up to K experts on other GPUs, and
the token rows travel by all-to-all exchanges (DeepSeek-V3 technical report
summary: "Problem setting and motivation", the all-to-all cost of
fine-grained routing; "Main ideas", DualPipe bullet; "Limitations", the SMs
given to the all-to-all).

One forward on every rank, over its own batch of tokens:

    moe_route, moe_permute      its tokens, all n_routed experts
    counts exchange             all-to-all of the n_routed loads
                                -> recv_counts [W, n_local]
    moe_ep_plan (host)          split sizes, expert-major grouping of the
                                received rows and its inverse
    dispatch exchange           all-to-all of the x_perm rows
    moe_gather_rows             the received rows, expert-major (regroup)
    up-projection, down-projection
    moe_gather_rows             back to the received order (ungroup)
    return exchange             all-to-all back -> y_perm in x_perm order
    moe_combine                 its tokens, as on one GPU

The shared expert runs on a side stream on the rank's own tokens. The bias
update needs the loads of the whole step: the counts are summed over the ranks
(dp.sync_load) before every rank applies the same update.

The exchanges are NCCL collectives (torch.distributed) between the library's
kernels; the host plan needs the split sizes, so a step reads 2*n_routed
int32 back to the host once. The stage methods (begin, plan, experts,
finish) let a caller put its own transport between them.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch
import torch.distributed as dist

from . import _lib as L
from . import dp
from .layer import MoELayer, _Timed


@dataclass
class ExchangePlan:
    """Host plan of one exchange, seen from one rank (moe_ep_plan's outputs)."""
    send_splits: list      # rows to each rank (x_perm blocks, rank order)
    recv_splits: list      # rows from each rank
    n_recv: int            # rows received
    group_offsets: torch.Tensor  # [n_local + 1] int32 (CPU): expert-major offsets
    regroup: torch.Tensor  # [n_recv] int32 (CPU): expert-major row -> received row
    ungroup: torch.Tensor  # [n_recv] int32 (CPU): received row -> expert-major row


def plan_exchange(local_counts: torch.Tensor, recv_counts: torch.Tensor, world: int,
                  n_local: int) -> ExchangePlan:
    """The plan of one exchange from this rank's loads (local_counts
    [world*n_local] int32) and the loads every rank routes to this rank's
    experts (recv_counts [world, n_local] int32); both CPU tensors."""
    local_counts = local_counts.to(torch.int32).contiguous()
    recv_counts = recv_counts.to(torch.int32).contiguous()
    n = int(recv_counts.sum())
    ss = torch.empty(world, dtype=torch.int64)
    rs = torch.empty(world, dtype=torch.int64)
    go = torch.empty(n_local + 1, dtype=torch.int32)
    rg = torch.empty(max(n, 1), dtype=torch.int32)
    ug = torch.empty(max(n, 1), dtype=torch.int32)
    got = L.moe_ep_plan(local_counts, recv_counts, world, n_local, n, ss, rs, go, rg, ug)
    if got != n:
        raise RuntimeError(f"moe_ep_plan counted {got} received rows, expected {n}")
    return ExchangePlan(ss.tolist(), rs.tolist(), n, go, rg[:n], ug[:n])


def exchange_counts(counts: torch.Tensor, group=None) -> torch.Tensor:
    """All-to-all of the per-expert loads [world*n_local] int32: chunk p of
    this rank's counts goes to rank p; chunk q of the result is what rank q
    routes to this rank's experts."""
    out = torch.empty_like(counts)
    dist.all_to_all_single(out, counts, group=group)
    return out


def dispatch_rows(x_perm: torch.Tensor, plan: ExchangePlan, out: torch.Tensor,
                  group=None) -> torch.Tensor:
    """All-to-all of the expert-contiguous token rows: x_perm's block of rows
    for rank p's experts goes to rank p; the rows received land in
    out[:n_recv], source-major."""
    rows = sum(plan.send_splits)
    dst = out[:plan.n_recv]
    dist.all_to_all_single(dst, x_perm[:rows], output_split_sizes=plan.recv_splits,
                           input_split_sizes=plan.send_splits, group=group)
    return dst


def return_rows(y_src: torch.Tensor, plan: ExchangePlan, out: torch.Tensor,
                group=None) -> torch.Tensor:
    """All-to-all back: the expert outputs of the rows received from rank q
    (in the order received) return to rank q, landing in x_perm order."""
    rows = sum(plan.send_splits)
    dst = out[:rows]
    dist.all_to_all_single(dst, y_src[:plan.n_recv], output_split_sizes=plan.send_splits,
                           input_split_sizes=plan.recv_splits, group=group)
    return dst


class ExpertParallelMoELayer(MoELayer):
    """A DeepSeekMoE layer whose routed experts are split over the ranks of
    `group` (bf16 forward). w1, w3 [·, I, d] and w2 [·, d, I] are either all
    n_routed experts (this rank keeps its slice) or only this rank's n_local.
    world/rank default to the group's; give them explicitly to build one
    rank's layer without a process group (the ranks then exchange through the
    caller's own transport between the stage methods)."""

    _merge_shared = False   # the shared expert stays in its own launches

    def __init__(self, centroids, bias, w1, w3, w2, shared=None, *, top_k: int,
                 routed_scale: float, gate_kind: str = "sigmoid", gamma: float = 0.001,
                 group=None, world: int | None = None, rank: int | None = None,
                 overlap_shared: bool = True, device="cuda"):
        self.group = group
        self.world = dist.get_world_size(group) if world is None else int(world)
        self.rank = dist.get_rank(group) if rank is None else int(rank)
        n_routed = centroids.shape[0]
        if n_routed % self.world:
            raise ValueError(f"{n_routed} routed experts do not split over {self.world} ranks")
        self.n_local = n_routed // self.world
        self.expert_lo = self.rank * self.n_local
        if w1.shape[0] == n_routed and self.n_local != n_routed:
            sl = slice(self.expert_lo, self.expert_lo + self.n_local)
            w1, w3, w2 = w1[sl], w3[sl], w2[sl]
        if w1.shape[0] != self.n_local:
            raise ValueError(f"expected {self.n_local} or {n_routed} experts, got {w1.shape[0]}")
        super().__init__(centroids, bias, w1, w3, w2, shared, top_k=top_k,
                         routed_scale=routed_scale, gate_kind=gate_kind, gamma=gamma,
                         overlap_shared=overlap_shared, device=device)
        self._cap = -1
        self._idx_copied = None   # event after the last upload of the plan's indices

    # ------------------------------------------------------------------ buffers
    def _ensure_recv(self, n: int) -> None:
        """Grow-only buffers for n received rows (rounded up to 256 rows)."""
        if n <= self._cap:
            return
        cap = max(256, (n + 255) // 256 * 256)
        dev, bf, d = self.device, torch.bfloat16, self.d
        # two row buffers, reused in stream order: x_recv holds the received
        # rows, then the expert-major down-projection output; y_src holds the
        # expert-major copy of the received rows, then the outputs in the
        # order received
        self.x_recv = torch.empty((cap, d), dtype=bf, device=dev)
        self.y_src = torch.empty((cap, d), dtype=bf, device=dev)
        self.h_recv = torch.empty((cap, self.inter), dtype=bf, device=dev)
        # group offsets, regroup, ungroup: one pinned host block, one copy
        self._idx_host = torch.empty(self.n_local + 1 + 2 * cap, dtype=torch.int32,
                                     pin_memory=True)
        self._idx_dev = torch.empty(self.n_local + 1 + 2 * cap, dtype=torch.int32, device=dev)
        self._cap = cap

    # ------------------------------------------------------------------ stages
    def begin(self, u, timers=None):
        """Route and dispatch-copy this rank's tokens (and start the shared
        expert on the side stream). Leaves the loads in self.counts."""
        assert u.dtype == torch.bfloat16 and u.is_contiguous() and u.device.type == "cuda"
        T = u.shape[0]
        self.allocate(T)
        ev = _Timed(timers)
        self._side_used = False
        if T > 0 and self.ws13 is not None and self.overlap_shared:
            side = self._fork()
            u.record_stream(side)
            with torch.cuda.stream(side):
                with ev("shared"):
                    self.shared_ffn(u)
            self._join_event.record(side)
            self._side_used = True
        with ev("route"):
            self.route(u)
        if T > 0:
            with ev("permute"):
                self.permute(u)

    def plan(self, local_counts: torch.Tensor, recv_counts: torch.Tensor) -> ExchangePlan:
        """Host plan from CPU loads; uploads its indices (one copy on the
        current stream) and sizes the receive buffers."""
        p = plan_exchange(local_counts, recv_counts.view(self.world, self.n_local), self.world,
                          self.n_local)
        if self._idx_copied is not None:
            # the previous upload must have left the pinned block before it
            # is rewritten (forward's host read already guarantees it; a
            # caller driving the stages itself may not)
            self._idx_copied.synchronize()
        self._ensure_recv(p.n_recv)
        nl, n = self.n_local, p.n_recv
        h = self._idx_host
        h[:nl + 1] = p.group_offsets
        h[nl + 1:nl + 1 + n] = p.regroup
        h[nl + 1 + n:nl + 1 + 2 * n] = p.ungroup
        self._idx_dev[:nl + 1 + 2 * n].copy_(h[:nl + 1 + 2 * n], non_blocking=True)
        if self._idx_copied is None:
            self._idx_copied = torch.cuda.Event()
        self._idx_copied.record()
        self._goff = self._idx_dev[:nl + 1]
        self._regroup = self._idx_dev[nl + 1:nl + 1 + n]
        self._ungroup = self._idx_dev[nl + 1 + n:nl + 1 + 2 * n]
        return p

    def experts(self, plan: ExchangePlan, x_recv=None, timers=None) -> torch.Tensor:
        """This rank's experts on the received rows (x_recv, default
        self.x_recv); returns their outputs in the order received."""
        n = plan.n_recv
        x = self.x_recv if x_recv is None else x_recv
        ev = _Timed(timers)
        if n > 0:
            # The rows are copied into expert-major order rather than read in
            # place by the gathered up-projection: that form is bound by its
            # TMA request rate, the copy by HBM bandwidth (far cheaper).
            x_exp, y_exp = self.y_src, self.x_recv
            with ev("regroup"):
                L.moe_gather_rows(x, n, self._regroup, n, self.d, x_exp)
            with ev("up"):
                L.moe_expert_up_swiglu(x_exp, self._goff, self.n_local, n, self.d, self.inter,
                                       self.w13, self.h_recv)
            with ev("down"):
                L.moe_expert_down(self.h_recv, self._goff, self.n_local, n, self.inter, self.d,
                                  self.w2, y_exp)
            with ev("ungroup"):
                L.moe_gather_rows(y_exp, n, self._ungroup, n, self.d, self.y_src)
        return self.y_src[:n]

    def finish(self, u, residual: bool = True, out=None, timers=None):
        """Combine this rank's tokens from self.y_perm (x_perm order)."""
        T = u.shape[0]
        dst = self.out if out is None else out
        assert dst.shape == (T, self.d) and dst.dtype == torch.bfloat16 and dst.is_contiguous()
        ev = _Timed(timers)
        if T > 0:
            if self._side_used:
                torch.cuda.current_stream().wait_event(self._join_event)
            elif self.ws13 is not None:
                with ev("shared"):
                    self.shared_ffn(u)
            with ev("combine"):
                self.combine(u, residual, dst)
        return dst

    # ------------------------------------------------------------------ forward
    def forward(self, u, residual: bool = True, out=None, train: bool = False, timers=None):
        """h' for this rank's tokens u [T, d] (bf16, device). Every rank of
        the group must call it (the exchanges are collectives), with any T."""
        if train:
            raise ValueError("the expert-parallel layer runs the forward only")
        self.begin(u, timers)
        ev = _Timed(timers)
        with ev("exchange_counts"):
            recv = exchange_counts(self.counts, self.group)
        loads = torch.cat([self.counts, recv]).cpu()
        p = self.plan(loads[:self.n_routed], loads[self.n_routed:])
        with ev("dispatch"):
            dispatch_rows(self.x_perm, p, self.x_recv, self.group)
        y_src = self.experts(p, timers=timers)
        with ev("return"):
            return_rows(y_src, p, self.y_perm, self.group)
        self.last_plan = p
        return self.finish(u, residual, out, timers)

    def step(self, u):
        """forward, then the bias update from the loads summed over the ranks."""
        out = self.forward(u)
        if self.gate_kind == "sigmoid":
            c = self.counts.clone()
            T_all = dp.sync_load(c, u.shape[0], self.group)
            self.update_bias(c, T_all)
        return out

    # route (1 + a memset), permute (3), regroup, up, down, ungroup, shared
    # FFN (2), combine; the exchanges are NCCL's
    def launches_per_step(self) -> int:
        n = (2 if self.route_split else 1) + 3 + 4 + 1
        if self.ws13 is not None:
            n += 2
        if self.gate_kind == "sigmoid":
            n += 1
        return n


class PeerExpertParallelMoELayer(MoELayer):
    """Expert parallelism with the token rows moved through peer memory by the
    library's own kernels, planned on the device (bf16 forward).

    Rank p holds the routed experts [p*n_local, (p+1)*n_local), as in
    ExpertParallelMoELayer; the centroids, the bias and the shared expert are
    replicated. One forward on every rank (all ranks call it with the same T):

        moe_route, moe_permute_index   this rank's tokens, no row copy
        all-gather of the loads        all_counts [W, N_r] (NCCL, on the device)
        moe_ep_plan_device             rows' destinations, own group offsets,
                                       loads summed over the ranks
        moe_ep_dispatch_p2p            each token row stored into its experts'
                                       owners' receive buffers
        barrier                        (a one-element all-reduce)
        up- and down-projection        on the receive buffer, expert-major
        barrier
        moe_ep_combine_p2p             each token's K outputs read back from
                                       the owners, gate-weighted, + shared + u

    Nothing is read back to the host. The receive buffers hold recv_capacity
    rows (default W*T*K, every rank's every row: no step can overflow); the
    other ranks' buffers are mapped with CUDA IPC, which needs PyTorch's
    default CUDA allocator (expandable segments have no IPC handles). With world/rank given and no
    group the layer is one of several ranks emulated in one process: the
    caller links them with link_emulated_ranks and drives the stages (begin,
    plan, dispatch, experts, finish) in rank order, which needs no kernel to
    wait on another."""

    _merge_shared = False   # the shared expert stays in its own launches

    def __init__(self, centroids, bias, w1, w3, w2, shared=None, *, top_k: int,
                 routed_scale: float, gate_kind: str = "sigmoid", gamma: float = 0.001,
                 group=None, world: int | None = None, rank: int | None = None,
                 recv_capacity: int | None = None, micro_batches: int = 1,
                 overlap_shared: bool = True, device="cuda"):
        if micro_batches not in (1, 2):
            raise ValueError("micro_batches must be 1 or 2")
        self.micro_batches = int(micro_batches)
        self.group = group
        self.emulated = world is not None and group is None
        self.world = dist.get_world_size(group) if world is None else int(world)
        self.rank = dist.get_rank(group) if rank is None else int(rank)
        n_routed = centroids.shape[0]
        if n_routed % self.world:
            raise ValueError(f"{n_routed} routed experts do not split over {self.world} ranks")
        self.n_local = n_routed // self.world
        self.expert_lo = self.rank * self.n_local
        if w1.shape[0] == n_routed and self.n_local != n_routed:
            sl = slice(self.expert_lo, self.expert_lo + self.n_local)
            w1, w3, w2 = w1[sl], w3[sl], w2[sl]
        if w1.shape[0] != self.n_local:
            raise ValueError(f"expected {self.n_local} or {n_routed} experts, got {w1.shape[0]}")
        super().__init__(centroids, bias, w1, w3, w2, shared, top_k=top_k,
                         routed_scale=routed_scale, gate_kind=gate_kind, gamma=gamma,
                         fused_gather=True, overlap_shared=overlap_shared, device=device)
        self.recv_capacity_arg = recv_capacity
        self._mapped = []          # IPC bases opened on this GPU
        self._recv_T = -1
        self._mb = None            # the two micro-batch halves (micro_batches == 2)
        self._comm = None

    # ------------------------------------------------------------------ buffers
    def allocate(self, T: int) -> None:
        super().allocate(T)
        if T == self._recv_T:
            return
        dev, bf = self.device, torch.bfloat16
        cap = (int(self.recv_capacity_arg) if self.recv_capacity_arg is not None
               else max(1, self.world * T * self.top_k))
        self._unmap_peers()
        self.recv_capacity = cap
        self.x_recv = torch.empty((cap, self.d), dtype=bf, device=dev)
        self.h_recv = torch.empty((cap, self.inter), dtype=bf, device=dev)
        self.y_recv = torch.empty((cap, self.d), dtype=bf, device=dev)
        i32 = torch.int32
        self.all_counts = torch.zeros((self.world, self.n_routed), dtype=i32, device=dev)
        self.dest_row = torch.empty(self.n_routed, dtype=i32, device=dev)
        self.goff = torch.empty(self.n_local + 1, dtype=i32, device=dev)
        self.global_counts = torch.empty(self.n_routed, dtype=i32, device=dev)
        self._barrier_t = torch.zeros(1, dtype=i32, device=dev)
        self._recv_T = T
        if not self.emulated:
            self._map_peers()

    def _unmap_peers(self):
        if not self._mapped:
            return
        # every rank closes its mappings before any rank frees the buffers
        for base in self._mapped:
            L.moe_ipc_close_handle(base)
        self._mapped = []
        dist.barrier(group=self.group)

    def _map_peers(self):
        """Pointer tables of the ranks' receive and output buffers as seen
        from this GPU (one all-gather of the IPC handles)."""
        xs, ys = [0] * self.world, [0] * self.world
        xs[self.rank], ys[self.rank] = self.x_recv.data_ptr(), self.y_recv.data_ptr()
        if self.world > 1:
            mine = (L.moe_ipc_get_handle(self.x_recv), L.moe_ipc_get_handle(self.y_recv))
            allh = [None] * self.world
            dist.all_gather_object(allh, mine, group=self.group)
            for q in range(self.world):
                if q == self.rank:
                    continue
                (hx, ox), (hy, oy) = allh[q]
                bx, by = L.moe_ipc_open_handle(hx), L.moe_ipc_open_handle(hy)
                self._mapped += [bx, by]
                xs[q], ys[q] = bx + ox, by + oy
        self.set_peer_tables(xs, ys)

    def set_peer_tables(self, x_ptrs, y_ptrs):
        """Device tables of the W receive (x) and output (y) buffer addresses."""
        self.peer_x = torch.tensor(x_ptrs, dtype=torch.int64, device=self.device)
        self.peer_y = torch.tensor(y_ptrs, dtype=torch.int64, device=self.device)

    # ------------------------------------------------------------------ stages
    def begin(self, u, timers=None):
        """Route this rank's tokens and compute their dispatch rows (and start
        the shared expert on the side stream). Leaves the loads in self.counts."""
        assert u.dtype == torch.bfloat16 and u.is_contiguous() and u.device.type == "cuda"
        T = u.shape[0]
        self.allocate(T)
        ev = _Timed(timers)
        self._side_used = False
        if T > 0 and self.ws13 is not None and self.overlap_shared:
            side = self._fork()
            u.record_stream(side)
            with torch.cuda.stream(side):
                with ev("shared"):
                    self.shared_ffn(u)
            self._join_event.record(side)
            self._side_used = True
        with ev("route"):
            self.route(u)
        with ev("permute"):
            self.permute(u)

    def plan(self, add_counts=None):
        """Device plan from self.all_counts (every rank's loads); add_counts:
        an earlier micro-batch's summed loads, folded into global_counts."""
        L.moe_ep_plan_device(self.all_counts, self.world, self.n_local, self.rank,
                             self.recv_capacity, self.dest_row, self.goff, self.global_counts,
                             add_counts)

    def dispatch(self, u, timers=None):
        with _Timed(timers)("dispatch"):
            L.moe_ep_dispatch_p2p(u, self.topk_idx, self.pos, self.offsets, self.dest_row,
                                  u.shape[0], self.d, self.n_routed, self.top_k, self.world,
                                  self.peer_x, self.recv_capacity)

    def experts(self, timers=None):
        """This rank's experts on its receive buffer (the group offsets come
        from the device plan; rows past them are never touched)."""
        ev = _Timed(timers)
        cap = self.recv_capacity
        with ev("up"):
            L.moe_expert_up_swiglu(self.x_recv, self.goff, self.n_local, cap, self.d, self.inter,
                                   self.w13, self.h_recv)
        with ev("down"):
            L.moe_expert_down(self.h_recv, self.goff, self.n_local, cap, self.inter, self.d,
                              self.w2, self.y_recv)

    def finish(self, u, residual: bool = True, out=None, timers=None):
        T = u.shape[0]
        dst = self.out if out is None else out
        assert dst.shape == (T, self.d) and dst.dtype == torch.bfloat16 and dst.is_contiguous()
        ev = _Timed(timers)
        if T > 0:
            if self._side_used:
                torch.cuda.current_stream().wait_event(self._join_event)
            elif self.ws13 is not None:
                with ev("shared"):
                    self.shared_ffn(u)
            with ev("combine"):
                L.moe_ep_combine_p2p(self.peer_y, self.topk_idx, self.pos, self.offsets,
                                     self.dest_row, self.topk_gate, self.shared_out,
                                     u if residual else None, T, self.d, self.n_routed,
                                     self.top_k, self.world, self.recv_capacity, dst)
        return dst

    def _barrier(self):
        dist.all_reduce(self._barrier_t, group=self.group)

    # ------------------------------------------------------------------ forward
    def forward(self, u, residual: bool = True, out=None, train: bool = False, timers=None):
        """h' for this rank's tokens u [T, d] (bf16, device). Every rank of the
        group calls it with the same T (the exchanges are collectives)."""
        if train:
            raise ValueError("the expert-parallel layer runs the forward only")
        if self.emulated:
            raise RuntimeError("an emulated rank is driven through its stages")
        if self.micro_batches == 2 and u.shape[0] >= 2:
            return self._forward_two(u, residual, out, timers)
        self.begin(u, timers)
        with _Timed(timers)("exchange_counts"):
            dist.all_gather_into_tensor(self.all_counts.view(-1), self.counts, group=self.group)
        self.plan()
        self.dispatch(u, timers)
        self._barrier()
        self.experts(timers)
        self._barrier()
        self._step_counts = self.global_counts
        self._step_T = u.shape[0]
        return self.finish(u, residual, out, timers)

    def micro_batch_halves(self):
        """The two halves of a two-micro-batch step: this layer and a second
        one sharing its weights, bias and process group, with buffers of its
        own (each half holds the first or second half of the tokens)."""
        if self._mb is None:
            import copy
            other = copy.copy(self)
            other._mb = None
            other._side = None           # its own side stream and events
            other._T = other._recv_T = -1
            other._mapped = []
            other.micro_batches = 1
            self._mb = (self, other)
        return self._mb

    def _forward_two(self, u, residual, out, timers):
        """Two micro-batches, the exchange of one beside the expert GEMMs of
        the other (the overlap the technical report arranges with DualPipe):

            main:  begin A, begin B | all-gather, plan, dispatch A, barrier
            comm:                     all-gather, plan, dispatch B, barrier
            main:  experts A   (beside B's dispatch)
            comm:  barrier, combine A   (beside B's experts)
            main:  experts B, barrier, combine B; then waits for comm

        The collectives are issued in the same order on every rank."""
        T = u.shape[0]
        T1 = T // 2
        A, B = self.micro_batch_halves()
        if out is None:
            if getattr(self, "_out_full", None) is None or self._out_full.shape[0] != T:
                self._out_full = torch.empty((T, self.d), dtype=torch.bfloat16,
                                             device=self.device)
            out = self._out_full
        assert out.shape == (T, self.d) and out.dtype == torch.bfloat16 and out.is_contiguous()
        dst = out
        uA, uB = u[:T1], u[T1:]
        oA, oB = dst[:T1], dst[T1:]
        cur = torch.cuda.current_stream()
        if self._comm is None:
            self._comm = torch.cuda.Stream(device=self.device)
        comm = self._comm
        # u and the output are used on the comm stream too
        u.record_stream(comm)
        dst.record_stream(comm)
        A.begin(uA, timers)
        B.begin(uB)
        dist.all_gather_into_tensor(A.all_counts.view(-1), A.counts, group=self.group)
        A.plan()
        A.dispatch(uA, timers)
        A._barrier()
        comm.wait_stream(cur)
        with torch.cuda.stream(comm):
            dist.all_gather_into_tensor(B.all_counts.view(-1), B.counts, group=self.group)
            B.plan(add_counts=A.global_counts)
            B.dispatch(uB)
            B._barrier()
            b_ready = torch.cuda.Event()
            b_ready.record(comm)
        A.experts(timers)
        a_done = torch.cuda.Event()
        a_done.record(cur)
        with torch.cuda.stream(comm):
            comm.wait_event(a_done)
            A._barrier()
            A.finish(uA, residual, oA)
        cur.wait_event(b_ready)
        B.experts()
        B._barrier()
        B.finish(uB, residual, oB)
        cur.wait_stream(comm)
        self._step_counts = B.global_counts
        self._step_T = T
        return dst

    def update_bias(self, counts=None, T=None):
        """End-of-step bias update from the loads summed over the ranks (the
        device plan's global_counts; with two micro-batches the second one's,
        which includes the first's) and the tokens of all ranks."""
        T_all = self.world * getattr(self, "_step_T", self._T) if T is None else T
        c = getattr(self, "_step_counts", self.global_counts) if counts is None else counts
        L.moe_bias_update(c, self.bias, self.n_routed, T_all, self.top_k, self.gamma)

    def step(self, u):
        out = self.forward(u)
        if self.gate_kind == "sigmoid":
            self.update_bias()
        return out

    # route (1 + a memset), permute index (2), plan, dispatch, up, down, shared
    # FFN (2), combine; the all-gather and the barriers are NCCL's
    def launches_per_step(self) -> int:
        n = (2 if self.route_split else 1) + 2 + 1 + 1 + 2 + 1
        if self.ws13 is not None:
            n += 2
        n *= self.micro_batches
        if self.gate_kind == "sigmoid":
            n += 1
        return n

    def close(self):
        """Unmap the other ranks' buffers (collective: every rank calls it)."""
        self._unmap_peers()
        if self._mb is not None:
            self._mb[1]._unmap_peers()


def link_emulated_ranks(layers) -> None:
    """Point every emulated rank's peer tables at the buffers of all of them
    (ranks emulated in one process on one GPU, in rank order)."""
    xs = [lay.x_recv.data_ptr() for lay in layers]
    ys = [lay.y_recv.data_ptr() for lay in layers]
    for lay in layers:
        lay.set_peer_tables(xs, ys)
