#!/usr/bin/env python
"""Benchmark of the DeepSeekMoE layer forward on B200: routed tokens/s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config v3p] [--impl ours|reference]

A step is one pass of the whole hot path over one batch of T tokens:
route (gate GEMM + sigmoid + biased top-K + gates + counts) -> permute ->
routed expert FFN (up-projection + SwiGLU, down-projection) -> shared expert
FFN -> combine with the residual -> bias update. With N > 1 (torchrun, one
rank per GPU) every rank runs its own batch of T tokens (data parallel, weak
scaling) and the per-expert counts are summed over ranks with one NCCL
all-reduce before the bias update, so the bias stays identical everywhere.

Rank 0 prints one JSON line. `value` is the whole-job throughput (all ranks'
tokens / max-over-ranks device time) with inputs resident in HBM; `e2e` is the
same metric through the public API with the batch copied from pinned host
memory and the output copied back inside the timed region; `roofline` is the
routed expert up-projection kernel (the dominant launch) against the measured
burst bf16 tensor peak (the sustained peak and the nominal rate at the run's
median SM clock beside it); `routing` counts the batch's near-ties and checks
the first timed step's expert indices against fp64 keys; `cpu_baseline` is the
fp64 oracle on a bounded sample. The default V3-prefill run then times, in the
same process, V3 decode (HBM roofline over the expert weights it touches), its
softmax-gate form and FP8 prefill (`variants`). `--gpus N` started as one
process re-launches itself as N ranks. `--impl reference` times the oracle
alone as the reference arm.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "routed tokens/sec per DeepSeekMoE layer on 1 B200; % of tensor/HBM roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        d["_source"] = "measured"
        return d
    d = dict(FALLBACK_PEAKS)
    d["_source"] = "fallback"
    return d


def cublas_fp8_tflops(dev, n: int = 8192, reps: int = 10) -> float:
    """Best-of-`reps` rate of one cuBLAS E4M3 GEMM (torch._scaled_mm, n^3, fp32
    scales, bf16 out), as context for the FP8 roofline; measured on `dev`."""
    import torch
    a = torch.randn(n, n, device=dev).to(torch.float8_e4m3fn)
    b = torch.randn(n, n, device=dev).to(torch.float8_e4m3fn).t()
    one = torch.ones((), device=dev)
    best = float("inf")
    for _ in range(reps + 2):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
        e1.record()
        torch.cuda.synchronize()
        best = min(best, e0.elapsed_time(e1))
    return 2.0 * n ** 3 / (best * 1e-3) / 1e12


def kernel_source_sha() -> str:
    h = hashlib.sha256()
    for f in ("ptx.cuh", "gemm.cuh", "gemm2sm.cuh"):
        h.update(open(os.path.join(ROOT, "mixture_experts_layer_58_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str):
    """DRAM bytes per launch of the up-projection kernel from the committed ncu
    summary, or None if absent or taken on different kernel source."""
    p = os.path.join(ROOT, "profiles", "expert_up_swiglu_traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    if d.get("source_sha") != kernel_source_sha() or d.get("workload") != workload:
        return None
    return d.get("bytes_per_launch")


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.proc is None:
            return
        time.sleep(0.2)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def oracle_sample(cfg, u_host, e_host, b_host, expert_fn, shared_list, n_tokens):
    """The oracle's full layer (route, routed + shared FFN, combine) on the
    first n_tokens of the batch. Returns seconds."""
    from oracle import moe_oracle as om
    t0 = time.perf_counter()
    u = u_host[:n_tokens]
    out, _ = om.layer(u, e_host, b_host if cfg.gate_kind == "sigmoid" else None, expert_fn,
                      shared_list, cfg.top_k, cfg.routed_scale, cfg.gate_kind)
    assert out.shape[0] == n_tokens
    return time.perf_counter() - t0


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [p.get("num_threads", 1) for p in threadpool_info() if p.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:  # noqa: BLE001
        return 1


def make_expert_fn(cfg, W_host=None):
    from mixture_experts_layer_58_b200 import synth
    cache = {}

    def fn(i):
        if i not in cache:
            if W_host is not None:
                ws = (W_host[0][i], W_host[1][i], W_host[2][i])
            else:
                ws = synth.expert_weights(cfg, i, "cuda" if cfg.weights_on_gpu else "cpu")
            cache.clear()
            cache[i] = tuple(w.float().cpu().numpy() for w in ws)
        return cache[i]
    return fn


# ----------------------------------------------------------------------------- reference arm
def run_reference(args, cfg, rank):
    """The fp64 oracle on the host cores as the reference arm, on this arm's
    workload and metric: each step is the oracle's full layer over a bounded
    sample of the batch's tokens."""
    import torch
    from mixture_experts_layer_58_b200 import synth
    if rank != 0:
        return
    u, e, b = synth.tokens(cfg), synth.centroids(cfg), synth.bias(cfg)
    shared = synth.shared_weights(cfg, "cuda" if cfg.weights_on_gpu else "cpu")
    shared_list = [tuple(w.float().cpu().numpy() for w in shared)] if shared is not None else []
    expert_fn = make_expert_fn(cfg)
    # size the per-step sample so the whole run stays within ~2 minutes
    probe = oracle_sample(cfg, u, e, b, expert_fn, shared_list, 1)
    budget = 120.0 / max(1, args.steps + args.warmup)
    n = int(max(1, min(cfg.T, budget / max(probe, 1e-3))))
    for _ in range(args.warmup):
        oracle_sample(cfg, u, e, b, expert_fn, shared_list, n)
    times = [oracle_sample(cfg, u, e, b, expert_fn, shared_list, n) for _ in range(args.steps)]
    sec = sum(times) / len(times)
    tps = n / sec
    cores = blas_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": tps, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": sec * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": cfg.name, "T": cfg.T, "d": cfg.d, "n_routed": cfg.n_routed,
                   "top_k": cfg.top_k, "n_shared": cfg.n_shared, "inter": cfg.inter,
                   "routed_scale": cfg.routed_scale, "gate": cfg.gate_kind,
                   "sample_tokens_per_step": n},
        "cpu_baseline": {"value": tps, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"oracle full layer on the first {n} of {cfg.T} tokens per "
                                   f"step (expert weights copied from the GPU on demand)"},
        "e2e": {"value": tps, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    del torch


# ----------------------------------------------------------------------------- our arm
def run_train(args, cfg, rank, world, local, dev):
    """Training step of the layer: forward (train=True), backward from a
    seeded dL/dh', bias update. Value = routed tokens per second of whole
    steps; roofline of the larger of the two biggest backward GEMMs (the
    routed up-projection dgrad dx = dac W13 and the W13 weight gradient,
    2 T K (2I) d flops each), timed with CUDA events inside the timed steps."""
    import torch
    import torch.distributed as dist
    from mixture_experts_layer_58_b200 import dp, synth
    from mixture_experts_layer_58_b200.layer import MoELayer
    if cfg.fp8:
        raise SystemExit("train mode runs the bf16 layer")
    T, K, d, I = cfg.T, cfg.top_k, cfg.d, cfg.inter
    W1, W3, W2 = synth.all_expert_weights(cfg, "cuda")
    lay = MoELayer(synth.centroids(cfg), synth.bias(cfg), W1, W3, W2,
                   synth.shared_weights(cfg, "cuda"), top_k=K, routed_scale=cfg.routed_scale,
                   gate_kind=cfg.gate_kind, gamma=cfg.gamma, device=dev)
    del W1, W3, W2
    torch.cuda.empty_cache()
    u_host = synth.tokens(cfg)
    g = torch.Generator().manual_seed(1234 + rank)
    dout_host = (torch.randn(T, d, generator=g) * 0.05).bfloat16()
    u = u_host.to(dev)
    dout = dout_host.to(dev)
    stream = torch.cuda.current_stream()

    def step(timers=None):
        lay.forward(u, train=True)
        lay.backward(dout, timers)
        if world > 1:
            # data parallel: average the weight gradients over the ranks
            dp.allreduce_grads([lay.grad_w13, lay.grad_w2, lay.grad_centroids,
                                getattr(lay, "grad_ws13", None), getattr(lay, "grad_ws2", None)])
        if cfg.gate_kind == "sigmoid":
            if world > 1:
                lay.update_bias(lay.counts, dp.sync_load(lay.counts, T))
            else:
                lay.update_bias()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if L_status() != 0:
        raise SystemExit("device timeout during warm-up")
    timers = {}
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        t0.record(stream)
        for _ in range(args.steps):
            step(timers)
        t1.record(stream)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
    ms = t0.elapsed_time(t1)
    if world > 1:
        tt = torch.tensor([ms], device=dev)
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        ms = float(tt.item())
    if L_status() != 0:
        raise SystemExit("device timeout during the timed region")
    ms_step = ms / args.steps
    kms = {n: sum(a.elapsed_time(b) for a, b in v) / len(v) for n, v in timers.items()}
    kname = max(kms, key=kms.get)
    flops = 2.0 * T * K * 2 * I * d
    pk = peaks()
    clocks = clk.summary()
    fwd_flops = T * cfg.flops_per_token()
    # backward: dgrad and wgrad of every forward GEMM except the router's
    # (2x the expert FLOPs), plus O(T K d) elementwise work
    step_flops = fwd_flops + 2 * (fwd_flops - 2.0 * T * d * cfg.n_routed)

    # e2e: the batch and dL/dh' from pinned host memory, du back, every step
    u_pin, dout_pin = u_host.pin_memory(), dout_host.pin_memory()
    du_pin = torch.empty((T, d), dtype=torch.bfloat16).pin_memory()

    def e2e_step():
        u.copy_(u_pin, non_blocking=True)
        dout.copy_(dout_pin, non_blocking=True)
        step()
        du_pin.copy_(lay.du, non_blocking=True)

    for _ in range(args.warmup):
        e2e_step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    if world > 1:
        tt = torch.tensor([e2e_ms], device=dev)
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        e2e_ms = float(tt.item())
    if rank == 0:
        print(json.dumps({
            "metric": "routed tokens/sec per DeepSeekMoE layer training step (forward + backward "
                      "+ bias update) on 1 B200",
            "value": T * world / (ms_step * 1e-3), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded; random-init weights of the layer shape)",
            "config": {"workload": cfg.name, "mode": "train", "T": T, "d": d,
                       "n_routed": cfg.n_routed, "top_k": K, "inter": I,
                       "parallelism": f"dp{world}" if world > 1 else "single",
                       "l2": "inputs larger than L2"},
            "step_tflops": step_flops / (ms_step * 1e-3) / 1e12,
            "roofline": {**tensor_roofline(flops, kms[kname], pk, clocks), "traffic": None,
                         "kernel": {"dx": "grouped_dgrad_bf16_kernel<store> (moe_expert_up_backward)",
                                    "dw13": "grouped_wgrad_bf16_kernel (moe_expert_wgrad, dW13)"}[kname],
                         "other_ms": kms},
            "e2e": {"value": T * world / (e2e_ms / args.steps * 1e-3), "unit": "tokens/s",
                    "h2d_bytes_per_step": 2 * T * d * 2, "d2h_bytes_per_step": T * d * 2,
                    "api": "MoELayer.forward(train=True) + MoELayer.backward"},
            "gpu_launches": args.steps * (lay.launches_per_step() + lay.launches_per_backward()),
            "clocks": clocks,
        }), flush=True)


def L_status() -> int:
    from mixture_experts_layer_58_b200 import _lib as L
    return L.moe_get_device_status()


# per-SM dense bf16 MMA rate of sm_100a: an M=128, N=256, K=16 tcgen05.mma
# (1 M flop) issues every 128 clocks on one SM
BF16_FLOP_PER_CLK_PER_SM = 8192
NUM_SMS = 148


def tensor_roofline(flops, kernel_ms, pk, clocks, fp8=False):
    """Achieved TFLOP/s of a kernel against the measured peaks: `frac` is
    against the burst bf16 peak (a kernel timed inside a step of tens of ms
    runs at burst clocks), with the sustained peak and the nominal tensor
    rate at the run's median SM clock beside it. FP8 takes 2x (the nominal
    fp8/bf16 ratio of sm_100a's tensor cores)."""
    ratio = 2.0 if fp8 else 1.0
    achieved = flops / (kernel_ms * 1e-3) / 1e12
    burst = pk["bf16_tflops"] * ratio
    sust = (pk.get("bf16_tflops_sustained") or pk["bf16_tflops"]) * ratio
    out = {"bound": "tensor", "achieved": achieved, "peak": burst, "unit": "TFLOP/s",
           "frac": achieved / burst, "frac_of_sustained": achieved / sust,
           "peak_sustained": sust, "kernel_ms": kernel_ms,
           "peak_source": f"{pk['_source']} bf16_tflops (burst)"
                          + (" x 2 (nominal fp8/bf16)" if fp8 else "")}
    mhz = (clocks or {}).get("sm_mhz")
    if mhz:
        nominal = NUM_SMS * BF16_FLOP_PER_CLK_PER_SM * ratio * mhz * 1e6 / 1e12
        out["nominal_at_median_clock"] = nominal
        out["frac_of_nominal_at_median_clock"] = achieved / nominal
    return out


# What bounds the FP8 expert GEMM below its tensor roofline (measured with
# diagnostic builds in one process): the promotion warps, which read each
# 128-K block's fp32 products from TMEM and fold them into the accumulators
# with the block's two scales on the CUDA cores. Without those FMAs the same
# kernel ran the up-projection of a Zipf mix in 5.09 ms instead of 6.92 ms.
FP8_LIMIT = ("promotion warps (each 128-K block's products read from TMEM and scaled into "
             "fp32 accumulators on the CUDA cores): without their FMAs the up-projection "
             "measured 1.36x faster; the tensor pipe is not the bound")


def routing_check(u, e, b, kind, K, idx_gpu):
    """Statistic of one routed batch: near-ties (a token whose K+1 largest
    selection keys, taken in fp64 from the same bf16 inputs and fp32 bias,
    hold an adjacent pair closer than 1e-5) and, outside them, tokens whose
    GPU selection differs from the fp64 top-K. Computed with torch fp64 on
    the device; a report, not the product path."""
    import torch
    z = u.double() @ e.double().T
    key = torch.sigmoid(z) + (b.double()[None, :] if b is not None else 0.0) \
        if kind == "sigmoid" else z
    top = torch.topk(key, K + 1, dim=1)
    gaps = top.values[:, :-1] - top.values[:, 1:]
    near = (gaps < 1e-5).any(dim=1)
    want = top.indices[:, :K].to(torch.int32)
    bad = (want != idx_gpu).any(dim=1) & ~near
    return {"tokens": int(u.shape[0]), "near_ties": int(near.sum()),
            "index_mismatch_outside_near_ties": int(bad.sum()),
            "keys": "fp64 (torch on the device) from the bf16 u, e and the fp32 bias "
                    "of the first timed step"}


def bias_step(lay, cfg, T, world, ep_mode):
    """The end-of-step bias update: this batch's loads on one GPU; the loads
    summed over the ranks otherwise (the peer-memory expert-parallel layer
    has them from its device plan already)."""
    from mixture_experts_layer_58_b200 import dp
    if cfg.gate_kind != "sigmoid":
        return
    if hasattr(lay, "global_counts"):
        lay.update_bias()
    elif world > 1 or ep_mode:
        lay.update_bias(lay.counts, dp.sync_load(lay.counts, T))
    else:
        lay.update_bias()


def time_forward(lay, u, cfg, args, world, ep_mode, local, stream, graph=None):
    """W warm-up steps, then K timed steps between barriers and device
    syncs (CUDA events on the launching stream, clocks sampled throughout).
    A step is the forward plus the bias update. Returns the timings and the
    routing of the first and last timed steps."""
    import torch
    import torch.distributed as dist
    from mixture_experts_layer_58_b200 import _lib as L
    from mixture_experts_layer_58_b200 import dp
    T = u.shape[0]
    timers, recv_rows, snap = {}, [], {}
    want_graph = getattr(args, "graph", False) if graph is None else graph
    use_graph = want_graph and world == 1 and not ep_mode
    if use_graph:
        # one CUDA graph per step (forward + bias update), reading u in place
        try:
            lay.capture(T, u=u, bias_update=(cfg.gate_kind == "sigmoid"))
        except RuntimeError as exc:            # capture refused: time the eager steps
            print(f"CUDA graph capture failed ({exc}); timing eager steps", file=sys.stderr)
            use_graph = False
            torch.cuda.synchronize()

    def step(i=None):
        if use_graph:
            lay.replay(u)
        else:
            lay.forward(u, timers=timers if i is not None else None)
        if i == 0:
            snap["idx0"] = lay.topk_idx.clone()
            snap["counts0"] = lay.counts.clone()
        if i is not None and i == args.steps - 1:
            snap["counts1"] = lay.counts.clone()
        if ep_mode and i is not None and hasattr(lay, "last_plan"):
            recv_rows.append(lay.last_plan.n_recv)
        if not use_graph:
            bias_step(lay, cfg, T, world, ep_mode)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if L.moe_get_device_status() != 0:
        raise SystemExit("device timeout during warm-up")
    bias0 = lay.bias.clone()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        t0.record(stream)
        for i in range(args.steps):
            step(i)
        t1.record(stream)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
    ms = t0.elapsed_time(t1)
    if world > 1 or ep_mode:
        tt = torch.tensor([ms], device=u.device)
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        ms = float(tt.item())
    if L.moe_get_device_status() != 0:
        raise SystemExit("device timeout during the timed region")
    if use_graph:
        # stage times from eager steps after the timed region (a graph
        # records no events between its kernels)
        for _ in range(max(3, min(args.steps, 5))):
            lay.forward(u, timers=timers)
            bias_step(lay, cfg, T, world, ep_mode)
        torch.cuda.synchronize()
    stage_ms = {n: sum(a.elapsed_time(b) for a, b in v) / len(v) for n, v in timers.items()}
    return {"ms_step": ms / args.steps, "stage_ms": stage_ms, "clocks": clk.summary(),
            "recv_rows": recv_rows, "bias0": bias0, "graph": use_graph, **snap}


def decode_hbm(cfg, counts, ms_step, pk):
    """HBM roofline of a decode-sized step: the bytes it must move at least,
    i.e. the W1/W3/W2 of every routed expert the batch touched and of the
    shared expert(s), the centroids, and the activations (u in, x_perm and
    y_perm written and read, h written and read, out written)."""
    T, K, d, I = cfg.T, cfg.top_k, cfg.d, cfg.inter
    wb = 1 if cfg.fp8 else 2
    touched = int((counts > 0).sum())
    weights = (touched * 3 * I * d + 3 * cfg.shared_inter * d) * wb
    acts = (T * d * 2 + 2 * T * K * d * 2 + 2 * T * K * I * 2 + T * d * 2
            + cfg.n_routed * d * 2)
    byts = weights + acts
    gbs = byts / (ms_step * 1e-3) / 1e9
    return {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
            "frac": gbs / pk["hbm_gbs"], "bytes_per_step": byts,
            "expert_weight_bytes": weights, "experts_touched": touched,
            "peak_source": f"{pk['_source']} hbm_gbs", "time": "whole layer step"}


def up_kernel_roofline(cfg, lay, t, pk, up_rows, recorded):
    """Roofline of the dominant launch, the routed up-projection + SwiGLU:
    tensor-bound for prefill-sized groups, HBM-bound (its W13 slabs) for
    decode-sized ones."""
    T, K, d, I = cfg.T, cfg.top_k, cfg.d, cfg.inter
    up_ms = t["stage_ms"]["up"]
    kname = ("grouped_gemm_fp8_kernel<SwiGLU> (moe_expert_up_swiglu_fp8)" if cfg.fp8 else
             "grouped_gemm_bf16_pair_kernel<SwiGLU, gather> (moe_expert_up_swiglu_gather)"
             if lay.fused_gather else
             "grouped_gemm bf16 <SwiGLU>, CTA-pair or 1-CTA tiles by group size "
             "(moe_expert_up_swiglu)")
    if T * K < 256 * cfg.n_routed:
        touched = int((t["counts1"] > 0).sum())
        wbytes = (1 if cfg.fp8 else 2) * 2 * I * d
        up_bytes = touched * wbytes + T * K * d * (1 if cfg.fp8 else 2) + T * K * I * 2
        gbs = up_bytes / (up_ms * 1e-3) / 1e9
        return {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": gbs / pk["hbm_gbs"], "traffic": recorded, "kernel": kname,
                "kernel_ms": up_ms, "bytes_per_launch": up_bytes, "experts_touched": touched,
                "peak_source": f"{pk['_source']} hbm_gbs"}
    r = tensor_roofline(2.0 * up_rows * d * 2 * I, up_ms, pk, t["clocks"], cfg.fp8)
    r.update({"traffic": recorded, "kernel": kname})
    return r


def variant_line(name, args, dev, local, stream, pk):
    """One more workload timed in the same process (decode, its softmax-gate
    form, FP8 prefill): device time per step, stages, rooflines and the
    routing statistic of its first timed step."""
    import torch
    from mixture_experts_layer_58_b200 import synth
    from mixture_experts_layer_58_b200.layer import MoELayer
    cfg = synth.CONFIGS[name]
    W1, W3, W2 = synth.all_expert_weights(cfg, "cuda")
    e_host, b_host = synth.centroids(cfg), synth.bias(cfg)
    lay = MoELayer(e_host, b_host, W1, W3, W2, synth.shared_weights(cfg, "cuda"),
                   top_k=cfg.top_k, routed_scale=cfg.routed_scale, gate_kind=cfg.gate_kind,
                   gamma=cfg.gamma, fp8=cfg.fp8, split_route=args.split_route,
                   shared_grouped=args.shared_grouped, device=dev)
    del W1, W3, W2
    torch.cuda.empty_cache()
    u = synth.tokens(cfg).to(dev)
    lay.allocate(cfg.T)
    # decode-sized batches: one CUDA graph per step (the launches are a
    # visible part of a 3 ms step); prefill: eager (measured equal)
    decode = cfg.T * cfg.top_k < 256 * cfg.n_routed
    t = time_forward(lay, u, cfg, args, 1, False, local, stream,
                     graph=(args.graph or decode))
    T, K = cfg.T, cfg.top_k
    line = {"workload": cfg.name, "T": T, "gate": cfg.gate_kind,
            "dtype": "e4m3 (fp32 promotion)" if cfg.fp8 else "bf16",
            "ms_per_step": t["ms_step"], "value": T / (t["ms_step"] * 1e-3),
            "unit": "tokens/s", "steps": args.steps, "warmup": args.warmup,
            "stage_ms": t["stage_ms"], "clocks": t["clocks"],
            "launch": "one CUDA graph per step" if t["graph"] else "eager",
            "gpu_launches": args.steps * lay.launches_per_step(),
            "max_expert_load": {"first_timed_step": int(t["counts0"].max()),
                                "last_timed_step": int(t["counts1"].max())}}
    line["routing"] = routing_check(u, lay.centroids, t["bias0"] if cfg.gate_kind == "sigmoid"
                                    else None, cfg.gate_kind, K, t["idx0"])
    line["roofline"] = up_kernel_roofline(cfg, lay, t, pk, T * K, None)
    if T * K < 256 * cfg.n_routed:
        line["layer_hbm"] = decode_hbm(cfg, t["counts1"].cpu(), t["ms_step"], pk)
    else:
        lt = T * cfg.flops_per_token() / (t["ms_step"] * 1e-3) / 1e12
        line["layer_tflops"] = lt
        line["layer_frac_of_tensor_peak"] = lt / (pk["bf16_tflops"] * (2 if cfg.fp8 else 1))
    if cfg.fp8:
        line["roofline"]["limit"] = FP8_LIMIT
        try:
            line["roofline"]["cublas_fp8_tflops_live"] = cublas_fp8_tflops(dev)
        except (RuntimeError, AttributeError) as exc:   # context only
            line["roofline"]["cublas_fp8_tflops_live"] = f"not measured: {exc}"[:120]
    del lay, u
    torch.cuda.empty_cache()
    return line


def relaunch_ranks(args, argv):
    """`bench.py --gpus N` (N > 1) started as one plain process: start N ranks
    on this node with torch.distributed.run (one per GPU, rendezvous on
    127.0.0.1) and return their exit status."""
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes", "1",
           "--nproc-per-node", str(args.gpus), "--master-addr", "127.0.0.1",
           "--master-port", str(port), os.path.abspath(__file__), *argv]
    return subprocess.call(cmd)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="v3p")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--mode", default="five-call",
                    choices=["five-call", "fused", "scatter", "scatter-combine", "train"],
                    help="five-call: route, permute (copy), grouped FFN, combine, bias update; "
                         "fused: the up-projection gathers the token rows itself (bf16; measured "
                         "slower: the TMA gathers are request-rate bound); scatter: the "
                         "down-projection applies the gates and writes slot-ordered rows, the "
                         "combine adds adjacent rows (bf16); scatter-combine: the same, with the "
                         "combine in the down-projection's epilogue too (bf16); train: forward "
                         "with saved "
                         "pre-activations + backward + bias update (bf16)")
    ap.add_argument("--no-overlap", action="store_true",
                    help="run the shared expert after the routed experts on one stream")
    ap.add_argument("--shared-join", default="auto", choices=["auto", "early", "late"],
                    help="where the overlapped shared expert rejoins: before the routed GEMMs "
                         "(early), before the combine (late), or by group size (auto)")
    ap.add_argument("--graph", action="store_true",
                    help="replay each step (forward + bias update) as one CUDA graph (1 GPU)")
    ap.add_argument("--shared-grouped", action="store_true",
                    help="the shared expert as the last group of the routed grouped GEMMs "
                         "instead of its own launches beside the route and dispatch")
    ap.add_argument("--split-route", default="auto", choices=["auto", "on", "off"],
                    help="gate GEMM split over K with a separate top-K pass (on), in one "
                         "fused pass (off), or split for batches of at most 2048 tokens (auto)")
    ap.add_argument("--parallel", default="dp", choices=["dp", "ep", "ep-p2p"],
                    help="dp: every rank holds all experts, its own batch; ep: the routed "
                         "experts split over the ranks, token rows exchanged by NCCL "
                         "all-to-all; ep-p2p: the same split, rows stored into and read back "
                         "from the owners' buffers by the library's kernels over peer memory, "
                         "planned on the device (bf16 forward, five-call mode)")
    ap.add_argument("--micro-batches", type=int, default=1, choices=[1, 2],
                    help="ep-p2p: split each step's tokens in two, the exchange of one "
                         "beside the expert GEMMs of the other")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-variants", action="store_true",
                    help="skip the decode and FP8 workloads timed after V3 prefill")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    argv = sys.argv[1:]
    args = ap.parse_args(argv)
    args.warmup = max(args.warmup, 3)
    if args.gpus < 1:
        raise SystemExit("--gpus must be >= 1")

    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        sys.exit(relaunch_ranks(args, argv))
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}: launch one rank per GPU")

    from mixture_experts_layer_58_b200 import synth
    cfg = synth.CONFIGS[args.config]

    if args.impl == "reference":
        run_reference(args, cfg, rank)
        return

    import torch
    import torch.distributed as dist
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    ep_mode = args.parallel in ("ep", "ep-p2p")
    if ep_mode and (cfg.fp8 or args.mode != "five-call"):
        raise SystemExit("--parallel ep runs the bf16 five-call forward")
    if world > 1 or ep_mode:
        from datetime import timedelta
        if world == 1:
            os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
            if "MASTER_PORT" not in os.environ:
                import socket
                with socket.socket() as sk:          # a free port for the one-rank group
                    sk.bind(("127.0.0.1", 0))
                    os.environ["MASTER_PORT"] = str(sk.getsockname()[1])
            os.environ.setdefault("RANK", "0")
            os.environ.setdefault("WORLD_SIZE", "1")
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    from mixture_experts_layer_58_b200 import _lib as L
    from mixture_experts_layer_58_b200 import build, dp
    from mixture_experts_layer_58_b200.layer import MoELayer
    build.build()
    if args.mode == "train":
        run_train(args, cfg, rank, world, local, dev)
        return
    L.load()

    # ---- inputs: same workload on every rank, each rank its own batch (seed + rank)
    rcfg = cfg.replace(seed=cfg.seed + rank) if world > 1 else cfg
    u_host = synth.tokens(rcfg)
    e_host, b_host = synth.centroids(cfg), synth.bias(cfg)
    W1, W3, W2 = synth.all_expert_weights(cfg, "cuda" if cfg.weights_on_gpu else "cpu")
    shared = synth.shared_weights(cfg, "cuda" if cfg.weights_on_gpu else "cpu")
    if ep_mode:
        from mixture_experts_layer_58_b200.ep import (ExpertParallelMoELayer,
                                                      PeerExpertParallelMoELayer)
        if args.parallel == "ep-p2p":
            lay = PeerExpertParallelMoELayer(e_host, b_host, W1, W3, W2, shared, top_k=cfg.top_k,
                                             routed_scale=cfg.routed_scale,
                                             gate_kind=cfg.gate_kind, gamma=cfg.gamma,
                                             micro_batches=args.micro_batches,
                                             overlap_shared=not args.no_overlap, device=dev)
        else:
            lay = ExpertParallelMoELayer(e_host, b_host, W1, W3, W2, shared, top_k=cfg.top_k,
                                         routed_scale=cfg.routed_scale, gate_kind=cfg.gate_kind,
                                         gamma=cfg.gamma, overlap_shared=not args.no_overlap,
                                         device=dev)
    else:
        lay = MoELayer(e_host, b_host, W1, W3, W2, shared, top_k=cfg.top_k,
                       routed_scale=cfg.routed_scale, gate_kind=cfg.gate_kind, gamma=cfg.gamma,
                       fp8=cfg.fp8, fused_gather=(args.mode == "fused"),
                       fused_scatter=(args.mode == "scatter"),
                       fused_combine=(args.mode == "scatter-combine"),
                       overlap_shared=not args.no_overlap, shared_join=args.shared_join,
                       split_route=args.split_route, shared_grouped=args.shared_grouped,
                       device=dev)
    W_host = None if cfg.weights_on_gpu else (W1, W3, W2)
    del W1, W3, W2
    torch.cuda.empty_cache()
    T, K, d, I = cfg.T, cfg.top_k, cfg.d, cfg.inter
    u = u_host.to(dev)
    lay.allocate(T)
    stream = torch.cuda.current_stream()

    t = time_forward(lay, u, cfg, args, world, ep_mode, local, stream)
    ms_step = t["ms_step"]
    value = T * world / (ms_step * 1e-3)
    counts = t["counts1"].cpu()
    routing = (routing_check(u, lay.centroids, t["bias0"] if cfg.gate_kind == "sigmoid" else None,
                             cfg.gate_kind, K, t["idx0"]) if not ep_mode else None)

    # ---- e2e: host batch in pinned memory -> device, forward, output back.
    # Copies run on their own stream into double buffers, so step i+1's
    # upload and step i-1's download overlap step i's kernels; every step's
    # upload and download is inside the timed region.
    u_pin = u_host.pin_memory()
    out_pin = [torch.empty((T, d), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    u_buf = [torch.empty_like(u) for _ in range(2)]
    o_buf = [torch.empty_like(u) for _ in range(2)]
    copy = torch.cuda.Stream(device=dev)
    up_done = [torch.cuda.Event() for _ in range(2)]
    fwd_done = [torch.cuda.Event() for _ in range(2)]
    down_done = [torch.cuda.Event() for _ in range(2)]

    def barrier():
        if world > 1:
            dist.barrier()

    def upload(i):
        b = i % 2
        with torch.cuda.stream(copy):
            copy.wait_event(fwd_done[b])          # buffer b free again
            u_buf[b].copy_(u_pin, non_blocking=True)
            up_done[b].record(copy)

    def e2e_run(n):
        for b in range(2):
            fwd_done[b].record(stream)
            down_done[b].record(stream)
        upload(0)
        for i in range(n):
            b = i % 2
            if i + 1 < n:
                upload(i + 1)
            stream.wait_event(up_done[b])
            stream.wait_event(down_done[b])       # o_buf[b] downloaded
            lay.forward(u_buf[b], out=o_buf[b])
            bias_step(lay, cfg, T, world, ep_mode)
            fwd_done[b].record(stream)
            with torch.cuda.stream(copy):
                copy.wait_event(fwd_done[b])
                out_pin[b].copy_(o_buf[b], non_blocking=True)
                down_done[b].record(copy)
        stream.wait_stream(copy)

    e2e_run(args.warmup)
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    e2e_run(args.steps)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = e0.elapsed_time(e1)
    if world > 1 or ep_mode:
        tt = torch.tensor([e2e_ms], device=dev)
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        e2e_ms = float(tt.item())
    e2e_value = T * world / (e2e_ms / args.steps * 1e-3)

    # ---- roofline of the dominant kernel (routed up-projection + SwiGLU)
    pk = peaks()
    # the routed rows this rank's up-projection processes: its own T*K rows,
    # or under expert parallelism the rows its experts received
    if t["recv_rows"]:
        up_rows = sum(t["recv_rows"]) / len(t["recv_rows"])
    elif hasattr(lay, "goff"):
        up_rows = int(lay.goff[-1])          # the last step's received rows (read after timing)
    else:
        up_rows = T * K
    # the recorded counters are those of the single-GPU launch
    roofline = up_kernel_roofline(cfg, lay, t, pk, up_rows,
                                  None if ep_mode else recorded_traffic(cfg.name))
    if cfg.fp8:
        roofline["limit"] = FP8_LIMIT
        try:
            roofline["cublas_fp8_tflops_live"] = cublas_fp8_tflops(dev)
        except (RuntimeError, AttributeError) as exc:   # context only
            roofline["cublas_fp8_tflops_live"] = f"not measured: {exc}"[:120]
    layer_flops = T * cfg.flops_per_token()
    layer_tflops = layer_flops / (ms_step * 1e-3) / 1e12

    result = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "e4m3 (fp32 promotion)" if cfg.fp8 else "bf16",
        "data": "synthetic (seeded; random-init weights of the V3 layer shape)",
        "config": {"workload": cfg.name, "T": T, "d": d, "n_routed": cfg.n_routed, "top_k": K,
                   "n_shared": cfg.n_shared, "inter": I, "routed_scale": cfg.routed_scale,
                   "gate": cfg.gate_kind, "global_batch_tokens": T * world,
                   "mode": ("expert-parallel over peer memory: rows stored into and read "
                            "back from the owners' buffers by the library's kernels, plan on "
                            "the device" + (", two micro-batches, the exchange of one beside "
                                            "the expert GEMMs of the other"
                                            if args.micro_batches == 2 else "")
                            if args.parallel == "ep-p2p" else
                            "expert-parallel: NCCL all-to-all dispatch/return, rows "
                            "regrouped by expert on the receiving rank" if ep_mode else
                            "fused gather" if lay.fused_gather else
                            "fused scatter and combine" if lay.fused_combine else
                            "fused scatter" if lay.fused_scatter else "five-call"),
                   "launch": "one CUDA graph per step" if t["graph"] else "eager",
                   "route": ("gate GEMM split over K, then a warp-per-token top-K pass"
                             if lay.route_split else "gate GEMM and top-K in one fused pass"),
                   "shared_expert": ("group N_r of the routed grouped GEMMs (its rows "
                                     "appended by the dispatch)"
                                     if getattr(lay, "shared_in_grouped", False) else
                                     f"side stream, overlapped, joins {lay.shared_join}"
                                     if lay.overlap_shared else "after the routed experts"),
                   "parallelism": (f"ep{world}" if ep_mode else
                                   f"dp{world}" if world > 1 else "single"),
                   "l2": "inputs larger than L2 (22.6 GB of expert weights streamed per step)"
                   if cfg.weights_on_gpu else "L2 not flushed: small workload",
                   "bias": "updated at the end of every step (the timed work), so the load "
                           "drifts toward balance over the steps",
                   "max_expert_load": {"first_timed_step": int(t["counts0"].max()),
                                       "last_timed_step": int(counts.max())},
                   "mean_expert_load": T * K / cfg.n_routed},
        "layer_tflops": layer_tflops,
        "layer_frac_of_bf16_peak": layer_tflops / pk["bf16_tflops"],
        "layer_frac_of_tensor_peak": layer_tflops / (pk["bf16_tflops"] * (2 if cfg.fp8 else 1)),
        "layer_frac_of_nominal_at_median_clock": (
            layer_tflops / (NUM_SMS * BF16_FLOP_PER_CLK_PER_SM * (2 if cfg.fp8 else 1)
                            * t["clocks"]["sm_mhz"] * 1e6 / 1e12)
            if t["clocks"].get("sm_mhz") else None),
        "target": "layer >= 60 % of the burst tensor peak (bf16 V3 prefill: <= "
                  f"{T * cfg.flops_per_token() / (0.6 * pk['bf16_tflops'] * 1e12) * 1e3:.2f} ms)",
        "roofline": roofline,
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": T * d * 2,
                "d2h_bytes_per_step": T * d * 2, "api": type(lay).__name__ + ".forward",
                "copies": "pinned host, own stream, overlapped with neighbouring steps"},
        "stage_ms": t["stage_ms"],
        "gpu_launches": args.steps * lay.launches_per_step(),
        "clocks": t["clocks"],
    }
    if routing is not None:
        result["routing"] = routing
    if T * K < 256 * cfg.n_routed:
        result["layer_hbm"] = decode_hbm(cfg, counts, ms_step, pk)

    # ---- CPU baseline: the oracle on a bounded sample (rank 0, N = 1 only)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        expert_fn = make_expert_fn(cfg, W_host)
        shared_list = ([tuple(w.float().cpu().numpy() for w in shared)]
                       if shared is not None else [])
        probe = oracle_sample(cfg, u_host, e_host, b_host, expert_fn, shared_list, 1)
        n = int(max(1, min(T, args.cpu_seconds / max(probe, 1e-3))))
        sec = oracle_sample(cfg, u_host, e_host, b_host, expert_fn, shared_list, n)
        result["cpu_baseline"] = {
            "value": n / sec, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"oracle full layer (fp64) on the first {n} of {T} tokens, {sec:.1f} s; "
                      f"host has {os.cpu_count()} cores"}

    # ---- the other V3-shape workloads, same process, after the headline line's
    # measurements: decode (HBM-bound), its softmax-gate form, FP8 prefill
    if (cfg.name == "v3p" and world == 1 and not ep_mode and args.mode == "five-call"
            and not args.no_variants):
        del lay, u, u_buf, o_buf
        torch.cuda.empty_cache()
        result["variants"] = {n: variant_line(n, args, dev, local, stream, pk)
                              for n in ("v3d", "v3d_softmax", "v3p_fp8")}

    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1 or ep_mode:
        if hasattr(lay, "close"):
            lay.close()
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
