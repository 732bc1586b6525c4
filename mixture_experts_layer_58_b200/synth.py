"""Seeded synthetic inputs for the DeepSeekMoE layer.

This module only draws numbers: it holds none of the layer's arithmetic (no
affinity, no top-k, no gate, no FFN). The CUDA path and the fp64 oracle both
consume what it returns, so a parity test compares the two on the very same
bf16 values.

Workloads (shapes from the DeepSeek-V3 technical-report summary, xyznot.com,
"Main ideas": 1 shared + 256 routed experts, 8 active; the model-architecture
page, deepseekmodel.com, MTP listing: hidden size 7168):

  tiny         T=64    d=256  N_r=16  K=4 N_s=1 I=128  S=1.0 b~U(-0.01,0.01)
  mid          T=4096  d=2048 N_r=64  K=6 N_s=2 I=1408 S=1.0 b=0, 16 bias steps
  v3p          T=16384 d=7168 N_r=256 K=8 N_s=1 I=2048 S=2.5 b~U(-0.05,0.05),
               Zipf(1.1)-skewed centroids (hottest expert ~10x the mean load)
  v3d          T=128   same shapes as v3p, uniform routing, S=2.5
  v3d_softmax  v3d with the softmax-over-top-k gate, no bias, S=1.0
  v3p_fp8      v3p inputs; FP8 E4M3 expert weights (128x128 blocks) and
               activations (1x128 tiles)
  v3p_small    profiling-size case with the V3 expert shapes: T=4096, 32 experts
  v3p_small_fp8  the same in the FP8 variant

Distributions: u ~ N(0,1); centroids and all expert / shared weights
~ N(0, 0.02^2) (0.02 is the standard deviation); every float tensor is drawn
in fp32 from a seeded torch generator and rounded once to bf16.

Skew (v3p): e_i = n_i + alpha * w_i * v with n_i ~ N(0,0.02^2) per element,
v a fixed random unit vector (seed 1), w_i = rank_i^-1.1 over a seeded random
permutation of the experts (rank 1 = hottest). alpha was found once by
bisection on the oracle's routing of the seed-0 batch so that the most loaded
expert receives about 10 * T*K/N_r tokens; the value is stored below
(oracle/calibrate_zipf.py reproduces it).

Where the weights live: for the small workloads they are drawn on the host so
that CPU-only tests can use them; for the V3-shape workloads (22.6 GB of bf16
expert weights) each expert is drawn directly on the GPU by torch's CUDA
generator with a per-expert seed, and a parity test copies the slices it needs
back to the host. The CPU and CUDA generators produce different streams, so a
tensor's values depend on the device it was drawn on; every test takes all
values for both sides from one draw.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass

import torch

# alpha for the v3p centroid skew (bisection result, see module docstring).
V3P_ZIPF_ALPHA = 6.515


@dataclass(frozen=True)
class MoEConfig:
    name: str
    T: int                 # tokens in the batch
    d: int                 # hidden size
    n_routed: int          # N_r
    top_k: int             # K_r
    n_shared: int          # N_s
    inter: int             # SwiGLU intermediate width I of one expert
    routed_scale: float    # S, multiplies the normalised gates
    gate_kind: str = "sigmoid"      # "sigmoid" (bias-adjusted) or "softmax" (top-k logits)
    bias_lo: float = 0.0
    bias_hi: float = 0.0
    zipf_s: float = 0.0             # 0 = no skew
    zipf_alpha: float = 0.0
    gamma: float = 0.001
    bias_steps: int = 1
    fp8: bool = False
    seed: int = 0
    weights_on_gpu: bool = False    # draw expert weights on the CUDA device

    def replace(self, **kw) -> "MoEConfig":
        return dataclasses.replace(self, **kw)

    @property
    def shared_inter(self) -> int:
        return self.n_shared * self.inter

    def flops_per_token(self) -> float:
        """Algorithmic multiply-add flops of one token through the layer:
        gate GEMM + K routed SwiGLU FFNs + the shared FFN(s)."""
        gate = 2.0 * self.d * self.n_routed
        ffn = 2.0 * self.d * 3 * self.inter          # W1, W3 (d->I) and W2 (I->d)
        return gate + ffn * (self.top_k + self.n_shared)


CONFIGS = {
    "tiny": MoEConfig("tiny", T=64, d=256, n_routed=16, top_k=4, n_shared=1, inter=128,
                      routed_scale=1.0, bias_lo=-0.01, bias_hi=0.01, bias_steps=1),
    "mid": MoEConfig("mid", T=4096, d=2048, n_routed=64, top_k=6, n_shared=2, inter=1408,
                     routed_scale=1.0, bias_steps=16),
    "v3p": MoEConfig("v3p", T=16384, d=7168, n_routed=256, top_k=8, n_shared=1, inter=2048,
                     routed_scale=2.5, bias_lo=-0.05, bias_hi=0.05, zipf_s=1.1,
                     zipf_alpha=V3P_ZIPF_ALPHA, weights_on_gpu=True),
    "v3d": MoEConfig("v3d", T=128, d=7168, n_routed=256, top_k=8, n_shared=1, inter=2048,
                     routed_scale=2.5, bias_lo=-0.05, bias_hi=0.05, weights_on_gpu=True),
    "v3d_softmax": MoEConfig("v3d_softmax", T=128, d=7168, n_routed=256, top_k=8, n_shared=1,
                             inter=2048, routed_scale=1.0, gate_kind="softmax",
                             weights_on_gpu=True),
    # profiling-size case of the V3 expert shapes (32 experts, ~5 GB on the device)
    "v3p_small": MoEConfig("v3p_small", T=4096, d=7168, n_routed=32, top_k=8, n_shared=1,
                           inter=2048, routed_scale=2.5, bias_lo=-0.05, bias_hi=0.05,
                           weights_on_gpu=True),
    "v3p_fp8": MoEConfig("v3p_fp8", T=16384, d=7168, n_routed=256, top_k=8, n_shared=1,
                         inter=2048, routed_scale=2.5, bias_lo=-0.05, bias_hi=0.05, zipf_s=1.1,
                         zipf_alpha=V3P_ZIPF_ALPHA, fp8=True, weights_on_gpu=True),
    # profiling-size case of the FP8 variant
    "v3p_small_fp8": MoEConfig("v3p_small_fp8", T=4096, d=7168, n_routed=32, top_k=8,
                               n_shared=1, inter=2048, routed_scale=2.5, bias_lo=-0.05,
                               bias_hi=0.05, fp8=True, weights_on_gpu=True),
}

# Per-tensor seed streams (added to 1000 * cfg.seed).
_S_U, _S_CENT, _S_BIAS, _S_SKEW, _S_SHARED, _S_EXPERT = 1, 2, 3, 4, 5, 100


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _normal_bf16(shape, std: float, seed: int, device="cpu") -> torch.Tensor:
    g = _gen(device, seed)
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(torch.bfloat16)


def tokens(cfg: MoEConfig, T: int | None = None) -> torch.Tensor:
    """u [T, d] bf16 on the host, u ~ N(0,1). T defaults to cfg.T; a smaller T
    returns the first T rows of the same draw."""
    u = _normal_bf16((cfg.T, cfg.d), 1.0, 1000 * cfg.seed + _S_U)
    return u if T is None else u[:T].contiguous()


def zipf_direction(cfg: MoEConfig):
    """(v, w): v a unit vector [d] (fp32) and w [N_r] the Zipf weight of each
    expert, w_i = rank_i^-s over a seeded random permutation."""
    g = _gen("cpu", 1)
    v = torch.randn(cfg.d, generator=g, dtype=torch.float64)
    v = v / v.norm()
    perm = torch.randperm(cfg.n_routed, generator=g)
    rank = torch.empty(cfg.n_routed, dtype=torch.float64)
    rank[perm] = torch.arange(1, cfg.n_routed + 1, dtype=torch.float64)
    w = rank.pow(-cfg.zipf_s)
    return v, w


def centroids(cfg: MoEConfig, alpha: float | None = None) -> torch.Tensor:
    """e [N_r, d] bf16 on the host. With cfg.zipf_s > 0 a shared direction
    scaled by alpha * w_i is added before the bf16 rounding."""
    g = _gen("cpu", 1000 * cfg.seed + _S_CENT)
    e = torch.randn((cfg.n_routed, cfg.d), generator=g, dtype=torch.float32) * 0.02
    if cfg.zipf_s > 0.0:
        a = cfg.zipf_alpha if alpha is None else alpha
        v, w = zipf_direction(cfg)
        e = (e.double() + a * w[:, None] * v[None, :]).float()
    return e.to(torch.bfloat16)


def bias(cfg: MoEConfig) -> torch.Tensor:
    """b [N_r] fp32 on the host, U(bias_lo, bias_hi) (all zero when lo == hi == 0)."""
    if cfg.bias_lo == 0.0 and cfg.bias_hi == 0.0:
        return torch.zeros(cfg.n_routed, dtype=torch.float32)
    g = _gen("cpu", 1000 * cfg.seed + _S_BIAS)
    r = torch.rand(cfg.n_routed, generator=g, dtype=torch.float32)
    return (cfg.bias_lo + (cfg.bias_hi - cfg.bias_lo) * r).float()


def expert_weights(cfg: MoEConfig, e: int, device="cpu"):
    """(w1 [I,d], w3 [I,d], w2 [d,I]) bf16 of routed expert e, drawn on `device`."""
    base = 1000 * cfg.seed + _S_EXPERT + 3 * e
    I, d = cfg.inter, cfg.d
    return (_normal_bf16((I, d), 0.02, base, device),
            _normal_bf16((I, d), 0.02, base + 1, device),
            _normal_bf16((d, I), 0.02, base + 2, device))


def shared_weights(cfg: MoEConfig, device="cpu"):
    """(ws1 [N_s*I, d], ws3 [N_s*I, d], ws2 [d, N_s*I]) bf16. Shared expert j
    owns rows j*I:(j+1)*I of ws1/ws3 and columns j*I:(j+1)*I of ws2."""
    if cfg.n_shared == 0:
        return None
    base = 1000 * cfg.seed + _S_SHARED * 10
    I, d = cfg.shared_inter, cfg.d
    return (_normal_bf16((I, d), 0.02, base, device),
            _normal_bf16((I, d), 0.02, base + 1, device),
            _normal_bf16((d, I), 0.02, base + 2, device))


def all_expert_weights(cfg: MoEConfig, device="cpu"):
    """Stacked (W1 [N_r,I,d], W3 [N_r,I,d], W2 [N_r,d,I]) bf16 on `device`,
    expert e equal to expert_weights(cfg, e, device)."""
    I, d, n = cfg.inter, cfg.d, cfg.n_routed
    W1 = torch.empty((n, I, d), dtype=torch.bfloat16, device=device)
    W3 = torch.empty((n, I, d), dtype=torch.bfloat16, device=device)
    W2 = torch.empty((n, d, I), dtype=torch.bfloat16, device=device)
    for e in range(n):
        a, b, c = expert_weights(cfg, e, device)
        W1[e].copy_(a)
        W3[e].copy_(b)
        W2[e].copy_(c)
    return W1, W3, W2
