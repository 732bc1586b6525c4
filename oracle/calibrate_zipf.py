"""Find alpha for the Zipf-skewed V3-shape prefill centroids.

e_i = N(0, 0.02^2) + alpha * w_i * v (see mixture_experts_layer_58_b200/synth.py);
alpha is bisected so that, under the oracle's routing of the seed-0 batch
(bias included), the most loaded expert receives about 10x the mean load
T*K/N_r. Run once: `python -m oracle.calibrate_zipf`; the printed alpha is the
constant stored in synth.py. Calls only the oracle and the input generator.
"""
from __future__ import annotations

import sys
import time

import numpy as np

from oracle import moe_oracle as om


def max_load(cfg, u64, alpha: float) -> int:
    from mixture_experts_layer_58_b200 import synth
    e = synth.centroids(cfg, alpha=alpha)
    b = synth.bias(cfg)
    r = om.route(u64, e, b, cfg.top_k, cfg.routed_scale, cfg.gate_kind)
    return int(r.counts.max())


def main(target_ratio: float = 10.0, iters: int = 18) -> float:
    from mixture_experts_layer_58_b200 import synth
    cfg = synth.CONFIGS["v3p"]
    u64 = synth.tokens(cfg).float().numpy().astype(np.float64)
    target = target_ratio * cfg.T * cfg.top_k / cfg.n_routed
    lo, hi = 0.0, 1.0
    while max_load(cfg, u64, hi) < target:
        hi *= 2.0
    for _ in range(iters):
        mid = 0.5 * (lo + hi)
        t0 = time.time()
        m = max_load(cfg, u64, mid)
        print(f"alpha={mid:.6f} max_load={m} target={target:.0f} ({time.time() - t0:.1f}s)",
              file=sys.stderr)
        if m < target:
            lo = mid
        else:
            hi = mid
    alpha = float(f"{hi:.4g}")
    print(f"alpha={alpha} max_load={max_load(cfg, u64, alpha)}")
    return alpha


if __name__ == "__main__":
    main()
