"""Choose the dual-window scale of each workload so that the oracle's mask
density meets the workload's target, and store the scales.

Run once:  python -m oracle.calibrate_windows
Writes workloads/window_scales.json. It calls only the oracle and the seeded
generators (inputs drawn on the CPU); nothing here touches the CUDA path.
Density = kept (query tile, key tile) pairs / (heads * Nt^2), window mask
OR'd with the score selection where the workload has one.
"""
import json
import math
import os
import sys

import numpy as np

from workloads import CONFIGS, make_qkv, window_params
from . import sta_oracle as O

OUT = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "workloads", "window_scales.json")


def _select_mask(cfg):
    q, k, _ = make_qkv(cfg, device="cpu")
    T, H, W = cfg.T, cfg.H, cfg.W
    _, _, nt, _ = O.tile_grid(T, H, W)
    sel = np.zeros((cfg.heads, nt, nt), dtype=bool)
    scale = 1.0 / math.sqrt(cfg.d)
    for h in range(cfg.heads):
        qt = O.reorder_fwd(q[:, :, h:h + 1].float().numpy(), T, H, W)
        kt = O.reorder_fwd(k[:, :, h:h + 1].float().numpy(), T, H, W)
        _, p = O.block_scores(O.pool(qt, T, H, W), O.pool(kt, T, H, W), scale)
        sel[h] = O.select(p[0, 0], cfg.top_p, cfg.k_min)
        print(f"  head {h}: select density {sel[h].mean():.4f}", file=sys.stderr)
    return sel


def _density(cfg, scale, base):
    w = window_params(cfg, scale)
    m = O.window_mask(w, cfg.group_lo, cfg.T, cfg.H, cfg.W)
    if base is not None:
        m |= base
    return float(m.mean())


def calibrate(cfg, target, base):
    lo, hi = 0.0, 4.0
    for _ in range(30):
        mid = 0.5 * (lo + hi)
        if _density(cfg, mid, base) < target:
            lo = mid
        else:
            hi = mid
    # the density is a step function of the scale: take the closer side
    dlo, dhi = _density(cfg, lo, base), _density(cfg, hi, base)
    return (lo, dlo) if abs(dlo - target) <= abs(dhi - target) else (hi, dhi)


def main():
    out = {}
    for idx, cfg in CONFIGS.items():
        if not cfg.window_density:
            continue
        base = _select_mask(cfg) if cfg.use_scores else None
        if base is not None:
            out[f"{idx}_select_density"] = float(base.mean())
        scales = []
        for target in cfg.window_density:
            s, dens = calibrate(cfg, target, base)
            print(f"config {idx}: target {target:.3f} -> scale {s:.6f}, density {dens:.4f}", file=sys.stderr)
            scales.append({"target": target, "scale": s, "density": dens})
        out[str(idx)] = scales
    with open(OUT, "w") as f:
        json.dump(out, f, indent=1)
    print(f"wrote {OUT}", file=sys.stderr)


if __name__ == "__main__":
    main()
