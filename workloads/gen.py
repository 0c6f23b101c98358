"""Seeded generators for Q, K, V and per-head dual-window parameters.

Q and K carry spatio-temporal structure through random-Fourier features of
the token position, so that pooled block scores concentrate near the query
tile the way the pages describe video-DiT heads (Compact Attention, Fig. 2:
heads concentrate attention mass in coarse local / axial regions).

Recipe (per head h, token at frame t, row y, column x):
  p        = (t, y / 8, x / 8)                      position in tile units
  omega_m  ~ N(0, I_3 / ell_h^2),  b_m ~ U[0, 2 pi)  for m = 1..32
  phi(p)   = [cos(omega_m . p + b_m), sin(omega_m . p + b_m)]_m / sqrt(32)
  q = a R phi(p) + 0.5 eps,   k = a R phi(p) + 0.5 eps',   a^2 = 40 sqrt(d)
  v ~ N(0, 1)
with R (d x 64) orthonormal columns from the QR factor of a Gaussian matrix.
The amplitude makes the pooled self-pair logit about 40: with it, top-p 0.95
alone keeps about 8% of the key tiles of the 75,600-token layer, so that the
dual windows bring the union to the intended ~15%.
Everything is rounded to bf16 once. Random numbers come from torch's
generator seeded with the workload seed, on the device the caller names.
"""
import math

import numpy as np
import torch

from .configs import WorkloadConfig, tile_counts

N_FREQ = 32
LOGIT_SCALE = 40.0  # a^2 / sqrt(d)


def _ells(cfg: WorkloadConfig, g: torch.Generator, device) -> list:
    if cfg.ell_fixed:
        return [float(cfg.ell[h % len(cfg.ell)]) for h in range(cfg.heads)]
    lo, hi = cfg.ell
    u = torch.rand(cfg.heads, generator=g, device=device, dtype=torch.float64)
    return [float(lo + (hi - lo) * x) for x in u.cpu().tolist()]


@torch.no_grad()
def make_qkv(cfg: WorkloadConfig, device="cpu", dtype=torch.bfloat16, amplitude=None):
    """Return Q, K, V in raster layout [B, L, heads, d] (bf16), L = T*H*W.

    The raster token index is (t*H + y)*W + x.
    """
    device = torch.device(device)
    g = torch.Generator(device=device)
    g.manual_seed(int(cfg.seed))
    B, L, Hh, d = cfg.B, cfg.L, cfg.heads, cfg.d
    a = math.sqrt(LOGIT_SCALE * math.sqrt(d)) if amplitude is None else float(amplitude)
    ells = _ells(cfg, g, device)

    t = torch.arange(cfg.T, device=device, dtype=torch.float32)
    y = torch.arange(cfg.H, device=device, dtype=torch.float32) / 8.0
    x = torch.arange(cfg.W, device=device, dtype=torch.float32) / 8.0
    pos = torch.stack(torch.meshgrid(t, y, x, indexing="ij"), dim=-1).reshape(L, 3)

    q = torch.empty(B, L, Hh, d, device=device, dtype=dtype)
    k = torch.empty(B, L, Hh, d, device=device, dtype=dtype)
    v = torch.empty(B, L, Hh, d, device=device, dtype=dtype)
    for b in range(B):
        for h in range(Hh):
            omega = torch.randn(N_FREQ, 3, generator=g, device=device) / ells[h]
            phase = torch.rand(N_FREQ, generator=g, device=device) * (2.0 * math.pi)
            ang = pos @ omega.T + phase
            phi = torch.cat([torch.cos(ang), torch.sin(ang)], dim=1) / math.sqrt(N_FREQ)
            gauss = torch.randn(d, 2 * N_FREQ, generator=g, device=device)
            rot, _ = torch.linalg.qr(gauss)  # d x 64, orthonormal columns
            base = a * (phi @ rot.T)
            q[b, :, h, :] = (base + 0.5 * torch.randn(L, d, generator=g, device=device)).to(dtype)
            k[b, :, h, :] = (base + 0.5 * torch.randn(L, d, generator=g, device=device)).to(dtype)
            v[b, :, h, :] = torch.randn(L, d, generator=g, device=device).to(dtype)
    return q, k, v


@torch.no_grad()
def perturb_step(master: torch.Tensor, g: torch.Generator):
    """One reuse step: X <- 0.95 X + 0.31 N(0, 1), on an fp32 master copy.

    Returns the updated fp32 master and its bf16 rounding.
    """
    noise = torch.randn(master.shape, generator=g, device=master.device, dtype=torch.float32)
    master = 0.95 * master + 0.31 * noise
    return master, master.to(torch.bfloat16)


def fixed_windows_tiny(cfg: WorkloadConfig) -> np.ndarray:
    """Windows of the tiny case: for |dt| = 0 a local window of radius 1 tile
    and an axial window spanning the whole tile row; nothing for |dt| >= 1
    (groups (0, 1), the last group being open-ended)."""
    _, nw, _, _ = tile_counts(cfg.T, cfg.H, cfg.W)
    w = np.full((cfg.heads, 2, 4), -1, dtype=np.int32)
    w[:, 0, :] = (1, 1, 0, nw - 1)
    return w


KINDS = ("local", "axial_x", "axial_y", "cross", "global")

_SCALES = None


def window_scale(workload: str, which: int = 0) -> float:
    """Window scale meeting the workload's density target number `which`
    (stored by the calibration script beside the oracle)."""
    global _SCALES
    if _SCALES is None:
        import json
        import os
        with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "window_scales.json")) as f:
            _SCALES = json.load(f)
    return float(_SCALES[workload][which]["scale"])


def window_params(cfg: WorkloadConfig, scale: float) -> np.ndarray:
    """Per-head dual-window extents, int32 [heads, G, 4] = (ry1, rx1, ry2, rx2).

    Each head draws one of the five kinds of Compact Attention's Table III
    (locality / cross / global, time-variant or time-invariant) and a size
    jitter; `scale` grows every extent together (0 gives one tile per frame).
    Extents are half-widths in tiles; -1 switches a window off.
    """
    nh, nw, _, _ = tile_counts(cfg.T, cfg.H, cfg.W)
    G = len(cfg.group_lo)
    rng = np.random.Generator(np.random.PCG64(1000 + cfg.seed))
    out = np.full((cfg.heads, G, 4), -1, dtype=np.int32)
    for h in range(cfg.heads):
        kind = int(rng.integers(0, len(KINDS)))
        jitter = float(rng.uniform(0.6, 1.4))
        time_variant = bool(rng.random() < 0.5)
        gamma = float(rng.uniform(0.35, 0.8)) if time_variant else 1.0
        for gi in range(G):
            f = scale * jitter * gamma ** gi

            def ey(c):
                return min(nh - 1, int(math.floor(c * f * nh)))

            def ex(c):
                return min(nw - 1, int(math.floor(c * f * nw)))

            if KINDS[kind] == "local":
                w = (ey(0.5), ex(0.5), -1, -1)
            elif KINDS[kind] == "axial_x":
                w = (ey(0.25), ex(0.25), ey(0.08), ex(2.0))
            elif KINDS[kind] == "axial_y":
                w = (ey(0.25), ex(0.25), ey(2.0), ex(0.08))
            elif KINDS[kind] == "cross":
                w = (ey(0.08), ex(2.0), ey(2.0), ex(0.08))
            else:
                w = (ey(1.0), ex(1.0), -1, -1)
            out[h, gi, :] = w
    return out
