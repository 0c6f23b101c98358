"""Workload shapes of the five synthetic layers.

Shapes follow the video-DiT layers the Compact Attention page measures on
(Wan2.1 at "80K" tokens, 40 heads; Table II) and the ~110K-token 720p
HunyuanVideo case on the AdaSpa page (abstract), with d = 128.
Each entry is plain data: grid size, heads, head dim, and the mask recipe.
"""
from dataclasses import dataclass, field
from typing import Optional, Tuple


@dataclass(frozen=True)
class WorkloadConfig:
    name: str
    B: int
    heads: int
    d: int
    T: int
    H: int
    W: int
    seed: int
    # mask recipe
    use_scores: bool
    top_p: float = 0.0
    k_min: int = 0
    group_lo: Tuple[int, ...] = (0,)
    # window density targets (fraction of (query tile, key tile) pairs)
    window_density: Tuple[float, ...] = ()
    # length scale range of the random-Fourier features, in tiles
    ell: Tuple[float, ...] = (1.0, 12.0)
    ell_fixed: bool = False
    # fixed-density sweep (reuse config): fraction of key tiles per row
    fixed_densities: Tuple[float, ...] = ()
    reuse_steps: int = 0
    note: str = ""

    @property
    def L(self) -> int:
        return self.T * self.H * self.W


def tile_counts(T: int, H: int, W: int):
    """Number of 1x8x8 tiles along (t, y, x) and in total; padded length."""
    nh = -(-H // 8)
    nw = -(-W // 8)
    nt = T * nh * nw
    return nh, nw, nt, 64 * nt


CONFIGS = {
    "tiny": WorkloadConfig(
        name="tiny_4x16x16_h2_d64", B=1, heads=2, d=64, T=4, H=16, W=16, seed=0,
        use_scores=True, top_p=0.9, k_min=2, group_lo=(0, 1),
        ell=(2.0, 6.0), ell_fixed=True,
        note="tiny reference case; fixed local 1x1 + full-row axial window"),
    "dit480p": WorkloadConfig(
        name="dit480p_21x30x52_h40_d128_win25", B=1, heads=40, d=128, T=21, H=30, W=52, seed=1,
        use_scores=False, group_lo=(0, 1, 4), window_density=(0.25,),
        note="dual-window masks only, ~25% density"),
    "dit720p": WorkloadConfig(
        name="dit720p_21x45x80_h40_d128_p95k8_d15", B=1, heads=40, d=128, T=21, H=45, W=80, seed=2,
        use_scores=True, top_p=0.95, k_min=8, group_lo=(0, 1, 4), window_density=(0.15,),
        note="online top-p 0.95 / k_min 8 OR dual windows, ~15% overall density"),
    "dit720p_129f": WorkloadConfig(
        name="dit720p129f_33x45x80_h24_d128_win", B=1, heads=24, d=128, T=33, H=45, W=80, seed=3,
        use_scores=False, group_lo=(0, 1, 3, 7), window_density=(0.05, 0.10, 0.20, 0.30),
        note="dual-window masks, 4 temporal groups, density sweep"),
    "reuse480p": WorkloadConfig(
        name="reuse_21x30x52_h40_d128", B=1, heads=40, d=128, T=21, H=30, W=52, seed=4,
        use_scores=True, top_p=0.0, group_lo=(0,),
        fixed_densities=(0.05, 0.10, 0.25, 0.50, 1.00), reuse_steps=10,
        note="mask built once at step 0 and reused over 10 perturbed steps"),
}
