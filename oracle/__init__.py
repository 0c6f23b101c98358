"""CPU oracle for block-sparse 3D-tile attention (test infrastructure).

A plain, slow fp64 numpy restatement of what the hot path computes: token
reorder into 1x8x8 tiles, mean-pooled block scores, hybrid top-p / k_min
selection, the per-head deformable dual-window mask, CSR emission and
masked softmax attention. It shares no code with the CUDA library and is
never used by it: only the tests, the smoke check and the benchmark's CPU
baseline import this package.

Sources (pages on block-sparse attention for video diffusion transformers):
  * Compact Attention (abstract; Fig. 1(3), Fig. 3, Fig. 4; Table III):
    tile-aligned masks, dual windows per temporal-distance group, masks
    loaded into block-sparse attention kernels.
  * Rectified SpaAttn (abstract): pooled query-key block scores.
  * SCOPE review (Eqs. (7)-(8) as quoted; abstract): hybrid top-p / fixed
    top-k selection; Eqs. (9)-(10): the online per-head top-k floor.
  * AdaSpa (abstract): exact block importance from a cached log-sum-exp.
  * Compact Attention Figs. 3-5: recall-driven offline window search.
  * Rectified SpaAttn (abstract): rectified attention, skipped tiles
    recovered from pooled keys and values (reading stated in the module).
  * The query-tile pairing the library emits with a mask (no counterpart in
    the pages; a scheduling choice of its attention kernels, restated so
    that the GPU's output can be checked).

Parity pins: every function here is checked in tests/test_oracle.py
against closed forms, textbook routines (torch SDPA in fp64, scipy
softmax, stable argsort) or brute force; none of the pages prints a worked
numeric example for this path, so no pin comes from a printed value.
"""
from .sta_oracle import (  # noqa: F401
    TILE,
    tile_grid,
    tiled_row_of_raster,
    valid_rows,
    reorder_fwd,
    reorder_inv,
    pool,
    block_scores,
    select_row,
    select,
    head_topk_floor,
    select_with_head_floor,
    tile_sizes,
    window_mask,
    build_mask,
    mask_to_csr,
    attention_rows,
    attention_all,
    block_mass,
    search_windows,
    pooled_kv,
    rectified_attention_rows,
    SEARCH_MOVES,
    PAIR_OFFSETS,
    default_pairs,
    pairs_union,
    pair_query_tiles,
)
