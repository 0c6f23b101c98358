"""Runs every entry point of the library on small seeded cases and saves the
outputs and device statuses to an .npz file (argv[1]). The checked-build
test runs it twice, once with STA_CHECKED=1 (libsta_debug.so: device-side
bounds checks compiled in) and once with the product library, and compares.
Needs a GPU; imports nothing from the oracle."""
import os
import sys

import numpy as np
import torch

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import block_sparse_attention_28_b200 as sta  # noqa: E402
from workloads import make_qkv, window_params  # noqa: E402
from workloads.configs import WorkloadConfig  # noqa: E402

out = {}


def keep(name, t):
    out[name] = t.detach().cpu().numpy() if isinstance(t, torch.Tensor) else np.asarray(t)


def status(name):
    torch.cuda.synchronize()
    out["status_" + name] = np.int64(sta.sta_get_device_error())


def tiled(x, B, Hh, d, g):
    y = torch.zeros((B, Hh, sta.sta_tiled_len(g), d), dtype=torch.bfloat16, device="cuda")
    sta.sta_reorder(x, y, B, Hh, d, g)
    return y


def case(tag, T, H, W, Hh, d, top_p, k_min, seed, G=2, head_floor=False):
    cfg = WorkloadConfig(name=tag, B=1, heads=Hh, d=d, T=T, H=H, W=W, seed=seed, use_scores=True,
                         group_lo=(0, 2)[:G])
    q, k, v = (x.cuda() for x in make_qkv(cfg, device="cpu"))
    B, g = 1, sta.grid(T, H, W)
    nt = sta.sta_num_tiles(g)
    qt, kt, vt = (tiled(x, B, Hh, d, g) for x in (q, k, v))
    back = torch.zeros_like(q)
    sta.sta_reorder(qt, back, B, Hh, d, g, inverse=True)
    status(tag + "_reorder")
    keep(tag + "_qt", qt.view(torch.int16))
    keep(tag + "_back", back.view(torch.int16))

    win = torch.from_numpy(window_params(cfg, 0.5)).cuda()
    params = sta.mask_params(top_p, k_min, True, 0.0, cfg.group_lo, win, head_floor=head_floor)
    bufs = sta.build_mask(qt, kt, B, Hh, d, g, params, sta.MaskBuffers(B, Hh, d, g, "cuda", True, True))
    status(tag + "_build")
    nnz = int(bufs.nnz.item())
    keep(tag + "_row_ptr", bufs.row_ptr)
    keep(tag + "_col_idx", bufs.col_idx[:nnz])
    keep(tag + "_mask", bufs.block_mask)
    keep(tag + "_probs", bufs.block_probs)

    rb = sta.MaskBuffers(B, Hh, d, g, "cuda")
    sta.build_mask(q, k, B, Hh, d, g, params, rb, raster=True)
    status(tag + "_build_raster")
    keep(tag + "_col_idx_raster", rb.col_idx[: int(rb.nnz.item())])

    mb = sta.MaskBuffers(B, Hh, d, g, "cuda")
    mb.ws_bytes = sta.sta_build_mask_workspace_min(B, Hh, d, g)
    mb.workspace = torch.empty(max(1, mb.ws_bytes), dtype=torch.uint8, device="cuda")
    sta.build_mask(qt, kt, B, Hh, d, g, params, mb)
    status(tag + "_build_min_ws")
    keep(tag + "_col_idx_min_ws", mb.col_idx[: int(mb.nnz.item())])

    rp, ci = bufs.row_ptr, bufs.col_idx
    o = torch.zeros_like(qt)
    lse = torch.zeros(qt.shape[:3], dtype=torch.float32, device="cuda")
    sta.sta_attn_fwd(qt, kt, vt, o, lse, rp, ci, B, Hh, d, g)
    status(tag + "_attn")
    keep(tag + "_o", o.view(torch.int16))
    keep(tag + "_lse", lse)

    o_r = torch.zeros_like(q)
    lse_r = torch.zeros_like(lse)
    sta.sta_attn_fwd_raster(q, k, v, o_r, lse_r, rp, ci, B, Hh, d, g)
    status(tag + "_attn_raster")
    keep(tag + "_o_raster", o_r.view(torch.int16))

    mass = torch.zeros((B, Hh, nt, nt), dtype=torch.float32, device="cuda")
    o_m = torch.zeros_like(qt)
    lse_m = torch.zeros_like(lse)
    sta.sta_attn_fwd_block_mass(qt, kt, vt, o_m, lse_m, rp, ci, lse, mass, B, Hh, d, g)
    status(tag + "_block_mass")
    keep(tag + "_mass", mass)

    ws_bytes = sta.sta_rectified_workspace(B, Hh, d, g)
    ws = torch.empty(max(1, ws_bytes), dtype=torch.uint8, device="cuda")
    o_x = torch.zeros_like(qt)
    lse_x = torch.zeros_like(lse)
    sta.sta_attn_fwd_rectified(qt, kt, vt, o_x, lse_x, rp, ci, ws, ws_bytes, B, Hh, d, g)
    status(tag + "_rectified")
    keep(tag + "_o_rect", o_x.view(torch.int16))

    # the overlap pairing of the query tiles and the paired calls
    qp = torch.full((B * Hh, 2 * ((nt + 1) // 2)), -7, dtype=torch.int32, device="cuda")
    pb = sta.MaskBuffers(B, Hh, d, g, "cuda")
    sta.build_mask(qt, kt, B, Hh, d, g, sta.mask_params(0.0, max(1, nt // 8), True, 0.0, cfg.group_lo,
                                                        query_pairs=qp), pb)
    status(tag + "_build_pairs")
    keep(tag + "_query_pairs", qp)
    o_p = torch.zeros_like(qt)
    sta.sta_attn_fwd_paired(qt, kt, vt, o_p, None, pb.row_ptr, pb.col_idx, qp, B, Hh, d, g)
    status(tag + "_attn_paired")
    keep(tag + "_o_paired", o_p.view(torch.int16))
    o_pr = torch.zeros_like(q)
    sta.sta_attn_fwd_raster_paired(q, k, v, o_pr, None, pb.row_ptr, pb.col_idx, qp, B, Hh, d, g)
    status(tag + "_attn_raster_paired")
    keep(tag + "_o_raster_paired", o_pr.view(torch.int16))

    w_out = torch.zeros((B * Hh, len(cfg.group_lo), 4), dtype=torch.int32, device="cuda")
    stats = torch.zeros((B * Hh, 2), dtype=torch.float32, device="cuda")
    sta.sta_search_windows(mass, B, Hh, g, cfg.group_lo, 0.9, 0.5, w_out, stats)
    status(tag + "_search")
    keep(tag + "_windows", w_out)


if __name__ == "__main__":
    out["debug_build"] = np.int64(sta.sta_debug_build())
    case("ragged128", 3, 19, 37, 3, 128, 0.9, 2, 11)
    case("small64", 4, 16, 16, 2, 64, 0.8, 3, 12, head_floor=True)
    case("onetile", 1, 8, 8, 1, 128, 0.5, 1, 13, G=1)
    np.savez(sys.argv[1], **out)
    print("saved", len(out), "arrays")
