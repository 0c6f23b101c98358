"""Saving and loading the reusable part of a built mask (the CSR lists, the
window extents and the query-tile pairing), so that a mask built at one
denoising step can be stored and used again at later steps or in a later
process (mask reuse across steps: Compact Attention Fig. 3). Plain file I/O
with torch.save / torch.load; nothing of the method is computed here.
"""
import torch

FORMAT = "sta-mask-v1"


def save_mask(path, bufs, B, heads, d, grid, windows=None, group_lo=None, query_pairs=None):
    """Write the CSR of `bufs` (a MaskBuffers filled by build_mask), trimmed to
    its nnz, with the sizes it belongs to and, when given, the window extents
    [heads, G, 4], their group bounds and the query-tile pairing."""
    nnz = int(bufs.nnz.item())
    blob = {
        "format": FORMAT,
        "B": int(B), "heads": int(heads), "d": int(d),
        "grid": (int(grid.T), int(grid.H), int(grid.W)),
        "row_ptr": bufs.row_ptr.detach().cpu(),
        "col_idx": bufs.col_idx[:nnz].detach().cpu(),
        "nnz": nnz,
        "windows": None if windows is None else windows.detach().cpu(),
        "group_lo": None if group_lo is None else tuple(int(x) for x in group_lo),
        "query_pairs": None if query_pairs is None else query_pairs.detach().cpu(),
    }
    torch.save(blob, path)


def load_mask(path, device="cuda"):
    """Read a file of save_mask. Returns a dict with the sizes and the tensors
    on `device`: row_ptr, col_idx (capacity B*heads*Nt*Nt, as sta_build_mask
    writes it, the first nnz entries filled), nnz (device int64 [1]), and
    windows / query_pairs when saved."""
    blob = torch.load(path, map_location="cpu", weights_only=True)  # tensors and plain values only
    if blob.get("format") != FORMAT:
        raise ValueError(f"{path}: not a saved sta mask")
    T, H, W = blob["grid"]
    nt = T * ((H + 7) // 8) * ((W + 7) // 8)
    R = blob["B"] * blob["heads"] * nt
    if blob["row_ptr"].numel() != R + 1 or int(blob["row_ptr"][-1]) != blob["nnz"]:
        raise ValueError(f"{path}: CSR does not match its sizes")
    col_idx = torch.empty(max(1, R * nt), dtype=torch.int32, device=device)
    col_idx[: blob["nnz"]] = blob["col_idx"].to(device)
    out = dict(blob)
    out["row_ptr"] = blob["row_ptr"].to(device)
    out["col_idx"] = col_idx
    out["nnz"] = torch.tensor([blob["nnz"]], dtype=torch.int64, device=device)
    for k in ("windows", "query_pairs"):
        if blob[k] is not None:
            out[k] = blob[k].to(device)
    return out
