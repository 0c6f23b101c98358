"""Saving and loading a built mask (block_sparse_attention_28_b200.maskio): the
CSR, windows and pairing come back unchanged; a reused mask gives the same
attention as the mask it was saved from."""
import types

import pytest
import torch


@pytest.fixture(scope="module")
def sta():
    import block_sparse_attention_28_b200 as mod

    return mod


def test_round_trip_on_the_host(sta, tmp_path):
    from block_sparse_attention_28_b200 import maskio

    T, H, W, B, heads = 2, 16, 24, 1, 2
    g = sta.grid(T, H, W)
    nt = sta.sta_num_tiles(g)
    R = B * heads * nt
    counts = torch.arange(R) % 3 + 1
    row_ptr = torch.zeros(R + 1, dtype=torch.int32)
    row_ptr[1:] = torch.cumsum(counts, 0)
    nnz = int(row_ptr[-1])
    col_idx = torch.full((R * nt,), -5, dtype=torch.int32)
    col_idx[:nnz] = torch.cat([torch.arange(int(c)) for c in counts]).int()
    bufs = types.SimpleNamespace(row_ptr=row_ptr, col_idx=col_idx, nnz=torch.tensor([nnz]))
    win = torch.randint(-1, 3, (heads, 2, 4), dtype=torch.int32)
    pairs = torch.arange(B * heads * 2 * ((nt + 1) // 2), dtype=torch.int32).view(B * heads, -1) % nt
    p = tmp_path / "mask.pt"
    maskio.save_mask(p, bufs, B, heads, 64, g, windows=win, group_lo=(0, 1), query_pairs=pairs)
    m = maskio.load_mask(p, device="cpu")
    assert (m["B"], m["heads"], m["d"], m["grid"]) == (B, heads, 64, (T, H, W))
    assert torch.equal(m["row_ptr"], row_ptr) and torch.equal(m["col_idx"][:nnz], col_idx[:nnz])
    assert m["col_idx"].numel() == R * nt and int(m["nnz"][0]) == nnz
    assert torch.equal(m["windows"], win) and m["group_lo"] == (0, 1) and torch.equal(m["query_pairs"], pairs)


def test_a_foreign_file_is_refused(sta, tmp_path):
    from block_sparse_attention_28_b200 import maskio

    p = tmp_path / "x.pt"
    torch.save({"format": "something else"}, p)
    with pytest.raises(ValueError):
        maskio.load_mask(p, device="cpu")


@pytest.mark.gpu
def test_a_reloaded_mask_gives_the_same_attention(sta, tmp_path):
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from block_sparse_attention_28_b200 import maskio
    from workloads import make_qkv
    from workloads.configs import WorkloadConfig

    T, H, W, heads, B, d = 3, 19, 37, 2, 1, 128
    cfg = WorkloadConfig(name="m", B=B, heads=heads, d=d, T=T, H=H, W=W, seed=21, use_scores=True)
    q, k, v = (x.cuda() for x in make_qkv(cfg, device="cpu"))
    g = sta.grid(T, H, W)
    nt = sta.sta_num_tiles(g)
    qp = torch.empty((B * heads, 2 * ((nt + 1) // 2)), dtype=torch.int32, device="cuda")
    params = sta.mask_params(0.0, max(1, nt // 10), True, query_pairs=qp)
    bufs = sta.build_mask(q, k, B, heads, d, g, params, sta.MaskBuffers(B, heads, d, g, "cuda"), raster=True)
    o1 = torch.empty_like(q)
    sta.sta_attn_fwd_raster_paired(q, k, v, o1, None, bufs.row_ptr, bufs.col_idx, qp, B, heads, d, g)
    p = tmp_path / "mask.pt"
    maskio.save_mask(p, bufs, B, heads, d, g, query_pairs=qp)
    m = maskio.load_mask(p)
    o2 = torch.empty_like(q)
    sta.sta_attn_fwd_raster_paired(q, k, v, o2, None, m["row_ptr"], m["col_idx"], m["query_pairs"], B, heads, d, g)
    torch.cuda.synchronize()
    assert sta.sta_get_device_error() == sta.STA_OK
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
