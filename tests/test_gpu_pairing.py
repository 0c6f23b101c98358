"""GPU: the query-tile pairing that sta_build_mask emits (sta_mask_params.
query_pairs) equals the oracle's pairing of the same final mask, bit for bit;
the paired attention calls match the oracle's attention and the raster form
equals the tiled one; a pair index out of range is reported, not faulted."""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle as O

pytestmark = pytest.mark.gpu

ATOL_MAX, ATOL_MEAN = 2e-2, 2e-3
GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "pair_cases.json")


@pytest.fixture(scope="module")
def sta():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    import block_sparse_attention_28_b200 as mod

    return mod


@pytest.fixture(scope="module")
def gp(sta):
    import _gpu_path

    return _gpu_path


def _build_with_pairs(sta, g, B, Hh, params_kw, q=None, k=None, d=128):
    nt = sta.sta_num_tiles(g)
    qp = torch.full((B * Hh, 2 * ((nt + 1) // 2)), -7, dtype=torch.int32, device="cuda")
    bufs = sta.MaskBuffers(B, Hh, d, g, "cuda", with_mask=True)
    sta.build_mask(q, k, B, Hh, d, g, sta.mask_params(query_pairs=qp, **params_kw), bufs)
    torch.cuda.synchronize()
    assert sta.sta_get_device_error() == sta.STA_OK
    return qp.cpu().numpy(), bufs.block_mask.cpu().numpy().astype(bool), bufs


def _check_against_oracle(qp, mask, T, H, W):
    B, Hh = mask.shape[:2]
    for b in range(B):
        for h in range(Hh):
            want = O.pair_query_tiles(mask[b, h], T, H, W)
            assert np.array_equal(qp[b * Hh + h], want), (b, h, qp[b * Hh + h][:16], want[:16])


def test_pairing_golden_cases_on_the_gpu(sta):
    """The hand-derived cases, as masks given through caller block scores
    (1 for a listed tile, 0 otherwise; top-p just below 1 keeps exactly the
    listed tiles)."""
    for case in json.load(open(GOLDEN))["cases"]:
        T, H, W = case["T"], case["H"], case["W"]
        g = sta.grid(T, H, W)
        nt = sta.sta_num_tiles(g)
        sc = torch.zeros((1, 1, nt, nt), dtype=torch.float32)
        for i, l in enumerate(case["lists"]):
            sc[0, 0, i, l] = 1.0
        qp, mask, _ = _build_with_pairs(sta, g, 1, 1, dict(top_p=0.9999, k_min=0, use_scores=True,
                                                           block_scores=sc.cuda()))
        assert np.array_equal(mask[0, 0], sc[0, 0].numpy() > 0), case["name"]
        assert qp[0].tolist() == case["pairs"], (case["name"], qp[0].tolist())


@pytest.mark.parametrize("T,H,W,Hh,B,rho", [(3, 19, 37, 3, 1, 0.05), (3, 19, 37, 3, 1, 0.3), (4, 16, 24, 2, 2, 0.1),
                                            (21, 30, 52, 2, 1, 0.05), (21, 30, 52, 2, 1, 0.1), (5, 8, 8, 4, 1, 0.5)])
def test_pairing_of_top_k_masks_equals_the_oracle(sta, T, H, W, Hh, B, rho):
    """Top-k masks of random block scores at low to medium density (the mask
    reuse layer's kind), ragged grids, several heads and batch entries."""
    g = sta.grid(T, H, W)
    nt = sta.sta_num_tiles(g)
    gen = torch.Generator(device="cuda").manual_seed(T * 131 + W + int(rho * 100))
    sc = torch.rand((B, Hh, nt, nt), generator=gen, device="cuda")
    qp, mask, _ = _build_with_pairs(sta, g, B, Hh, dict(top_p=0.0, k_min=max(1, round(rho * nt)),
                                                        use_scores=True, block_scores=sc))
    _check_against_oracle(qp, mask, T, H, W)


def test_pairing_of_window_masks_equals_the_oracle(sta):
    """Window-only masks (no scores): frame partners share most of their
    lists, so the default pairing is usually kept."""
    from workloads.configs import WorkloadConfig
    from workloads import window_params

    T, H, W, Hh = 6, 40, 56, 4
    cfg = WorkloadConfig(name="w", B=1, heads=Hh, d=128, T=T, H=H, W=W, seed=3, use_scores=False,
                         group_lo=(0, 1, 3))
    win = torch.from_numpy(window_params(cfg, 0.4)).cuda()
    qp, mask, _ = _build_with_pairs(sta, sta.grid(T, H, W), 1, Hh, dict(use_scores=False, group_lo=cfg.group_lo,
                                                                         windows=win))
    _check_against_oracle(qp, mask, T, H, W)


@pytest.mark.parametrize("d", [64, 128])
def test_paired_attention_matches_the_oracle(sta, gp, d):
    """Attention over a top-k mask with the emitted pairing: the tiled output
    matches the oracle, the raster output equals the tiled one bit for bit,
    and the pairing differs from the default on this mask (so the test runs
    the caller's pairs)."""
    from workloads.configs import WorkloadConfig
    from workloads import make_qkv

    T, H, W, Hh, B = 3, 19, 37, 2, 1
    cfg = WorkloadConfig(name="p", B=B, heads=Hh, d=d, T=T, H=H, W=W, seed=5, use_scores=True)
    q, k, v = (x.cuda() for x in make_qkv(cfg, device="cpu"))
    g = sta.grid(T, H, W)
    nt = sta.sta_num_tiles(g)
    qt, kt, vt = (gp.reorder(x, B, Hh, d, g) for x in (q, k, v))
    qp_np, mask, bufs = _build_with_pairs(sta, g, B, Hh, dict(top_p=0.0, k_min=max(1, nt // 12), use_scores=True),
                                          qt, kt, d)
    dflt = np.array([i for p in O.default_pairs(T, H, W) for i in p])
    assert any(not np.array_equal(qp_np[h], dflt) for h in range(Hh))
    qp = torch.from_numpy(qp_np).cuda()
    o = torch.full_like(qt, float("nan"))
    lse = torch.full(qt.shape[:3], float("nan"), dtype=torch.float32, device="cuda")
    sta.sta_attn_fwd_paired(qt, kt, vt, o, lse, bufs.row_ptr, bufs.col_idx, qp, B, Hh, d, g)
    o_r = torch.full_like(q, float("nan"))
    lse_r = torch.full_like(lse, float("nan"))
    sta.sta_attn_fwd_raster_paired(q, k, v, o_r, lse_r, bufs.row_ptr, bufs.col_idx, qp, B, Hh, d, g)
    torch.cuda.synchronize()
    assert sta.sta_get_device_error() == sta.STA_OK
    back = torch.zeros_like(q)
    sta.sta_reorder(o, back, B, Hh, d, g, inverse=True)
    torch.cuda.synchronize()
    assert torch.equal(back.view(torch.int16), o_r.view(torch.int16))
    rp, ci, _ = gp.csr_np(bufs)
    o_ref, l_ref = O.attention_all(gp.to_np64(qt), gp.to_np64(kt), gp.to_np64(vt), rp, ci, T, H, W,
                                   1.0 / math.sqrt(d))
    valid = O.valid_rows(T, H, W)
    mx, mean = gp.attn_errors(o, o_ref, valid)
    assert mx <= ATOL_MAX and mean <= ATOL_MEAN, (mx, mean)
    lg = lse.cpu().numpy()[:, :, valid]
    lr = l_ref[:, :, valid]
    assert np.allclose(lg, lr, rtol=1e-5, atol=1e-4)


def test_pair_index_out_of_range_is_reported(sta, gp):
    """A tile index past Nt in the caller's pairs: STA_ERR_BAD_MASK from the
    device error word, the other pairs still computed, the context usable."""
    T, H, W, Hh, B, d = 2, 16, 16, 1, 1, 64
    g = sta.grid(T, H, W)
    nt = sta.sta_num_tiles(g)
    x = torch.randn((B, Hh, sta.sta_tiled_len(g), d), device="cuda").to(torch.bfloat16)
    rp = torch.arange(0, nt + 1, dtype=torch.int32, device="cuda")
    ci = torch.arange(0, nt, dtype=torch.int32, device="cuda")  # each tile lists itself
    pairs = torch.tensor([[i for p in O.default_pairs(T, H, W) for i in p]], dtype=torch.int32).cuda()
    pairs[0, 2] = nt + 5
    o = torch.zeros_like(x)
    sta.sta_attn_fwd_paired(x, x, x, o, None, rp, ci, pairs, B, Hh, d, g)
    assert sta.sta_get_device_error() == sta.STA_ERR_BAD_MASK
    o2 = torch.zeros_like(x)
    sta.sta_attn_fwd(x, x, x, o2, None, rp, ci, B, Hh, d, g)
    assert sta.sta_get_device_error() == sta.STA_OK
    # the pairs that were valid give what the default call gives
    a, b = int(pairs[0, 0]), int(pairs[0, 1])
    for t in (a, b):
        assert torch.equal(o[0, 0, 64 * t:64 * t + 64], o2[0, 0, 64 * t:64 * t + 64])


def test_csr_validation(sta, gp):
    """sta_validate_csr: a mask the library built passes; each kind of
    corruption of a caller's CSR is reported as STA_ERR_BAD_MASK, and the
    offsets are checked against the column capacity before any column is
    read."""
    T, H, W, Hh, B, d = 3, 19, 37, 2, 1, 128
    g = sta.grid(T, H, W)
    nt = sta.sta_num_tiles(g)
    gen = torch.Generator(device="cuda").manual_seed(4)
    sc = torch.rand((B, Hh, nt, nt), generator=gen, device="cuda")
    bufs = sta.MaskBuffers(B, Hh, d, g, "cuda")
    sta.build_mask(None, None, B, Hh, d, g, sta.mask_params(0.0, 5, True, block_scores=sc), bufs)
    torch.cuda.synchronize()
    assert sta.sta_get_device_error() == sta.STA_OK
    nnz = int(bufs.nnz.item())
    sta.sta_validate_csr(bufs.row_ptr, bufs.col_idx, B, Hh, g)
    assert sta.sta_get_device_error() == sta.STA_OK
    sta.sta_validate_csr(bufs.row_ptr, bufs.col_idx, B, Hh, g, col_capacity=nnz)
    assert sta.sta_get_device_error() == sta.STA_OK

    def corrupt(fn, cap=None):
        rp, ci = bufs.row_ptr.clone(), bufs.col_idx.clone()
        fn(rp, ci)
        sta.sta_validate_csr(rp, ci, B, Hh, g, col_capacity=cap)
        return sta.sta_get_device_error()

    def swap_cols(rp, ci):
        a = int(rp[7])
        ci[a], ci[a + 1] = ci[a + 1].clone(), ci[a].clone()

    def dup_col(rp, ci):
        a = int(rp[9])
        ci[a + 1] = ci[a]

    cases = {
        "first offset not zero": lambda rp, ci: rp.__setitem__(0, 1),
        "offsets decrease": lambda rp, ci: rp.__setitem__(5, int(rp[4]) - 1),
        "column past Nt": lambda rp, ci: ci.__setitem__(int(rp[3]), nt),
        "negative column": lambda rp, ci: ci.__setitem__(int(rp[3]), -1),
        "columns out of order": swap_cols,
        "repeated column": dup_col,
    }
    for name, fn in cases.items():
        assert corrupt(fn) == sta.STA_ERR_BAD_MASK, name
    # offsets beyond the column capacity: refused before the columns are read
    assert corrupt(lambda rp, ci: None, cap=nnz - 1) == sta.STA_ERR_BAD_MASK
