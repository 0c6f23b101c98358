"""Parity of the CUDA path (through the C ABI) with the fp64 oracle.

Bars: reorder, CSR lists and byte masks bit-exact; block probabilities within
a bound derived from the GPU's fp32 arithmetic; attention output within
max-abs 2e-2 and mean-abs 2e-3 of the oracle, LSE within 1e-3, with masks
built from identical block probabilities (the oracle's selection runs on the
GPU's exported P).
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
from workloads import CONFIGS, fixed_windows_tiny, make_qkv, window_params, window_scale

pytestmark = pytest.mark.gpu

ATOL_MAX, ATOL_MEAN, LSE_TOL = 2e-2, 2e-3, 1e-3


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


def _rand_raster(B, L, Hh, d, seed, scale=1.0, device="cuda"):
    g = torch.Generator(device=device).manual_seed(seed)
    return (torch.randn(B, L, Hh, d, generator=g, device=device) * scale).to(torch.bfloat16)


def _structured(T, H, W, Hh, d, seed, B=1):
    """Small Q, K, V with the workload recipe (RFF positions + noise)."""
    from workloads.configs import WorkloadConfig

    cfg = WorkloadConfig(name="t", B=B, heads=Hh, d=d, T=T, H=H, W=W, seed=seed, use_scores=True)
    return [x.cuda() for x in make_qkv(cfg, device="cpu")]


# ------------------------------------------------------------------ reorder
@pytest.mark.parametrize("T,H,W,d,B,Hh", [(4, 16, 16, 64, 1, 2), (3, 13, 19, 128, 2, 3),
                                          (2, 9, 10, 64, 1, 1), (1, 8, 8, 128, 1, 5)])
def test_reorder_bit_exact(sta, gp, T, H, W, d, B, Hh):
    g = sta.grid(T, H, W)
    x = _rand_raster(B, T * H * W, Hh, d, seed=T * 100 + H)
    xt = gp.reorder(x, B, Hh, d, g)
    want = O.reorder_fwd(gp.to_np64(x), T, H, W)
    got = gp.to_np64(xt)
    assert np.array_equal(got, want)  # also: pad rows are exactly zero
    back = torch.full_like(x, float("nan"))
    sta.sta_reorder(xt, back, B, Hh, d, g, inverse=True)
    assert torch.equal(back.view(torch.int16), x.view(torch.int16))


def test_reorder_full_size_720p(sta, gp):
    cfg = CONFIGS["dit720p"]
    B, Hh, d, T, H, W = cfg.B, cfg.heads, cfg.d, cfg.T, cfg.H, cfg.W
    g = sta.grid(T, H, W)
    x = _rand_raster(B, cfg.L, Hh, d, seed=7)
    xt = gp.reorder(x, B, Hh, d, g)
    rows = O.tiled_row_of_raster(T, H, W)
    rng = np.random.default_rng(0)
    sample = rng.choice(cfg.L, 4096, replace=False)
    got = xt[0][:, torch.from_numpy(rows[sample]).cuda(), :]
    want = x[0][torch.from_numpy(sample).cuda()].transpose(0, 1)
    assert torch.equal(got.view(torch.int16), want.view(torch.int16))
    valid = torch.from_numpy(O.valid_rows(T, H, W)).cuda()
    assert int(valid.sum()) == cfg.L
    assert torch.count_nonzero(xt[:, :, ~valid, :].float()) == 0
    back = torch.empty_like(x)
    sta.sta_reorder(xt, back, B, Hh, d, g, inverse=True)
    assert torch.equal(back.view(torch.int16), x.view(torch.int16))


# --------------------------------------------------------------- build_mask
def _assert_near_threshold(own, gpu, p_ref, bound, top_p):
    """Every (row, tile) where the oracle's own selection (on the fp64 P) and
    the selection on the GPU's P differ is one the P error bound explains:
    - a near-tie: its P lies within twice the bound of the P of a boundary
      tile of the row (the last kept or the first dropped in the oracle's
      order), so the two orders may swap them; or
    - a near-threshold prefix: 0 < top_p < 1 and the integer mass of the tiles
      ahead of it in the oracle's order lies within the mass error of the
      threshold, tol = 2 * sum_j (bound_j * 2^24 + 1) + 1 (the error of any
      prefix sum of w = floor(P * 2^24), plus that of thr = ceil(top_p * W)),
      so one side's prefix reaches the threshold one tile before the other's.
    Returns the largest |prefix - thr| / W met among the near-threshold ones."""
    worst = 0.0
    for idx in np.argwhere(own != gpu):
        row = tuple(idx[:-1])
        t = idx[-1]
        p, b = p_ref[row], bound[row]
        order = np.lexsort((np.arange(p.size), -p))  # P descending, ties to the lower index
        pos = np.empty(p.size, dtype=np.int64)
        pos[order] = np.arange(p.size)
        m = int(own[row].sum())  # the oracle keeps order[:m]
        edge = [order[m - 1]] if m > 0 else []
        edge += [order[m]] if m < p.size else []
        near_tie = any(abs(p[t] - p[e]) <= 2.0 * max(b[t], b[e]) for e in edge)
        w = np.floor(p * 2.0 ** 24)
        W = w.sum()
        tp = float(np.float32(top_p))
        thr = math.ceil(tp * W)
        ahead = w[order[:pos[t]]].sum()
        tol = 2.0 * (b * 2.0 ** 24 + 1.0).sum() + 1.0
        near_mass = 0.0 < tp < 1.0 and abs(ahead - thr) <= tol
        assert near_tie or near_mass, (row, t, m, pos[t], ahead - thr, tol)
        if near_mass and not near_tie:
            worst = max(worst, abs(ahead - thr) / W)
    return worst


def _check_mask(sta, gp, qt, kt, B, Hh, d, T, H, W, top_p, k_min, use_scores, win, group_lo,
                check_probs=True, sm_scale=0.0):
    g = sta.grid(T, H, W)
    win_d = torch.from_numpy(win).cuda() if win is not None else None
    params = sta.mask_params(top_p, k_min, use_scores, sm_scale, group_lo, win_d)
    bufs = gp.build(qt, kt, B, Hh, d, g, params)
    torch.cuda.synchronize()
    assert sta.sta_get_device_error() == sta.STA_OK
    rp, ci, nnz = gp.csr_np(bufs)
    nt = sta.sta_num_tiles(g)
    mask = np.zeros((B, Hh, nt, nt), dtype=bool)
    probs = bufs.block_probs.cpu().numpy()
    if use_scores:
        mask |= O.select(probs, top_p, k_min)
        if check_probs:
            scale = sm_scale if sm_scale != 0.0 else 1.0 / math.sqrt(d)
            qb, kb = O.pool(gp.to_np64(qt), T, H, W), O.pool(gp.to_np64(kt), T, H, W)
            _, p_ref = O.block_scores(qb, kb, scale)
            bound = gp.prob_bound(qb, kb, scale, p_ref)
            assert np.all(np.abs(probs - p_ref) <= bound)
            assert np.max(np.abs(probs - p_ref) / bound) <= gp.PROB_ERR_CEILING
            # the oracle's own end-to-end mask differs only at near-threshold
            # tiles: a P within the error bound of a boundary tile's P (a
            # near-tie), or a prefix mass within the derived mass error of
            # the threshold
            own = O.select(p_ref, top_p, k_min)
            sel_gpu = O.select(probs, top_p, k_min)
            assert (own != sel_gpu).mean() < 1e-3
            _assert_near_threshold(own, sel_gpu, p_ref, bound, top_p)
    else:
        assert np.all(probs == 0)
    if win is not None:
        mask |= O.window_mask(win, group_lo, T, H, W)[None]
    rp_o, ci_o = O.mask_to_csr(mask)
    assert np.array_equal(rp, rp_o)
    assert nnz == ci_o.size and np.array_equal(ci, ci_o)
    assert np.array_equal(bufs.block_mask.cpu().numpy().astype(bool), mask)
    return bufs, mask


def test_build_mask_tiny_config(sta, gp):
    cfg = CONFIGS["tiny"]
    q, k, _ = (x.cuda() for x in make_qkv(cfg, device="cpu"))
    g = sta.grid(cfg.T, cfg.H, cfg.W)
    qt, kt = gp.reorder(q, 1, cfg.heads, cfg.d, g), gp.reorder(k, 1, cfg.heads, cfg.d, g)
    _check_mask(sta, gp, qt, kt, 1, cfg.heads, cfg.d, cfg.T, cfg.H, cfg.W, cfg.top_p, cfg.k_min, True,
                fixed_windows_tiny(cfg), cfg.group_lo)


@pytest.mark.parametrize("top_p,k_min,use_scores,with_win", [
    (0.7, 3, True, True), (0.95, 8, True, False), (1.0, 0, True, False), (0.0, 0, True, False),
    (0.0, 5, True, True), (0.5, 100, True, False), (0.0, 0, False, True), (0.3, 1, True, True)])
@pytest.mark.parametrize("d", [64, 128])
def test_build_mask_ragged(sta, gp, top_p, k_min, use_scores, with_win, d):
    T, H, W, Hh, B = 3, 19, 37, 3, 2  # 3 x 3 x 5 = 45 tiles, partial tiles on two edges
    rng = np.random.default_rng(d + int(100 * top_p) + k_min)
    q, k, _ = _structured(T, H, W, Hh, d, seed=11, B=B)
    g = sta.grid(T, H, W)
    qt, kt = gp.reorder(q, B, Hh, d, g), gp.reorder(k, B, Hh, d, g)
    win = None
    if with_win:
        win = rng.integers(-1, 3, size=(Hh, 3, 4)).astype(np.int32)
    _check_mask(sta, gp, qt, kt, B, Hh, d, T, H, W, top_p, k_min, use_scores, win, (0, 1, 3))


@pytest.mark.parametrize("d", [64, 128])
def test_build_mask_several_key_blocks(sta, gp, d):
    """Nt = 175 tiles: two 128-tile key blocks of the tensor-core scores, the
    query range split over several CTAs, and rows of S whose length is not a
    multiple of four (scalar stores)."""
    T, H, W, Hh, B = 5, 40, 50, 2, 1  # 5 x 5 x 7 tiles
    q, k, _ = _structured(T, H, W, Hh, d, seed=41, B=B)
    g = sta.grid(T, H, W)
    assert sta.sta_num_tiles(g) == 175
    qt, kt = gp.reorder(q, B, Hh, d, g), gp.reorder(k, B, Hh, d, g)
    rng = np.random.default_rng(d)
    win = rng.integers(-1, 3, size=(Hh, 3, 4)).astype(np.int32)
    _check_mask(sta, gp, qt, kt, B, Hh, d, T, H, W, 0.9, 4, True, win, (0, 1, 3))


@pytest.mark.parametrize("sm_scale", [0.05, 0.5])
def test_build_mask_custom_scale(sta, gp, sm_scale):
    """A caller-given score scale reaches the pooled scores (tensor-core
    layout): P within its bound of the oracle's at that scale, CSR equal to
    the oracle's selection on the GPU's P."""
    T, H, W, Hh, B, d = 3, 19, 37, 3, 2, 128
    q, k, _ = _structured(T, H, W, Hh, d, seed=17, B=B)
    g = sta.grid(T, H, W)
    qt, kt = gp.reorder(q, B, Hh, d, g), gp.reorder(k, B, Hh, d, g)
    _check_mask(sta, gp, qt, kt, B, Hh, d, T, H, W, 0.8, 2, True, None, (0,), sm_scale=sm_scale)


def test_build_mask_window_only_full_480p(sta, gp):
    cfg = CONFIGS["dit480p"]
    g = sta.grid(cfg.T, cfg.H, cfg.W)
    win = window_params(cfg, window_scale("dit480p", 0))
    win_d = torch.from_numpy(win).cuda()
    params = sta.mask_params(0.0, 0, False, 0.0, cfg.group_lo, win_d)
    bufs = gp.build(None, None, 1, cfg.heads, cfg.d, g, params, with_mask=False, with_probs=False)
    rp, ci, nnz = gp.csr_np(bufs)
    mask = O.window_mask(win, cfg.group_lo, cfg.T, cfg.H, cfg.W)[None]
    rp_o, ci_o = O.mask_to_csr(mask)
    assert np.array_equal(rp, rp_o) and np.array_equal(ci, ci_o)
    assert abs(nnz / mask.size - 0.25) < 0.01


def test_build_mask_full_720p_sampled_rows(sta, gp):
    """The headline layer: full-size build; the oracle's selection on the GPU's
    P for sampled rows, plus the windows, must give the same CSR rows."""
    cfg = CONFIGS["dit720p"]
    B, Hh, d, T, H, W = cfg.B, cfg.heads, cfg.d, cfg.T, cfg.H, cfg.W
    g = sta.grid(T, H, W)
    q, k, _ = make_qkv(cfg, device="cuda")
    qt, kt = gp.reorder(q, B, Hh, d, g), gp.reorder(k, B, Hh, d, g)
    del q, k
    win = window_params(cfg, window_scale("dit720p", 0))
    params = sta.mask_params(cfg.top_p, cfg.k_min, True, 0.0, cfg.group_lo, torch.from_numpy(win).cuda())
    bufs = gp.build(qt, kt, B, Hh, d, g, params, with_mask=False, with_probs=True)
    torch.cuda.synchronize()
    rp, ci, nnz = gp.csr_np(bufs)
    nt = sta.sta_num_tiles(g)
    rng = np.random.default_rng(2)
    heads = rng.choice(Hh, 3, replace=False)
    wm = O.window_mask(win[heads], cfg.group_lo, T, H, W)
    for hi, h in enumerate(heads):
        rows = rng.choice(nt, 40, replace=False)
        probs = bufs.block_probs[0, h, torch.from_numpy(rows).cuda()].cpu().numpy()
        for ri, qtile in enumerate(rows):
            keep = O.select_row(probs[ri], cfg.top_p, cfg.k_min) | wm[hi, qtile]
            r = h * nt + qtile
            assert np.array_equal(ci[rp[r]:rp[r + 1]], np.nonzero(keep)[0]), (h, qtile)
    density = nnz / (B * Hh * nt * nt)
    assert 0.10 < density < 0.20, density


# ------------------------------------------------------------------ attention
def _attn_check(sta, gp, qt, kt, vt, rp_t, ci_t, B, Hh, d, T, H, W, sm_scale=0.0, rows=None):
    g = sta.grid(T, H, W)
    o, lse = gp.attn(qt, kt, vt, rp_t, ci_t, B, Hh, d, g, sm_scale)
    torch.cuda.synchronize()
    assert sta.sta_get_device_error() == sta.STA_OK
    rp, ci = rp_t.cpu().numpy(), ci_t.cpu().numpy()
    scale = sm_scale if sm_scale else 1.0 / math.sqrt(d)
    nt = sta.sta_num_tiles(g)
    if rows is None:
        rows = range(B * Hh * nt)
    q64, k64, v64 = gp.to_np64(qt), gp.to_np64(kt), gp.to_np64(vt)
    res = O.attention_rows(q64, k64, v64, rp, ci, T, H, W, scale, rows)
    o_np = o.float().cpu().numpy()
    lse_np = lse.cpu().numpy()
    errs = []
    for r, qrows, o_ref, lse_ref in res:
        bh, _ = divmod(r, nt)
        b, h = divmod(bh, Hh)
        got = o_np[b, h, qrows]
        errs.append(np.abs(got - o_ref).ravel())
        gl = lse_np[b, h, qrows]
        fin = np.isfinite(lse_ref)
        assert np.all(np.isneginf(gl[~fin]))
        assert np.all(np.abs(gl[fin] - lse_ref[fin]) <= LSE_TOL * np.maximum(1.0, np.abs(lse_ref[fin])))
    err = np.concatenate(errs)
    assert np.isfinite(err).all()
    assert err.max() <= ATOL_MAX and err.mean() <= ATOL_MEAN, (err.max(), err.mean())
    return o, lse, err


def test_attn_tiny_config(sta, gp):
    cfg = CONFIGS["tiny"]
    B, Hh, d, T, H, W = cfg.B, cfg.heads, cfg.d, cfg.T, cfg.H, cfg.W
    g = sta.grid(T, H, W)
    q, k, v = (x.cuda() for x in make_qkv(cfg, device="cpu"))
    qt, kt, vt = (gp.reorder(x, B, Hh, d, g) for x in (q, k, v))
    win = torch.from_numpy(fixed_windows_tiny(cfg)).cuda()
    bufs = gp.build(qt, kt, B, Hh, d, g, sta.mask_params(cfg.top_p, cfg.k_min, True, 0.0, cfg.group_lo, win))
    _attn_check(sta, gp, qt, kt, vt, bufs.row_ptr, bufs.col_idx, B, Hh, d, T, H, W)


def _custom_csr(mask):
    rp, ci = O.mask_to_csr(mask)
    return torch.from_numpy(rp).cuda(), torch.from_numpy(np.ascontiguousarray(ci) if ci.size else
                                                         np.zeros(1, np.int32)).cuda()


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("kind", ["random", "dense", "empty_rows", "single_tile", "edge_tiles"])
def test_attn_ragged_masks(sta, gp, d, kind):
    T, H, W, Hh, B = 3, 19, 37, 2, 2  # 45 tiles: odd count, so the last CTA has one tile
    g = sta.grid(T, H, W)
    nt = sta.sta_num_tiles(g)
    q, k, v = _structured(T, H, W, Hh, d, seed=5, B=B)
    qt, kt, vt = (gp.reorder(x, B, Hh, d, g) for x in (q, k, v))
    rng = np.random.default_rng(len(kind) + d)
    if kind == "random":
        mask = rng.random((B, Hh, nt, nt)) < 0.3
    elif kind == "dense":
        mask = np.ones((B, Hh, nt, nt), dtype=bool)
    elif kind == "empty_rows":
        mask = rng.random((B, Hh, nt, nt)) < 0.2
        mask[:, :, ::3] = False  # whole rows empty, including both halves of some CTAs
        mask[0, 0, 0:2] = False
    elif kind == "single_tile":
        mask = np.zeros((B, Hh, nt, nt), dtype=bool)
        for r in range(nt):
            mask[:, :, r, (r * 7) % nt] = True
    else:  # only the partial tiles at the right / bottom edges
        nh, nw = (H + 7) // 8, (W + 7) // 8
        edge = [t for t in range(nt) if (t % nw) == nw - 1 or ((t // nw) % nh) == nh - 1]
        mask = np.zeros((B, Hh, nt, nt), dtype=bool)
        mask[..., edge] = True
    rp, ci = _custom_csr(mask)
    _attn_check(sta, gp, qt, kt, vt, rp, ci, B, Hh, d, T, H, W, sm_scale=0.11 if d == 64 else 0.0)


def test_attn_dense_large_logits(sta, gp):
    """Dense mask on an unpadded grid with a large score scale, so that the
    running max moves by more than the lazy-rescale threshold many times."""
    T, H, W, Hh, B, d = 2, 32, 48, 2, 1, 128
    g = sta.grid(T, H, W)
    nt = sta.sta_num_tiles(g)
    q, k, v = _structured(T, H, W, Hh, d, seed=9)
    qt, kt, vt = (gp.reorder(x, B, Hh, d, g) for x in (q, k, v))
    rp, ci = _custom_csr(np.ones((B, Hh, nt, nt), dtype=bool))
    _attn_check(sta, gp, qt, kt, vt, rp, ci, B, Hh, d, T, H, W, sm_scale=0.35)


def test_attn_full_720p_sampled_rows(sta, gp):
    """The headline layer end to end: full-size build and attention as timed by
    the benchmark; the oracle recomputes sampled rows on the GPU's CSR."""
    cfg = CONFIGS["dit720p"]
    B, Hh, d, T, H, W = cfg.B, cfg.heads, cfg.d, cfg.T, cfg.H, cfg.W
    g = sta.grid(T, H, W)
    q, k, v = make_qkv(cfg, device="cuda")
    qt, kt, vt = (gp.reorder(x, B, Hh, d, g) for x in (q, k, v))
    del q, k, v
    win = torch.from_numpy(window_params(cfg, window_scale("dit720p", 0))).cuda()
    bufs = gp.build(qt, kt, B, Hh, d, g, sta.mask_params(cfg.top_p, cfg.k_min, True, 0.0, cfg.group_lo, win),
                    with_mask=False, with_probs=False)
    nt = sta.sta_num_tiles(g)
    rng = np.random.default_rng(3)
    rows = sorted(rng.choice(B * Hh * nt, 48, replace=False).tolist())
    _attn_check(sta, gp, qt, kt, vt, bufs.row_ptr, bufs.col_idx, B, Hh, d, T, H, W, rows=rows)


def test_attn_reuse_steps(sta, gp):
    """Mask built once from step-0 inputs, reused after 10 perturbed steps."""
    cfg = CONFIGS["reuse480p"]
    B, Hh, d, T, H, W = cfg.B, 8, cfg.d, cfg.T, cfg.H, cfg.W
    from dataclasses import replace

    c8 = replace(cfg, heads=Hh)
    g = sta.grid(T, H, W)
    nt = sta.sta_num_tiles(g)
    q, k, v = make_qkv(c8, device="cuda")
    qt, kt, vt = (gp.reorder(x, B, Hh, d, g) for x in (q, k, v))
    kmin = int(round(0.10 * nt))
    bufs = gp.build(qt, kt, B, Hh, d, g, sta.mask_params(0.0, kmin, True), with_mask=False, with_probs=False)
    rp, ci, nnz = gp.csr_np(bufs)
    assert nnz == B * Hh * nt * kmin
    gen = torch.Generator(device="cuda").manual_seed(44)
    mq, mk = q.float(), k.float()
    from workloads import perturb_step

    for _ in range(cfg.reuse_steps):
        mq, qb = perturb_step(mq, gen)
        mk, kb = perturb_step(mk, gen)
    qt10, kt10 = gp.reorder(qb, B, Hh, d, g), gp.reorder(kb, B, Hh, d, g)
    rng = np.random.default_rng(4)
    rows = sorted(rng.choice(B * Hh * nt, 24, replace=False).tolist())
    _attn_check(sta, gp, qt, kt, vt, bufs.row_ptr, bufs.col_idx, B, Hh, d, T, H, W, rows=rows)
    _attn_check(sta, gp, qt10, kt10, vt, bufs.row_ptr, bufs.col_idx, B, Hh, d, T, H, W, rows=rows)


def test_attn_bad_column_index_is_reported(sta, gp):
    T, H, W, Hh, B, d = 2, 16, 16, 1, 1, 64
    g = sta.grid(T, H, W)
    nt = sta.sta_num_tiles(g)
    q, k, v = _structured(T, H, W, Hh, d, seed=3)
    qt, kt, vt = (gp.reorder(x, B, Hh, d, g) for x in (q, k, v))
    mask = np.ones((B, Hh, nt, nt), dtype=bool)
    rp, ci = _custom_csr(mask)
    ci[3] = nt + 5  # out of range: skipped and reported, never read
    sta.sta_get_device_error()
    o, lse = gp.attn(qt, kt, vt, rp, ci, B, Hh, d, g)
    assert sta.sta_get_device_error() == sta.STA_ERR_BAD_MASK
    assert sta.sta_get_device_error() == sta.STA_OK  # the word was cleared
    assert torch.isfinite(o.float()).all()


# ------------------------------------------------- full-size workload coverage
@pytest.mark.parametrize("which", [0, 1, 2, 3])
def test_build_mask_window_only_full_129_frames(sta, gp, which):
    """129-frame layer (24 heads, 1,980 tiles per head), four temporal groups,
    each density target: the whole CSR against the oracle's window mask."""
    cfg = CONFIGS["dit720p_129f"]
    g = sta.grid(cfg.T, cfg.H, cfg.W)
    win = window_params(cfg, window_scale("dit720p_129f", which))
    params = sta.mask_params(0.0, 0, False, 0.0, cfg.group_lo, torch.from_numpy(win).cuda())
    bufs = gp.build(None, None, 1, cfg.heads, cfg.d, g, params, with_mask=False, with_probs=False)
    rp, ci, nnz = gp.csr_np(bufs)
    mask = O.window_mask(win, cfg.group_lo, cfg.T, cfg.H, cfg.W)[None]
    rp_o, ci_o = O.mask_to_csr(mask)
    assert np.array_equal(rp, rp_o) and np.array_equal(ci, ci_o)
    assert abs(nnz / mask.size - cfg.window_density[which]) < 0.01


def test_attn_full_129_frames_sampled_rows(sta, gp):
    cfg = CONFIGS["dit720p_129f"]
    B, Hh, d, T, H, W = cfg.B, cfg.heads, cfg.d, cfg.T, cfg.H, cfg.W
    g = sta.grid(T, H, W)
    q, k, v = make_qkv(cfg, device="cuda")
    qt, kt, vt = (gp.reorder(x, B, Hh, d, g) for x in (q, k, v))
    del q, k, v
    win = torch.from_numpy(window_params(cfg, window_scale("dit720p_129f", 2))).cuda()
    bufs = gp.build(None, None, B, Hh, d, g, sta.mask_params(0.0, 0, False, 0.0, cfg.group_lo, win),
                    with_mask=False, with_probs=False)
    nt = sta.sta_num_tiles(g)
    rng = np.random.default_rng(5)
    rows = sorted(rng.choice(B * Hh * nt, 24, replace=False).tolist())
    _attn_check(sta, gp, qt, kt, vt, bufs.row_ptr, bufs.col_idx, B, Hh, d, T, H, W, rows=rows)


def test_attn_full_480p_sampled_rows(sta, gp):
    cfg = CONFIGS["dit480p"]
    B, Hh, d, T, H, W = cfg.B, cfg.heads, cfg.d, cfg.T, cfg.H, cfg.W
    g = sta.grid(T, H, W)
    q, k, v = make_qkv(cfg, device="cuda")
    qt, kt, vt = (gp.reorder(x, B, Hh, d, g) for x in (q, k, v))
    del q, k, v
    win = torch.from_numpy(window_params(cfg, window_scale("dit480p", 0))).cuda()
    bufs = gp.build(None, None, B, Hh, d, g, sta.mask_params(0.0, 0, False, 0.0, cfg.group_lo, win),
                    with_mask=False, with_probs=False)
    nt = sta.sta_num_tiles(g)
    rng = np.random.default_rng(6)
    rows = sorted(rng.choice(B * Hh * nt, 32, replace=False).tolist())
    _attn_check(sta, gp, qt, kt, vt, bufs.row_ptr, bufs.col_idx, B, Hh, d, T, H, W, rows=rows)


def test_attn_reuse_all_densities_full(sta, gp):
    """Reuse layer, all 40 heads: masks of every density built once from step-0
    inputs (fixed count per row, selection exact against the oracle on the
    GPU's P for sampled rows), attention after 0 and 10 perturbed steps; the
    100% run is the dense-mask reference of the same kernel."""
    from workloads import perturb_step

    cfg = CONFIGS["reuse480p"]
    B, Hh, d, T, H, W = cfg.B, cfg.heads, cfg.d, cfg.T, cfg.H, cfg.W
    g = sta.grid(T, H, W)
    nt = sta.sta_num_tiles(g)
    q, k, v = make_qkv(cfg, device="cuda")
    qt, kt, vt = (gp.reorder(x, B, Hh, d, g) for x in (q, k, v))
    gen = torch.Generator(device="cuda").manual_seed(404)
    mq, mk = q.float(), k.float()
    for _ in range(cfg.reuse_steps):
        mq, qb = perturb_step(mq, gen)
        mk, kb = perturb_step(mk, gen)
    qt10, kt10 = gp.reorder(qb, B, Hh, d, g), gp.reorder(kb, B, Hh, d, g)
    del q, k, mq, mk, qb, kb
    rng = np.random.default_rng(7)
    for rho in cfg.fixed_densities:
        kmin = int(round(rho * nt))
        bufs = gp.build(qt, kt, B, Hh, d, g, sta.mask_params(0.0, kmin, True), with_mask=False, with_probs=True)
        rp, ci, nnz = gp.csr_np(bufs)
        assert nnz == B * Hh * nt * kmin
        rows = sorted(rng.choice(B * Hh * nt, 6, replace=False).tolist())
        for r in rows:
            bh, qtile = divmod(r, nt)
            p_row = bufs.block_probs.view(-1, nt)[r].cpu().numpy()
            assert np.array_equal(ci[rp[r]:rp[r + 1]], np.nonzero(O.select_row(p_row, 0.0, kmin))[0])
        bufs.block_probs = None
        _attn_check(sta, gp, qt, kt, vt, bufs.row_ptr, bufs.col_idx, B, Hh, d, T, H, W, rows=rows)
        _attn_check(sta, gp, qt10, kt10, vt, bufs.row_ptr, bufs.col_idx, B, Hh, d, T, H, W, rows=rows)


# ---------------------------------------------- per-head top-k floor (SCOPE f1)
def _floor_mask(probs, top_p, k_min, sizes):
    B, Hh, nt, _ = probs.shape
    out = np.zeros((B, Hh, nt, nt), dtype=bool)
    for b in range(B):
        for h in range(Hh):
            out[b, h] = O.select_with_head_floor(probs[b, h], top_p, k_min, sizes)[0]
    return out


@pytest.mark.parametrize("d", [64, 128])
def test_build_mask_head_floor_ragged(sta, gp, d):
    T, H, W, Hh, B = 3, 19, 37, 3, 2  # partial tiles: the cluster sizes n_c differ
    q, k, _ = _structured(T, H, W, Hh, d, seed=21, B=B)
    g = sta.grid(T, H, W)
    qt, kt = gp.reorder(q, B, Hh, d, g), gp.reorder(k, B, Hh, d, g)
    rng = np.random.default_rng(d)
    win = rng.integers(-1, 2, size=(Hh, 3, 4)).astype(np.int32)
    params = sta.mask_params(0.6, 1, True, 0.0, (0, 1, 3), torch.from_numpy(win).cuda(), head_floor=True)
    bufs = gp.build(qt, kt, B, Hh, d, g, params)
    torch.cuda.synchronize()
    rp, ci, nnz = gp.csr_np(bufs)
    probs = bufs.block_probs.cpu().numpy()
    sizes = O.tile_sizes(T, H, W)
    mask = _floor_mask(probs, 0.6, 1, sizes) | O.window_mask(win, (0, 1, 3), T, H, W)[None]
    rp_o, ci_o = O.mask_to_csr(mask)
    assert np.array_equal(rp, rp_o) and np.array_equal(ci, ci_o)
    assert np.array_equal(bufs.block_mask.cpu().numpy().astype(bool), mask)
    # the floor only adds tiles
    base = O.select(probs, 0.6, 1)
    assert (_floor_mask(probs, 0.6, 1, sizes) >= base).all()


def test_build_mask_head_floor_720p_sampled_heads(sta, gp):
    cfg = CONFIGS["dit720p"]
    B, Hh, d, T, H, W = cfg.B, cfg.heads, cfg.d, cfg.T, cfg.H, cfg.W
    g = sta.grid(T, H, W)
    q, k, _ = make_qkv(cfg, device="cuda")
    qt, kt = gp.reorder(q, B, Hh, d, g), gp.reorder(k, B, Hh, d, g)
    del q, k
    win = window_params(cfg, window_scale("dit720p", 0))
    params = sta.mask_params(cfg.top_p, cfg.k_min, True, 0.0, cfg.group_lo, torch.from_numpy(win).cuda(),
                             head_floor=True)
    bufs = gp.build(qt, kt, B, Hh, d, g, params, with_mask=False, with_probs=True)
    torch.cuda.synchronize()
    rp, ci, nnz = gp.csr_np(bufs)
    nt = sta.sta_num_tiles(g)
    sizes = O.tile_sizes(T, H, W)
    for h in (3, 29):
        probs = bufs.block_probs[0, h].cpu().numpy()
        keep, k_head = O.select_with_head_floor(probs, cfg.top_p, cfg.k_min, sizes)
        keep |= O.window_mask(win[h:h + 1], cfg.group_lo, T, H, W)[0]
        for qtile in range(0, nt, 7):
            r = h * nt + qtile
            assert np.array_equal(ci[rp[r]:rp[r + 1]], np.nonzero(keep[qtile])[0]), (h, qtile, k_head)


# ---------------------------------------- LSE-cached block importance (AdaSpa f3)
def _mass_check(sta, gp, qt, kt, vt, rp_t, ci_t, lse_cached, B, Hh, d, T, H, W, rows, sm_scale=0.0):
    g = sta.grid(T, H, W)
    nt = sta.sta_num_tiles(g)
    o_ref, lse_ref = gp.attn(qt, kt, vt, rp_t, ci_t, B, Hh, d, g, sm_scale)
    o = torch.full_like(qt, float("nan"))
    lse = torch.full(qt.shape[:3], float("nan"), dtype=torch.float32, device=qt.device)
    mass = torch.full((B, Hh, nt, nt), float("nan"), dtype=torch.float32, device=qt.device)
    sta.sta_attn_fwd_block_mass(qt, kt, vt, o, lse, rp_t, ci_t, lse_cached, mass, B, Hh, d, g, sm_scale)
    torch.cuda.synchronize()
    assert sta.sta_get_device_error() == sta.STA_OK
    # the attention outputs are those of sta_attn_fwd, bit for bit
    assert torch.equal(o.view(torch.int16), o_ref.view(torch.int16))
    assert torch.equal(lse, lse_ref)
    rp, ci = rp_t.cpu().numpy(), ci_t.cpu().numpy()
    res = O.block_mass(gp.to_np64(qt), gp.to_np64(kt), lse_cached.double().cpu().numpy(), rp, ci, T, H, W,
                       sm_scale, rows)
    m_np = mass.view(-1, nt).cpu().numpy()
    listed = np.zeros_like(m_np, dtype=bool)
    for r in range(m_np.shape[0]):
        listed[r, ci[rp[r]:rp[r + 1]]] = True
    assert np.all(m_np[~listed] == 0)
    for r, (tiles, want) in res.items():
        got = m_np[r, tiles]
        assert np.allclose(got, want, rtol=2e-4, atol=1e-9), (r, np.abs(got - want).max())
    return mass, lse


def test_block_mass_tiny_dense_exact_lse(sta, gp):
    """Dense list and the exact LSE of the same inputs: masses match the
    oracle and every row sums to one."""
    cfg = CONFIGS["tiny"]
    B, Hh, d, T, H, W = cfg.B, cfg.heads, cfg.d, cfg.T, cfg.H, cfg.W
    g = sta.grid(T, H, W)
    nt = sta.sta_num_tiles(g)
    q, k, v = (x.cuda() for x in make_qkv(cfg, device="cpu"))
    qt, kt, vt = (gp.reorder(x, B, Hh, d, g) for x in (q, k, v))
    rp, ci = _custom_csr(np.ones((B, Hh, nt, nt), dtype=bool))
    _, lse_exact = gp.attn(qt, kt, vt, rp, ci, B, Hh, d, g)
    mass, _ = _mass_check(sta, gp, qt, kt, vt, rp, ci, lse_exact, B, Hh, d, T, H, W, range(B * Hh * nt))
    sums = mass.sum(-1).cpu().numpy()
    assert np.allclose(sums, 1.0, atol=1e-4)


@pytest.mark.parametrize("d", [64, 128])
def test_block_mass_ragged_sparse_stale_lse(sta, gp, d):
    """Ragged grid, random lists (odd tile count), a cached LSE from perturbed
    inputs; then the selection on the masses is bit-exact."""
    T, H, W, Hh, B = 3, 19, 37, 2, 2
    g = sta.grid(T, H, W)
    nt = sta.sta_num_tiles(g)
    q, k, v = _structured(T, H, W, Hh, d, seed=31, B=B)
    qt, kt, vt = (gp.reorder(x, B, Hh, d, g) for x in (q, k, v))
    rng = np.random.default_rng(d + 1)
    mask = rng.random((B, Hh, nt, nt)) < 0.4
    rp, ci = _custom_csr(mask)
    q2 = (q.float() * 0.95 + 0.3 * torch.randn(q.shape, device="cuda")).to(torch.bfloat16)
    _, lse_stale = gp.attn(gp.reorder(q2, B, Hh, d, g), kt, vt, rp, ci, B, Hh, d, g)
    mass, _ = _mass_check(sta, gp, qt, kt, vt, rp, ci, lse_stale, B, Hh, d, T, H, W, range(B * Hh * nt))
    # selection on the exact masses
    params = sta.mask_params(0.8, 2, True, block_scores=mass)
    bufs = gp.build(None, None, B, Hh, d, g, params)
    rp_g, ci_g, nnz = gp.csr_np(bufs)
    used = np.clip(mass.cpu().numpy(), 0.0, 1.0).astype(np.float32)
    assert np.array_equal(bufs.block_probs.cpu().numpy(), used)
    rp_o, ci_o = O.mask_to_csr(O.select(used.astype(np.float64), 0.8, 2))
    assert np.array_equal(rp_g, rp_o) and np.array_equal(ci_g, ci_o)


def test_block_mass_720p_dense_sampled_rows(sta, gp):
    """The headline layer, dense list, exact LSE: sampled rows of masses."""
    cfg = CONFIGS["dit720p"]
    B, Hh, d, T, H, W = cfg.B, cfg.heads, cfg.d, cfg.T, cfg.H, cfg.W
    g = sta.grid(T, H, W)
    nt = sta.sta_num_tiles(g)
    q, k, v = make_qkv(cfg, device="cuda")
    qt, kt, vt = (gp.reorder(x, B, Hh, d, g) for x in (q, k, v))
    del q, k, v
    R = B * Hh * nt
    rp = (torch.arange(R + 1, device="cuda", dtype=torch.int64) * nt).to(torch.int32)
    ci = torch.arange(nt, device="cuda", dtype=torch.int32).repeat(R)
    _, lse_exact = gp.attn(qt, kt, vt, rp, ci, B, Hh, d, g)
    rng = np.random.default_rng(9)
    rows = sorted(rng.choice(R, 4, replace=False).tolist())
    mass, _ = _mass_check(sta, gp, qt, kt, vt, rp, ci, lse_exact, B, Hh, d, T, H, W, rows)
    sums = mass.view(-1, nt)[torch.tensor(rows, device="cuda")].sum(-1).cpu().numpy()
    assert np.allclose(sums, 1.0, atol=1e-4)


# ------------------------------------------ the two select passes, same P
@pytest.mark.parametrize("top_p,k_min,floor", [(0.95, 8, False), (0.6, 1, False), (0.0, 37, False),
                                               (0.9, 4, True), (1.0, 0, False)])
def test_register_select_equals_general_select_on_the_same_p(sta, gp, top_p, k_min, floor):
    """The select pass that holds the row in registers (rows from the scores)
    and the general one (caller block scores, 64-bit sums) reach the same CSR
    on the same P: the build's exported P fed back as block_scores (values in
    [0, 1], so the clamp changes nothing), with windows, on a 720p-shaped grid
    of 4 heads."""
    T, H, W, Hh, d = 21, 45, 80, 4, 128
    g = sta.grid(T, H, W)
    q, k, _ = _structured(T, H, W, Hh, d, seed=77)
    rng = np.random.default_rng(5)
    win = torch.from_numpy(rng.integers(-1, 3, size=(Hh, 3, 4)).astype(np.int32)).cuda()
    bufs = sta.MaskBuffers(1, Hh, d, g, "cuda", with_mask=True, with_probs=True)
    sta.build_mask(q, k, 1, Hh, d, g, sta.mask_params(top_p, k_min, True, 0.0, (0, 1, 4), win, floor), bufs,
                   raster=True)
    P = bufs.block_probs.clone()
    again = sta.MaskBuffers(1, Hh, d, g, "cuda", with_mask=True, with_probs=True)
    sta.build_mask(None, None, 1, Hh, d, g,
                   sta.mask_params(top_p, k_min, True, 0.0, (0, 1, 4), win, floor, block_scores=P), again)
    torch.cuda.synchronize()
    assert sta.sta_get_device_error() == sta.STA_OK
    assert torch.equal(again.block_probs.view(torch.int32), P.view(torch.int32))
    n = int(bufs.nnz.item())
    assert n == int(again.nnz.item())
    assert torch.equal(bufs.row_ptr, again.row_ptr) and torch.equal(bufs.col_idx[:n], again.col_idx[:n])
    assert torch.equal(bufs.block_mask, again.block_mask)


def test_caller_block_scores_with_row_mass_beyond_32_bits(sta, gp):
    """Caller block scores need not sum to one: rows of 1980 values in
    [0.5, 1] carry ~2^34 of integer mass, beyond 32 bits. The selection (top-p
    and the count floor) equals the oracle's, which sums in exact integers."""
    T, H, W, Hh = 33, 45, 80, 2
    g = sta.grid(T, H, W)
    nt = sta.sta_num_tiles(g)
    gen = torch.Generator(device="cuda").manual_seed(9)
    sc = (0.5 + 0.5 * torch.rand((1, Hh, nt, nt), generator=gen, device="cuda")).float()
    sc[0, 0, 3, :] = 1.0  # a row of ties
    sc[0, 1, 5, ::7] = 0.0
    for top_p, k_min in ((0.7, 3), (0.3, 900), (0.999, 0)):
        bufs = sta.MaskBuffers(1, Hh, 128, g, "cuda", with_mask=True)
        sta.build_mask(None, None, 1, Hh, 128, g, sta.mask_params(top_p, k_min, True, block_scores=sc), bufs)
        torch.cuda.synchronize()
        assert sta.sta_get_device_error() == sta.STA_OK
        want = O.select(sc.cpu().numpy().astype(np.float64), top_p, k_min)
        assert np.array_equal(bufs.block_mask.cpu().numpy().astype(bool), want)
        rp, ci = O.mask_to_csr(want)
        got_rp, got_ci, nnz = gp.csr_np(bufs)
        assert np.array_equal(got_rp, rp) and np.array_equal(got_ci, ci)


def test_rows_longer_than_2048_tiles_take_the_general_select(sta, gp):
    """Nt = 2304 (a 36 x 64 x 64 grid): past the register pass's 2048-tile
    rows the general select pass runs; its CSR equals the oracle's selection
    on the GPU's P, and P is within the bound."""
    T, H, W, Hh, d = 36, 64, 64, 1, 64
    g = sta.grid(T, H, W)
    nt = sta.sta_num_tiles(g)
    assert nt > 2048
    q, k, _ = _structured(T, H, W, Hh, d, seed=3)
    qt, kt = gp.reorder(q, 1, Hh, d, g), gp.reorder(k, 1, Hh, d, g)
    bufs = gp.build(qt, kt, 1, Hh, d, g, sta.mask_params(0.9, 5, True))
    torch.cuda.synchronize()
    assert sta.sta_get_device_error() == sta.STA_OK
    probs = bufs.block_probs.cpu().numpy()
    rows = np.random.default_rng(0).choice(nt, 64, replace=False)
    want = O.select(probs[0, 0, rows].astype(np.float64), 0.9, 5)
    assert np.array_equal(bufs.block_mask.cpu().numpy()[0, 0, rows].astype(bool), want)
    scale = 1.0 / math.sqrt(d)
    qb, kb = O.pool(gp.to_np64(qt), T, H, W), O.pool(gp.to_np64(kt), T, H, W)
    _, p_ref = O.block_scores(qb[:, :, rows], kb, scale)
    bound = gp.prob_bound(qb[:, :, rows], kb, scale, p_ref)
    assert np.all(np.abs(probs[:, :, rows] - p_ref) <= bound)
    assert np.max(np.abs(probs[:, :, rows] - p_ref) / bound) <= gp.PROB_ERR_CEILING


# ------------------------------------------------ pooled means (a2), directly
def _rna_tf32(x32):
    """fp32 -> the nearest tf32 (10 explicit mantissa bits), ties away from
    zero: half a tf32 unit added to the magnitude bits, then the 13 low bits
    cleared (the sign bit is untouched)."""
    u = np.ascontiguousarray(x32, dtype=np.float32).view(np.uint32)
    return ((u + np.uint32(0x1000)) & np.uint32(0xFFFFE000)).view(np.float32)


def _pooled_from_ws(sta, ws, B, Hh, d, g, ws_bytes):
    nt = sta.sta_num_tiles(g)
    R = B * Hh * nt
    off = sta.sta_build_mask_pooled_offsets(B, Hh, d, g, ws_bytes)

    def at(o):
        return ws[o:o + R * d * 4].view(torch.float32).view(B, Hh, nt, d).cpu().numpy()

    return at(off[0]), at(off[1]), (at(off[2]) if off[2] else None), (at(off[3]) if off[3] else None)


@pytest.mark.parametrize("T,H,W,Hh,d,B,raster,full_ws", [
    (3, 19, 37, 3, 128, 2, True, True), (3, 19, 37, 3, 128, 2, False, True),
    (3, 19, 37, 3, 128, 2, False, False), (5, 24, 37, 6, 64, 1, True, True),
    (2, 9, 10, 10, 128, 1, True, False), (1, 8, 8, 1, 64, 1, False, True)])
def test_pooled_means_bit_exact(sta, gp, T, H, W, Hh, d, B, raster, full_ws):
    """q-bar and k-bar as the mask build leaves them in its workspace, against
    the oracle's fp64 tile means: both sides sum the bf16 values exactly and
    divide by the real-token count in fp64, so the GPU's one rounding to fp32
    gives fp32(oracle mean) bit for bit; in the tensor-core layout the two
    stored parts are tf32(x) and tf32(x - tf32(x)), round to nearest, ties
    away (ragged grids, partial head boxes, raster and tiled pooling)."""
    g = sta.grid(T, H, W)
    q, k, _ = _structured(T, H, W, Hh, d, seed=41 + H, B=B)
    src = (q, k) if raster else (gp.reorder(q, B, Hh, d, g), gp.reorder(k, B, Hh, d, g))
    ws_bytes = (sta.sta_build_mask_workspace if full_ws else sta.sta_build_mask_workspace_min)(B, Hh, d, g)
    bufs = sta.MaskBuffers(B, Hh, d, g, "cuda")
    ws = torch.full((ws_bytes,), 0xFF, dtype=torch.uint8, device="cuda")
    params = sta.mask_params(0.9, 2, True)
    fn = sta.sta_build_mask_raster if raster else sta.sta_build_mask
    fn(src[0], src[1], B, Hh, d, g, params, bufs.row_ptr, bufs.col_idx, bufs.nnz, None, None, ws, ws_bytes)
    torch.cuda.synchronize()
    assert sta.sta_get_device_error() == sta.STA_OK
    qb, kb, qlo, klo = _pooled_from_ws(sta, ws, B, Hh, d, g, ws_bytes)
    for got, lo, x in ((qb, qlo, q), (kb, klo, k)):
        want = O.pool(O.reorder_fwd(gp.to_np64(x), T, H, W), T, H, W).astype(np.float32)
        if full_ws:
            hi = _rna_tf32(want)
            assert np.array_equal(got.view(np.uint32), hi.view(np.uint32))
            assert np.array_equal(lo.view(np.uint32), _rna_tf32(want - hi).view(np.uint32))
        else:
            assert lo is None
            assert np.array_equal(got.view(np.uint32), want.view(np.uint32))


def test_pooled_means_bit_exact_720p_sampled_heads(sta, gp):
    """The 720p layer in the benchmark's launch configuration (raster pooling
    through the TMA ring, full workspace): three sampled heads, every tile."""
    cfg = CONFIGS["dit720p"]
    B, Hh, d, T, H, W = cfg.B, cfg.heads, cfg.d, cfg.T, cfg.H, cfg.W
    g = sta.grid(T, H, W)
    q, k, _ = make_qkv(cfg, device="cuda")
    ws_bytes = sta.sta_build_mask_workspace(B, Hh, d, g)
    bufs = sta.MaskBuffers(B, Hh, d, g, "cuda")
    ws = torch.full((ws_bytes,), 0xFF, dtype=torch.uint8, device="cuda")
    params = sta.mask_params(cfg.top_p, cfg.k_min, True)
    sta.sta_build_mask_raster(q, k, B, Hh, d, g, params, bufs.row_ptr, bufs.col_idx, bufs.nnz, None, None, ws,
                              ws_bytes)
    torch.cuda.synchronize()
    assert sta.sta_get_device_error() == sta.STA_OK
    qb, kb, qlo, klo = _pooled_from_ws(sta, ws, B, Hh, d, g, ws_bytes)
    heads = [0, 17, 39]
    for got, lo, x in ((qb, qlo, q), (kb, klo, k)):
        sub = gp.to_np64(x[:, :, heads, :])
        want = O.pool(O.reorder_fwd(sub, T, H, W), T, H, W).astype(np.float32)
        hi = _rna_tf32(want)
        assert np.array_equal(got[:, heads].view(np.uint32), hi.view(np.uint32))
        assert np.array_equal(lo[:, heads].view(np.uint32), _rna_tf32(want - hi).view(np.uint32))


# ------------------------------------------ recall-driven window search (f2)
def _local_masses(T, H, W, shapes):
    """One [Nt, Nt] row-normalised mass per (st, sy, sx) spread of a Gaussian
    in tile distance (local-looking heads of different shape)."""
    nh, nw, nt, _ = O.tile_grid(T, H, W)
    idx = np.arange(nt)
    t, y, x = idx // (nh * nw), (idx // nw) % nh, idx % nw
    out = []
    for st, sy, sx in shapes:
        d2 = st * (t[:, None] - t[None]) ** 2 + sy * (y[:, None] - y[None]) ** 2 + sx * (x[:, None] - x[None]) ** 2
        m = np.exp(-d2)
        out.append(m / m.sum(1, keepdims=True))
    return np.stack(out)


def _search_check(sta, masses32, B, Hh, T, H, W, group_lo, tau, lam, heads=None):
    """Run the GPU search on fp32 masses [B*Hh, Nt, Nt]; compare the windows
    (exactly) and the stats with the oracle on the same fp32 values."""
    g = sta.grid(T, H, W)
    G = len(group_lo)
    mass_t = torch.from_numpy(masses32).cuda()
    win = torch.full((B * Hh, G, 4), 12345, dtype=torch.int32, device="cuda")
    stats = torch.full((B * Hh, 2), float("nan"), dtype=torch.float32, device="cuda")
    sta.sta_search_windows(mass_t, B, Hh, g, group_lo, tau, lam, win, stats)
    torch.cuda.synchronize()
    assert sta.sta_get_device_error() == sta.STA_OK
    win_np, st_np = win.cpu().numpy(), stats.cpu().numpy()
    for bh in (range(B * Hh) if heads is None else heads):
        want, st = O.search_windows(masses32[bh].astype(np.float64), T, H, W, group_lo, tau, lam)
        assert np.array_equal(win_np[bh], want), (bh, win_np[bh].tolist(), want.tolist())
        assert st_np[bh, 0] == np.float32(st["recall"]), (bh, st_np[bh, 0], st["recall"])
        assert st_np[bh, 1] == np.float32(st["density"]), (bh, st_np[bh, 1], st["density"])
    return win_np, st_np


@pytest.mark.parametrize("tau,lam", [(0.9, 1.0), (0.97, 0.5), (0.8, 2.0), (1.0, 1.0), (0.0, 0.0)])
def test_search_windows_synthetic_heads(sta, tau, lam):
    """Ragged grid, three groups, local heads of several shapes plus the
    degenerate ones (all mass on the own tile; no mass at all; uniform)."""
    T, H, W = 4, 24, 40
    nt = O.tile_grid(T, H, W)[2]
    local = _local_masses(T, H, W, [(2.0, 1.0, 0.3), (0.2, 0.05, 2.0), (5.0, 3.0, 3.0), (0.05, 0.5, 0.01)])
    extra = np.stack([np.eye(nt), np.zeros((nt, nt)), np.full((nt, nt), 1.0 / nt)])
    masses = np.concatenate([local, extra]).astype(np.float32)  # B = 1, 7 heads
    _search_check(sta, masses, 1, masses.shape[0], T, H, W, (0, 1, 3), tau, lam)


def test_search_windows_batch_and_single_group(sta):
    """B = 2 with one open-ended group on an odd tile grid."""
    T, H, W = 3, 19, 37
    masses = _local_masses(T, H, W, [(1.0, 0.5, 0.5), (0.1, 2.0, 0.1), (3.0, 0.02, 0.02), (0.5, 0.5, 0.05)])
    _search_check(sta, masses.astype(np.float32), 2, 2, T, H, W, (0,), 0.9, 1.0)


def test_search_windows_on_480p_block_masses(sta, gp):
    """The 480p layer: exact block masses of the dense attention (fused LSE
    path), then the search for every head; sampled heads match the oracle
    window for window, and every head's windows meet the recall target."""
    cfg = CONFIGS["dit480p"]
    B, Hh, d, T, H, W = cfg.B, cfg.heads, cfg.d, cfg.T, cfg.H, cfg.W
    g = sta.grid(T, H, W)
    nt = sta.sta_num_tiles(g)
    q, k, v = make_qkv(cfg, device="cuda")
    qt, kt, vt = (gp.reorder(x, B, Hh, d, g) for x in (q, k, v))
    del q, k, v
    R = B * Hh * nt
    rp = (torch.arange(R + 1, device="cuda", dtype=torch.int64) * nt).to(torch.int32)
    ci = torch.arange(nt, device="cuda", dtype=torch.int32).repeat(R)
    _, lse_exact = gp.attn(qt, kt, vt, rp, ci, B, Hh, d, g)
    o = torch.empty_like(qt)
    lse = torch.empty_like(lse_exact)
    mass = torch.empty((B, Hh, nt, nt), dtype=torch.float32, device="cuda")
    sta.sta_attn_fwd_block_mass(qt, kt, vt, o, lse, rp, ci, lse_exact, mass, B, Hh, d, g)
    torch.cuda.synchronize()
    masses = mass.view(B * Hh, nt, nt).cpu().numpy()
    tau, lam = 0.9, 1.0
    win, st = _search_check(sta, masses, B, Hh, T, H, W, cfg.group_lo, tau, lam, heads=(0, 17, 39))
    for bh in range(B * Hh):
        keep = O.window_mask(win[bh][None], cfg.group_lo, T, H, W)[0]
        w = np.floor(np.clip(masses[bh].astype(np.float64), 0, 1) * 2 ** 24)
        assert w[keep].sum() >= math.ceil(float(np.float32(tau)) * w.sum())
        assert st[bh, 1] == np.float32(keep.mean())


def test_search_windows_golden_cases(sta, golden_dir):
    """The hand-derived cases of the search (lambda choosing the cheap move,
    tau stopping one move early, a tie across groups, a cross grown out of two
    full windows): the kernel reaches the stated windows, recall and density."""
    import _search_cases as SC

    for case in SC.load(golden_dir):
        T, H, W = case["grid"]
        nt = O.tile_grid(T, H, W)[2]
        G = len(case["group_lo"])
        g = sta.grid(T, H, W)
        m = torch.from_numpy(SC.mass(case).astype(np.float32)[None]).cuda()
        win = torch.full((1, G, 4), 12345, dtype=torch.int32, device="cuda")
        stats = torch.full((1, 2), float("nan"), dtype=torch.float32, device="cuda")
        sta.sta_search_windows(m, 1, 1, g, tuple(case["group_lo"]), case["tau"], case["lambda"], win, stats)
        torch.cuda.synchronize()
        assert sta.sta_get_device_error() == sta.STA_OK
        assert win[0].cpu().tolist() == case["windows"], case["name"]
        st = stats[0].cpu().numpy()
        assert st[0] == np.float32(case["covered_units"] / case["total_units"]), case["name"]
        assert st[1] == np.float32(case["pairs"] / (nt * nt)), case["name"]


def test_search_windows_rejects_bad_groups(sta):
    g = sta.grid(4, 24, 40)
    nt = O.tile_grid(4, 24, 40)[2]
    m = torch.zeros((1, nt, nt), device="cuda")
    out = torch.empty((1, 2, 4), dtype=torch.int32, device="cuda")
    for lo, tau in (((1, 2), 0.9), ((0, 0), 0.9), ((0, 2), 1.5), ((0,) * 9, 0.9)):
        with pytest.raises(sta.StaError):
            sta.sta_search_windows(m, 1, 1, g, lo, tau, 1.0, out)


@pytest.mark.parametrize("floor", [False, True])
@pytest.mark.parametrize("d", [64, 128])
def test_build_mask_fused_and_tensor_core_layouts(sta, gp, floor, d):
    """The minimum workspace runs the fused pass (scores as fp32 FMA chains),
    the full one the tensor-core scores and a separate select pass. For each
    layout: P within that layout's own error bound of the oracle's P; the CSR
    and the byte mask equal to the oracle's selection (with the per-head
    floor when asked) on that layout's own P, OR the windows; without the
    floor, the selection differs from the oracle's own only at near-threshold
    tiles. The full layout without block_probs (rows in the workspace) gives
    the same CSR as with them."""
    T, H, W, Hh, B = 5, 24, 37, 3, 2
    g = sta.grid(T, H, W)
    q, k, _ = _structured(T, H, W, Hh, d, seed=23, B=B)
    qt, kt = (gp.reorder(x, B, Hh, d, g) for x in (q, k))
    nh, nw, nt, _ = O.tile_grid(T, H, W)
    win = np.tile(np.array([[[1, 1, 0, nw - 1], [0, 0, -1, -1]]], dtype=np.int32), (Hh, 1, 1))
    win_t = torch.from_numpy(win).cuda()
    top_p, k_min, glo = 0.8, 3, (0, 2)
    params = sta.mask_params(top_p, k_min, True, 0.0, glo, win_t, head_floor=floor)
    scale = 1.0 / math.sqrt(d)
    qb, kb = O.pool(gp.to_np64(qt), T, H, W), O.pool(gp.to_np64(kt), T, H, W)
    _, p_ref = O.block_scores(qb, kb, scale)
    wmask = O.window_mask(win, glo, T, H, W)[None]
    sizes = O.tile_sizes(T, H, W)
    own = O.select(p_ref, top_p, k_min)

    def run(ws_bytes, with_probs):
        bufs = sta.MaskBuffers(B, Hh, d, g, "cuda", True, with_probs)
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
        sta.sta_build_mask(qt, kt, B, Hh, d, g, params, bufs.row_ptr, bufs.col_idx, bufs.nnz, bufs.block_mask,
                           bufs.block_probs, ws, ws_bytes)
        torch.cuda.synchronize()
        assert sta.sta_get_device_error() == sta.STA_OK
        return bufs

    for fused in (True, False):
        ws_bytes = (sta.sta_build_mask_workspace_min if fused else sta.sta_build_mask_workspace)(B, Hh, d, g)
        bufs = run(ws_bytes, True)
        probs = bufs.block_probs.cpu().numpy()
        bound = gp.prob_bound(qb, kb, scale, p_ref, fused=fused)
        assert np.all(np.abs(probs.astype(np.float64) - p_ref) <= bound)
        assert np.max(np.abs(probs.astype(np.float64) - p_ref) / bound) <= gp.PROB_ERR_CEILING
        sel = _floor_mask(probs, top_p, k_min, sizes) if floor else O.select(probs, top_p, k_min)
        mask = sel | wmask
        assert np.array_equal(bufs.block_mask.cpu().numpy().astype(bool), mask)
        rp, ci, nnz = gp.csr_np(bufs)
        rp_o, ci_o = O.mask_to_csr(mask)
        assert np.array_equal(rp, rp_o) and np.array_equal(ci, ci_o)
        if not floor:
            _assert_near_threshold(own, sel, p_ref, bound, top_p)
        if not fused:
            other = run(ws_bytes, False)
            assert torch.equal(other.row_ptr, bufs.row_ptr)
            assert torch.equal(other.col_idx[:nnz], bufs.col_idx[:nnz])
            assert torch.equal(other.block_mask, bufs.block_mask)


# ------------------------------------------ raster-layout path (no reorder)
def _raster_vs_tiled(sta, gp, q, k, v, B, Hh, d, T, H, W, params, rows_check=None):
    """Mask and attention through the raster entry points equal, bit for bit,
    the tiled path followed by the inverse reorder; returns the raster O."""
    g = sta.grid(T, H, W)
    qt, kt, vt = (gp.reorder(x, B, Hh, d, g) for x in (q, k, v))
    bt = gp.build(qt, kt, B, Hh, d, g, params, with_mask=True, with_probs=True)
    br = sta.MaskBuffers(B, Hh, d, g, "cuda", True, True)
    sta.build_mask(q, k, B, Hh, d, g, params, br, raster=True)
    torch.cuda.synchronize()
    assert int(bt.nnz.item()) == int(br.nnz.item())
    nnz = int(bt.nnz.item())
    assert torch.equal(bt.row_ptr, br.row_ptr) and torch.equal(bt.col_idx[:nnz], br.col_idx[:nnz])
    assert torch.equal(bt.block_mask, br.block_mask)
    assert torch.equal(bt.block_probs, br.block_probs)
    o_t, lse_t = gp.attn(qt, kt, vt, bt.row_ptr, bt.col_idx, B, Hh, d, g)
    o_back = torch.full_like(q, float("nan"))
    sta.sta_reorder(o_t, o_back, B, Hh, d, g, inverse=True)
    o_r = torch.full_like(q, float("nan"))
    lse_r = torch.full_like(lse_t, float("nan"))
    sta.sta_attn_fwd_raster(q, k, v, o_r, lse_r, br.row_ptr, br.col_idx, B, Hh, d, g)
    torch.cuda.synchronize()
    assert sta.sta_get_device_error() == sta.STA_OK
    assert torch.equal(o_r.view(torch.int16), o_back.view(torch.int16))  # every raster row written
    valid = torch.from_numpy(O.valid_rows(T, H, W)).cuda()
    assert torch.equal(lse_r[:, :, valid], lse_t[:, :, valid])
    return o_r


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("T,H,W,Hh,B", [(3, 19, 37, 2, 2), (4, 16, 16, 3, 1), (2, 9, 10, 1, 1), (5, 24, 13, 2, 1),
                                        (3, 11, 20, 6, 1), (2, 8, 24, 10, 2)])
def test_raster_path_equals_tiled(sta, gp, d, T, H, W, Hh, B):
    """Raster and tiled calls agree bit for bit, and the raster output matches
    the oracle. Head counts below, at and above one pooling box (4 heads at
    d = 128, 8 at d = 64), with a partial last box."""
    q, k, v = _structured(T, H, W, Hh, d, seed=T * 7 + W, B=B)
    nh, nw, _, _ = O.tile_grid(T, H, W)
    win = np.zeros((Hh, 2, 4), dtype=np.int32)
    win[:, 0] = (1, 1, 0, nw - 1)
    win[:, 1] = (0, 0, -1, -1)
    win_t = torch.from_numpy(win).cuda()  # params holds only its pointer: keep it alive
    params = sta.mask_params(0.8, 2, True, 0.0, (0, 1), win_t)
    o_r = _raster_vs_tiled(sta, gp, q, k, v, B, Hh, d, T, H, W, params)
    # and against the oracle directly, on the raster output
    g = sta.grid(T, H, W)
    bt = gp.build(gp.reorder(q, B, Hh, d, g), gp.reorder(k, B, Hh, d, g), B, Hh, d, g, params)
    rp, ci, _ = gp.csr_np(bt)
    o_ref, _ = O.attention_all(*(O.reorder_fwd(gp.to_np64(x), T, H, W) for x in (q, k, v)), rp, ci, T, H, W,
                               1.0 / math.sqrt(d))
    want = O.reorder_inv(o_ref, T, H, W)
    err = np.abs(gp.to_np64(o_r) - want)
    assert err.max() <= ATOL_MAX and err.mean() <= ATOL_MEAN


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("T,H,W", [(1, 5, 3), (1, 20, 30), (2, 3, 40), (3, 1, 1), (7, 8, 8)])
def test_degenerate_grids(sta, gp, d, T, H, W):
    """One tile, one frame, tiles one token high, one token per frame, whole
    tiles only: raster and tiled calls agree bit for bit and match the oracle."""
    Hh, B = 2, 1
    q, k, v = _structured(T, H, W, Hh, d, seed=H * 31 + W, B=B)
    nh, nw, nt, _ = O.tile_grid(T, H, W)
    win_t = torch.from_numpy(np.tile(np.array([[1, 1, 0, nw - 1]], dtype=np.int32), (Hh, 1, 1))).cuda()
    params = sta.mask_params(0.9, 1, True, 0.0, (0,), win_t)
    o_r = _raster_vs_tiled(sta, gp, q, k, v, B, Hh, d, T, H, W, params)
    g = sta.grid(T, H, W)
    bt = gp.build(gp.reorder(q, B, Hh, d, g), gp.reorder(k, B, Hh, d, g), B, Hh, d, g, params)
    rp, ci, _ = gp.csr_np(bt)
    o_ref, _ = O.attention_all(*(O.reorder_fwd(gp.to_np64(x), T, H, W) for x in (q, k, v)), rp, ci, T, H, W,
                               1.0 / math.sqrt(d))
    err = np.abs(gp.to_np64(o_r) - O.reorder_inv(o_ref, T, H, W))
    assert err.max() <= ATOL_MAX and err.mean() <= ATOL_MEAN


def test_raster_path_equals_tiled_720p(sta, gp):
    """The headline layer: raster mask and attention equal the tiled path."""
    cfg = CONFIGS["dit720p"]
    B, Hh, d, T, H, W = cfg.B, cfg.heads, cfg.d, cfg.T, cfg.H, cfg.W
    q, k, v = make_qkv(cfg, device="cuda")
    win = torch.from_numpy(window_params(cfg, window_scale("dit720p", 0))).cuda()
    params = sta.mask_params(cfg.top_p, cfg.k_min, True, 0.0, cfg.group_lo, win)
    _raster_vs_tiled(sta, gp, q, k, v, B, Hh, d, T, H, W, params)


# ---------------------------------------------- rectified attention (f4)
def _rect(sta, qt, kt, vt, rp, ci, B, Hh, d, g, sm_scale=0.0):
    ws_bytes = sta.sta_rectified_workspace(B, Hh, d, g)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    o = torch.full_like(qt, float("nan"))
    lse = torch.full(qt.shape[:3], float("nan"), dtype=torch.float32, device="cuda")
    sta.sta_attn_fwd_rectified(qt, kt, vt, o, lse, rp, ci, ws, ws_bytes, B, Hh, d, g, sm_scale)
    torch.cuda.synchronize()
    assert sta.sta_get_device_error() == sta.STA_OK
    return o, lse


def _rect_check(sta, gp, qt, kt, vt, rp_t, ci_t, B, Hh, d, T, H, W, rows):
    """Rows of the GPU's rectified attention against the oracle, one head at
    a time (the oracle pools the whole head's K and V)."""
    g = sta.grid(T, H, W)
    o, lse = _rect(sta, qt, kt, vt, rp_t, ci_t, B, Hh, d, g)
    nt = sta.sta_num_tiles(g)
    rp, ci = rp_t.cpu().numpy(), ci_t.cpu().numpy()
    by_head = {}
    for r in rows:
        by_head.setdefault(int(r) // nt, []).append(int(r) % nt)
    errs = []
    for bh, qts in sorted(by_head.items()):
        b, h = divmod(bh, Hh)
        one = [gp.to_np64(x[b:b + 1, h:h + 1]) for x in (qt, kt, vt)]
        rp_h = rp[bh * nt:(bh + 1) * nt + 1] - rp[bh * nt]
        ci_h = ci[rp[bh * nt]:rp[(bh + 1) * nt]]
        o_np = gp.to_np64(o[b, h])
        l_np = lse[b, h].double().cpu().numpy()
        for _, qrows, o_ref, l_ref in O.rectified_attention_rows(*one, rp_h, ci_h, T, H, W, 0.0, qts):
            errs.append(np.abs(o_np[qrows] - o_ref).ravel())
            assert np.all(np.abs(l_np[qrows] - l_ref) <= LSE_TOL * np.maximum(1.0, np.abs(l_ref)))
    err = np.concatenate(errs)
    assert np.isfinite(err).all()
    assert err.max() <= ATOL_MAX and err.mean() <= ATOL_MEAN, (err.max(), err.mean())
    return o, lse


def test_rectified_with_every_tile_listed_equals_plain(sta, gp):
    """All tiles listed: every pooled column is masked and the output is that
    of sta_attn_fwd, bit for bit."""
    T, H, W, Hh, B, d = 3, 19, 37, 2, 2, 128
    g = sta.grid(T, H, W)
    nt = sta.sta_num_tiles(g)
    q, k, v = _structured(T, H, W, Hh, d, seed=5, B=B)
    qt, kt, vt = (gp.reorder(x, B, Hh, d, g) for x in (q, k, v))
    rp, ci = _custom_csr(np.ones((B, Hh, nt, nt), dtype=bool))
    o_p, l_p = gp.attn(qt, kt, vt, rp, ci, B, Hh, d, g)
    o_r, l_r = _rect(sta, qt, kt, vt, rp, ci, B, Hh, d, g)
    valid = torch.from_numpy(O.valid_rows(T, H, W)).cuda()
    assert torch.equal(o_r[:, :, valid].view(torch.int16), o_p[:, :, valid].view(torch.int16))
    assert torch.equal(l_r[:, :, valid], l_p[:, :, valid])


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("density", [0.0, 0.1, 0.5])
def test_rectified_ragged_sparse(sta, gp, d, density):
    """Ragged grid (odd tile count, partial tiles, Nt not a multiple of 64),
    random lists incl. empty rows: every row against the oracle."""
    T, H, W, Hh, B = 3, 19, 37, 2, 2
    g = sta.grid(T, H, W)
    nt = sta.sta_num_tiles(g)
    q, k, v = _structured(T, H, W, Hh, d, seed=11, B=B)
    qt, kt, vt = (gp.reorder(x, B, Hh, d, g) for x in (q, k, v))
    rng = np.random.default_rng(int(density * 100) + d)
    mask = rng.random((B, Hh, nt, nt)) < density
    mask[0, 0, 3] = False  # an empty row
    rp, ci = _custom_csr(mask)
    _rect_check(sta, gp, qt, kt, vt, rp, ci, B, Hh, d, T, H, W, range(B * Hh * nt))


def test_rectified_720p_sampled_rows(sta, gp):
    """The headline layer with its own mask: sampled rows against the oracle."""
    cfg = CONFIGS["dit720p"]
    B, Hh, d, T, H, W = cfg.B, cfg.heads, cfg.d, cfg.T, cfg.H, cfg.W
    g = sta.grid(T, H, W)
    nt = sta.sta_num_tiles(g)
    q, k, v = make_qkv(cfg, device="cuda")
    qt, kt, vt = (gp.reorder(x, B, Hh, d, g) for x in (q, k, v))
    del q, k, v
    win = torch.from_numpy(window_params(cfg, window_scale("dit720p", 0))).cuda()
    params = sta.mask_params(cfg.top_p, cfg.k_min, True, 0.0, cfg.group_lo, win)
    bufs = gp.build(qt, kt, B, Hh, d, g, params, with_mask=False, with_probs=False)
    rng = np.random.default_rng(17)
    rows = sorted(rng.choice(B * Hh * nt, 6, replace=False).tolist())
    nnz = int(bufs.nnz.item())
    _rect_check(sta, gp, qt, kt, vt, bufs.row_ptr, bufs.col_idx[:max(nnz, 1)], B, Hh, d, T, H, W, rows)
    del qt, kt, vt


def test_step_replays_from_a_cuda_graph(sta, gp):
    """The raster mask build and attention launch nothing that breaks stream
    capture (no allocation, no host synchronisation): a captured step replays
    with the same outputs as the eager calls."""
    T, H, W, Hh, B, d = 4, 30, 44, 4, 1, 128
    g = sta.grid(T, H, W)
    q, k, v = _structured(T, H, W, Hh, d, seed=41, B=B)
    nh, nw, nt, _ = O.tile_grid(T, H, W)
    win_t = torch.from_numpy(np.tile(np.array([[[1, 2, 0, nw - 1], [0, 0, -1, -1]]], dtype=np.int32),
                                     (Hh, 1, 1))).cuda()
    params = sta.mask_params(0.9, 2, True, 0.0, (0, 1), win_t)
    bufs = sta.MaskBuffers(B, Hh, d, g, "cuda")
    o_eager = torch.empty_like(q)
    sta.build_mask(q, k, B, Hh, d, g, params, bufs, raster=True)
    sta.sta_attn_fwd_raster(q, k, v, o_eager, None, bufs.row_ptr, bufs.col_idx, B, Hh, d, g)
    torch.cuda.synchronize()
    rp_eager = bufs.row_ptr.clone()
    o = torch.zeros_like(q)
    bufs.row_ptr.zero_()
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        sta.build_mask(q, k, B, Hh, d, g, params, bufs, raster=True)
        sta.sta_attn_fwd_raster(q, k, v, o, None, bufs.row_ptr, bufs.col_idx, B, Hh, d, g)
    for _ in range(2):
        graph.replay()
    torch.cuda.synchronize()
    assert sta.sta_get_device_error() == sta.STA_OK
    assert torch.equal(bufs.row_ptr, rp_eager)
    assert torch.equal(o.view(torch.int16), o_eager.view(torch.int16))
    del graph


def test_tma_stream_probe_runs_and_checks_arguments(sta):
    from block_sparse_attention_28_b200 import probe

    buf = torch.zeros(8 << 20, dtype=torch.uint8, device="cuda")
    probe.sta_probe_tma_stream(buf, 2, 4, 20)  # first launch loads the module
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    probe.sta_probe_tma_stream(buf, 2, 4, 200)
    e1.record()
    torch.cuda.synchronize()
    assert probe.sta_probe_get_device_error() == sta.STA_OK
    moved = torch.cuda.get_device_properties(0).multi_processor_count * 2 * 200 * 16384
    assert moved / (e0.elapsed_time(e1) * 1e-3) > 1e12  # well above 1 TB/s from L2
    with pytest.raises(sta.StaError):
        probe.sta_probe_tma_stream(buf, 2, 7, 10)  # more than 6 loads in flight
    with pytest.raises(sta.StaError):
        probe.sta_probe_tma_stream(buf, 8, 6, 10)  # does not fit in shared memory


# ------------------------------------------------------- failure detection
def test_bounded_wait_reports_timeout_and_context_survives(sta, gp):
    """The pipeline's bounded wait, on a barrier nothing completes, gives up
    after its limit and reports STA_ERR_TIMEOUT; the context keeps working."""
    sta.sta_get_device_error()
    sta.sta_selftest_wait_timeout(2_000_000)  # about a millisecond of SM cycles
    assert sta.sta_get_device_error() == sta.STA_ERR_TIMEOUT
    assert sta.sta_get_device_error() == sta.STA_OK
    test_attn_tiny_config(sta, gp)  # a full attention call still runs and matches


def _timeout_case(sta, gp):
    """A small layer (4 heads, d = 128, 4 x 40 x 48 grid, every key tile
    listed) in raster and tiled form."""
    B, Hh, d, T, H, W = 1, 4, 128, 4, 40, 48
    g = sta.grid(T, H, W)
    nt = sta.sta_num_tiles(g)
    q, k, v = _structured(T, H, W, Hh, d, seed=31)
    R = B * Hh * nt
    rp = (torch.arange(R + 1, device="cuda", dtype=torch.int64) * nt).to(torch.int32)
    ci = torch.arange(nt, device="cuda", dtype=torch.int32).repeat(R)
    return B, Hh, d, g, q, k, v, rp, ci


def test_attention_waits_run_out_drain_and_the_context_survives(sta, gp):
    """With the pipeline wait limit cut to 1,000 SM cycles (shorter than a
    tile load or a softmax step), the attention kernel's own waits run out:
    the call reports STA_ERR_TIMEOUT and no fault, the CTAs drain their copies
    and MMAs and free TMEM, and a call with the default limit afterwards, on
    the same context, gives output bit-identical to one made before."""
    B, Hh, d, g, q, k, v, rp, ci = _timeout_case(sta, gp)
    o_ref, lse_ref = torch.empty_like(q), torch.empty(B, Hh, sta.sta_tiled_len(g), device="cuda")
    sta.sta_attn_fwd_raster(q, k, v, o_ref, lse_ref, rp, ci, B, Hh, d, g)
    assert sta.sta_get_device_error() == sta.STA_OK
    assert sta.sta_get_wait_limit() == 2_000_000_000
    try:
        sta.sta_set_wait_limit(1000)
        assert sta.sta_get_wait_limit() == 1000
        o = torch.zeros_like(q)
        sta.sta_attn_fwd_raster(q, k, v, o, None, rp, ci, B, Hh, d, g)
        assert sta.sta_get_device_error() == sta.STA_ERR_TIMEOUT
    finally:
        sta.sta_set_wait_limit(0)
    assert sta.sta_get_wait_limit() == 2_000_000_000
    assert sta.sta_get_device_error() == sta.STA_OK
    o2, lse2 = torch.full_like(q, float("nan")), torch.full_like(lse_ref, float("nan"))
    sta.sta_attn_fwd_raster(q, k, v, o2, lse2, rp, ci, B, Hh, d, g)
    assert sta.sta_get_device_error() == sta.STA_OK
    assert torch.equal(o2.view(torch.int16), o_ref.view(torch.int16))
    assert torch.equal(lse2.view(torch.int32), lse_ref.view(torch.int32))


def test_mask_build_waits_run_out_drain_and_the_context_survives(sta, gp):
    """The same for the mask build's pipelined kernels (the raster pooling's
    TMA ring and the tensor-core scores): at a 1,000-cycle limit the build
    reports STA_ERR_TIMEOUT without a fault, and with the default limit it then
    gives the CSR, byte mask and P of a build made before, bit for bit."""
    B, Hh, d, g, q, k, _, _, _ = _timeout_case(sta, gp)
    params = sta.mask_params(0.9, 4, True)

    def build():
        bufs = sta.MaskBuffers(B, Hh, d, g, "cuda", with_mask=True, with_probs=True)
        sta.build_mask(q, k, B, Hh, d, g, params, bufs, raster=True)
        return bufs

    ref = build()
    assert sta.sta_get_device_error() == sta.STA_OK
    try:
        sta.sta_set_wait_limit(1000)
        build()
        assert sta.sta_get_device_error() == sta.STA_ERR_TIMEOUT
    finally:
        sta.sta_set_wait_limit(0)
    assert sta.sta_get_device_error() == sta.STA_OK
    again = build()
    assert sta.sta_get_device_error() == sta.STA_OK
    n = int(ref.nnz.item())
    assert n == int(again.nnz.item())
    assert torch.equal(again.row_ptr, ref.row_ptr) and torch.equal(again.col_idx[:n], ref.col_idx[:n])
    assert torch.equal(again.block_mask, ref.block_mask)
    assert torch.equal(again.block_probs.view(torch.int32), ref.block_probs.view(torch.int32))


def test_wait_limit_is_checked_on_the_host(sta):
    for bad in (1, 999, 2_000_000_001, -5):
        with pytest.raises(sta.StaError):
            sta.sta_set_wait_limit(bad)
    assert sta.sta_get_wait_limit() == 2_000_000_000


@pytest.mark.parametrize("a_tmem", [False, True])
def test_mma_rate_probe(sta, a_tmem):
    """The MMA-rate probe runs on every SM and reports a cost per MMA that
    respects the tensor core's dense peak (4096 bf16 multiply-adds per SM per
    clock): no width is measured faster than that bound."""
    from block_sparse_attention_28_b200 import probe

    iters = 1024
    for n in (64, 128, 256):
        cyc = probe.sta_probe_mma_rate(n, a_tmem, iters)
        torch.cuda.synchronize()
        assert probe.sta_probe_get_device_error() == sta.STA_OK
        assert cyc.numel() == torch.cuda.get_device_properties(0).multi_processor_count
        assert bool((cyc > 0).all())
        per = cyc.double() / iters
        floor = 128 * n * 16 / 4096  # cycles of the multiply-adds alone at the peak
        assert float(per.min()) >= 0.98 * floor
        assert float(per.max()) < 20 * floor
