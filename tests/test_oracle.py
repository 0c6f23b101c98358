"""Pins for the fp64 oracle: closed forms, textbook routines, brute force.

None of these call the CUDA path. Each test is chosen so that a plausible
slip in the oracle (a dropped pad exclusion, a wrong tile index, a flipped
comparison, a transposed operand, an off-by-one in the threshold) fails it.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import scipy.special
import torch

import oracle as O
from oracle import sta_oracle

import _search_cases as SC

RNG = np.random.default_rng(12345)


def _bf16_exact(shape, rng, scale=1.0):
    x = torch.from_numpy(rng.standard_normal(shape) * scale).to(torch.bfloat16)
    return x.to(torch.float64).numpy()


# ----------------------------------------------------------------- layout
def test_tile_grid_matches_workload_table():
    # Sizes of the five workloads (padded to whole 1x8x8 tiles).
    assert O.tile_grid(4, 16, 16) == (2, 2, 16, 1024)
    assert O.tile_grid(21, 30, 52) == (4, 7, 588, 37632)
    assert O.tile_grid(21, 45, 80) == (6, 10, 1260, 80640)
    assert O.tile_grid(33, 45, 80) == (6, 10, 1980, 126720)


def test_reorder_golden(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "reorder_cases.json")))
    T, H, W = g["grid"]["T"], g["grid"]["H"], g["grid"]["W"]
    assert O.tile_grid(T, H, W) == (g["grid"]["NH"], g["grid"]["NW"], g["grid"]["Nt"], g["grid"]["Lpad"])
    rows = O.tiled_row_of_raster(T, H, W)
    for tok in g["tokens"]:
        i = (tok["t"] * H + tok["y"]) * W + tok["x"]
        assert rows[i] == tok["row"], tok
    v = O.valid_rows(T, H, W).reshape(-1, 64).sum(axis=1)
    assert v.tolist() == g["valid_rows_per_tile"]


@pytest.mark.parametrize("T,H,W", [(2, 9, 10), (3, 13, 19), (1, 16, 8), (2, 1, 1)])
def test_reorder_tiles_are_spatial_blocks(T, H, W):
    """Every tile holds the tokens of one frame inside one 8x8 block, row-major;
    pad rows are zero; the map is a bijection onto the real rows."""
    nh, nw, nt, lpad = O.tile_grid(T, H, W)
    L = T * H * W
    t, y, x = np.meshgrid(np.arange(T), np.arange(H), np.arange(W), indexing="ij")
    # encode coordinates (+1 so that pads, which are 0, are distinguishable)
    x_r = np.stack([t.ravel() + 1, y.ravel() + 1, x.ravel() + 1], axis=1).astype(np.float64)
    x_r = x_r.reshape(1, L, 1, 3)
    xt = O.reorder_fwd(x_r, T, H, W)[0, 0]  # [Lpad, 3]
    assert xt.shape == (lpad, 3)
    real = xt[:, 0] > 0
    assert real.sum() == L
    assert np.all(xt[~real] == 0)
    tiles = xt.reshape(nt, 64, 3)
    for n in range(nt):
        tn, tyn, txn = n // (nh * nw), (n // nw) % nh, n % nw
        for r in range(64):
            if tiles[n, r, 0] == 0:
                # a pad row must be outside the grid
                yy, xx = 8 * tyn + r // 8, 8 * txn + r % 8
                assert yy >= H or xx >= W
                continue
            tt, yy, xx = (tiles[n, r] - 1).astype(int)
            assert tt == tn
            assert yy == 8 * tyn + r // 8 and xx == 8 * txn + r % 8
    back = O.reorder_inv(O.reorder_fwd(x_r, T, H, W), T, H, W)
    assert np.array_equal(back, x_r)


def test_reorder_roundtrip_multihead():
    T, H, W = 3, 11, 17
    x = _bf16_exact((2, T * H * W, 3, 8), RNG)
    xt = O.reorder_fwd(x, T, H, W)
    assert xt.shape == (2, 3, O.tile_grid(T, H, W)[3], 8)
    assert np.array_equal(O.reorder_inv(xt, T, H, W), x)
    # heads and batches do not mix: head h of the tiled tensor holds only head h
    for b in range(2):
        for h in range(3):
            assert np.array_equal(O.reorder_inv(xt[b:b + 1, h:h + 1], T, H, W)[0, :, 0], x[b, :, h])


# ---------------------------------------------------------------- pooling
def test_pool_closed_form_linear_field():
    """x(t, y, x) = a + b t + c y + e x: the mean over the real tokens of tile
    (t, ty, tx) with vy x vx real tokens is a + b t + c (8 ty + (vy-1)/2)
    + e (8 tx + (vx-1)/2) (arithmetic series)."""
    T, H, W = 3, 13, 21
    a, bb, c, e = 0.5, -1.25, 0.75, 2.0
    t, y, x = np.meshgrid(np.arange(T), np.arange(H), np.arange(W), indexing="ij")
    f = (a + bb * t + c * y + e * x).ravel()
    xr = f.reshape(1, -1, 1, 1)
    p = O.pool(O.reorder_fwd(xr, T, H, W), T, H, W)[0, 0, :, 0]
    nh, nw, nt, _ = O.tile_grid(T, H, W)
    for n in range(nt):
        tn, ty, tx = n // (nh * nw), (n // nw) % nh, n % nw
        vy, vx = min(8, H - 8 * ty), min(8, W - 8 * tx)
        want = a + bb * tn + c * (8 * ty + (vy - 1) / 2) + e * (8 * tx + (vx - 1) / 2)
        assert abs(p[n] - want) < 1e-12


def test_pool_excludes_pads():
    T, H, W = 2, 9, 10
    xr = np.ones((1, T * H * W, 2, 4))
    p = O.pool(O.reorder_fwd(xr, T, H, W), T, H, W)
    assert np.allclose(p, 1.0, atol=0, rtol=1e-15)


def test_pooled_score_is_mean_of_token_pair_logits():
    """scale * qbar . kbar equals the mean over all (query token, key token)
    pairs of scale * q . k (bilinearity), computed here by brute force."""
    T, H, W, d = 2, 9, 10, 6
    q = _bf16_exact((1, T * H * W, 1, d), RNG)
    k = _bf16_exact((1, T * H * W, 1, d), RNG)
    qt, kt = O.reorder_fwd(q, T, H, W), O.reorder_fwd(k, T, H, W)
    s, p = O.block_scores(O.pool(qt, T, H, W), O.pool(kt, T, H, W), 0.3)
    valid = O.valid_rows(T, H, W)
    nt = O.tile_grid(T, H, W)[2]
    for a in range(nt):
        for b in range(nt):
            qa = [qt[0, 0, r] for r in range(64 * a, 64 * a + 64) if valid[r]]
            kb = [kt[0, 0, r] for r in range(64 * b, 64 * b + 64) if valid[r]]
            tot = 0.0
            for u in qa:
                for w in kb:
                    tot += float(np.dot(u, w))
            assert abs(s[0, 0, a, b] - 0.3 * tot / (len(qa) * len(kb))) < 1e-10
    assert np.allclose(p[0, 0], scipy.special.softmax(s[0, 0], axis=-1), rtol=1e-13, atol=1e-15)
    assert np.allclose(p.sum(-1), 1.0, atol=1e-13)


# -------------------------------------------------------------- selection
def test_select_golden(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "select_cases.json")))
    for case in g["cases"]:
        keep = O.select_row(np.array(case["p"]), case["top_p"], case["k_min"])
        assert sorted(np.nonzero(keep)[0].tolist()) == case["keep"], case["name"]


def test_select_top_p_one_keeps_all():
    p = scipy.special.softmax(RNG.standard_normal((5, 37)) * 3, axis=-1)
    for row in p:
        assert O.select_row(row, 1.0, 0).all()
        assert O.select_row(row, 1.5, 0).all()


def test_select_top_p_zero_is_stable_topk():
    p = scipy.special.softmax(RNG.standard_normal((6, 29)) * 2, axis=-1)
    p[0, 3] = p[0, 7]  # a tie
    for row in p:
        for k in (0, 1, 5, 29, 40):
            keep = O.select_row(row, 0.0, k)
            want = np.argsort(-row, kind="stable")[: min(k, row.size)]
            assert sorted(np.nonzero(keep)[0].tolist()) == sorted(want.tolist())


def test_select_minimal_by_brute_force():
    """On Nt = 12, the kept set (k_min = 0) is a smallest subset whose integer
    mass reaches the threshold, and it is the prefix of the stated order."""
    nt = 12
    for trial in range(6):
        row = scipy.special.softmax(RNG.standard_normal(nt) * (1 + trial), axis=-1)
        for top_p in (0.3, 0.6, 0.9, 0.97):
            keep = O.select_row(row, top_p, 0)
            w = np.floor(row * 2 ** 24).astype(np.int64)
            thr = math.ceil(float(np.float32(top_p)) * float(w.sum()))
            best = None
            for m in range(nt + 1):
                if any(w[list(c)].sum() >= thr for c in itertools.combinations(range(nt), m)):
                    best = m
                    break
            assert keep.sum() == best
            assert w[keep].sum() >= thr
            order = sorted(range(nt), key=lambda j: (-row[j], j))
            assert set(np.nonzero(keep)[0]) == set(order[:best])


def test_select_monotone_in_top_p_and_k_min():
    row = scipy.special.softmax(RNG.standard_normal(50) * 2, axis=-1)
    prev = np.zeros(50, dtype=bool)
    for tp in np.linspace(0, 1, 21):
        for km in (0, 3, 10):
            keep = O.select_row(row, tp, km)
            assert (O.select_row(row, tp, km + 1) >= keep).all()
        keep0 = O.select_row(row, tp, 0)
        assert (keep0 >= prev).all()
        prev = keep0


# ----------------------------------------------------------------- window
def _window_count_closed_form(windows, group_lo, T, H, W, h, qt):
    """Row count as a sum over frames of |R1 u R2| = |R1| + |R2| - |R1 n R2|
    for two clipped rectangles centred on the query tile (inclusion-exclusion),
    independent of the oracle's per-pair test."""
    nh, nw, _, _ = O.tile_grid(T, H, W)
    tq, yq, xq = qt // (nh * nw), (qt // nw) % nh, qt % nw

    def span(c, r, n):
        if r < 0:
            return 0
        return min(n - 1, c + r) - max(0, c - r) + 1

    total = 0
    for tk in range(T):
        dt = abs(tq - tk)
        gs = [g for g in range(len(group_lo)) if group_lo[g] <= dt]
        if not gs:
            continue
        ry1, rx1, ry2, rx2 = windows[h, max(gs)]
        a1 = span(yq, ry1, nh) * span(xq, rx1, nw)
        a2 = span(yq, ry2, nh) * span(xq, rx2, nw)
        ry3 = min(ry1, ry2) if min(ry1, rx1, ry2, rx2) >= 0 else -1
        rx3 = min(rx1, rx2) if ry3 >= 0 else -1
        a3 = span(yq, ry3, nh) * span(xq, rx3, nw)
        total += a1 + a2 - a3
    return total


def test_window_counts_closed_form():
    T, H, W = 5, 40, 56  # 5 x 5 x 7 tiles
    windows = np.array([
        [[1, 1, 0, 6], [0, 1, -1, -1], [-1, -1, -1, -1]],
        [[2, 0, 0, 3], [1, 1, 4, 0], [0, 0, 0, 0]],
        [[4, 6, -1, -1], [-1, -1, 2, 2], [1, 0, 0, 1]],
    ], dtype=np.int32)
    group_lo = [0, 1, 3]
    m = O.window_mask(windows, group_lo, T, H, W)
    nt = O.tile_grid(T, H, W)[2]
    for h in range(3):
        for qt in range(nt):
            assert m[h, qt].sum() == _window_count_closed_form(windows, group_lo, T, H, W, h, qt)
        assert np.array_equal(m[h], m[h].T)  # |dt|, |dy|, |dx| are symmetric


def test_window_tiny_separates_local_and_axial():
    """2 x 4 x 6 tile grid: local radius 1 plus full-row axial window for
    |dt| = 0, nothing for |dt| >= 1: row count = 3x3-clipped block + rest of
    the row, all in the query's own frame."""
    T, H, W = 2, 32, 48
    nh, nw, nt, _ = O.tile_grid(T, H, W)
    windows = np.array([[[1, 1, 0, nw - 1], [-1, -1, -1, -1]]], dtype=np.int32)
    m = O.window_mask(windows, [0, 1], T, H, W)[0]
    # the last group is open-ended: one group [0] alone covers every frame
    m_all = O.window_mask(windows[:, :1], [0], T, H, W)[0]
    assert m_all.sum() == T * m.sum()
    for qt in range(nt):
        tq, yq, xq = qt // (nh * nw), (qt // nw) % nh, qt % nw
        ny = min(nh - 1, yq + 1) - max(0, yq - 1) + 1
        nx = min(nw - 1, xq + 1) - max(0, xq - 1) + 1
        assert m[qt].sum() == ny * nx + (nw - nx)
        # nothing in the other frame
        other = [k for k in range(nt) if k // (nh * nw) != tq]
        assert not m[qt, other].any()


def test_window_monotone_in_extent():
    T, H, W = 3, 24, 40
    base = np.array([[[1, 1, 0, 2], [0, 0, -1, -1]]], dtype=np.int32)
    m0 = O.window_mask(base, [0, 1], T, H, W)
    for h_ in range(2):
        for c in range(4):
            wider = base.copy()
            wider[0, h_, c] += 1
            assert (O.window_mask(wider, [0, 1], T, H, W) >= m0).all()


# -------------------------------------------------------------------- CSR
def test_csr_invariants():
    mask = RNG.random((2, 3, 9, 9)) < 0.3
    mask[0, 1, 4] = False  # an empty row
    rp, ci = O.mask_to_csr(mask)
    assert rp[0] == 0 and rp[-1] == ci.size == mask.sum()
    assert np.all(np.diff(rp) >= 0)
    flat = mask.reshape(-1, 9)
    for r in range(flat.shape[0]):
        cols = ci[rp[r]:rp[r + 1]]
        assert np.all(np.diff(cols) > 0)
        assert set(cols.tolist()) == set(np.nonzero(flat[r])[0].tolist())


def test_build_mask_union_of_parts():
    T, H, W, d = 3, 16, 24, 8
    q = _bf16_exact((1, T * H * W, 2, d), RNG, 2.0)
    k = _bf16_exact((1, T * H * W, 2, d), RNG, 2.0)
    qt, kt = O.reorder_fwd(q, T, H, W), O.reorder_fwd(k, T, H, W)
    win = np.array([[[0, 0, -1, -1], [-1, -1, -1, -1]], [[1, 0, 0, 2], [0, 0, -1, -1]]], dtype=np.int32)
    res = O.build_mask(qt, kt, T, H, W, True, 0.8, 2, win, [0, 1])
    only_sel = O.build_mask(qt, kt, T, H, W, True, 0.8, 2, None, None)
    only_win = O.build_mask(qt, kt, T, H, W, False, 0.0, 0, win, [0, 1])
    assert np.array_equal(res["mask"], only_sel["mask"] | only_win["mask"])
    assert np.array_equal(only_sel["mask"], O.select(res["probs"], 0.8, 2))
    assert (only_sel["mask"].sum(-1) >= 2).all()


# -------------------------------------------------------------- attention
def _sdpa64(q, k, v, scale):
    import torch.nn.functional as F
    tq = torch.from_numpy(q)[None, None]
    tk = torch.from_numpy(k)[None, None]
    tv = torch.from_numpy(v)[None, None]
    return F.scaled_dot_product_attention(tq, tk, tv, scale=scale)[0, 0].numpy()


def test_dense_mask_equals_sdpa():
    """A full mask reproduces dense softmax attention (torch SDPA, fp64)."""
    T, H, W, d = 2, 16, 16, 16
    q = _bf16_exact((1, T * H * W, 1, d), RNG)
    k = _bf16_exact((1, T * H * W, 1, d), RNG)
    v = _bf16_exact((1, T * H * W, 1, d), RNG)
    qt, kt, vt = (O.reorder_fwd(a, T, H, W) for a in (q, k, v))
    nt = O.tile_grid(T, H, W)[2]
    rp, ci = O.mask_to_csr(np.ones((1, 1, nt, nt), dtype=bool))
    Ot, lse = O.attention_all(qt, kt, vt, rp, ci, T, H, W, 0.0)
    o_r = O.reorder_inv(Ot, T, H, W)[0, :, 0]
    ref = _sdpa64(q[0, :, 0], k[0, :, 0], v[0, :, 0], 1 / math.sqrt(d))
    assert np.allclose(o_r, ref, atol=1e-12, rtol=1e-12)
    s = q[0, :, 0] @ k[0, :, 0].T / math.sqrt(d)
    lse_ref = scipy.special.logsumexp(s, axis=1)
    assert np.allclose(O.reorder_inv(lse[..., None], T, H, W)[0, :, 0, 0], lse_ref, atol=1e-12)


def test_dense_mask_ragged_grid_equals_sdpa_over_real_tokens():
    T, H, W, d = 2, 9, 13, 8
    q = _bf16_exact((1, T * H * W, 1, d), RNG)
    k = _bf16_exact((1, T * H * W, 1, d), RNG)
    v = _bf16_exact((1, T * H * W, 1, d), RNG)
    qt, kt, vt = (O.reorder_fwd(a, T, H, W) for a in (q, k, v))
    nt = O.tile_grid(T, H, W)[2]
    rp, ci = O.mask_to_csr(np.ones((1, 1, nt, nt), dtype=bool))
    Ot, _ = O.attention_all(qt, kt, vt, rp, ci, T, H, W, 0.7)
    ref = _sdpa64(q[0, :, 0], k[0, :, 0], v[0, :, 0], 0.7)
    assert np.allclose(O.reorder_inv(Ot, T, H, W)[0, :, 0], ref, atol=1e-12)


def test_attention_weights_convex():
    """With V = 1 every output is exactly 1 (weights sum to one); outputs lie in
    the per-coordinate range of the attended values."""
    T, H, W, d = 2, 16, 24, 8
    q = _bf16_exact((1, T * H * W, 2, d), RNG, 3.0)
    k = _bf16_exact((1, T * H * W, 2, d), RNG, 3.0)
    v = _bf16_exact((1, T * H * W, 2, d), RNG)
    qt, kt, vt = (O.reorder_fwd(a, T, H, W) for a in (q, k, v))
    nt = O.tile_grid(T, H, W)[2]
    mask = RNG.random((1, 2, nt, nt)) < 0.4
    mask[0, 0, 0] = False
    rp, ci = O.mask_to_csr(mask)
    ones = np.ones_like(vt)
    res1 = O.attention_rows(qt, kt, ones, rp, ci, T, H, W, 0.0, range(2 * nt))
    for r, qrows, o, lse in res1:
        if rp[r + 1] > rp[r]:
            assert np.allclose(o, 1.0, atol=1e-12)
        else:
            assert np.all(o == 0) and np.all(np.isneginf(lse))
    res = O.attention_rows(qt, kt, vt, rp, ci, T, H, W, 0.0, range(2 * nt))
    for r, qrows, o, lse in res:
        tiles = ci[rp[r]:rp[r + 1]]
        if tiles.size == 0:
            continue
        h = r // nt
        rows = (tiles[:, None] * 64 + np.arange(64)).ravel()
        vv = vt[0, h, rows]
        assert np.all(o <= vv.max(axis=0) + 1e-12) and np.all(o >= vv.min(axis=0) - 1e-12)


def test_single_tile_list_is_plain_softmax():
    T, H, W, d = 1, 16, 16, 16
    q = _bf16_exact((1, T * H * W, 1, d), RNG, 2.0)
    k = _bf16_exact((1, T * H * W, 1, d), RNG, 2.0)
    v = _bf16_exact((1, T * H * W, 1, d), RNG)
    qt, kt, vt = (O.reorder_fwd(a, T, H, W) for a in (q, k, v))
    rp = np.array([0, 1, 2, 3, 4], dtype=np.int32)
    ci = np.array([3, 0, 2, 1], dtype=np.int32)
    res = O.attention_rows(qt, kt, vt, rp, ci, T, H, W, 0.25, range(4))
    for r, qrows, o, lse in res:
        kk = kt[0, 0, 64 * ci[r]:64 * ci[r] + 64]
        vv = vt[0, 0, 64 * ci[r]:64 * ci[r] + 64]
        s = qt[0, 0, qrows] @ kk.T * 0.25
        assert np.allclose(o, scipy.special.softmax(s, axis=1) @ vv, atol=1e-12)
        assert np.allclose(lse, scipy.special.logsumexp(s, axis=1), atol=1e-12)


# ------------------------------------------------- per-head top-k floor (f1)
def test_head_floor_golden(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "head_floor_cases.json")))
    for c in g["floor_cases"]:
        assert O.head_topk_floor(c["counts"], c["sizes"]) == c["k_head"], c["why"]
    sc = g["select_case"]
    P = np.array(sc["p"])
    base = np.stack([O.select_row(r, sc["top_p"], sc["k_min"]) for r in P])
    assert [np.nonzero(r)[0].tolist() for r in base] == sc["base_keep"]
    keep, k_head = O.select_with_head_floor(P, sc["top_p"], sc["k_min"], sc["sizes"])
    assert k_head == sc["k_head"]
    assert [np.nonzero(r)[0].tolist() for r in keep] == sc["keep"]


def test_head_floor_properties():
    """The floor never removes a tile, leaves rows at or above k_head alone,
    brings every other row to exactly min(k_head, Nt), and with all base
    counts equal changes nothing."""
    rng = np.random.default_rng(8)
    for trial in range(5):
        P = scipy.special.softmax(rng.standard_normal((20, 31)) * (1 + trial), axis=-1)
        sizes = rng.integers(1, 65, size=20)
        base = np.stack([O.select_row(r, 0.8, 2) for r in P])
        keep, k_head = O.select_with_head_floor(P, 0.8, 2, sizes)
        assert (keep >= base).all()
        bc = base.sum(1)
        want = np.where(bc >= k_head, bc, min(k_head, 31))
        assert np.array_equal(keep.sum(1), want)
        assert k_head == -(-int((sizes * bc).sum()) // int(sizes.sum()))
    P = np.full((4, 8), 1 / 8)
    keep, k_head = O.select_with_head_floor(P, 0.5, 0, [64] * 4)
    assert k_head == 4 and np.array_equal(keep, np.stack([O.select_row(r, 0.5, 0) for r in P]))


def test_tile_sizes():
    assert O.tile_sizes(2, 9, 10).tolist() == [64, 16, 8, 2] * 2


# ------------------------------------------- LSE-cached block importance (f3)
def test_block_mass_is_block_sum_of_dense_softmax():
    """With the exact LSE and every tile listed, the block masses are the block
    sums of the dense softmax matrix (scipy), averaged over the query tile's
    real tokens; every row of masses sums to one."""
    T, H, W, d = 2, 9, 13, 8  # ragged tiles
    q = _bf16_exact((1, T * H * W, 1, d), RNG, 2.0)
    k = _bf16_exact((1, T * H * W, 1, d), RNG, 2.0)
    v = _bf16_exact((1, T * H * W, 1, d), RNG)
    qt, kt, vt = (O.reorder_fwd(a, T, H, W) for a in (q, k, v))
    nh, nw, nt, _ = O.tile_grid(T, H, W)
    rp, ci = O.mask_to_csr(np.ones((1, 1, nt, nt), dtype=bool))
    _, lse = O.attention_all(qt, kt, vt, rp, ci, T, H, W, 0.4)
    res = O.block_mass(qt, kt, lse, rp, ci, T, H, W, 0.4, range(nt))
    valid = O.valid_rows(T, H, W)
    real = np.nonzero(valid)[0]
    P = scipy.special.softmax(qt[0, 0, real] @ kt[0, 0, real].T * 0.4, axis=1)
    tile_of = real // 64
    for r in range(nt):
        tiles, masses = res[r]
        assert abs(masses.sum() - 1.0) < 1e-12
        rows_r = tile_of == r
        for kt_i, mval in zip(tiles, masses):
            want = P[np.ix_(rows_r, tile_of == kt_i)].sum() / rows_r.sum()
            assert abs(mval - want) < 1e-12


def test_block_mass_with_stale_lse_scales_by_the_lse_gap():
    """A cached LSE larger by delta scales every mass by exp(-delta)."""
    T, H, W, d = 1, 16, 16, 8
    q = _bf16_exact((1, T * H * W, 1, d), RNG)
    k = _bf16_exact((1, T * H * W, 1, d), RNG)
    qt, kt = O.reorder_fwd(q, T, H, W), O.reorder_fwd(k, T, H, W)
    nt = O.tile_grid(T, H, W)[2]
    rp, ci = O.mask_to_csr(np.ones((1, 1, nt, nt), dtype=bool))
    lse = np.zeros((1, 1, 64 * nt))
    a = O.block_mass(qt, kt, lse, rp, ci, T, H, W, 0.0, range(nt))
    b = O.block_mass(qt, kt, lse + 0.5, rp, ci, T, H, W, 0.0, range(nt))
    for r in range(nt):
        assert np.allclose(b[r][1], a[r][1] * math.exp(-0.5), rtol=1e-13)


# ------------------------------------------------ recall-driven window search (f2)
def _coverage(win, group_lo, T, H, W, mass):
    m = O.window_mask(np.asarray(win)[None], group_lo, T, H, W)[0]
    w = np.floor(np.clip(mass, 0, 1) * 2 ** 24).astype(np.int64)
    return m, int(w[m].sum()), int(w.sum())


def _search_case_result(search, case):
    T, H, W = case["grid"]
    win, st = search(SC.mass(case), T, H, W, tuple(case["group_lo"]), case["tau"], case["lambda"])
    nt = O.tile_grid(T, H, W)[2]
    return dict(moves=list(st["moves"]), windows=win.tolist(), covered_units=st["covered"] / SC.UNIT,
                total_units=st["total"] / SC.UNIT, pairs=round(st["density"] * nt * nt))


def test_window_search_golden(golden_dir):
    """Hand-derived move sequences (Compact Attention Figs. 3-4 as read): lambda
    choosing the cheap move, the same masses at lambda = 0, tau stopping the
    descent one move early, an exact tie of J across groups, and a cross grown
    out of two full windows by moves that uncover nothing."""
    for case in SC.load(golden_dir):
        got = _search_case_result(O.search_windows, case)
        assert got == {k: case[k] for k in SC.FIELDS}, (case["name"], got)


# Each planted mistake is a plausible slip in the step rule; each must change
# the outcome of at least one golden case.
SEARCH_MUTANTS = {
    "first admissible move instead of the best": ("if best is None or J > best[0]:", "if best is None:"),
    "lambda term with the wrong sign": ("- lam * (lost", "+ lam * (lost"),
    "ties to the highest index": ("J > best[0]", "J >= best[0]"),
    "recall bound strict": ("if covered - lost < thr:", "if covered - lost <= thr:"),
    "no cost constraint": ("if J < 0.0:", "if False:"),
    "a move must uncover a pair": ("if covered - lost < thr:", "if removed == 0 or covered - lost < thr:"),
    "lambda term dropped": ("- lam * (lost / float(total) if total else 0.0)", ""),
    "removed pairs not normalised": ("removed / float(nt * nt)", "float(removed)"),
}


def _mutant(old, new):
    import inspect

    src = inspect.getsource(O.search_windows)
    assert src.count(old) == 1, old
    ns = dict(vars(sta_oracle))
    exec(compile(src.replace(old, new), "<mutant>", "exec"), ns)
    return ns["search_windows"]


@pytest.mark.parametrize("name", sorted(SEARCH_MUTANTS))
def test_window_search_planted_mistakes_fail_the_golden_cases(golden_dir, name):
    search = _mutant(*SEARCH_MUTANTS[name])
    wrong = 0
    for case in SC.load(golden_dir):
        wrong += _search_case_result(search, case) != {k: case[k] for k in SC.FIELDS}
    assert wrong >= 1, name


def test_window_search_keeps_everything_at_full_recall_with_dense_mass():
    """tau = 1 and every pair carries mass: no pair can go, so the mask stays
    full; only the moves that uncover nothing run (the first window of every
    group is switched off one extent at a time)."""
    rng = np.random.default_rng(1)
    T, H, W = 3, 24, 32
    nh, nw, nt, _ = O.tile_grid(T, H, W)
    mass = rng.random((nt, nt)) + 0.1
    mass /= mass.sum(1, keepdims=True)
    win, st = O.search_windows(mass, T, H, W, (0, 1), 1.0, 1.0)
    assert st["recall"] == 1.0 and st["density"] == 1.0
    assert (win == np.array([-1, -1, nh - 1, nw - 1])).all()
    # group 0's ry1 steps first (index 0), then its rx1, then group 1's
    assert st["moves"] == [0] * nh + [1] * nw + [6] * nh + [7] * nw


def test_window_search_diagonal_mass_shrinks_to_the_own_tile():
    """All mass on the query's own tile: at tau = 1 the search removes every
    other pair (closed form: density 1/Nt, recall 1)."""
    T, H, W = 3, 24, 32
    nt = O.tile_grid(T, H, W)[2]
    mass = np.eye(nt)
    win, st = O.search_windows(mass, T, H, W, (0, 1), 1.0, 1.0)
    m, cov, tot = _coverage(win, (0, 1), T, H, W, mass)
    assert st["recall"] == 1.0 and cov == tot
    assert m.sum() == nt and np.array_equal(m, np.eye(nt, dtype=bool))


def test_window_search_zero_target_removes_everything():
    rng = np.random.default_rng(2)
    T, H, W = 2, 16, 24
    nt = O.tile_grid(T, H, W)[2]
    mass = rng.random((nt, nt))
    win, st = O.search_windows(mass, T, H, W, (0, 1), 0.0, 0.0)
    assert st["density"] == 0.0 and st["recall"] == 0.0
    assert (win == -1).all()


def test_window_search_result_is_feasible_and_locally_final():
    """On local-looking masses: the final recall (recomputed from the windows)
    meets tau, and no single move of the move set meets both constraints
    (recall >= tau and J >= 0), checked by direct enumeration."""
    T, H, W = 4, 24, 40
    nh, nw, nt, _ = O.tile_grid(T, H, W)
    idx = np.arange(nt)
    t, y, x = idx // (nh * nw), (idx // nw) % nh, idx % nw
    d2 = (t[:, None] - t[None]) ** 2 * 2.0 + (y[:, None] - y[None]) ** 2 + 0.3 * (x[:, None] - x[None]) ** 2
    mass = np.exp(-d2)
    mass /= mass.sum(1, keepdims=True)
    group_lo = (0, 1, 3)
    for tau, lam in ((0.9, 1.0), (0.97, 0.5), (0.8, 2.0), (0.9, 0.0)):
        win, st = O.search_windows(mass, T, H, W, group_lo, tau, lam)
        m, cov, tot = _coverage(win, group_lo, T, H, W, mass)
        thr = math.ceil(float(np.float32(tau)) * tot)
        assert cov == st["covered"] and cov >= thr
        assert st["density"] == m.mean() < 1.0
        for g in range(len(group_lo)):
            for ext in O.SEARCH_MOVES:
                cand = win.astype(np.int64).copy()
                if any(cand[g, e] <= -1 for e in ext):
                    continue
                for e in ext:
                    cand[g, e] -= 1
                m2, cov2, _ = _coverage(cand, group_lo, T, H, W, mass)
                removed = int((m & ~m2).sum())
                J = removed / float(nt * nt) - float(np.float32(lam)) * (cov - cov2) / float(tot)
                assert cov2 < thr or J < 0.0, (tau, lam, g, ext)


# ------------------------------------------- rectified attention (f4 reading)
def _tile_constant(T, H, W, Hh, d, rng, scale=1.0):
    """Raster [1, L, Hh, d] whose real tokens of each 1x8x8 tile share one
    bf16-exact vector (so a tile's mean equals each of its tokens)."""
    nh, nw, nt, _ = O.tile_grid(T, H, W)
    per_tile = torch.from_numpy(rng.standard_normal((nt, Hh, d)) * scale).to(torch.bfloat16).double().numpy()
    t, y, x = np.meshgrid(np.arange(T), np.arange(H), np.arange(W), indexing="ij")
    tile = ((t * nh + y // 8) * nw + x // 8).reshape(-1)
    return per_tile[tile][None]


def test_rectified_with_every_tile_listed_is_plain_attention():
    T, H, W, d = 2, 9, 13, 8
    q = _bf16_exact((1, T * H * W, 1, d), RNG, 2.0)
    k = _bf16_exact((1, T * H * W, 1, d), RNG, 2.0)
    v = _bf16_exact((1, T * H * W, 1, d), RNG)
    qt, kt, vt = (O.reorder_fwd(a, T, H, W) for a in (q, k, v))
    nt = O.tile_grid(T, H, W)[2]
    rp, ci = O.mask_to_csr(np.ones((1, 1, nt, nt), dtype=bool))
    plain = O.attention_rows(qt, kt, vt, rp, ci, T, H, W, 0.0, range(nt))
    rect = O.rectified_attention_rows(qt, kt, vt, rp, ci, T, H, W, 0.0, range(nt))
    for (r1, q1, o1, l1), (r2, q2, o2, l2) in zip(plain, rect):
        assert r1 == r2 and np.array_equal(q1, q2)
        assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


@pytest.mark.parametrize("density", [0.0, 0.3, 0.7])
def test_rectified_is_exact_when_tiles_are_constant(density):
    """If every token of a tile carries the tile's key and value, a skipped
    tile's pooled term (multiplicity x exp(q.k_bar), value v_bar) is exactly
    its tokens' contribution: for any mask the rectified output and LSE equal
    dense attention over all real tokens (torch SDPA in fp64, scipy logsumexp).
    Ragged grid, so multiplicities differ between tiles."""
    rng = np.random.default_rng(int(density * 10) + 3)
    T, H, W, d, Hh = 3, 11, 19, 8, 2
    q = _bf16_exact((1, T * H * W, Hh, d), rng, 1.5)
    k = _tile_constant(T, H, W, Hh, d, rng, 1.5)
    v = _tile_constant(T, H, W, Hh, d, rng)
    qt, kt, vt = (O.reorder_fwd(a, T, H, W) for a in (q, k, v))
    nt = O.tile_grid(T, H, W)[2]
    mask = rng.random((1, Hh, nt, nt)) < density
    rp, ci = O.mask_to_csr(mask)
    res = O.rectified_attention_rows(qt, kt, vt, rp, ci, T, H, W, 0.0, range(Hh * nt))
    Ot = np.full(qt.shape, np.nan)
    Lt = np.full(qt.shape[:3], np.nan)
    for r, qrows, o, lse in res:
        h, _ = divmod(r, nt)
        Ot[0, h, qrows] = o
        Lt[0, h, qrows] = lse
    o_r = O.reorder_inv(Ot, T, H, W)[0]
    l_r = O.reorder_inv(Lt[..., None], T, H, W)[0, :, :, 0]
    for h in range(Hh):
        ref = _sdpa64(q[0, :, h], k[0, :, h], v[0, :, h], 1 / math.sqrt(d))
        assert np.allclose(o_r[:, h], ref, atol=1e-10, rtol=1e-10)
        lse_ref = scipy.special.logsumexp(q[0, :, h] @ k[0, :, h].T / math.sqrt(d), axis=1)
        assert np.allclose(l_r[:, h], lse_ref, atol=1e-10)


def test_rectified_weights_sum_to_one_and_pool_over_real_tokens():
    """V = 1 gives exactly 1 (kept and pooled weights share one normaliser);
    the pooled key and value of a partial tile average only its real tokens."""
    T, H, W, d = 2, 10, 12, 8
    q = _bf16_exact((1, T * H * W, 1, d), RNG, 2.0)
    k = _bf16_exact((1, T * H * W, 1, d), RNG, 2.0)
    qt, kt = (O.reorder_fwd(a, T, H, W) for a in (q, k))
    vt = O.reorder_fwd(np.ones((1, T * H * W, 1, d)), T, H, W)
    nt = O.tile_grid(T, H, W)[2]
    mask = RNG.random((1, 1, nt, nt)) < 0.4
    rp, ci = O.mask_to_csr(mask)
    for _, _, o, _ in O.rectified_attention_rows(qt, kt, vt, rp, ci, T, H, W, 0.0, range(nt)):
        assert np.allclose(o, 1.0, atol=1e-12)
    kb, vb, n = O.pooled_kv(kt, vt, T, H, W)
    assert n.sum() == T * H * W and np.allclose(vb, 1.0)
    # tile 1 is cut by the right edge (W = 12): 8 x 4 real tokens
    real = kt[0, 0, 64:128][O.valid_rows(T, H, W)[64:128]]
    assert real.shape[0] == n[1] == 32 and np.allclose(kb[0, 0, 1], real.mean(0))


# ---------------------------------------------------------------- query-tile pairing
def _pair_cases(golden_dir):
    import json

    return json.load(open(os.path.join(golden_dir, "pair_cases.json")))["cases"]


def _lists_mask(lists):
    nt = len(lists)
    m = np.zeros((nt, nt), dtype=bool)
    for i, l in enumerate(lists):
        m[i, list(l)] = True
    return m


def test_pairing_golden(golden_dir):
    """Hand-derived pairings: equal lists found across non-frame neighbours,
    the frame pairing kept on a tie, left-overs paired in ascending order, the
    tie order of equal weights, and an odd tile count."""
    for case in _pair_cases(golden_dir):
        got = O.pair_query_tiles(_lists_mask(case["lists"]), case["T"], case["H"], case["W"])
        assert got.tolist() == case["pairs"], (case["name"], got.tolist())


PAIR_MUTANTS = {
    "ties to the higher smaller tile": ("edges.append((-w, min(a, b), max(a, b)))",
                                        "edges.append((-w, -min(a, b), max(a, b)))"),
    "lightest pairs first": ("edges.append((-w, min(a, b), max(a, b)))", "edges.append((w, min(a, b), max(a, b)))"),
    "greedy kept on a tie with the frame pairing": ("if pairs_union(mask, pairs) >= pairs_union(mask, dflt):",
                                                    "if pairs_union(mask, pairs) > pairs_union(mask, dflt):"),
    "left-overs paired from the top": ("left = [v for v in range(nt) if mate[v] < 0]",
                                       "left = [v for v in range(nt) if mate[v] < 0][::-1]"),
    "no frame-pairing fallback": ("pairs = dflt", "pass"),
}


def _pair_mutant(old, new):
    import inspect

    src = inspect.getsource(O.pair_query_tiles)
    assert src.count(old) == 1, old
    ns = dict(vars(sta_oracle))
    exec(compile(src.replace(old, new), "<mutant>", "exec"), ns)
    return ns["pair_query_tiles"]


@pytest.mark.parametrize("name", sorted(PAIR_MUTANTS))
def test_pairing_planted_mistakes_fail_the_golden_cases(golden_dir, name):
    fn = _pair_mutant(*PAIR_MUTANTS[name])
    wrong = 0
    for case in _pair_cases(golden_dir):
        wrong += fn(_lists_mask(case["lists"]), case["T"], case["H"], case["W"]).tolist() != case["pairs"]
    assert wrong >= 1, name


def test_pairing_is_a_partition_never_worse_than_the_default():
    """Random top-k masks on ragged grids: every tile appears exactly once,
    ceil(Nt/2) pairs, and the total union is at most the default pairing's.
    The greedy part is maximal: no two tiles left over (before the
    left-over pairing) are candidate partners."""
    rng = np.random.default_rng(7)
    for T, H, W, k in ((3, 19, 37, 3), (4, 16, 24, 2), (1, 40, 40, 5), (5, 8, 8, 2)):
        nh, nw, nt, _ = O.tile_grid(T, H, W)
        scores = rng.random((nt, nt))
        mask = np.zeros((nt, nt), dtype=bool)
        np.put_along_axis(mask, np.argsort(-scores, axis=1)[:, :k], True, axis=1)
        flat = O.pair_query_tiles(mask, T, H, W)
        assert flat.size == 2 * ((nt + 1) // 2)
        tiles = flat[flat >= 0]
        assert sorted(tiles.tolist()) == list(range(nt))
        pairs = [(int(flat[2 * i]), int(flat[2 * i + 1])) for i in range(flat.size // 2)]
        assert O.pairs_union(mask, pairs) <= O.pairs_union(mask, O.default_pairs(T, H, W))
        # brute-force: the sequential greedy over every candidate pair, by
        # exhaustive scan for the heaviest free pair each time
        cand = {}
        for a in range(nt):
            t, rem = divmod(a, nh * nw)
            y, x = divmod(rem, nw)
            for dt, dy, dx in O.PAIR_OFFSETS:
                if t + dt < T and 0 <= y + dy < nh and 0 <= x + dx < nw:
                    b = ((t + dt) * nh + y + dy) * nw + x + dx
                    cand[(min(a, b), max(a, b))] = int((mask[a] & mask[b]).sum())
        free = set(range(nt))
        matched = []
        while True:
            live = [(w, e) for e, w in cand.items() if e[0] in free and e[1] in free]
            if not live:
                break
            w, e = max(live, key=lambda we: (we[0], -we[1][0], -we[1][1]))
            matched.append(e)
            free -= set(e)
        if pairs != O.default_pairs(T, H, W):
            for e in matched:
                assert e in pairs, (T, H, W, e)


def test_default_pairs_cover_every_tile():
    for T, H, W in ((1, 8, 8), (2, 8, 24), (3, 19, 37), (5, 17, 9)):
        nt = O.tile_grid(T, H, W)[2]
        dp = O.default_pairs(T, H, W)
        assert len(dp) == (nt + 1) // 2
        tiles = sorted(t for p in dp for t in p if t >= 0)
        assert tiles == list(range(nt))
