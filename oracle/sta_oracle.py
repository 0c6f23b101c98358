"""fp64 CPU oracle (test infrastructure only; see the package docstring).

Readings taken where the pages leave a step open are stated beside each
function. Arrays are numpy; floating-point work is float64 on values that
are exactly the bf16 inputs.
"""
import math

import numpy as np

TILE = (1, 8, 8)  # tokens per tile along (t, y, x); 64 tokens
TILE_TOKENS = 64
MASS_ONE = 1 << 24  # fixed-point unit of the selection mass


# --------------------------------------------------------------------------
# Token layout (Compact Attention abstract: "tile-aligned mask family";
# Table III "Cubic" component).
# Reading: 1x8x8 tiles; tiles numbered in (t, tile-row, tile-column) raster
# order; tokens inside a tile row-major in (y, x); heads moved to dim 1;
# grids not divisible by 8 are padded with zero rows at the right / bottom.
# --------------------------------------------------------------------------
def tile_grid(T, H, W):
    """(NH, NW, Nt, Lpad) for a T x H x W token grid."""
    nh = (H + 7) // 8
    nw = (W + 7) // 8
    nt = T * nh * nw
    return nh, nw, nt, TILE_TOKENS * nt


def tiled_row_of_raster(T, H, W):
    """For each raster token i = (t*H + y)*W + x, its row in the tiled layout."""
    nh, nw, _, _ = tile_grid(T, H, W)
    out = np.empty(T * H * W, dtype=np.int64)
    i = 0
    for t in range(T):
        for y in range(H):
            for x in range(W):
                n = (t * nh + y // 8) * nw + x // 8
                out[i] = TILE_TOKENS * n + (y % 8) * 8 + (x % 8)
                i += 1
    return out


def valid_rows(T, H, W):
    """Boolean [Lpad]: True where the tiled row holds a real token."""
    _, _, _, lpad = tile_grid(T, H, W)
    v = np.zeros(lpad, dtype=bool)
    v[tiled_row_of_raster(T, H, W)] = True
    return v


def reorder_fwd(x, T, H, W):
    """Raster [B, L, heads, d] -> tiled [B, heads, Lpad, d]; pad rows are 0."""
    x = np.asarray(x)
    B, L, Hh, d = x.shape
    assert L == T * H * W
    _, _, _, lpad = tile_grid(T, H, W)
    out = np.zeros((B, Hh, lpad, d), dtype=x.dtype)
    rows = tiled_row_of_raster(T, H, W)
    out[:, :, rows, :] = np.transpose(x, (0, 2, 1, 3))
    return out


def reorder_inv(xt, T, H, W):
    """Tiled [B, heads, Lpad, d] -> raster [B, L, heads, d]; pad rows dropped."""
    xt = np.asarray(xt)
    rows = tiled_row_of_raster(T, H, W)
    return np.ascontiguousarray(np.transpose(xt[:, :, rows, :], (0, 2, 1, 3)))


# --------------------------------------------------------------------------
# Pooled block scores (Rectified SpaAttn abstract: weights recovered from the
# pooled query-key).
# Reading: the mean over the real tokens of each tile (pads excluded); score
# scale 1/sqrt(d) unless given; softmax over all key tiles of the row.
# --------------------------------------------------------------------------
def pool(xt, T, H, W):
    """Tiled [B, heads, Lpad, d] -> per-tile means [B, heads, Nt, d] (fp64)."""
    xt = np.asarray(xt)
    B, Hh, lpad, d = xt.shape
    _, _, nt, lp = tile_grid(T, H, W)
    assert lpad == lp
    valid = valid_rows(T, H, W).reshape(nt, TILE_TOKENS)
    cnt = valid.sum(axis=1).astype(np.float64)
    out = np.empty((B, Hh, nt, d), dtype=np.float64)
    for b in range(B):
        for h in range(Hh):
            tiles = xt[b, h].astype(np.float64).reshape(nt, TILE_TOKENS, d)
            s = np.einsum("nr,nrd->nd", valid.astype(np.float64), tiles)
            out[b, h] = s / cnt[:, None]
    return out


def block_scores(qbar, kbar, scale):
    """S = scale * qbar kbar^T and its row softmax P, both [B, heads, Nt, Nt]."""
    qbar = np.asarray(qbar, dtype=np.float64)
    kbar = np.asarray(kbar, dtype=np.float64)
    s = np.einsum("bhqd,bhkd->bhqk", qbar, kbar) * float(scale)
    m = s.max(axis=-1, keepdims=True)
    e = np.exp(s - m)
    p = e / e.sum(axis=-1, keepdims=True)
    return s, p


# --------------------------------------------------------------------------
# Hybrid top-p / fixed top-k selection (SCOPE review, Eqs. (7)-(8) as quoted:
# keep the smallest set reaching mass rho, with a fixed floor of keys).
# Reading, at tile granularity:
#   order  : key tiles by P descending, ties to the lower key-tile index;
#   mass   : w_j = floor(P_j * 2^24) (integers, exact in any summation order);
#   thr    : ceil(double(top_p) * double(sum_j w_j)), top_p taken as float32;
#   m_p    : smallest m whose first m tiles reach thr; Nt if top_p >= 1,
#            0 if top_p <= 0;
#   keep   : the first max(m_p, min(k_min, Nt)) tiles of the order.
# --------------------------------------------------------------------------
def select_row(p_row, top_p, k_min):
    """Boolean [Nt] keep-set for one row of block probabilities."""
    p = np.asarray(p_row, dtype=np.float64)
    nt = p.shape[0]
    order = sorted(range(nt), key=lambda j: (-p[j], j))
    w = [int(math.floor(float(p[j]) * MASS_ONE)) for j in range(nt)]
    total = sum(w)
    tp = float(np.float32(top_p))
    if tp >= 1.0:
        m_p = nt
    elif tp <= 0.0:
        m_p = 0
    else:
        thr = math.ceil(tp * float(total))
        acc = 0
        m_p = nt
        for m in range(nt + 1):
            if acc >= thr:
                m_p = m
                break
            if m < nt:
                acc += w[order[m]]
    m = max(m_p, min(int(k_min), nt))
    keep = np.zeros(nt, dtype=bool)
    keep[order[:m]] = True
    return keep


def select(P, top_p, k_min):
    """Row-wise select() over the last axis of P."""
    P = np.asarray(P)
    flat = P.reshape(-1, P.shape[-1])
    out = np.stack([select_row(r, top_p, k_min) for r in flat])
    return out.reshape(P.shape)


# --------------------------------------------------------------------------
# Online per-head top-k floor (SCOPE review, Eqs. (9)-(10) as quoted: the
# head's floor is the cluster-size-weighted mean of the base retained counts,
# and clusters below it are extended to it).
# Reading, at tile granularity: a cluster is a query tile, its size n_c the
# number of real tokens in it, its base count b_c the size of the hybrid
# top-p / k_min selection; k_head = ceil(sum n_c b_c / sum n_c) over the query
# tiles of the head; a row keeps the first max(b_c, min(k_head, Nt)) tiles of
# its order. The windows are OR'd in afterwards, as without the floor.
# --------------------------------------------------------------------------
def head_topk_floor(counts, sizes):
    """k_head = ceil(sum(n_c * b_c) / sum(n_c)) in exact integer arithmetic."""
    num = sum(int(n) * int(b) for n, b in zip(sizes, counts))
    den = sum(int(n) for n in sizes)
    return -(-num // den) if den else 0


def select_with_head_floor(P_head, top_p, k_min, sizes):
    """Selection of one head [Nt, Nt] with the per-head floor; returns
    (keep [Nt, Nt] bool, k_head)."""
    P_head = np.asarray(P_head)
    base = np.stack([select_row(r, top_p, k_min) for r in P_head])
    k_head = head_topk_floor(base.sum(axis=1), sizes)
    out = base.copy()
    for c in range(P_head.shape[0]):
        if base[c].sum() < k_head:
            out[c] = select_row(P_head[c], top_p, max(int(k_min), k_head))
    return out, k_head


def tile_sizes(T, H, W):
    """Real tokens per tile, [Nt]."""
    return valid_rows(T, H, W).reshape(-1, TILE_TOKENS).sum(axis=1)


# --------------------------------------------------------------------------
# Deformable dual window per temporal-distance group (Compact Attention
# Fig. 1(3), Fig. 4; Table III "Frame-group" and "Dual Window").
# Reading: in tile units, key tile kt is kept for query tile qt of head h iff
# group g (the last g with group_lo[g] <= |dt|) exists and
#   (|dy| <= ry1 and |dx| <= rx1) or (|dy| <= ry2 and |dx| <= rx2)
# with (ry1, rx1, ry2, rx2) = windows[h, g]; -1 switches a window off;
# rectangles are centred on the query tile and clipped at the grid edge.
# --------------------------------------------------------------------------
def window_mask(windows, group_lo, T, H, W):
    """Boolean [heads, Nt, Nt] dual-window mask."""
    windows = np.asarray(windows, dtype=np.int64)
    Hh, G, four = windows.shape
    assert four == 4 and len(group_lo) == G
    nh, nw, nt, _ = tile_grid(T, H, W)
    idx = np.arange(nt)
    tt, ty, tx = idx // (nh * nw), (idx // nw) % nh, idx % nw
    dt = np.abs(tt[:, None] - tt[None, :])
    dy = np.abs(ty[:, None] - ty[None, :])
    dx = np.abs(tx[:, None] - tx[None, :])
    grp = np.full((nt, nt), -1, dtype=np.int64)
    for g in range(G):
        grp[dt >= int(group_lo[g])] = g
    out = np.zeros((Hh, nt, nt), dtype=bool)
    for h in range(Hh):
        for g in range(G):
            ry1, rx1, ry2, rx2 = windows[h, g]
            in_g = grp == g
            w1 = (dy <= ry1) & (dx <= rx1)
            w2 = (dy <= ry2) & (dx <= rx2)
            out[h] |= in_g & (w1 | w2)
    return out


def mask_to_csr(mask):
    """Boolean [..., Nt, Nt] -> (row_ptr int32 [R+1], col_idx int32 [nnz]);
    rows are the flattened leading axes, columns ascending."""
    m = np.asarray(mask, dtype=bool)
    nt = m.shape[-1]
    flat = m.reshape(-1, nt)
    counts = flat.sum(axis=1)
    row_ptr = np.zeros(flat.shape[0] + 1, dtype=np.int64)
    row_ptr[1:] = np.cumsum(counts)
    cols = [np.nonzero(r)[0] for r in flat]
    col_idx = np.concatenate(cols) if cols else np.zeros(0, dtype=np.int64)
    return row_ptr.astype(np.int32), col_idx.astype(np.int32)


def build_mask(q_tiled, k_tiled, T, H, W, use_scores, top_p, k_min,
               windows=None, group_lo=None, sm_scale=0.0, head_floor=False):
    """Full mask construction: pool, score, select (with the per-head top-k
    floor when head_floor), OR windows, emit CSR.

    Returns dict(mask [B,heads,Nt,Nt] bool, probs [B,heads,Nt,Nt] fp64 or
    None, row_ptr, col_idx).
    """
    q_tiled = np.asarray(q_tiled)
    B, Hh, _, d = q_tiled.shape
    _, _, nt, _ = tile_grid(T, H, W)
    scale = float(sm_scale) if sm_scale else 1.0 / math.sqrt(d)
    mask = np.zeros((B, Hh, nt, nt), dtype=bool)
    probs = None
    if use_scores:
        qbar = pool(q_tiled, T, H, W)
        kbar = pool(k_tiled, T, H, W)
        _, probs = block_scores(qbar, kbar, scale)
        if head_floor:
            sizes = tile_sizes(T, H, W)
            for b in range(B):
                for h in range(Hh):
                    mask[b, h] |= select_with_head_floor(probs[b, h], top_p, k_min, sizes)[0]
        else:
            mask |= select(probs, top_p, k_min)
    if windows is not None:
        mask |= window_mask(windows, group_lo, T, H, W)[None]
    row_ptr, col_idx = mask_to_csr(mask)
    return dict(mask=mask, probs=probs, row_ptr=row_ptr, col_idx=col_idx)


# --------------------------------------------------------------------------
# Masked softmax attention over the listed key tiles (Compact Attention
# Fig. 3: precomputed masks loaded into block-sparse attention kernels).
# Definition: for each real query token of query tile qt,
#   o = sum_j softmax_j(scale * q . k_j) v_j,  LSE = log sum_j exp(scale q.k_j)
# over the real tokens j of the listed key tiles. An empty list gives o = 0
# and LSE = -inf. Padded query rows are not defined and not returned.
# --------------------------------------------------------------------------
def attention_rows(q_tiled, k_tiled, v_tiled, row_ptr, col_idx, T, H, W,
                   sm_scale, rows):
    """Attention for the CSR rows listed in `rows` (flat (b*heads + h)*Nt + qt).

    Returns a list of (row, token_rows, O [n_q, d] fp64, LSE [n_q] fp64),
    token_rows being the tiled-layout rows of the real query tokens.
    """
    q_tiled = np.asarray(q_tiled)
    B, Hh, lpad, d = q_tiled.shape
    _, _, nt, _ = tile_grid(T, H, W)
    valid = valid_rows(T, H, W)
    scale = float(sm_scale) if sm_scale else 1.0 / math.sqrt(d)
    out = []
    for r in rows:
        r = int(r)
        bh, qt = divmod(r, nt)
        b, h = divmod(bh, Hh)
        qrows = np.arange(qt * 64, qt * 64 + 64)
        qrows = qrows[valid[qrows]]
        q = q_tiled[b, h, qrows].astype(np.float64)
        tiles = np.asarray(col_idx[int(row_ptr[r]):int(row_ptr[r + 1])], dtype=np.int64)
        if tiles.size == 0:
            out.append((r, qrows, np.zeros((qrows.size, d)), np.full(qrows.size, -np.inf)))
            continue
        krows = (tiles[:, None] * 64 + np.arange(64)[None, :]).reshape(-1)
        krows = krows[valid[krows]]
        k = np.asarray(k_tiled)[b, h, krows].astype(np.float64)
        v = np.asarray(v_tiled)[b, h, krows].astype(np.float64)
        s = (q @ k.T) * scale
        m = s.max(axis=1, keepdims=True)
        e = np.exp(s - m)
        z = e.sum(axis=1, keepdims=True)
        o = (e / z) @ v
        lse = (m + np.log(z))[:, 0]
        out.append((r, qrows, o, lse))
    return out


def attention_all(q_tiled, k_tiled, v_tiled, row_ptr, col_idx, T, H, W, sm_scale):
    """Attention for every row; returns O [B, heads, Lpad, d] (pad rows NaN)
    and LSE [B, heads, Lpad] (pad rows NaN)."""
    q_tiled = np.asarray(q_tiled)
    B, Hh, lpad, d = q_tiled.shape
    _, _, nt, _ = tile_grid(T, H, W)
    O = np.full((B, Hh, lpad, d), np.nan)
    LSE = np.full((B, Hh, lpad), np.nan)
    res = attention_rows(q_tiled, k_tiled, v_tiled, row_ptr, col_idx, T, H, W,
                         sm_scale, range(B * Hh * nt))
    for r, qrows, o, lse in res:
        bh, _ = divmod(r, nt)
        b, h = divmod(bh, Hh)
        O[b, h, qrows] = o
        LSE[b, h, qrows] = lse
    return O, LSE


# --------------------------------------------------------------------------
# Rectified attention (Rectified SpaAttn abstract: sparse attention inflates
# the weights of the kept (critical) tokens, by a factor set by the weight it
# drops, and loses the dropped (non-critical) tokens entirely; the fix
# reallocates the kept weights with pooled weights and recovers the dropped
# ones from the pooled query-key).
# Reading (the abstract gives no formula): every key tile the row does not
# list enters the softmax as one pooled key k_bar (mean of its real keys)
# with multiplicity n (its real token count) and value v_bar (mean of its
# real values); listed tiles enter token by token:
#   Z_keep = sum_{j in listed}   exp(scale * q.k_j)
#   Z_skip = sum_{t not listed}  n_t * exp(scale * q.k_bar_t)
#   o      = (sum_listed exp(scale q.k_j) v_j + sum_skip n_t exp(scale q.k_bar_t) v_bar_t)
#            / (Z_keep + Z_skip)
#   lse    = log(Z_keep + Z_skip)
# so the kept part is scaled by Z_keep / (Z_keep + Z_skip) (the reallocation)
# and the skipped tiles add their pooled estimate. No gate is applied (the
# abstract's gain-versus-error condition has no stated form).
# --------------------------------------------------------------------------
def pooled_kv(k_tiled, v_tiled, T, H, W):
    """Per-tile means of K and V over real tokens and the real-token counts:
    (k_bar [B, heads, Nt, d], v_bar [B, heads, Nt, d], n [Nt])."""
    kb = pool(k_tiled, T, H, W)
    vb = pool(v_tiled, T, H, W)
    return kb, vb, tile_sizes(T, H, W).astype(np.float64)


def rectified_attention_rows(q_tiled, k_tiled, v_tiled, row_ptr, col_idx, T, H, W, sm_scale, rows):
    """Rectified attention for the CSR rows in `rows`; same return format as
    attention_rows (row, token_rows, O, LSE)."""
    q_tiled = np.asarray(q_tiled)
    B, Hh, lpad, d = q_tiled.shape
    _, _, nt, _ = tile_grid(T, H, W)
    valid = valid_rows(T, H, W)
    scale = float(sm_scale) if sm_scale else 1.0 / math.sqrt(d)
    kbar, vbar, n = pooled_kv(k_tiled, v_tiled, T, H, W)
    out = []
    for r in rows:
        r = int(r)
        bh, qt = divmod(r, nt)
        b, h = divmod(bh, Hh)
        qrows = np.arange(qt * 64, qt * 64 + 64)
        qrows = qrows[valid[qrows]]
        q = q_tiled[b, h, qrows].astype(np.float64)
        tiles = np.asarray(col_idx[int(row_ptr[r]):int(row_ptr[r + 1])], dtype=np.int64)
        skip = np.setdiff1d(np.arange(nt), tiles)
        krows = (tiles[:, None] * 64 + np.arange(64)[None, :]).reshape(-1)
        krows = krows[valid[krows]]
        k = np.asarray(k_tiled)[b, h, krows].astype(np.float64)
        v = np.asarray(v_tiled)[b, h, krows].astype(np.float64)
        # logits of kept tokens, and of skipped tiles with log-multiplicity
        s_keep = (q @ k.T) * scale
        s_skip = (q @ kbar[b, h, skip].T) * scale + np.log(n[skip])[None, :]
        s = np.concatenate([s_keep, s_skip], axis=1)
        vals = np.concatenate([v, vbar[b, h, skip]], axis=0)
        if s.shape[1] == 0:
            out.append((r, qrows, np.zeros((qrows.size, d)), np.full(qrows.size, -np.inf)))
            continue
        m = s.max(axis=1, keepdims=True)
        e = np.exp(s - m)
        z = e.sum(axis=1, keepdims=True)
        out.append((r, qrows, (e / z) @ vals, (m + np.log(z))[:, 0]))
    return out


# --------------------------------------------------------------------------
# LSE-cached exact block importance (AdaSpa abstract: exact block importance
# computed during a full-attention step with a cached log-sum-exp, then
# reused for the block-sparse steps that follow).
# Reading: for query tile qt and listed key tile kt,
#   mass(qt, kt) = (1 / n_q) * sum_i sum_j exp(scale * q_i . k_j - lse_i)
# over the real query tokens i of qt (n_q of them) and the real key tokens j of
# kt, with lse the cached per-token log-sum-exp (natural log); a token with
# lse = -inf contributes nothing. With the exact LSE of the same inputs and
# every tile listed, each row of masses sums to one.
# --------------------------------------------------------------------------
def block_mass(q_tiled, k_tiled, lse, row_ptr, col_idx, T, H, W, sm_scale, rows):
    """Masses for the listed (row, key tile) pairs of the CSR rows in `rows`.

    Returns {row: (tiles, masses)} with masses fp64 aligned to tiles."""
    q_tiled = np.asarray(q_tiled)
    B, Hh, lpad, d = q_tiled.shape
    _, _, nt, _ = tile_grid(T, H, W)
    valid = valid_rows(T, H, W)
    scale = float(sm_scale) if sm_scale else 1.0 / math.sqrt(d)
    out = {}
    for r in rows:
        r = int(r)
        bh, qt = divmod(r, nt)
        b, h = divmod(bh, Hh)
        qrows = np.arange(qt * 64, qt * 64 + 64)
        qrows = qrows[valid[qrows]]
        q = q_tiled[b, h, qrows].astype(np.float64)
        l = np.asarray(lse)[b, h, qrows].astype(np.float64)
        live = np.isfinite(l)
        tiles = np.asarray(col_idx[int(row_ptr[r]):int(row_ptr[r + 1])], dtype=np.int64)
        masses = np.zeros(tiles.size)
        for i, kt in enumerate(tiles):
            krows = np.arange(kt * 64, kt * 64 + 64)
            krows = krows[valid[krows]]
            k = np.asarray(k_tiled)[b, h, krows].astype(np.float64)
            s = (q[live] @ k.T) * scale - l[live][:, None]
            masses[i] = np.exp(s).sum() / qrows.size
        out[r] = (tiles, masses)
    return out


# --------------------------------------------------------------------------
# Recall-driven window search (Compact Attention Fig. 3: offline search that
# iteratively shrinks the dual windows under the recall (tau) and cost
# (lambda) constraints; Fig. 4: starting from full coverage in every
# temporal-distance group, the dual windows are shrunk while the recall and
# shrink-penalty constraints hold; Fig. 5(c): recall target vs sparsity).
# Reading (the pages give no step rule):
#   masses : exact block importances of one head [Nt, Nt] (e.g. from an
#            LSE-cached dense step), as integers w = floor(min(max(m,0),1)*2^24);
#            W = sum w; recall of a window set = covered w / W;
#   start  : (ry1, rx1, ry2, rx2) = (NH-1, NW-1, NH-1, NW-1) in every group;
#   moves  : for each group g, in order: ry1-1, rx1-1, ry2-1, rx2-1,
#            (ry1-1, ry2-1), (rx1-1, rx2-1); an extent never goes below -1;
#   value  : J = removed / Nt^2 - lambda * lost / W (double, in that order),
#            removed / lost = pairs / mass the move uncovers;
#   admit  : covered - lost >= ceil(double(tau) * W)   (recall constraint)
#            and J >= 0                                (cost constraint);
#            a move that uncovers nothing (one window shrunk inside the
#            other) is admissible with J = 0: it is how the two windows,
#            equal at the start, come apart;
#   step   : the admissible move with the largest J, ties to the lowest move
#            index g*6 + m; stop when none is left (every move lowers an
#            extent, so the search ends).
# --------------------------------------------------------------------------
SEARCH_MOVES = ((0,), (1,), (2,), (3,), (0, 2), (1, 3))


def search_windows(mass, T, H, W, group_lo, tau, lam):
    """Greedy window search for one head; returns (windows [G,4] int32, stats)
    with stats = dict(recall, density, steps, covered, total, moves), moves
    being the applied move indices g*6 + m in order."""
    m = np.clip(np.asarray(mass, dtype=np.float64), 0.0, 1.0)
    w = np.floor(m * MASS_ONE).astype(np.int64)
    total = int(w.sum())
    nh, nw, nt, _ = tile_grid(T, H, W)
    G = len(group_lo)
    win = np.empty((G, 4), dtype=np.int64)
    win[:] = (nh - 1, nw - 1, nh - 1, nw - 1)
    thr = math.ceil(float(np.float32(tau)) * float(total))
    lam = float(np.float32(lam))
    cur = window_mask(win[None], group_lo, T, H, W)[0]
    covered = int(w[cur].sum())
    moves = []
    while True:
        best = None
        for g in range(G):
            for mi, ext in enumerate(SEARCH_MOVES):
                cand = win.copy()
                if any(cand[g, e] <= -1 for e in ext):
                    continue
                for e in ext:
                    cand[g, e] -= 1
                new = window_mask(cand[None], group_lo, T, H, W)[0]
                gone = cur & ~new
                removed = int(gone.sum())
                lost = int(w[gone].sum())
                if covered - lost < thr:
                    continue
                J = removed / float(nt * nt) - lam * (lost / float(total) if total else 0.0)
                if J < 0.0:
                    continue
                if best is None or J > best[0]:
                    best = (J, g * 6 + mi, cand, new, lost)
        if best is None:
            break
        _, idx, win, cur, lost = best
        covered -= lost
        moves.append(idx)
    stats = dict(recall=covered / total if total else 1.0, density=float(cur.mean()), steps=len(moves),
                 covered=covered, total=total, moves=moves)
    return win.astype(np.int32), stats


# --------------------------------------------------------------------------
# Query-tile pairing by list overlap. The pages have no counterpart: this is
# how the library groups two 64-token query tiles into one 128-row block of
# its attention kernels (Compact Attention Fig. 3: precomputed masks loaded
# into block-sparse kernels), and the attention result does not depend on it
# beyond fp32 summation order. Restated here because sta_build_mask emits
# it as an output (sta_mask_params.query_pairs).
# Rule: candidate pairs (a, a + o) for the offsets o of PAIR_OFFSETS inside
# the tile grid, weight |L_a n L_b| of the final key-tile lists; taken
# greedily in the order (weight descending, smaller tile ascending, larger
# tile ascending) when both tiles are free; tiles left over paired in
# ascending order, a last one alone; kept only if its total union
# sum |L_a u L_b| is below that of the default pairing (frames 2u, 2u+1 of
# one spatial tile; in a last odd frame, neighbours 2i, 2i+1), else the
# default pairing is returned. Pairs come in ascending order of their first
# tile (the default pairing in its own order).
# --------------------------------------------------------------------------
PAIR_OFFSETS = ([(1, dy, dx) for dy in (-1, 0, 1) for dx in (-1, 0, 1)]
                + [(0, 1, -1), (0, 1, 0), (0, 1, 1), (0, 0, 1), (2, 0, 0)])


def default_pairs(T, H, W):
    """The attention kernels' own pairing: list of (a, b or -1)."""
    nh, nw, nt, _ = tile_grid(T, H, W)
    tpf = nh * nw
    pairs = []
    for u in range(T // 2):
        for rem in range(tpf):
            a = 2 * u * tpf + rem
            pairs.append((a, a + tpf))
    if T % 2:
        base = (T - 1) * tpf
        for i in range(0, tpf, 2):
            a = base + i
            pairs.append((a, a + 1 if a + 1 < nt else -1))
    return pairs


def pairs_union(mask, pairs):
    """Total union size sum |L_a u L_b| over the pairs (|L_a| for a lone tile)."""
    total = 0
    for a, b in pairs:
        total += int((mask[a] | mask[b]).sum()) if b >= 0 else int(mask[a].sum())
    return total


def pair_query_tiles(mask, T, H, W):
    """mask: bool [Nt, Nt] of one head (row = query tile). Returns the pairs
    as a flat int array [2 * ceil(Nt/2)]."""
    mask = np.asarray(mask, dtype=bool)
    nh, nw, nt, _ = tile_grid(T, H, W)
    edges = []
    for a in range(nt):
        t, rem = divmod(a, nh * nw)
        y, x = divmod(rem, nw)
        for dt, dy, dx in PAIR_OFFSETS:
            t2, y2, x2 = t + dt, y + dy, x + dx
            if t2 < T and 0 <= y2 < nh and 0 <= x2 < nw:
                b = (t2 * nh + y2) * nw + x2
                w = int((mask[a] & mask[b]).sum())
                edges.append((-w, min(a, b), max(a, b)))
    edges.sort()
    mate = [-1] * nt
    for _, a, b in edges:
        if mate[a] < 0 and mate[b] < 0:
            mate[a], mate[b] = b, a
    left = [v for v in range(nt) if mate[v] < 0]
    pairs = []
    for i in range(0, len(left) - 1, 2):
        mate[left[i]], mate[left[i + 1]] = left[i + 1], left[i]
    for v in range(nt):
        if mate[v] < 0:
            pairs.append((v, -1))
        elif mate[v] > v:
            pairs.append((v, mate[v]))
    dflt = default_pairs(T, H, W)
    if pairs_union(mask, pairs) >= pairs_union(mask, dflt):
        pairs = dflt
    return np.array([i for p in pairs for i in p], dtype=np.int64)
