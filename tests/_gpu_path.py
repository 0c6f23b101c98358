"""Helpers for the GPU parity tests: run the CUDA path through the binding and
bring results back as numpy. Imported only by tests marked gpu."""
import math

import numpy as np
import torch

import block_sparse_attention_28_b200 as sta

DEV = "cuda"
U32 = 2.0 ** -24


def to_np64(x):
    return x.float().cpu().numpy().astype(np.float64)


def reorder(x, B, Hh, d, g):
    lpad = sta.sta_tiled_len(g)
    out = torch.full((B, Hh, lpad, d), float("nan"), dtype=torch.bfloat16, device=x.device)
    sta.sta_reorder(x, out, B, Hh, d, g)
    return out


def build(qt, kt, B, Hh, d, g, params, with_mask=True, with_probs=True):
    bufs = sta.MaskBuffers(B, Hh, d, g, qt.device if qt is not None else DEV, with_mask, with_probs)
    sta.build_mask(qt, kt, B, Hh, d, g, params, bufs)
    return bufs


def csr_np(bufs):
    nnz = int(bufs.nnz.item())
    return bufs.row_ptr.cpu().numpy(), bufs.col_idx[:nnz].cpu().numpy(), nnz


def attn(qt, kt, vt, row_ptr, col_idx, B, Hh, d, g, sm_scale=0.0):
    o = torch.full_like(qt, float("nan"))
    lse = torch.full(qt.shape[:3], float("nan"), dtype=torch.float32, device=qt.device)
    sta.sta_attn_fwd(qt, kt, vt, o, lse, row_ptr, col_idx, B, Hh, d, g, sm_scale)
    return o, lse


def prob_bound(qbar, kbar, scale, p_ref, fused=False):
    """Per-element bound on |P_gpu - P_oracle| from the GPU arithmetic.

    Both layouts round the pooled means once to fp32 (an exact fp64 sum). The
    score term differs:
    - fused (minimum workspace): a D-term sequential fp32 FMA chain,
      error <= gamma_D |q||k|;
    - tensor cores (full workspace): each mean x split as hi = tf32(x),
      lo = tf32(x - hi), so |x - hi - lo| <= 2^-22 |x|; the products
      lo*hi + hi*lo + hi*hi drop lo*lo, in all <= 3 * 2^-22 |q k|; the
      fp32 accumulator passes through 3*D/8 MMAs (K = 8 each), each taken to
      add at most 2 ulp (2^-22) of the sum of the magnitudes so far.
    A score error of at most E per row moves P by a factor within e^(+-2E).
    The softmax in fp32: e = ex2.approx(fma(s, log2 e, -round(m log2 e))),
    whose relative error is at most 2^-22 (ex2.approx) plus u (|s| + 2|m|)
    (the rounding of the argument, ln 2 log2 e = 1); Z summed lane by lane
    over ceil(Nt/32) terms, then by a 5-step butterfly (gamma_{ceil(Nt/32)+4});
    P = e * round(1/Z) (two roundings). So
      |P_gpu / P - 1| <= 2.2 E + 2 eps_exp + gamma_{ceil(Nt/32)+4} + 2u
    with eps_exp = 2^-22 + 3 u max_j |s_j|.
    Returns an array like p_ref."""
    d = qbar.shape[-1]
    if fused:
        gam = d * U32 / (1 - d * U32)
    else:
        gam = (3 * d / 8 + 3) * 2.0 ** -22
    cond = np.einsum("...qd,...kd->...qk", np.abs(qbar), np.abs(kbar)) * scale
    ds = (gam + 2.0 * U32) * cond  # score error bound per element
    E = ds.max(axis=-1, keepdims=True)
    nt = p_ref.shape[-1]
    s = np.einsum("...qd,...kd->...qk", qbar, kbar) * scale
    smax = np.abs(s).max(axis=-1, keepdims=True)
    eps_exp = 2.0 ** -22 + 3.0 * U32 * smax
    n = -(-nt // 32) + 4
    rel = 2.2 * E + 2.0 * eps_exp + n * U32 / (1 - n * U32) + 2.0 * U32
    return p_ref * rel + 1e-30


# Observed |P_gpu - P_oracle| / bound stays below 0.07 in every case the tests
# run (both layouts, d = 64 and 128, custom scales, the 720p grid); a
# regression of the score or softmax arithmetic by 10x would cross this.
PROB_ERR_CEILING = 0.2


def attn_errors(o_gpu_t, o_ref_t, valid_rows):
    """max-abs and mean-abs error over real token rows (tiled layout)."""
    a = to_np64(o_gpu_t)[:, :, valid_rows, :]
    b = o_ref_t[:, :, valid_rows, :]
    err = np.abs(a - b)
    return float(err.max()), float(err.mean())


def default_scale(d):
    return 1.0 / math.sqrt(d)
