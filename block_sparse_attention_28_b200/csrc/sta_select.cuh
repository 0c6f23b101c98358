// Row selection with the row in registers: the select pass of the mask build
// for rows of up to 2048 key tiles. Hybrid top-p / k_min selection (SCOPE
// review, Eqs. (7)-(8) as quoted) of a row of block probabilities, OR'd with
// the row's dual windows (Compact Attention Fig. 1(3), Fig. 4), written as a
// row bitset and its count.
//
// One warp per row, eight rows per CTA; lane l holds entries l + 32 i,
// i < NPL (NPL * 32 >= Nt). Everything per entry is done in registers by
// fully unrolled code:
//   softmax   P = 2^(s log2e - m log2e) * (1 / Z): one FFMA, one ex2.approx,
//             one FADD of the lane-strided sum and one FMUL per entry; Z is
//             summed lane by lane in index order, then over the lanes by a
//             butterfly, and 1/Z is rounded once (IEEE reciprocal);
//   threshold the pattern v of the last kept entry, found in two levels:
//             level 1, a private histogram per lane (no conflicts) of
//             (mass, count) over 32 bins of the exponent of P, gives the bin
//             where the weight from the top first reaches the target; the
//             entries of that bin are appended to per-lane candidate columns
//             in shared memory; level 2 is a radix select over the
//             candidates' remaining bits (256-bin histogram per pass);
//   bitset    one ballot per 32 entries (P > v, or P == v among the first
//             c ties by index), OR'd with the window bits.
// Every sum of masses and counts is an integer sum, so the result does not
// depend on the order of summation: it equals the selection the fallback
// select pass (score_select_kernel) computes on the same P.
#pragma once
#include "sta_mask.cuh"

namespace sta {
namespace sel {

constexpr int WARPS = 8;
constexpr int THREADS = 32 * WARPS;
constexpr int MAX_NPL = 64;  // rows of up to 2048 key tiles
constexpr uint32_t NONE = 0xFFFFFFFFu;  // "no level": nothing is kept by the threshold
constexpr int MASS_BASE = 103;          // exponent of 2^-24: the smallest P with mass >= 1
constexpr int COUNT_BASE = 96;          // counting: exponents below 97 share bin 0

// Per-warp shared memory in 32-bit words: the level-1 histograms
// [32 bins][32 lanes], aliased by the candidate columns [NPL][32]; the
// 256-bin histogram of level 2; the window bits of the row [wpr].
template <int NPL>
struct Ws {
  static constexpr int U = (32 * 32 > 32 * NPL) ? 32 * 32 : 32 * NPL;
  static constexpr int HIST = U;
  static constexpr int WIN = U + 256;
};

// Shared memory of select_rows_kernel<NPL>: window tables, then per warp.
inline size_t smem_bytes(int npl, int wpr, int T) {
  const int u = (32 > npl ? 32 : npl) * 32;
  const size_t tables = (size_t)((T + 3) & ~3) + 4 * STA_MAX_GROUPS;
  return (tables + (size_t)WARPS * (u + 256 + ((wpr + 3) & ~3))) * 4;
}

// Weight of a P pattern in level 1: mass w = floor(P 2^24) in bits 0-24 and
// a count of 1 in bits 25-31 (a lane adds at most NPL <= 64 entries to a bin,
// and its masses sum to at most 2^24 (1 + Nt 2^-24) < 2^25).
constexpr uint32_t CNT_ONE = 1u << 25;
constexpr uint32_t MASS_MASK = CNT_ONE - 1u;

// Level 1: private per-lane histograms over bin = exponent(P) - base,
// clamped to [0, 31] (mass: entries with no mass are left out, and base is
// the exponent of 2^-24, so the bins are exact exponents). Returns the bin
// b* where the weight at or above it first reaches `target` (scanning from
// the top bin) and the mass and count strictly above b*. target >= 1 and the
// row's total weight is >= target.
template <int NPL>
__device__ __forceinline__ void level1(const uint32_t (&pb)[NPL], int nt, int lane, bool mass, uint32_t target,
                                       uint32_t *h, int &bstar, uint32_t &mass_above, uint32_t &cnt_above) {
  const int base = mass ? MASS_BASE : COUNT_BASE;
#pragma unroll
  for (int b = 0; b < 32; ++b) h[b * 32 + lane] = 0u;
  __syncwarp();
#pragma unroll
  for (int i = 0; i < NPL; ++i) {
    if (32 * i + lane < nt) {
      const uint32_t b = pb[i];
      const uint32_t w = mass_of(__uint_as_float(b));
      int bin = (int)(b >> 23) - base;
      bin = bin < 0 ? 0 : (bin > 31 ? 31 : bin);
      if (!mass || w != 0u) atomicAdd(h + bin * 32 + lane, w + CNT_ONE);  // private column: no conflicts
    }
  }
  __syncwarp();
  // lane l totals bin l over the 32 columns, reading diagonally (conflict-free)
  uint32_t m = 0u, c = 0u;
#pragma unroll 8
  for (int t = 0; t < 32; ++t) {
    const uint32_t x = h[lane * 32 + ((lane + t) & 31)];
    m += x & MASS_MASK;
    c += x >> 25;
  }
  // weight at or above each bin (suffix sums from the top bin)
  const uint32_t own = mass ? m : c;
  uint32_t suf = own, sufc = c, sufm = m;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_down_sync(0xffffffffu, suf, o);
    const uint32_t yc = __shfl_down_sync(0xffffffffu, sufc, o);
    const uint32_t ym = __shfl_down_sync(0xffffffffu, sufm, o);
    if (lane + o < 32) {
      suf += y;
      sufc += yc;
      sufm += ym;
    }
  }
  const uint32_t hit = __ballot_sync(0xffffffffu, suf >= target);
  bstar = 31 - __clz((int)hit);
  mass_above = __shfl_sync(0xffffffffu, sufm - m, bstar);
  cnt_above = __shfl_sync(0xffffffffu, sufc - c, bstar);
  __syncwarp();  // the histograms are reused as candidate columns
}

// Appends the entries of bin b* to the lane's candidate column
// (cand[k * 32 + lane], k < returned count).
template <int NPL>
__device__ __forceinline__ int collect(const uint32_t (&pb)[NPL], int nt, int lane, bool mass, int bstar,
                                       uint32_t *cand) {
  const int base = mass ? MASS_BASE : COUNT_BASE;
  int k = 0;
#pragma unroll
  for (int i = 0; i < NPL; ++i) {
    const uint32_t b = pb[i];
    int bin = (int)(b >> 23) - base;
    bin = bin < 0 ? 0 : (bin > 31 ? 31 : bin);
    const bool in = (32 * i + lane < nt) && bin == bstar && (!mass || mass_of(__uint_as_float(b)) != 0u);
    if (in) cand[(k++) * 32 + lane] = b;
  }
  __syncwarp();
  return k;
}

// Level 2: radix select over the candidates, digit passes from `first`
// (0: bits 30-23, 1: 22-15, 2: 14-7, 3: 6-0): the largest pattern v whose
// weight at or above reaches `target`, and the weight of the candidates
// strictly above v. Per-warp 256-bin histogram; integer sums.
__device__ __forceinline__ void level2(const uint32_t *cand, int k, int first, uint32_t target, bool count_only,
                                       int lane, uint32_t *hist, uint32_t &v_out, uint32_t &above_out) {
  const int kmax = __reduce_max_sync(0xffffffffu, k);
  uint32_t prefix = 0u, pmask = 0u, above = 0u;
  if (first > 0) {
    // the candidates share the bits above the first pass: take them from any
    const int src = __ffs(__ballot_sync(0xffffffffu, k > 0)) - 1;
    const uint32_t any = __shfl_sync(0xffffffffu, k > 0 ? cand[lane] : 0u, src);
    pmask = first == 1 ? 0xFF800000u : (first == 2 ? 0xFFFF8000u : 0xFFFFFF80u);
    prefix = any & pmask;
  }
  for (int pass = first; pass < 4; ++pass) {
    const int shift = pass == 0 ? 23 : (pass == 1 ? 15 : (pass == 2 ? 7 : 0));
    const uint32_t dmask = pass == 3 ? 0x7Fu : 0xFFu;
#pragma unroll
    for (int i = 0; i < 8; ++i) hist[i * 32 + lane] = 0u;
    __syncwarp();
    for (int j = 0; j < kmax; ++j) {
      if (j < k) {
        const uint32_t b = cand[j * 32 + lane];
        const uint32_t add = count_only ? 1u : mass_of(__uint_as_float(b));
        if ((b & pmask) == prefix && add != 0u) atomicAdd(hist + ((b >> shift) & dmask), add);
      }
    }
    __syncwarp();
    // lane owns digits [8 lane, 8 lane + 8)
    uint32_t hb[8], own = 0u;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      hb[q] = hist[8 * lane + q];
      own += hb[q];
    }
    uint32_t suffix = own;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_down_sync(0xffffffffu, suffix, o);
      if (lane + o < 32) suffix += y;
    }
    uint32_t run = above + (suffix - own);
    int found = -1;
    uint32_t above_found = 0u;
#pragma unroll
    for (int q = 7; q >= 0; --q) {
      if (found < 0 && run + hb[q] >= target) {
        found = 8 * lane + q;
        above_found = run;
      }
      run += hb[q];
    }
    const uint32_t hit = __ballot_sync(0xffffffffu, found >= 0);
    const int src = 31 - __clz((int)hit);
    const int digit = __shfl_sync(0xffffffffu, found, src);
    above = __shfl_sync(0xffffffffu, above_found, src);
    prefix |= (uint32_t)digit << shift;
    pmask |= dmask << shift;
    __syncwarp();
  }
  v_out = prefix;
  above_out = above;
}

// Number of candidates strictly above v and equal to v (warp totals).
__device__ __forceinline__ void cand_counts(const uint32_t *cand, int k, uint32_t v, int lane, uint32_t &gt,
                                            uint32_t &eq) {
  uint32_t g = 0u, e = 0u;
  for (int j = 0; j < k; ++j) {
    const uint32_t b = cand[j * 32 + lane];
    g += b > v ? 1u : 0u;
    e += b == v ? 1u : 0u;
  }
  gt = __reduce_add_sync(0xffffffffu, g);
  eq = __reduce_add_sync(0xffffffffu, e);
}

// Selection by weight: the pattern v of the entry where the weight (mass or
// count) in P-descending order first reaches target, the number of entries
// strictly above v and equal to v, and the weight strictly above v.
template <int NPL>
__device__ __forceinline__ void threshold(const uint32_t (&pb)[NPL], int nt, int lane, bool mass, uint32_t target,
                                          uint32_t *wsm, uint32_t &v, uint32_t &n_gt, uint32_t &n_eq,
                                          uint32_t &w_above) {
  int bstar;
  uint32_t m_above, c_above;
  level1<NPL>(pb, nt, lane, mass, target, wsm, bstar, m_above, c_above);
  uint32_t *cand = wsm;
  const int k = collect<NPL>(pb, nt, lane, mass, bstar, cand);
  const uint32_t a1 = mass ? m_above : c_above;
  // bins above 0 are exact exponents; bin 0 of the count mode mixes exponents
  const int first = (!mass && bstar == 0) ? 0 : 1;
  uint32_t above_c;
  level2(cand, k, first, target - a1, !mass, lane, wsm + Ws<NPL>::HIST, v, above_c);
  uint32_t gt_c, eq_c;
  cand_counts(cand, k, v, lane, gt_c, eq_c);
  n_gt = c_above + gt_c;
  n_eq = eq_c;
  w_above = a1 + above_c;
  __syncwarp();
}

// One warp per row r = (b*heads + h)*Nt + q0 + warp; the row's scores
// (p_logits: softmax first) or block scores (clamped to [0, 1]) come from
// P_in. kmin_head (per-head floor, second pass) raises k_min; sel_count
// (first pass of the floor) records the selected count and skips the bitset.
template <int NPL>
__global__ void __launch_bounds__(THREADS, 2)
select_rows_kernel(const float *__restrict__ P_in, int p_logits, float *__restrict__ probs_out, int heads,
                   Geo g, float top_p, int k_min, int use_scores, const int *__restrict__ windows, int G,
                   GroupLo glo, unsigned int *__restrict__ bits, int *__restrict__ counts, int wpr,
                   const int *__restrict__ kmin_head, int *__restrict__ sel_count) {
  extern __shared__ __align__(16) uint32_t smw[];
  const int nt = g.Nt;
  const int bh = blockIdx.y;
  const int h = bh % heads;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int tpf = g.NH * g.NW;
  int *gtab = reinterpret_cast<int *>(smw);
  int *wtab = gtab + ((g.T + 3) & ~3);  // 4 ints per group
  uint32_t *wsm = reinterpret_cast<uint32_t *>(wtab + 4 * STA_MAX_GROUPS) +
                  warp * (Ws<NPL>::WIN + ((wpr + 3) & ~3));
  uint32_t *wwin = wsm + Ws<NPL>::WIN;

  if (windows != nullptr) {
    for (int dt = tid; dt < g.T; dt += THREADS) {
      int grp = -1;
      for (int gg = 0; gg < G; ++gg)
        if (dt >= glo.v[gg]) grp = gg;
      gtab[dt] = grp;
    }
    for (int i = tid; i < G * 4; i += THREADS) wtab[i] = windows[(long long)h * G * 4 + i];
  }
  __syncthreads();

  const int qt = blockIdx.x * WARPS + warp;
  if (qt >= nt) return;
  const long long row = (long long)bh * nt + qt;

  uint32_t v_f = NONE, c_f = 0u;  // keep P > v_f, plus the first c_f ties at v_f
  uint32_t eq_f = 0u;              // entries equal to v_f
  uint32_t pb[NPL];
  if (use_scores) {
    const float *src = P_in + row * nt;
    float s[NPL];
#pragma unroll
    for (int i = 0; i < NPL; ++i) s[i] = (32 * i + lane < nt) ? __ldcs(src + 32 * i + lane) : -INFINITY;
    if (p_logits) {
      float mx = -INFINITY;
#pragma unroll
      for (int i = 0; i < NPL; ++i) mx = fmaxf(mx, s[i]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const float ml = mx * LOG2E_F;
      float z = 0.0f;
#pragma unroll
      for (int i = 0; i < NPL; ++i) {
        s[i] = ex2_approx(fmaf(s[i], LOG2E_F, -ml));
        z += s[i];
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
      const float rz = __frcp_rn(z);
#pragma unroll
      for (int i = 0; i < NPL; ++i) s[i] *= rz;
    } else {
#pragma unroll
      for (int i = 0; i < NPL; ++i) s[i] = clamp_unit(s[i]);
    }
    if (probs_out != nullptr) {
      float *dst = probs_out + row * nt;
#pragma unroll
      for (int i = 0; i < NPL; ++i)
        if (32 * i + lane < nt) dst[32 * i + lane] = s[i];
    }
#pragma unroll
    for (int i = 0; i < NPL; ++i) pb[i] = __float_as_uint(s[i]);

    // per-head top-k floor (second pass): k_min raised to the head's floor
    const uint32_t kk = (uint32_t)min(kmin_head != nullptr ? max(k_min, kmin_head[bh]) : k_min, nt);
    uint32_t m_level = NONE, m_ties = 0u, m_eq = 0u;
    long long m_p = 0;
    if (top_p >= 1.0f) {
      m_level = 0u;  // every entry has P >= 0: keep all
      m_ties = NONE;
      m_p = nt;
    } else if (top_p > 0.0f) {
      uint32_t wsum = 0u;
#pragma unroll
      for (int i = 0; i < NPL; ++i)
        if (32 * i + lane < nt) wsum += mass_of(__uint_as_float(pb[i]));
      const uint32_t W = __reduce_add_sync(0xffffffffu, wsum);
      const uint32_t thr = (uint32_t)ceil((double)top_p * (double)W);
      if (thr > 0u) {
        uint32_t v, n_gt, n_eq, above;
        threshold<NPL>(pb, nt, lane, true, thr, wsm, v, n_gt, n_eq, above);
        const uint32_t wv = mass_of(__uint_as_float(v));
        m_level = v;
        m_ties = (thr - above + wv - 1u) / wv;  // tied entries at level v
        m_eq = n_eq;
        m_p = (long long)n_gt + m_ties;
      }
    }
    if ((long long)kk > m_p) {
      if (kk >= (uint32_t)nt) {
        v_f = 0u;  // every entry
        c_f = NONE;
      } else {
        uint32_t u, n_gt, n_eq, above;
        threshold<NPL>(pb, nt, lane, false, kk, wsm, u, n_gt, n_eq, above);
        v_f = u;
        c_f = kk - n_gt;
        eq_f = n_eq;
      }
    } else if (m_p > 0) {
      v_f = m_level;
      c_f = m_ties;
      eq_f = m_eq;
    }
    if (sel_count != nullptr) {
      if (lane == 0) sel_count[row] = (int)((long long)kk > m_p ? kk : m_p);
      return;
    }
  }

  // window tiles of the row, written as runs of bits: for each key frame, each
  // of the two rectangles and each tile row it covers, the tile columns within
  // the extent (clipped to the grid) are consecutive key tiles
  const int tq = qt / tpf, remq = qt - tq * tpf;
  const int yq = remq / g.NW, xq = remq - yq * g.NW;
  if (windows != nullptr) {
    for (int w = lane; w < wpr; w += 32) wwin[w] = 0u;
    __syncwarp();
    const int items = g.T * 2 * g.NH;
    for (int it = lane; it < items; it += 32) {
      const int y = it % g.NH, rect = (it / g.NH) & 1, tk = it / (2 * g.NH);
      const int grp = gtab[abs(tq - tk)];
      if (grp < 0) continue;
      const int4 w4 = reinterpret_cast<const int4 *>(wtab)[grp];
      const int ry = rect ? w4.z : w4.x, rx = rect ? w4.w : w4.y;
      if (ry < 0 || rx < 0 || abs(y - yq) > ry) continue;
      const int base = (tk * g.NH + y) * g.NW;
      const int k0 = base + max(0, xq - rx), k1 = base + min(g.NW - 1, xq + rx);
      for (int w = k0 >> 5; w <= (k1 >> 5); ++w) {
        const int lo = max(k0 - 32 * w, 0), hi = min(k1 - 32 * w, 31);
        atomicOr(wwin + w, (0xFFFFFFFFu >> (31 - hi + lo)) << lo);  // bits lo..hi
      }
    }
    __syncwarp();
  }

  // membership bits: one ballot per 32 entries; ties at v_f ranked by index
  // only when some tied entries are left out
  const bool all_ties = c_f == NONE || c_f >= eq_f;
  unsigned int *brow = bits + row * wpr;
  uint32_t ties_seen = 0u, mine[(NPL + 31) / 32];
#pragma unroll
  for (int q = 0; q < (NPL + 31) / 32; ++q) mine[q] = 0u;
  int total = 0;
#pragma unroll
  for (int i = 0; i < NPL; ++i) {
    if (32 * i >= nt) break;  // uniform: words past the row
    const bool valid = 32 * i + lane < nt;
    bool sel = false;
    if (use_scores && v_f != NONE) {
      if (all_ties) {
        sel = valid && pb[i] >= v_f;
      } else {
        const bool tie = valid && pb[i] == v_f;
        const uint32_t tmask = __ballot_sync(0xffffffffu, tie);
        const uint32_t before = __popc(tmask & ((1u << lane) - 1u));
        sel = valid && (pb[i] > v_f || (tie && ties_seen + before < c_f));
        ties_seen += __popc(tmask);
      }
    }
    const uint32_t word = __ballot_sync(0xffffffffu, sel) | (windows != nullptr ? wwin[i] : 0u);
    if (lane == (i & 31)) mine[i >> 5] = word;
    total += __popc(word);
  }
#pragma unroll
  for (int q = 0; q < (NPL + 31) / 32; ++q)
    if (32 * q + lane < wpr) brow[32 * q + lane] = mine[q];
  if (lane == 0) counts[row] = total;
}

}  // namespace sel
}  // namespace sta
