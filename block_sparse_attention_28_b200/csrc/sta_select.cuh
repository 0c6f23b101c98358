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

// Level 1 of the threshold search: a private histogram per lane (its own
// column of [32 bins][32 lanes], so no two lanes ever add to the same word)
// of the entries' weight over 32 bins of the exponent of P. By mass: bin =
// exponent - 103 for the entries with mass (P >= 2^-24, exponent 103 .. 127),
// each adding its mass w = floor(P 2^24) and a count of 1 packed as
// w + 2^25 (a lane's masses in a bin sum below 2^25). Entries of zero mass,
// the row's padding among them (P = 0), are left out. By count (top-k):
// bin = max(exponent - 96, 0), each valid entry adding a count of 1 (2^25).
constexpr uint32_t CNT_ONE = 1u << 25;
constexpr uint32_t MASS_MASK = CNT_ONE - 1u;

template <int NPL>
__device__ __forceinline__ void hist_mass(const uint32_t (&pb)[NPL], int lane, uint32_t *h) {
#pragma unroll
  for (int b = 0; b < 32; ++b) h[b * 32 + lane] = 0u;
  __syncwarp();
#pragma unroll
  for (int i = 0; i < NPL; ++i) {
    const uint32_t ex = pb[i] >> 23;
    if (ex >= (uint32_t)MASS_BASE)
      atomicAdd(h + (ex - MASS_BASE) * 32 + lane, mass_of(__uint_as_float(pb[i])) + CNT_ONE);
  }
  __syncwarp();
}

template <int NPL>
__device__ __forceinline__ void hist_count(const uint32_t (&pb)[NPL], int nv, int lane, uint32_t *h) {
#pragma unroll
  for (int b = 0; b < 32; ++b) h[b * 32 + lane] = 0u;
  __syncwarp();
#pragma unroll
  for (int i = 0; i < NPL; ++i) {
    if (i < nv) {
      const int bin = max((int)(pb[i] >> 23) - COUNT_BASE, 0);
      atomicAdd(h + bin * 32 + lane, CNT_ONE);
    }
  }
  __syncwarp();
}

// Lane l's total of bin l over the 32 columns (read diagonally: conflict-free),
// summed as packed words in 64 bits (mass below bit 25, count above).
__device__ __forceinline__ unsigned long long bin_total(const uint32_t *h, int lane) {
  unsigned long long acc = 0ull;
  const uint32_t *rowp = h + lane * 32;
#pragma unroll
  for (int t = 0; t < 32; ++t) acc += rowp[(lane + t) & 31];
  return acc;
}

// The bin b* where the weight at or above it, scanning down from the top bin,
// first reaches `target` (1 <= target <= total), with the weight and count
// strictly above b*.
__device__ __forceinline__ void find_bin(uint32_t own_w, uint32_t own_c, uint32_t target, int lane, int &bstar,
                                         uint32_t &w_above, uint32_t &c_above) {
  uint32_t suf = own_w, sufc = own_c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_down_sync(0xffffffffu, suf, o);
    const uint32_t yc = __shfl_down_sync(0xffffffffu, sufc, o);
    if (lane + o < 32) {
      suf += y;
      sufc += yc;
    }
  }
  const uint32_t hit = __ballot_sync(0xffffffffu, suf >= target);
  bstar = 31 - __clz((int)hit);
  w_above = __shfl_sync(0xffffffffu, suf - own_w, bstar);
  c_above = __shfl_sync(0xffffffffu, sufc - own_c, bstar);
}

// Level 2: radix select over the candidates (lane l's in cand[k * 32 + l],
// k < its count), digit passes from `first` (0: bits 30-23, 1: 22-15,
// 2: 14-7, 3: 6-0), `prefix0` holding the bits above the first pass: the
// largest pattern v whose weight at or above reaches `target`, and the weight
// of the candidates strictly above v. Per-warp 256-bin histogram; integer sums.
__device__ __forceinline__ void level2(const uint32_t *cand, int k, int first, uint32_t prefix0, uint32_t target,
                                       bool count_only, int lane, uint32_t *hist, uint32_t &v_out,
                                       uint32_t &above_out) {
  const int kmax = __reduce_max_sync(0xffffffffu, k);
  uint32_t prefix = prefix0, above = 0u;
  uint32_t pmask = first == 0 ? 0u : (first == 1 ? 0xFF800000u : (first == 2 ? 0xFFFF8000u : 0xFFFFFF80u));
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
        if ((b & pmask) == prefix) atomicAdd(hist + ((b >> shift) & dmask), add);
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

// Candidates strictly above v and equal to v (warp totals).
__device__ __forceinline__ void cand_counts(const uint32_t *cand, int k, uint32_t v, uint32_t &gt, uint32_t &eq,
                                            int lane) {
  uint32_t g = 0u, e = 0u;
  for (int j = 0; j < k; ++j) {
    const uint32_t b = cand[j * 32 + lane];
    g += b > v ? 1u : 0u;
    e += b == v ? 1u : 0u;
  }
  gt = __reduce_add_sync(0xffffffffu, g);
  eq = __reduce_add_sync(0xffffffffu, e);
}

// One warp per row r = (b*heads + h)*Nt + q0 + warp; the row's scores come
// from P_in (softmaxed here) unless the mask is window-only. kmin_head
// (per-head floor, second pass) raises k_min; sel_count (first pass of the
// floor) records the selected count and skips the bitset. Entries past Nt
// get P = 0: they carry no mass, so the top-p path needs no validity test;
// the count path (top-k) and a threshold at P = 0 test it explicitly.
template <int NPL>
__global__ void __launch_bounds__(THREADS, NPL <= 40 ? 3 : 2)
select_rows_kernel(const float *__restrict__ P_in, float *__restrict__ probs_out, int heads, Geo g, float top_p,
                   int k_min, int use_scores, const int *__restrict__ windows, int G, GroupLo glo,
                   unsigned int *__restrict__ bits, int *__restrict__ counts, int wpr,
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
  uint32_t *hist2 = wsm + Ws<NPL>::HIST;

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
  // checked build: this warp's shared-memory region lies inside the launch's
  const uint32_t warp_end = (uint32_t)(reinterpret_cast<const uint8_t *>(wwin + ((wpr + 3) & ~3)) -
                                       reinterpret_cast<const uint8_t *>(smw));
  if (!dbg_ok(warp_end <= dyn_smem_bytes() && wpr * 32 >= nt)) {
    if (lane == 0) counts[row] = 0;
    return;
  }
  const int nv = (nt - lane + 31) >> 5;  // valid entries of this lane: i < nv

  uint32_t v_f = NONE, c_f = 0u;  // keep P > v_f, plus the first c_f ties at v_f
  uint32_t eq_f = 0u;              // entries equal to v_f
  uint32_t pb[NPL];
  if (use_scores) {
    const float *src = P_in + row * nt;
    float s[NPL];
#pragma unroll
    for (int i = 0; i < NPL; ++i) s[i] = (i < nv) ? __ldcs(src + 32 * i + lane) : -INFINITY;
    float mx = -INFINITY;
#pragma unroll
    for (int i = 0; i + 1 < NPL; i += 2) mx = fmax3_f(mx, s[i], s[i + 1]);
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
    for (int i = 0; i < NPL; ++i) pb[i] = __float_as_uint(s[i] * rz);
    if (probs_out != nullptr) {
      float *dst = probs_out + row * nt;
#pragma unroll
      for (int i = 0; i < NPL; ++i)
        if (i < nv) dst[32 * i + lane] = __uint_as_float(pb[i]);
    }

    // per-head top-k floor (second pass): k_min raised to the head's floor
    const uint32_t kk = (uint32_t)min(kmin_head != nullptr ? max(k_min, kmin_head[bh]) : k_min, nt);
    uint32_t m_level = NONE, m_ties = 0u, m_eq = 0u;
    long long m_p = 0;
    if (top_p >= 1.0f) {
      m_level = 0u;  // every entry has P >= 0: keep all
      m_ties = NONE;
      m_p = nt;
    } else if (top_p > 0.0f) {
      hist_mass<NPL>(pb, lane, wsm);
      const unsigned long long tot = bin_total(wsm, lane);
      const uint32_t own_w = (uint32_t)(tot & MASS_MASK), own_c = (uint32_t)(tot >> 25);
      const uint32_t W = __reduce_add_sync(0xffffffffu, own_w);
      const uint32_t thr = (uint32_t)ceil((double)top_p * (double)W);
      __syncwarp();  // the histogram columns become candidate columns
      if (thr > 0u) {
        int bstar;
        uint32_t w_above, c_above;
        find_bin(own_w, own_c, thr, lane, bstar, w_above, c_above);
        // the entries of bin b*: exponent MASS_BASE + b*
        const uint32_t ex = (uint32_t)(MASS_BASE + bstar);
        int k = 0;
#pragma unroll
        for (int i = 0; i < NPL; ++i)
          if ((pb[i] >> 23) == ex) wsm[(k++) * 32 + lane] = pb[i];
        __syncwarp();
        uint32_t v, above_c, gt_c, eq_c;
        level2(wsm, k, 1, ex << 23, thr - w_above, false, lane, hist2, v, above_c);
        cand_counts(wsm, k, v, gt_c, eq_c, lane);
        const uint32_t above = w_above + above_c;
        const uint32_t wv = mass_of(__uint_as_float(v));
        m_level = v;
        m_ties = (thr - above + wv - 1u) / wv;  // tied entries at level v
        m_eq = eq_c;
        m_p = (long long)(c_above + gt_c) + m_ties;
        __syncwarp();
      }
    }
    if ((long long)kk > m_p) {
      if (kk >= (uint32_t)nt) {
        v_f = 0u;  // every entry
        c_f = NONE;
      } else {
        hist_count<NPL>(pb, nv, lane, wsm);
        const uint32_t own_c = (uint32_t)(bin_total(wsm, lane) >> 25);
        __syncwarp();
        int bstar;
        uint32_t c_above, c_above2;
        find_bin(own_c, own_c, kk, lane, bstar, c_above, c_above2);
        int k = 0;
#pragma unroll
        for (int i = 0; i < NPL; ++i)
          if (i < nv && max((int)(pb[i] >> 23) - COUNT_BASE, 0) == bstar) wsm[(k++) * 32 + lane] = pb[i];
        __syncwarp();
        // bins above 0 are exact exponents; bin 0 mixes the exponents below 97
        const int first = bstar == 0 ? 0 : 1;
        const uint32_t pre = bstar == 0 ? 0u : (uint32_t)(COUNT_BASE + bstar) << 23;
        uint32_t u, above_c, gt_c, eq_c;
        level2(wsm, k, first, pre, kk - c_above, true, lane, hist2, u, above_c);
        cand_counts(wsm, k, u, gt_c, eq_c, lane);
        v_f = u;
        c_f = kk - (c_above + gt_c);
        eq_f = eq_c;
        __syncwarp();
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

  // window tiles of the row, written as runs of bits: for each key frame and
  // each of the two rectangles, every tile row the rectangle covers holds a
  // run of consecutive key tiles (the columns within the extent, clipped to
  // the grid)
  const int tq = qt / tpf, remq = qt - tq * tpf;
  const int yq = remq / g.NW, xq = remq - yq * g.NW;
  if (windows != nullptr) {
    for (int w = lane; w < wpr; w += 32) wwin[w] = 0u;
    __syncwarp();
    for (int it = lane; it < 2 * g.T; it += 32) {
      const int rect = it & 1, tk = it >> 1;
      const int grp = gtab[abs(tq - tk)];
      if (grp < 0) continue;
      const int4 w4 = reinterpret_cast<const int4 *>(wtab)[grp];
      const int ry = rect ? w4.z : w4.x, rx = rect ? w4.w : w4.y;
      if (ry < 0 || rx < 0) continue;
      const int y0 = max(0, yq - ry), y1 = min(g.NH - 1, yq + ry);
      const int x0 = max(0, xq - rx), x1 = min(g.NW - 1, xq + rx);
      for (int y = y0; y <= y1; ++y) {
        const int base = (tk * g.NH + y) * g.NW;
        const int k0 = base + x0, k1 = base + x1;
        for (int w = k0 >> 5; w <= (k1 >> 5); ++w) {
          const int lo = max(k0 - 32 * w, 0), hi = min(k1 - 32 * w, 31);
          atomicOr(wwin + w, (0xFFFFFFFFu >> (31 - hi + lo)) << lo);  // bits lo..hi
        }
      }
    }
    __syncwarp();
  }

  // membership bits: one ballot per 32 entries; ties at v_f ranked by index
  // only when some tied entries are left out; entries past Nt (P = 0) can
  // only meet a threshold at P = 0, where validity is tested
  constexpr int NW32 = (NPL + 31) / 32;
  uint32_t mine[NW32];
#pragma unroll
  for (int q = 0; q < NW32; ++q) mine[q] = 0u;
  if (use_scores && v_f != NONE) {
    const bool all_ties = c_f == NONE || c_f >= eq_f;
    const bool test_valid = v_f == 0u;
    uint32_t ties_seen = 0u;
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
      if (32 * i >= nt) break;  // uniform: words past the row
      const bool valid = !test_valid || i < nv;
      bool sel;
      if (all_ties) {
        sel = valid && pb[i] >= v_f;
      } else {
        const bool tie = valid && pb[i] == v_f;
        const uint32_t tmask = __ballot_sync(0xffffffffu, tie);
        const uint32_t before = __popc(tmask & ((1u << lane) - 1u));
        sel = valid && (pb[i] > v_f || (tie && ties_seen + before < c_f));
        ties_seen += __popc(tmask);
      }
      const uint32_t word = __ballot_sync(0xffffffffu, sel);
      if (lane == (i & 31)) mine[i >> 5] = word;
    }
  }
  unsigned int *brow = bits + row * wpr;
  int total = 0;
#pragma unroll
  for (int q = 0; q < NW32; ++q) {
    const int w = 32 * q + lane;
    if (w < wpr) {
      const uint32_t word = mine[q] | (windows != nullptr ? wwin[w] : 0u);
      brow[w] = word;
      total += __popc(word);
    }
  }
  total = __reduce_add_sync(0xffffffffu, total);
  if (lane == 0) counts[row] = total;
}

}  // namespace sel
}  // namespace sta
