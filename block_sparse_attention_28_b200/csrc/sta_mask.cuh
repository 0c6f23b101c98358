// Online mask construction: pooled block scores (Rectified SpaAttn), hybrid
// top-p / k_min selection (SCOPE Eqs. (7)-(8) as quoted), OR'd with per-head
// dual windows per temporal-distance group (Compact Attention Fig. 1(3),
// Fig. 4), emitted as CSR lists (Compact Attention Fig. 3).
//
// Kernels, in launch order:
//   pool_kernel          tile means of tiled Q and K (HBM-bound, coalesced 16 B
//                        loads); the raster form pools with pool_tma_kernel
//                        (sta_pool.cuh)
//   score_tc_kernel      (sta_score.cuh, full workspace) the scores on the
//                        tensor cores, rows of S written to a row buffer
//   score_select_kernel  row softmax, selection, window test -> row bitsets;
//                        with the minimum workspace it also computes the
//                        scores (fp32 FMA chains, 16 query tiles per CTA)
//   scan_kernel          exclusive scan of the row counts -> row_ptr, nnz
//   fill_kernel          bitsets -> ascending col_idx (+ optional byte mask)
#pragma once
#include "sta_common.cuh"

namespace sta {

constexpr float MASS_ONE_F = 16777216.0f;  // 2^24, fixed-point unit of the mass

// fp32 rounded to the nearest tf32 (10 explicit mantissa bits, ties away
// from zero); the low 13 bits of the result are zero.
__device__ __forceinline__ float round_tf32(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return __uint_as_float(r);
}

// ---------------------------------------------------------------- pooling
// One warp per (b*heads + h, tile) of the tiled layout. Each lane owns one
// 16-byte chunk of a row and walks the tile's real rows; the sum is exact in
// fp64 (64 bf16 values whose magnitudes span less than 2^39), the mean is
// rounded once to fp32. With qlo / klo given, the mean x is
// stored split for the tensor-core scores: tf32(x) in qbar / kbar and
// tf32(x - tf32(x)) in qlo / klo (round to nearest, ties away).
template <int D>
__global__ void __launch_bounds__(256)
pool_kernel(const uint4 *__restrict__ q, const uint4 *__restrict__ k, float *__restrict__ qbar,
            float *__restrict__ kbar, float *__restrict__ qlo, float *__restrict__ klo,
            long long n_tiles_total, Geo g) {
  constexpr int CPR = D / 8;      // chunks per row
  constexpr int RPI = 32 / CPR;   // rows per warp step
  const long long warp_id = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const bool is_k = warp_id >= n_tiles_total;
  const long long idx = is_k ? warp_id - n_tiles_total : warp_id;
  if (idx >= n_tiles_total) return;
  const uint4 *src = is_k ? k : q;
  float *dst = is_k ? kbar : qbar;
  float *dst_lo = is_k ? klo : qlo;
  const long long bh = idx / g.Nt;
  const int n = (int)(idx % g.Nt);
  const long long tile = bh * g.Nt + n;  // output row of qbar / kbar
  const int tpf = g.NH * g.NW;
  const int t = n / tpf, rem = n - t * tpf;
  const int ty = rem / g.NW, tx = rem - ty * g.NW;
  const int vy = valid_extent(g.H, ty), vx = valid_extent(g.W, tx);
  const int sub = lane / CPR, c = lane - sub * CPR;
  auto row_chunk = [&](int r) -> const uint4 * { return src + (tile * 64 + r) * CPR; };
  double acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.0;
#pragma unroll 4
  for (int i = 0; i < 64 / RPI; ++i) {
    const int r = i * RPI + sub;
    if ((r >> 3) < vy && (r & 7) < vx) {
      const uint4 w = __ldcs(row_chunk(r) + c);
      const __nv_bfloat162 *p = reinterpret_cast<const __nv_bfloat162 *>(&w);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(p[e]);
        acc[2 * e] += (double)f.x;
        acc[2 * e + 1] += (double)f.y;
      }
    }
  }
#pragma unroll
  for (int off = CPR; off < 32; off <<= 1) {
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], off);
  }
  if (sub == 0) {
    const double cnt = (double)(vy * vx);
    float out[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) out[e] = (float)(acc[e] / cnt);
    if (dst_lo != nullptr) {
      float lo[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float hi = round_tf32(out[e]);
        lo[e] = round_tf32(out[e] - hi);  // x - hi is exact in fp32
        out[e] = hi;
      }
      float4 *ol = reinterpret_cast<float4 *>(dst_lo + tile * D + c * 8);
      ol[0] = make_float4(lo[0], lo[1], lo[2], lo[3]);
      ol[1] = make_float4(lo[4], lo[5], lo[6], lo[7]);
    }
    float4 *o = reinterpret_cast<float4 *>(dst + tile * D + c * 8);
    o[0] = make_float4(out[0], out[1], out[2], out[3]);
    o[1] = make_float4(out[4], out[5], out[6], out[7]);
  }
}

// Pooled K and V of the rectified attention: row (bh, kt) of kbar / vbar is
// the mean over the real tokens of tile kt (fp64 sum, rounded once to bf16),
// for kt < Nt; rows Nt .. ntp-1 are zero. One warp per (tensor, bh, kt).
template <int D>
__global__ void __launch_bounds__(256)
pool_kv_kernel(const uint4 *__restrict__ k, const uint4 *__restrict__ v, uint4 *__restrict__ kbar,
               uint4 *__restrict__ vbar, long long bh_total, int ntp, Geo g) {
  constexpr int CPR = D / 8;
  constexpr int RPI = 32 / CPR;
  const long long warp_id = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const long long rows = bh_total * ntp;
  const bool is_v = warp_id >= rows;
  const long long idx = is_v ? warp_id - rows : warp_id;
  if (idx >= rows) return;
  const long long bh = idx / ntp;
  const int kt = (int)(idx - bh * ntp);
  const uint4 *src = is_v ? v : k;
  uint4 *dst = (is_v ? vbar : kbar) + idx * CPR;
  const int sub = lane / CPR, c = lane - sub * CPR;
  if (kt >= g.Nt) {
    if (sub == 0) dst[c] = make_uint4(0u, 0u, 0u, 0u);
    return;
  }
  const int rem = kt % (g.NH * g.NW);
  const int ty = rem / g.NW, tx = rem - ty * g.NW;
  const int vy = valid_extent(g.H, ty), vx = valid_extent(g.W, tx);
  const uint4 *base = src + (bh * g.Nt + kt) * 64 * CPR;
  double acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.0;
  for (int i = 0; i < 64 / RPI; ++i) {
    const int r = i * RPI + sub;
    if ((r >> 3) < vy && (r & 7) < vx) {
      const uint4 w = base[r * CPR + c];
      const __nv_bfloat162 *p = reinterpret_cast<const __nv_bfloat162 *>(&w);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(p[e]);
        acc[2 * e] += (double)f.x;
        acc[2 * e + 1] += (double)f.y;
      }
    }
  }
#pragma unroll
  for (int off = CPR; off < 32; off <<= 1) {
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], off);
  }
  if (sub == 0) {
    const double cnt = (double)(vy * vx);
    uint32_t pk[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      __nv_bfloat162 b2 = __floats2bfloat162_rn((float)(acc[2 * e] / cnt), (float)(acc[2 * e + 1] / cnt));
      pk[e] = *reinterpret_cast<uint32_t *>(&b2);
    }
    dst[c] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
  }
}

// ------------------------------------------------------ scores + selection
constexpr int SEL_THREADS = 256;
constexpr int SEL_QB = 16;        // query tiles per CTA of the fused pass
constexpr int SEL_QB_SELECT = 8;  // rows per CTA of the select pass (one per warp)
// Modes of score_select_kernel:
//   SEL_FUSED   scores (fp32 FMA chains), softmax, selection and windows in
//               one CTA of 16 rows kept in shared memory (the minimum
//               workspace: no row buffer)
//   SEL_SELECT  softmax (when the rows hold scores), selection and windows
//               on rows read from P_in; no score code, so the CTA is small
//               and four fit on an SM
constexpr int SEL_FUSED = 0, SEL_SELECT = 1;
constexpr int SEL_KPT = 3;  // key tiles per thread in the fused score loop

struct GroupLo {
  int v[STA_MAX_GROUPS];
};

constexpr float LOG2E_F = 1.4426950408889634f;

// 2^x on the MUFU unit (ex2.approx.ftz.f32: relative error below 2^-22).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Three-input maximum (one instruction).
__device__ __forceinline__ float fmax3_f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// A caller-given block score clamped to [0, 1], with -0 taken to +0 (the
// selection orders P by its bit pattern).
__device__ __forceinline__ float clamp_unit(float x) { return __fadd_rn(fminf(fmaxf(x, 0.0f), 1.0f), 0.0f); }

__device__ __forceinline__ unsigned int warp_sum_u32(unsigned int x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// Row softmax in fp32 over Sr[0, nt): the maximum m, e = 2^(s log2e - m log2e)
// (one FFMA, ex2.approx), the sum Z in a fixed order (lane-strided partial
// sums in index order, then a butterfly over the lanes), P = e * (1 / Z) with
// the reciprocal rounded once. P replaces the scores in Sr and is copied to
// out when given. The register-resident select pass computes the same P bit
// for bit (same operations in the same order).
__device__ __forceinline__ void row_softmax(float *Sr, int nt, int lane, float *out) {
  float mx = -INFINITY;
  for (int j = lane; j < nt; j += 32) mx = fmaxf(mx, Sr[j]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  const float ml = mx * LOG2E_F;
  float sum = 0.0f;
  for (int j = lane; j < nt; j += 32) {
    const float e = ex2_approx(fmaf(Sr[j], LOG2E_F, -ml));
    Sr[j] = e;
    sum += e;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  const float rz = __frcp_rn(sum);
  for (int j = lane; j < nt; j += 32) {
    const float p = Sr[j] * rz;
    Sr[j] = p;
    if (out) out[j] = p;
  }
}

__device__ __forceinline__ unsigned int mass_of(float p) {
  return __float2uint_rd(p * MASS_ONE_F);  // exact: p in [0,1], scaling by 2^24
}

// Total mass (or count when `count_only`) of the row entries whose P bit
// pattern is >= `key`. P >= 0, so float bits order like the values. 64-bit:
// a row of caller-given block scores (each clamped to [0, 1], not normalised)
// can hold up to Nt * 2^24 of mass.
__device__ __forceinline__ unsigned long long mass_at_least(const float *row, int nt, unsigned int key,
                                                            bool count_only, int lane) {
  unsigned long long s = 0;
  for (int j = lane; j < nt; j += 32) {
    const float p = row[j];
    if (__float_as_uint(p) >= key) s += count_only ? 1u : mass_of(p);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  return s;
}

// Radix select over the P bit patterns (P >= 0, so the bits order like the
// values). Finds the largest pattern v with f(v) >= target, where
// f(v) = sum over entries with P >= v of (count_only ? 1 : mass), one digit at
// a time from the most significant (bits 30-23, 22-15, 14-7, 6-0), with a
// per-warp histogram of 256 bins in shared memory. Also returns f restricted
// to entries strictly above v. target must be >= 1 and f(0) >= target.
// All sums are 64-bit integers, so the result does not depend on summation
// order.
__device__ void radix_level(const float *row, int nt, unsigned long long target, bool count_only, int lane,
                            unsigned long long *hist, unsigned int &v_out, unsigned long long &above_out) {
  unsigned int prefix = 0u, pmask = 0u;
  unsigned long long above = 0ull;
#pragma unroll
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = pass == 0 ? 23 : (pass == 1 ? 15 : (pass == 2 ? 7 : 0));
    const unsigned int dmask = pass == 3 ? 0x7Fu : 0xFFu;
#pragma unroll
    for (int i = 0; i < 8; ++i) hist[i * 32 + lane] = 0ull;
    __syncwarp();
    for (int j = lane; j < nt; j += 32) {
      const unsigned int b = __float_as_uint(row[j]);
      // entries of zero mass add nothing to a mass histogram: no atomic
      const unsigned int add = count_only ? 1u : mass_of(__uint_as_float(b));
      if ((b & pmask) == prefix && add != 0u) atomicAdd(hist + ((b >> shift) & dmask), (unsigned long long)add);
    }
    __syncwarp();
    // lane owns digits [8*lane, 8*lane + 8)
    unsigned long long hb[8], own = 0ull;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      hb[k] = hist[8 * lane + k];
      own += hb[k];
    }
    unsigned long long suffix = own;  // digits owned by this lane and all higher lanes
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned long long y = __shfl_down_sync(0xffffffffu, suffix, o);
      if (lane + o < 32) suffix += y;
    }
    unsigned long long run = above + (suffix - own);
    int found = -1;
    unsigned long long above_found = 0ull;
#pragma unroll
    for (int k = 7; k >= 0; --k) {
      if (found < 0 && run + hb[k] >= target) {
        found = 8 * lane + k;
        above_found = run;
      }
      run += hb[k];
    }
    const unsigned int hit = __ballot_sync(0xffffffffu, found >= 0);
    const int src = 31 - __clz((int)hit);
    const int digit = __shfl_sync(0xffffffffu, found, src);
    above = __shfl_sync(0xffffffffu, above_found, src);
    prefix |= (unsigned int)digit << shift;
    pmask |= dmask << shift;
    __syncwarp();
  }
  v_out = prefix;
  above_out = above;
}

// One CTA per (b*heads + h, block of QB query tiles).
// Dynamic smem: qs [QB][D] fp32 (fused mode), S [QB][Nt] fp32 and the
// per-warp histograms (if use_scores), then the window tables.
// SEL_SELECT reads its rows from P_in: scores to be softmaxed when p_logits
// (the tensor-core score pass), else block scores clamped to [0, 1].
// SEL_SELECT CTAs are capped at four per SM by shared memory; saying so lets
// the compiler use the registers that occupancy leaves (56 instead of 40).
template <int D, int QB, int MODE>
__global__ void __launch_bounds__(SEL_THREADS, MODE == SEL_SELECT ? 4 : 1)
score_select_kernel(const float *__restrict__ qbar, const float *__restrict__ kbar, int heads, Geo g,
                    float scale, float top_p, int k_min, int use_scores,
                    const int *__restrict__ windows, int G, GroupLo glo,
                    unsigned int *__restrict__ bits, int *__restrict__ counts,
                    float *__restrict__ probs_out, int wpr, const int *__restrict__ kmin_head,
                    int *__restrict__ sel_count, const float *__restrict__ P_in, int p_logits) {
  constexpr bool HAS_SCORES = MODE == SEL_FUSED;
  extern __shared__ __align__(16) float sm[];
  const int nt = g.Nt;
  const int bh = blockIdx.y;
  const int h = bh % heads;
  const int q0 = blockIdx.x * QB;
  const int nq = min(QB, nt - q0);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int tpf = g.NH * g.NW;
  // shared memory: [qs], [S, histograms] if use_scores, then the window
  // tables and one row of window bits per warp (all 16-byte aligned: QB * nt
  // is a multiple of 8)
  float *qs = sm;
  float *S = qs + ((HAS_SCORES && use_scores) ? QB * D : 0);
  unsigned long long *hist = reinterpret_cast<unsigned long long *>(S + (use_scores ? QB * nt : 0));
  int *gtab = reinterpret_cast<int *>(hist + (use_scores ? (SEL_THREADS / 32) * 256 : 0));
  int *wtab = gtab + ((g.T + 3) & ~3);  // 4 ints per group
  unsigned int *wwin = reinterpret_cast<unsigned int *>(wtab + 4 * STA_MAX_GROUPS) + warp * wpr;
  unsigned long long *whist = hist + warp * 256;

  // Window tables, once per CTA: the temporal group of every |dt| and this
  // head's extents.
  if (windows != nullptr) {
    for (int dt = tid; dt < g.T; dt += SEL_THREADS) {
      int grp = -1;
      for (int gg = 0; gg < G; ++gg)
        if (dt >= glo.v[gg]) grp = gg;
      gtab[dt] = grp;
    }
    for (int i = tid; i < G * 4; i += SEL_THREADS) wtab[i] = windows[(long long)h * G * 4 + i];
  }
  __syncthreads();  // every warp reads the tables

  if (HAS_SCORES && use_scores && P_in == nullptr) {
    // Phase 1: S[i][kt] = scale * qbar[q0+i] . kbar[kt], sequential fp32 FMA over d.
    for (int e = tid; e < QB * D; e += SEL_THREADS) {
      const int i = e / D;
      qs[e] = (i < nq) ? qbar[((long long)bh * nt + q0 + i) * D + (e - i * D)] : 0.0f;
    }
    __syncthreads();
    // Each thread owns up to SEL_KPT key tiles (kt = base + tid + u * threads)
    // of a chunk, so every query value read from shared memory feeds
    // SEL_KPT FMAs; the passes split Nt into equal chunks. Every score is
    // still one sequential fp32 FMA chain over d.
    const int per_pass = SEL_THREADS * SEL_KPT;
    const int passes = (nt + per_pass - 1) / per_pass;
    const int chunk = (nt + passes - 1) / passes;
    for (int pass = 0; pass < passes; ++pass) {
      const int lo = pass * chunk, hi = min(nt, lo + chunk);
      const float4 *kr[SEL_KPT];
      bool on[SEL_KPT];
#pragma unroll
      for (int u = 0; u < SEL_KPT; ++u) {
        const int kt = lo + tid + u * SEL_THREADS;
        on[u] = kt < hi;
        kr[u] = reinterpret_cast<const float4 *>(kbar + ((long long)bh * nt + (on[u] ? kt : lo)) * D);
      }
      float acc[SEL_KPT][QB];
#pragma unroll
      for (int u = 0; u < SEL_KPT; ++u)
#pragma unroll
        for (int i = 0; i < QB; ++i) acc[u][i] = 0.0f;
      for (int d4 = 0; d4 < D / 4; ++d4) {
        float4 kv[SEL_KPT];
#pragma unroll
        for (int u = 0; u < SEL_KPT; ++u) kv[u] = __ldg(kr[u] + d4);
#pragma unroll
        for (int i = 0; i < QB; ++i) {
          const float4 qv = reinterpret_cast<const float4 *>(qs + i * D)[d4];
#pragma unroll
          for (int u = 0; u < SEL_KPT; ++u) {
            acc[u][i] = fmaf(qv.x, kv[u].x, acc[u][i]);
            acc[u][i] = fmaf(qv.y, kv[u].y, acc[u][i]);
            acc[u][i] = fmaf(qv.z, kv[u].z, acc[u][i]);
            acc[u][i] = fmaf(qv.w, kv[u].w, acc[u][i]);
          }
        }
      }
#pragma unroll
      for (int u = 0; u < SEL_KPT; ++u) {
        const int kt = lo + tid + u * SEL_THREADS;
        if (on[u]) {
#pragma unroll
          for (int i = 0; i < QB; ++i) S[i * nt + kt] = acc[u][i] * scale;
        }
      }
    }
    __syncthreads();
  }

  for (int i = warp; i < nq; i += SEL_THREADS / 32) {
    const int qt = q0 + i;
    const long long row = (long long)bh * nt + qt;
    float *Sr = S + i * nt;
    unsigned int v_f = 0xFFFFFFFFu;  // keep P > v_f, plus c_f ties at v_f
    unsigned int c_f = 0u;
    if (use_scores) {
      float *pout = probs_out ? probs_out + row * nt : nullptr;
      if (!HAS_SCORES && p_logits) {
        // Phase 2: scores of the tensor-core pass, then the row softmax (the
        // rows may be the caller's block_probs: each lane reads its entries
        // before it overwrites them with P)
        for (int j = lane; j < nt; j += 32) Sr[j] = P_in[row * nt + j];
        row_softmax(Sr, nt, lane, pout);
      } else if (!HAS_SCORES || P_in != nullptr) {
        // caller-supplied block scores (e.g. exact block masses), clamped to [0, 1]
        for (int j = lane; j < nt; j += 32) {
          const float p = clamp_unit(P_in[row * nt + j]);
          Sr[j] = p;
          if (pout) pout[j] = p;
        }
      } else {
        // Phase 2: row softmax of the fused pass's scores
        row_softmax(Sr, nt, lane, pout);
      }
      __syncwarp();
      // Phase 3: selection threshold as (level v_f, ties c_f).
      // per-head top-k floor (second pass): k_min raised to the head's floor
      const int kk = min(kmin_head != nullptr ? max(k_min, kmin_head[bh]) : k_min, nt);
      unsigned int m_p_level = 0xFFFFFFFFu, m_p_ties = 0u;
      long long m_p = 0;
      if (top_p >= 1.0f) {
        m_p_level = 0u;  // every entry has P >= 0: keep all
        m_p_ties = 0xFFFFFFFFu;
        m_p = nt;
      } else if (top_p > 0.0f) {
        const unsigned long long W = mass_at_least(Sr, nt, 0u, false, lane);
        const unsigned long long thr = (unsigned long long)ceil((double)top_p * (double)W);
        if (thr > 0ull) {
          unsigned int v;
          unsigned long long above;
          radix_level(Sr, nt, thr, false, lane, whist, v, above);
          const unsigned long long wv = mass_of(__uint_as_float(v));
          const unsigned int need = (unsigned int)((thr - above + wv - 1ull) / wv);  // tied entries at level v
          const unsigned int cnt_above = (unsigned int)mass_at_least(Sr, nt, v + 1u, true, lane);
          m_p_level = v;
          m_p_ties = need;
          m_p = (long long)cnt_above + need;
        }
      }
      if ((long long)kk > m_p) {
        unsigned int u;
        unsigned long long cnt_above;
        radix_level(Sr, nt, (unsigned long long)kk, true, lane, whist, u, cnt_above);
        v_f = u;
        c_f = (unsigned int)kk - (unsigned int)cnt_above;
      } else if (m_p > 0) {
        v_f = m_p_level;
        c_f = m_p_ties;
      }
      if (sel_count != nullptr && lane == 0) sel_count[row] = (int)((long long)kk > m_p ? kk : m_p);
    }
    // Phase 4: membership bits = selected OR window, one 32-bit word per lane step.
    const int tq = qt / tpf, remq = qt - tq * tpf;
    const int yq = remq / g.NW, xq = remq - yq * g.NW;
    if (windows != nullptr) {
      // The row's window tiles, written as runs of bits: for each key frame,
      // each of the two rectangles and each tile row it covers, the tile
      // columns within the extent (clipped to the grid) are consecutive
      // key tiles.
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
    unsigned int ties_seen = 0u;
    int total = 0;
    unsigned int *brow = bits + row * wpr;
    for (int w0 = 0; w0 < wpr; ++w0) {
      const int kt = w0 * 32 + lane;
      // Selection membership needs the index-ordered rank among ties: warp-wide.
      bool sel = false;
      if (use_scores && v_f != 0xFFFFFFFFu) {
        const unsigned int pb = (kt < nt) ? __float_as_uint(Sr[kt]) : 0u;
        const bool tie = (kt < nt) && (pb == v_f);
        const unsigned int tmask = __ballot_sync(0xffffffffu, tie);
        const unsigned int before = __popc(tmask & ((1u << lane) - 1u));
        sel = (kt < nt) && (pb > v_f || (tie && ties_seen + before < c_f));
        ties_seen += __popc(tmask);
      }
      const unsigned int word = __ballot_sync(0xffffffffu, sel) | (windows != nullptr ? wwin[w0] : 0u);
      if (lane == 0) brow[w0] = word;
      total += __popc(word);
    }
    if (lane == 0) counts[row] = total;
  }
}

// ------------------------------------------------ per-head top-k floor
// One CTA per (b*heads + h): k_head = ceil(sum_c n_c b_c / sum_c n_c), with
// b_c the selected count of query tile c and n_c its number of real tokens
// (SCOPE Eqs. (9)-(10) as quoted, query tiles as clusters). Integer sums.
constexpr int FLOOR_THREADS = 256;

__global__ void __launch_bounds__(FLOOR_THREADS)
head_floor_kernel(const int *__restrict__ sel_count, int *__restrict__ kfloor, Geo g) {
  __shared__ long long part[2][FLOOR_THREADS / 32];
  const int bh = blockIdx.x, tid = threadIdx.x;
  const int tpf = g.NH * g.NW;
  long long num = 0, den = 0;
  for (int qt = tid; qt < g.Nt; qt += FLOOR_THREADS) {
    const int rem = qt % tpf;
    const int ty = rem / g.NW, tx = rem - ty * g.NW;
    const long long n = (long long)valid_extent(g.H, ty) * valid_extent(g.W, tx);
    num += n * sel_count[(long long)bh * g.Nt + qt];
    den += n;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    num += __shfl_xor_sync(0xffffffffu, num, o);
    den += __shfl_xor_sync(0xffffffffu, den, o);
  }
  if ((tid & 31) == 0) {
    part[0][tid >> 5] = num;
    part[1][tid >> 5] = den;
  }
  __syncthreads();
  if (tid == 0) {
    long long N = 0, Dn = 0;
    for (int w = 0; w < FLOOR_THREADS / 32; ++w) {
      N += part[0][w];
      Dn += part[1][w];
    }
    kfloor[bh] = Dn > 0 ? (int)((N + Dn - 1) / Dn) : 0;
  }
}

// ---------------------------------------------------------------- scan
// Single CTA: row_ptr[0] = 0, row_ptr[r+1] = sum of counts[0..r]; nnz = total.
constexpr int SCAN_THREADS = 1024;
constexpr int SCAN_BATCH = 4;  // chunks of 4 * SCAN_THREADS counts whose loads are issued together

__device__ __forceinline__ int warp_incl_scan(int x, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  return x;
}

// Single-CTA exclusive scan of the row counts into row_ptr (row_ptr[0] = 0,
// row_ptr[r + 1] = sum of counts[0..r]) and nnz = the total. The counts are
// read in chunks of 4 per thread (4096 per chunk, coalesced), scanned with
// warp shuffles plus one pass over the 32 warp totals, and chained by a
// running carry. Integer sums: the result does not depend on the order.
__global__ void __launch_bounds__(SCAN_THREADS)
scan_kernel(const int *__restrict__ counts, int *__restrict__ row_ptr, long long *__restrict__ nnz,
            long long R) {
  __shared__ int wsum[SCAN_THREADS / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr long long CH = 4LL * SCAN_THREADS;
  long long carry = 0;
  if (tid == 0) row_ptr[0] = 0;
  for (long long base = 0; base < R; base += CH * SCAN_BATCH) {
    int v[SCAN_BATCH][4];
#pragma unroll
    for (int bch = 0; bch < SCAN_BATCH; ++bch) {
      const long long i0 = base + bch * CH + 4LL * tid;
#pragma unroll
      for (int e = 0; e < 4; ++e) v[bch][e] = (i0 + e < R) ? counts[i0 + e] : 0;
    }
#pragma unroll
    for (int bch = 0; bch < SCAN_BATCH; ++bch) {
      if (base + bch * CH >= R) break;  // uniform over the CTA
      int x[4];
      x[0] = v[bch][0];
#pragma unroll
      for (int e = 1; e < 4; ++e) x[e] = x[e - 1] + v[bch][e];
      const int incl = warp_incl_scan(x[3], lane);
      if (lane == 31) wsum[warp] = incl;
      __syncthreads();
      if (warp == 0) wsum[lane] = warp_incl_scan(wsum[lane], lane);
      __syncthreads();
      const long long pre = carry + (warp > 0 ? wsum[warp - 1] : 0) + (incl - x[3]);
      const long long i0 = base + bch * CH + 4LL * tid;
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (i0 + e < R) row_ptr[i0 + e + 1] = (int)(pre + x[e]);
      carry += wsum[SCAN_THREADS / 32 - 1];
      __syncthreads();  // wsum is rewritten by the next chunk
    }
  }
  if (tid == 0) *nnz = carry;
}

// ---------------------------------------------------------------- validate
// One warp per row of a caller's CSR: the offsets are read first and checked
// (row_ptr[0] == 0, non-decreasing, at most Nt entries per row, inside the
// column array's capacity), and only then the row's columns, which must be
// strictly ascending and in [0, Nt). Any violation sets DEV_ERR_BAD_MASK.
__global__ void __launch_bounds__(256)
validate_csr_kernel(const int *__restrict__ row_ptr, const int *__restrict__ col_idx, long long capacity,
                    long long R, int nt) {
  const long long row = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= R) return;
  const long long a0 = row_ptr[row], a1 = row_ptr[row + 1];
  bool bad = (row == 0 && a0 != 0) || a0 < 0 || a1 < a0 || a1 - a0 > nt || a1 > capacity;
  if (!bad) {
    for (long long i = a0 + lane; i < a1; i += 32) {
      const int c = col_idx[i];
      const int prev = (i > a0) ? col_idx[i - 1] : -1;
      if (c < 0 || c >= nt || c <= prev) bad = true;
    }
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) record_error(DEV_ERR_BAD_MASK);
}

// ---------------------------------------------------------------- fill
// One warp per row: word prefix popcounts -> ascending column indices.
__global__ void __launch_bounds__(256)
fill_kernel(const unsigned int *__restrict__ bits, const int *__restrict__ row_ptr,
            int *__restrict__ col_idx, unsigned char *__restrict__ block_mask, long long R, int nt,
            int wpr) {
  const long long row = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= R) return;
  const unsigned int *brow = bits + row * wpr;
  int base = row_ptr[row];
  // checked build: every index stays inside the row's own range of col_idx
  const int row_end = STA_DEBUG ? row_ptr[row + 1] : 0x7fffffff;
  for (int w0 = 0; w0 < wpr; w0 += 32) {
    const int w = w0 + lane;
    unsigned int word = (w < wpr) ? brow[w] : 0u;
    const int c = __popc(word);
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int pos = base + incl - c;
    if (block_mask && w < wpr) {
      unsigned char *bm = block_mask + row * nt + (long long)w * 32;
      const int lim = min(32, nt - w * 32);
      for (int b = 0; b < lim; ++b) bm[b] = (unsigned char)((word >> b) & 1u);
    }
    while (word) {
      const int b = __ffs(word) - 1;
      if (dbg_ok(pos < row_end && (long long)pos < R * nt && w * 32 + b < nt)) col_idx[pos] = w * 32 + b;
      ++pos;
      word &= word - 1u;
    }
    base += __shfl_sync(0xffffffffu, incl, 31);
  }
}

}  // namespace sta
