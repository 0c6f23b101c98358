// Query-tile pairing by list overlap. The attention kernels run two 64-token
// query tiles as one 128-row tensor-core tile over the union of their key
// lists, so a pair whose lists differ computes union steps one of its tiles
// does not need. The total work is sum over pairs of |L_a u L_b| =
// sum |L| - sum |L_a n L_b|: a matching of maximal total overlap minimises it.
// Here, per head: candidate partners are the spatio-temporal neighbours of a
// tile (14 forward offsets), weighted by the overlap of their final lists;
// the matching is greedy in a strict total order of the candidate pairs,
// computed as a locally-dominant matching (a free tile and its heaviest free
// candidate that choose each other are matched, round after round), which
// gives the sequential greedy result; the tiles left over are paired in
// ascending order; and the pairing is kept only if its total union is below
// that of the attention's default frame pairing.
//   pair_candidates_kernel  one warp per tile: the overlaps of its candidates
//                        from the row bitsets of the mask build (AND + popcount
//                        over words), sorted in the total order
//   pair_match_kernel    one CTA per head: the matching, the left-over tiles,
//                        the comparison with the frame pairing, the output
#pragma once
#include "sta_common.cuh"

namespace sta {
namespace pairq {

constexpr int NOFF = 14;
constexpr int MATCH_THREADS = 512;

// Offset k of the candidate set: (1, dy, dx) for dy, dx in {-1, 0, 1}
// (k = 0..8), (0, 1, dx) (k = 9..11), (0, 0, 1) (k = 12), (2, 0, 0) (k = 13).
__device__ __forceinline__ void offset(int k, int &dt, int &dy, int &dx) {
  if (k < 9) {
    dt = 1;
    dy = k / 3 - 1;
    dx = k % 3 - 1;
  } else if (k < 12) {
    dt = 0;
    dy = 1;
    dx = k - 10;
  } else if (k == 12) {
    dt = 0;
    dy = 0;
    dx = 1;
  } else {
    dt = 2;
    dy = 0;
    dx = 0;
  }
}

// Tile (t, y, x) + sign * offset k, or -1 outside the grid.
__device__ __forceinline__ int step(const Geo &g, int t, int y, int x, int k, int sign) {
  int dt, dy, dx;
  offset(k, dt, dy, dx);
  const int t2 = t + sign * dt, y2 = y + sign * dy, x2 = x + sign * dx;
  if (t2 < 0 || t2 >= g.T || y2 < 0 || y2 >= g.NH || x2 < 0 || x2 >= g.NW) return -1;
  return (t2 * g.NH + y2) * g.NW + x2;
}

// Strict total order of candidate pairs: larger weight first, then the lower
// smaller tile, then the lower larger tile. True if (w1, a1, b1) comes first.
__device__ __forceinline__ bool before(int w1, int a1, int b1, int w2, int a2, int b2) {
  const int lo1 = min(a1, b1), hi1 = max(a1, b1), lo2 = min(a2, b2), hi2 = max(a2, b2);
  if (w1 != w2) return w1 > w2;
  if (lo1 != lo2) return lo1 < lo2;
  return hi1 < hi2;
}

// One warp per tile v of a head: the overlaps |L_v n L_u| of its (up to
// 2 * NOFF) candidates u = v +- offset k (AND + popcount of the two row
// bitsets; the words of row v are loaded once), then the candidates in the
// total order into cand[(bh*Nt + v)*2*NOFF + rank], -1 after the last. Lane j
// holds candidate j; its rank is the number of candidates that come first.
__global__ void __launch_bounds__(256)
pair_candidates_kernel(const unsigned int *__restrict__ bits, int *__restrict__ cand, long long R, Geo g,
                       int wpr) {
  const long long row = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= R) return;
  const int v = (int)(row % g.Nt);
  const int tpf = g.NH * g.NW;
  const int t = v / tpf, rem = v - t * tpf;
  const int y = rem / g.NW, x = rem - y * g.NW;
  const unsigned int *rv = bits + row * wpr;
  const unsigned int v0 = lane < wpr ? rv[lane] : 0u;  // rows of up to 32 words in one load
  int my_u = -1, my_w = 0, n = 0;
#pragma unroll 1
  for (int j = 0; j < 2 * NOFF; ++j) {
    const int u = step(g, t, y, x, j >> 1, (j & 1) ? -1 : 1);
    if (u < 0) continue;  // uniform over the warp
    const unsigned int *ru = bits + (row - v + u) * wpr;
    int c = __popc(v0 & (lane < wpr ? ru[lane] : 0u));
    for (int i = lane + 32; i < wpr; i += 32) c += __popc(rv[i] & ru[i]);
    c = __reduce_add_sync(0xffffffffu, c);
    if (lane == n) {
      my_u = u;
      my_w = c;
    }
    ++n;
  }
  int rank = 0;
  for (int i = 0; i < n; ++i) {
    const int ui = __shfl_sync(0xffffffffu, my_u, i), wi = __shfl_sync(0xffffffffu, my_w, i);
    if (lane < n && i != lane && before(wi, v, ui, my_w, v, my_u)) ++rank;
  }
  int *out = cand + row * 2 * NOFF;
  if (lane < n && dbg_ok(rank < 2 * NOFF)) out[rank] = my_u;
  if (lane >= n && lane < 2 * NOFF) out[lane] = -1;
}

// The default pairing of the attention kernels: pair i -> (qtA, qtB), qtB
// = -1 past the last tile.
__device__ __forceinline__ void frame_pair(const Geo &g, int i, int &qa, int &qb) {
  const int tpf = g.NH * g.NW;
  const int pairs_t = (g.T / 2) * tpf;
  if (i < pairs_t) {
    const int u = i / tpf, rem = i - u * tpf;
    qa = 2 * u * tpf + rem;
    qb = qa + tpf;
  } else {
    qa = (g.T - 1) * tpf + 2 * (i - pairs_t);
    qb = qa + 1;
  }
  if (qb >= g.Nt) qb = -1;
}

// Exclusive prefix sum over the MATCH_THREADS threads of the block (all of
// them call it); returns this thread's offset and the total in `total`.
__device__ __forceinline__ int block_exclusive_scan(int x, int *tmp, int &total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) tmp[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int t = lane < MATCH_THREADS / 32 ? tmp[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    if (lane < MATCH_THREADS / 32) tmp[lane] = t;  // inclusive per warp
  }
  __syncthreads();
  total = tmp[MATCH_THREADS / 32 - 1];
  const int before = (warp > 0 ? tmp[warp - 1] : 0) + incl - x;
  __syncthreads();  // tmp is reused by the next call
  return before;
}

// One CTA per (b, h), on the candidate lists of pair_candidates_kernel: a
// round only advances each free tile's pointer past candidates that got
// matched, so a round costs a few loads per free tile however many rounds
// ties make. Shared memory: mate[Nt], best[Nt] (int32), ptr[Nt] (uint8).
__global__ void __launch_bounds__(MATCH_THREADS)
pair_match_kernel(const unsigned int *__restrict__ bits, const int *__restrict__ counts,
                  const int *__restrict__ cand, int *__restrict__ pairs, Geo g, int wpr) {
  extern __shared__ int psm[];
  const int nt = g.Nt;
  int *mate = psm;       // partner, -1 while free
  int *best = psm + nt;  // this round's choice
  uint8_t *ptr = reinterpret_cast<uint8_t *>(psm + 2 * nt);
  __shared__ long long cost[2];
  __shared__ int scan_tmp[MATCH_THREADS / 32];
  const int tid = threadIdx.x, lane = tid & 31;
  const long long r0 = (long long)blockIdx.x * nt;
  const int *ch = cand + r0 * 2 * NOFF;
  for (int v = tid; v < nt; v += MATCH_THREADS) {
    mate[v] = -1;
    ptr[v] = 0;
  }
  if (tid == 0) cost[0] = cost[1] = 0;
  __syncthreads();
  // locally-dominant matching: at most nt / 2 rounds (each round matches the
  // heaviest free candidate pair, if any)
  for (int round = 0; round <= nt / 2; ++round) {
    for (int v = tid; v < nt; v += MATCH_THREADS) {
      int bu = -1;
      if (mate[v] < 0) {
        const int *cv = ch + (long long)v * 2 * NOFF;
        int p = ptr[v];
        while (p < 2 * NOFF && cv[p] >= 0 && mate[cv[p]] >= 0) ++p;
        ptr[v] = (uint8_t)p;
        bu = (p < 2 * NOFF) ? cv[p] : -1;
      }
      best[v] = bu;
    }
    __syncthreads();
    int changed = 0;
    for (int v = tid; v < nt; v += MATCH_THREADS) {
      const int u = best[v];
      if (mate[v] < 0 && u >= 0 && best[u] == v) {
        mate[v] = u;
        changed = 1;
      }
    }
    if (!__syncthreads_or(changed)) break;
  }
  // tiles left over: paired in ascending order of their rank among the free
  // tiles (2i with 2i + 1; a last one alone); best[] now lists them by rank
  const int CH = (nt + MATCH_THREADS - 1) / MATCH_THREADS;  // tiles per thread, contiguous
  const int v0 = tid * CH, v1 = min(nt, v0 + CH);
  int nfree = 0;
  for (int v = v0; v < v1; ++v) nfree += mate[v] < 0;
  int total_free;
  int rank = block_exclusive_scan(nfree, scan_tmp, total_free);
  __syncthreads();  // every thread has read mate[] for the scan
  for (int v = v0; v < v1; ++v)
    if (mate[v] < 0) best[rank++] = v;
  __syncthreads();
  for (int r = 2 * tid; r < total_free; r += 2 * MATCH_THREADS) {
    const int a = best[r];
    if (r + 1 < total_free) {
      const int b = best[r + 1];
      mate[a] = b;
      mate[b] = a;
    } else {
      mate[a] = nt;  // alone (odd count): marked past the end
    }
  }
  __syncthreads();
  // total union of this pairing (pairs led by their lower tile) and of the
  // default pairing; a thread per pair, the overlap over the row words
  const int np = (nt + 1) / 2;
  long long c_greedy = 0, c_frame = 0;
  auto ovl = [&](int x, int y) {
    int c = 0;
    for (int i = 0; i < wpr; ++i) c += __popc(bits[(r0 + x) * wpr + i] & bits[(r0 + y) * wpr + i]);
    return c;
  };
  for (int v = tid; v < nt; v += MATCH_THREADS) {
    const int u = mate[v];
    if (u < v) continue;  // led by the partner
    const int ca = counts[r0 + v];
    c_greedy += (u >= nt) ? ca : ca + counts[r0 + u] - ovl(v, u);
  }
  for (int i = tid; i < np; i += MATCH_THREADS) {
    int qa, qb;
    frame_pair(g, i, qa, qb);
    const int ca = counts[r0 + qa];
    c_frame += (qb < 0) ? ca : ca + counts[r0 + qb] - ovl(qa, qb);
  }
  // a warp's sum is at most 32 (Nt/512 + 1) 2 Nt < 2^32 for every Nt whose
  // 9 Nt bytes of shared memory the launch allows
  c_greedy = __reduce_add_sync(0xffffffffu, (unsigned)c_greedy);
  c_frame = __reduce_add_sync(0xffffffffu, (unsigned)c_frame);
  if (lane == 0) {
    atomicAdd(reinterpret_cast<unsigned long long *>(&cost[0]), (unsigned long long)c_greedy);
    atomicAdd(reinterpret_cast<unsigned long long *>(&cost[1]), (unsigned long long)c_frame);
  }
  __syncthreads();
  int *out = pairs + (long long)blockIdx.x * 2 * np;
  if (cost[0] < cost[1]) {
    // pairs in ascending order of their lower tile: a leader's slot is the
    // number of leaders before it
    int nlead = 0;
    for (int v = v0; v < v1; ++v) nlead += mate[v] >= v;
    int total_lead;
    int slot = block_exclusive_scan(nlead, scan_tmp, total_lead);
    for (int v = v0; v < v1; ++v) {
      const int u = mate[v];
      if (u < v) continue;
      if (dbg_ok(slot < np)) {
        out[2 * slot] = v;
        out[2 * slot + 1] = (u >= nt) ? -1 : u;
      }
      ++slot;
    }
  } else {
    for (int i = tid; i < np; i += MATCH_THREADS) {
      int qa, qb;
      frame_pair(g, i, qa, qb);
      out[2 * i] = qa;
      out[2 * i + 1] = qb;
    }
  }
}

}  // namespace pairq
}  // namespace sta
