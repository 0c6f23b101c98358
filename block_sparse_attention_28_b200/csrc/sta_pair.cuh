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
//   pair_weights_kernel  one warp per (tile, offset): |L_a n L_b| from the row
//                        bitsets of the mask build (AND + popcount over words)
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

// Tile a + offset k, or -1 outside the grid.
__device__ __forceinline__ int neighbour(const Geo &g, int a, int k) {
  int dt, dy, dx;
  offset(k, dt, dy, dx);
  const int tpf = g.NH * g.NW;
  const int t = a / tpf, rem = a - t * tpf;
  const int y = rem / g.NW, x = rem - y * g.NW;
  const int t2 = t + dt, y2 = y + dy, x2 = x + dx;
  if (t2 >= g.T || y2 < 0 || y2 >= g.NH || x2 < 0 || x2 >= g.NW) return -1;
  return (t2 * g.NH + y2) * g.NW + x2;
}

// Tile a - offset k (the tile whose candidate k is a), or -1.
__device__ __forceinline__ int back_neighbour(const Geo &g, int a, int k) {
  int dt, dy, dx;
  offset(k, dt, dy, dx);
  const int tpf = g.NH * g.NW;
  const int t = a / tpf, rem = a - t * tpf;
  const int y = rem / g.NW, x = rem - y * g.NW;
  const int t2 = t - dt, y2 = y - dy, x2 = x - dx;
  if (t2 < 0 || y2 < 0 || y2 >= g.NH || x2 < 0 || x2 >= g.NW) return -1;
  return (t2 * g.NH + y2) * g.NW + x2;
}

// w[(bh*Nt + a)*NOFF + k] = |L_a n L_b| for b = a + offset k, -1 if b is off
// the grid.
__global__ void __launch_bounds__(256)
pair_weights_kernel(const unsigned int *__restrict__ bits, int *__restrict__ w, long long R, Geo g, int wpr) {
  const long long gw = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (gw >= R * NOFF) return;
  const long long row = gw / NOFF;
  const int k = (int)(gw - row * NOFF);
  const int a = (int)(row % g.Nt);
  const int b = neighbour(g, a, k);
  int c = 0;
  if (b >= 0) {
    const unsigned int *ra = bits + row * wpr;
    const unsigned int *rb = bits + (row - a + b) * wpr;
    for (int i = lane; i < wpr; i += 32) c += __popc(ra[i] & rb[i]);
    c = __reduce_add_sync(0xffffffffu, c);
  }
  if (lane == 0 && dbg_ok(gw < R * NOFF)) w[gw] = b >= 0 ? c : -1;
}

// Strict total order of candidate pairs: larger weight first, then the lower
// smaller tile, then the lower larger tile. True if (w1, a1, b1) comes first.
__device__ __forceinline__ bool before(int w1, int a1, int b1, int w2, int a2, int b2) {
  const int lo1 = min(a1, b1), hi1 = max(a1, b1), lo2 = min(a2, b2), hi2 = max(a2, b2);
  if (w1 != w2) return w1 > w2;
  if (lo1 != lo2) return lo1 < lo2;
  return hi1 < hi2;
}

// |L_a n L_b| of two rows of one head, by one warp.
__device__ __forceinline__ int overlap(const unsigned int *__restrict__ bits, long long r0, int a, int b, int wpr,
                                      int lane) {
  int c = 0;
  for (int i = lane; i < wpr; i += 32) c += __popc(bits[(r0 + a) * wpr + i] & bits[(r0 + b) * wpr + i]);
  return __reduce_add_sync(0xffffffffu, c);
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

// One CTA per (b, h). Shared memory: mate[Nt], best[Nt] (int32).
__global__ void __launch_bounds__(MATCH_THREADS)
pair_match_kernel(const unsigned int *__restrict__ bits, const int *__restrict__ w, const int *__restrict__ counts,
                  int *__restrict__ pairs, Geo g, int wpr) {
  extern __shared__ int psm[];
  const int nt = g.Nt;
  int *mate = psm;       // partner, -1 while free
  int *best = psm + nt;  // this round's choice
  __shared__ long long cost[2];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const long long r0 = (long long)blockIdx.x * nt;
  const int *wh = w + r0 * NOFF;
  for (int v = tid; v < nt; v += MATCH_THREADS) mate[v] = -1;
  if (tid == 0) cost[0] = cost[1] = 0;
  __syncthreads();
  // locally-dominant matching: at most nt / 2 rounds (each round matches the
  // heaviest free candidate pair, if any)
  for (int round = 0; round <= nt / 2; ++round) {
    for (int v = tid; v < nt; v += MATCH_THREADS) {
      int bu = -1, bw = 0;
      if (mate[v] < 0) {
        for (int k = 0; k < NOFF; ++k) {
          const int u = neighbour(g, v, k);
          if (u >= 0 && mate[u] < 0) {
            const int wt = wh[(long long)v * NOFF + k];
            if (bu < 0 || before(wt, v, u, bw, v, bu)) {
              bu = u;
              bw = wt;
            }
          }
          const int u2 = back_neighbour(g, v, k);
          if (u2 >= 0 && mate[u2] < 0) {
            const int wt = wh[(long long)u2 * NOFF + k];
            if (bu < 0 || before(wt, v, u2, bw, v, bu)) {
              bu = u2;
              bw = wt;
            }
          }
        }
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
  // tiles left over: paired in ascending order (serial; Nt is small)
  if (tid == 0) {
    int prev = -1;
    for (int v = 0; v < nt; ++v) {
      if (mate[v] >= 0) continue;
      if (prev < 0) {
        prev = v;
      } else {
        mate[prev] = v;
        mate[v] = prev;
        prev = -1;
      }
    }
    if (prev >= 0) mate[prev] = nt;  // alone (odd count): marked past the end
  }
  __syncthreads();
  // total union of this pairing (pairs led by their lower tile) and of the
  // default pairing, one warp per pair
  const int np = (nt + 1) / 2;
  const int nwarps = MATCH_THREADS / 32;
  long long c_greedy = 0, c_frame = 0;
  for (int v = warp; v < nt; v += nwarps) {
    const int u = mate[v];
    if (u < v) continue;  // led by the partner
    const int ca = counts[r0 + v];
    c_greedy += (u >= nt) ? ca : ca + counts[r0 + u] - overlap(bits, r0, v, u, wpr, lane);
  }
  for (int i = warp; i < np; i += nwarps) {
    int qa, qb;
    frame_pair(g, i, qa, qb);
    const int ca = counts[r0 + qa];
    c_frame += (qb < 0) ? ca : ca + counts[r0 + qb] - overlap(bits, r0, qa, qb, wpr, lane);
  }
  if (lane == 0) {
    atomicAdd(reinterpret_cast<unsigned long long *>(&cost[0]), (unsigned long long)c_greedy);
    atomicAdd(reinterpret_cast<unsigned long long *>(&cost[1]), (unsigned long long)c_frame);
  }
  __syncthreads();
  int *out = pairs + (long long)blockIdx.x * 2 * np;
  if (cost[0] < cost[1]) {
    // pairs in ascending order of their lower tile: the rank of a leader is
    // the number of leaders before it (serial count; Nt is small)
    if (tid == 0) {
      int i = 0;
      for (int v = 0; v < nt; ++v) {
        const int u = mate[v];
        if (u < v) continue;
        if (dbg_ok(i < np)) {
          out[2 * i] = v;
          out[2 * i + 1] = (u >= nt) ? -1 : u;
        }
        ++i;
      }
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
