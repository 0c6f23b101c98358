// Recall-driven dual-window search (Compact Attention Fig. 3: the offline
// search shrinks the dual windows under the recall (tau) and cost (lambda)
// constraints; Fig. 4: it starts from full coverage in every
// temporal-distance group). One CTA per (b*heads + h) runs the whole greedy in
// shared memory, with no round trip to the host:
//   masses  w = floor(min(max(m, 0), 1) * 2^24) (exact integer sums);
//   start   (ry1, rx1, ry2, rx2) = (NH-1, NW-1, NH-1, NW-1) in every group;
//   moves   per group g: ry1-1, rx1-1, ry2-1, rx2-1, (ry1-1, ry2-1),
//           (rx1-1, rx2-1); an extent never goes below -1;
//   value   J = removed / Nt^2 - lambda * lost / W (double, no contraction);
//   admit   covered - lost >= ceil(double(tau) * W) and J >= 0; a move that
//           uncovers nothing (one window shrunk inside the other) has J = 0,
//           which is how the two windows, equal at the start, come apart;
//   step    the admissible move with the largest J, ties to the lowest index
//           g*6 + m; stop when none is left.
#pragma once
#include "sta_common.cuh"

namespace sta {

constexpr int SEARCH_THREADS = 1024;
constexpr int SEARCH_MOVES = 6;

__device__ __forceinline__ void search_move(int m, int (&w)[4]) {
  // decrement the extents a move names (see the table above)
  if (m == 0 || m == 4) w[0] -= 1;
  if (m == 1 || m == 5) w[1] -= 1;
  if (m == 2 || m == 4) w[2] -= 1;
  if (m == 3 || m == 5) w[3] -= 1;
}

__device__ __forceinline__ bool search_move_valid(int m, const int (&w)[4]) {
  const bool a = (m == 0 || m == 4) ? w[0] > -1 : true;
  const bool b = (m == 1 || m == 5) ? w[1] > -1 : true;
  const bool c = (m == 2 || m == 4) ? w[2] > -1 : true;
  const bool d = (m == 3 || m == 5) ? w[3] > -1 : true;
  return a && b && c && d;
}

__device__ __forceinline__ bool covers(int dy, int dx, int ry1, int rx1, int ry2, int rx2) {
  return (dy <= ry1 && dx <= rx1) || (dy <= ry2 && dx <= rx2);
}

__device__ __forceinline__ unsigned long long search_mass(float m) {
  return (unsigned long long)__float2uint_rd(fminf(fmaxf(m, 0.0f), 1.0f) * 16777216.0f);
}

// dynamic smem: kcoord [Nt] packed (t << 20 | y << 10 | x), gtab [T]
__global__ void __launch_bounds__(SEARCH_THREADS)
search_windows_kernel(const float *__restrict__ mass, Geo g, int G, GroupLo glo, float tau,
                      float lambda, int *__restrict__ windows_out, float *__restrict__ stats_out) {
  extern __shared__ unsigned int ssm[];
  __shared__ int win[STA_MAX_GROUPS][4];
  __shared__ unsigned long long red_mass[SEARCH_MOVES][SEARCH_THREADS / 32];
  __shared__ unsigned int red_cnt[SEARCH_MOVES][SEARCH_THREADS / 32];
  __shared__ unsigned long long mv_lost[STA_MAX_GROUPS][SEARCH_MOVES];
  __shared__ unsigned int mv_removed[STA_MAX_GROUPS][SEARCH_MOVES];
  __shared__ int done;
  __shared__ int dirty;  // group whose moves must be re-evaluated (-1: all)
  const int nt = g.Nt, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nwarps = SEARCH_THREADS / 32;
  const long long bh = blockIdx.x;
  const float *M = mass + bh * (long long)nt * nt;
  unsigned int *kcoord = ssm;
  int *gtab = reinterpret_cast<int *>(ssm + nt);
  const int tpf = g.NH * g.NW;
  for (int k = tid; k < nt; k += SEARCH_THREADS) {
    const int t = k / tpf, rem = k - t * tpf;
    const int y = rem / g.NW, x = rem - y * g.NW;
    kcoord[k] = ((unsigned)t << 20) | ((unsigned)y << 10) | (unsigned)x;
  }
  for (int dt = tid; dt < g.T; dt += SEARCH_THREADS) {
    int grp = -1;
    for (int gg = 0; gg < G; ++gg)
      if (dt >= glo.v[gg]) grp = gg;
    gtab[dt] = grp;
  }
  if (tid < G * 4) win[tid / 4][tid % 4] = (tid % 2 == 0) ? g.NH - 1 : g.NW - 1;
  if (tid == 0) {
    done = 0;
    dirty = -1;
  }
  // total integer mass W (every pair is covered at the start)
  unsigned long long tot = 0;
  for (int q = warp; q < nt; q += nwarps)
    for (int k = lane; k < nt; k += 32) tot += search_mass(M[(long long)q * nt + k]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
  if (lane == 0) red_mass[0][warp] = tot;
  __syncthreads();
  unsigned long long total = 0;
  for (int w = 0; w < nwarps; ++w) total += red_mass[0][w];
  __syncthreads();
  const unsigned long long thr = (unsigned long long)ceil((double)tau * (double)total);
  unsigned long long covered = total;
  unsigned long long covered_pairs = (unsigned long long)nt * nt;
  const int max_steps = G * (2 * g.NH + 2 * g.NW + 4);

  for (int step = 0; step < max_steps && !done; ++step) {
    // A move of group g changes only pairs whose |dt| falls in g, so the other
    // groups' move costs from earlier steps still hold: only the group the
    // last step moved is scanned again (all groups on the first step).
    const int only = dirty;
    for (int gi = 0; gi < G; ++gi) {
      if (only >= 0 && gi != only) continue;
      const int ry1 = win[gi][0], rx1 = win[gi][1], ry2 = win[gi][2], rx2 = win[gi][3];
      int cand[SEARCH_MOVES][4];
#pragma unroll
      for (int mi = 0; mi < SEARCH_MOVES; ++mi) {
        cand[mi][0] = ry1; cand[mi][1] = rx1; cand[mi][2] = ry2; cand[mi][3] = rx2;
        search_move(mi, cand[mi]);
      }
      unsigned int cnt[SEARCH_MOVES] = {0u, 0u, 0u, 0u, 0u, 0u};
      unsigned long long lost[SEARCH_MOVES] = {0ull, 0ull, 0ull, 0ull, 0ull, 0ull};
      for (int q = warp; q < nt; q += nwarps) {
        const unsigned int qc = kcoord[q];
        const int tq = (int)(qc >> 20), yq = (int)((qc >> 10) & 1023u), xq = (int)(qc & 1023u);
        for (int k = lane; k < nt; k += 32) {
          const unsigned int kc = kcoord[k];
          const int dt = abs(tq - (int)(kc >> 20));
          if (gtab[dt] != gi) continue;
          const int dy = abs(yq - (int)((kc >> 10) & 1023u)), dx = abs(xq - (int)(kc & 1023u));
          if (!covers(dy, dx, ry1, rx1, ry2, rx2)) continue;
          const unsigned long long wgt = search_mass(M[(long long)q * nt + k]);
#pragma unroll
          for (int mi = 0; mi < SEARCH_MOVES; ++mi) {
            if (!covers(dy, dx, cand[mi][0], cand[mi][1], cand[mi][2], cand[mi][3])) {
              cnt[mi] += 1u;
              lost[mi] += wgt;
            }
          }
        }
      }
#pragma unroll
      for (int mi = 0; mi < SEARCH_MOVES; ++mi) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          cnt[mi] += __shfl_xor_sync(0xffffffffu, cnt[mi], o);
          lost[mi] += __shfl_xor_sync(0xffffffffu, lost[mi], o);
        }
        if (lane == 0) {
          red_cnt[mi][warp] = cnt[mi];
          red_mass[mi][warp] = lost[mi];
        }
      }
      __syncthreads();
      if (tid < SEARCH_MOVES) {
        unsigned int c = 0u;
        unsigned long long l = 0ull;
        for (int w = 0; w < nwarps; ++w) {
          c += red_cnt[tid][w];
          l += red_mass[tid][w];
        }
        mv_removed[gi][tid] = c;
        mv_lost[gi][tid] = l;
      }
      __syncthreads();
    }
    if (tid == 0) {
      int best = -1;
      double bestJ = 0.0;
      for (int gi = 0; gi < G; ++gi) {
        const int cur[4] = {win[gi][0], win[gi][1], win[gi][2], win[gi][3]};
        for (int mi = 0; mi < SEARCH_MOVES; ++mi) {
          if (!search_move_valid(mi, cur)) continue;
          const unsigned int removed = mv_removed[gi][mi];
          const unsigned long long l = mv_lost[gi][mi];
          if (l > covered || covered - l < thr) continue;  // recall constraint
          const double a = (double)removed / (double)((long long)nt * nt);
          const double b = total ? (double)l / (double)total : 0.0;
          // a - lambda * b with two roundings (a fused multiply-add could
          // change the sign of a J near zero)
          const double J = __dsub_rn(a, __dmul_rn((double)lambda, b));
          if (J < 0.0) continue;  // cost constraint
          if (best < 0 || J > bestJ) {
            best = gi * SEARCH_MOVES + mi;
            bestJ = J;
          }
        }
      }
      if (best < 0) {
        done = 1;
      } else {
        const int gi = best / SEARCH_MOVES, mi = best % SEARCH_MOVES;
        int w4[4] = {win[gi][0], win[gi][1], win[gi][2], win[gi][3]};
        search_move(mi, w4);
        for (int e = 0; e < 4; ++e) win[gi][e] = w4[e];
        covered -= mv_lost[gi][mi];
        covered_pairs -= mv_removed[gi][mi];
        dirty = gi;
      }
    }
    __syncthreads();
  }
  if (tid < G * 4) windows_out[bh * G * 4 + tid] = win[tid / 4][tid % 4];
  if (tid == 0 && stats_out != nullptr) {
    stats_out[bh * 2 + 0] = total ? (float)((double)covered / (double)total) : 1.0f;
    stats_out[bh * 2 + 1] = (float)((double)covered_pairs / ((double)nt * nt));
  }
}

}  // namespace sta
