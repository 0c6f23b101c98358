// Token reorder between raster order and 1x8x8 tiles (Compact Attention:
// tile-aligned masks; Table III "Cubic" tiles). A pure permutation copy, so
// the kernel is bound by HBM bandwidth: every 16-byte chunk is read once and
// written once, with 2D grids so that all index math stays in 32 bits.
#pragma once
#include "sta_common.cuh"

namespace sta {

constexpr int REORDER_THREADS = 256;
constexpr int REORDER_UNROLL = 4;

// Forward: dst tiled [B, heads, Lpad, D] <- src raster [B, L, heads, D].
// grid.y = b*heads + h; each thread moves REORDER_UNROLL 16-byte chunks of
// one head's tiled rows. Pad rows (outside the grid) are written as zero.
template <int D>
__global__ void __launch_bounds__(REORDER_THREADS)
reorder_fwd_kernel(const uint4 *__restrict__ src, uint4 *__restrict__ dst, int heads, Geo g) {
  constexpr int CPR = D / 8;  // 16-byte chunks per row
  const int bh = blockIdx.y;
  const int b = bh / heads, h = bh - b * heads;
  const long long L = (long long)g.T * g.H * g.W;
  const unsigned int per_head = (unsigned int)g.Lpad * CPR;
  const uint4 *src_b = src + (long long)b * L * heads * CPR;
  uint4 *dst_bh = dst + (long long)bh * per_head;
  const unsigned int base = blockIdx.x * (REORDER_THREADS * REORDER_UNROLL) + threadIdx.x;
  const int tiles_per_frame = g.NH * g.NW;
  uint4 v[REORDER_UNROLL];
#pragma unroll
  for (int u = 0; u < REORDER_UNROLL; ++u) {
    const unsigned int idx = base + u * REORDER_THREADS;
    v[u] = make_uint4(0u, 0u, 0u, 0u);
    if (idx < per_head) {
      const unsigned int c = idx % CPR, lrow = idx / CPR;
      const unsigned int n = lrow >> 6, r = lrow & 63u;
      const unsigned int t = n / tiles_per_frame, rem = n - t * tiles_per_frame;
      const unsigned int ty = rem / g.NW, tx = rem - ty * g.NW;
      const unsigned int y = ty * 8 + (r >> 3), x = tx * 8 + (r & 7u);
      if (y < (unsigned)g.H && x < (unsigned)g.W) {
        const long long i = ((long long)t * g.H + y) * g.W + x;
        v[u] = __ldcs(src_b + (i * heads + h) * CPR + c);
      }
    }
  }
#pragma unroll
  for (int u = 0; u < REORDER_UNROLL; ++u) {
    const unsigned int idx = base + u * REORDER_THREADS;
    if (idx < per_head) __stcs(dst_bh + idx, v[u]);
  }
}

// Inverse: dst raster [B, L, heads, D] <- src tiled [B, heads, Lpad, D].
// grid.y = b; each thread moves REORDER_UNROLL chunks of the raster output.
template <int D>
__global__ void __launch_bounds__(REORDER_THREADS)
reorder_inv_kernel(const uint4 *__restrict__ src, uint4 *__restrict__ dst, int heads, Geo g) {
  constexpr int CPR = D / 8;
  const int b = blockIdx.y;
  const unsigned int HW = (unsigned)g.H * g.W;
  const unsigned long long per_b = (unsigned long long)g.T * HW * heads * CPR;
  const unsigned long long base =
      (unsigned long long)blockIdx.x * (REORDER_THREADS * REORDER_UNROLL) + threadIdx.x;
  const uint4 *src_b = src + (long long)b * heads * g.Lpad * CPR;
  uint4 *dst_b = dst + (long long)b * per_b;
  uint4 v[REORDER_UNROLL];
#pragma unroll
  for (int u = 0; u < REORDER_UNROLL; ++u) {
    const unsigned long long idx = base + u * REORDER_THREADS;
    if (idx < per_b) {
      const unsigned int c = (unsigned int)(idx % CPR);
      const unsigned long long t2 = idx / CPR;
      const unsigned int h = (unsigned int)(t2 % heads);
      const unsigned int i = (unsigned int)(t2 / heads);
      const unsigned int t = i / HW, rem = i - t * HW;
      const unsigned int y = rem / g.W, x = rem - y * g.W;
      const unsigned int n = (t * g.NH + (y >> 3)) * g.NW + (x >> 3);
      const unsigned int lrow = n * 64 + (y & 7u) * 8 + (x & 7u);
      v[u] = __ldcs(src_b + ((long long)h * g.Lpad + lrow) * CPR + c);
    }
  }
#pragma unroll
  for (int u = 0; u < REORDER_UNROLL; ++u) {
    const unsigned long long idx = base + u * REORDER_THREADS;
    if (idx < per_b) __stcs(dst_b + idx, v[u]);
  }
}

template <int D>
inline cudaError_t launch_reorder(const void *src, void *dst, int B, int heads, const Geo &g,
                                  bool inverse, cudaStream_t s) {
  constexpr int CPR = D / 8;
  const long long per_block = (long long)REORDER_THREADS * REORDER_UNROLL;
  if (!inverse) {
    const long long per_head = g.Lpad * CPR;
    dim3 grid((unsigned)((per_head + per_block - 1) / per_block), (unsigned)(B * heads));
    reorder_fwd_kernel<D><<<grid, REORDER_THREADS, 0, s>>>(
        static_cast<const uint4 *>(src), static_cast<uint4 *>(dst), heads, g);
  } else {
    const long long per_b = (long long)g.T * g.H * g.W * heads * CPR;
    dim3 grid((unsigned)((per_b + per_block - 1) / per_block), (unsigned)B);
    reorder_inv_kernel<D><<<grid, REORDER_THREADS, 0, s>>>(
        static_cast<const uint4 *>(src), static_cast<uint4 *>(dst), heads, g);
  }
  return cudaGetLastError();
}

}  // namespace sta
