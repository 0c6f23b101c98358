// Shared definitions of the libsta CUDA library (single translation unit).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/sta.h"

namespace sta {

// Device error word: bit flags, read and cleared by sta_get_device_error().
enum : unsigned int {
  DEV_ERR_TIMEOUT = 1u,
  DEV_ERR_BAD_MASK = 2u,
  DEV_ERR_BOUNDS = 4u,  // checked build only: an index or address failed its check
};

__device__ unsigned int g_dev_error;

__device__ __forceinline__ void record_error(unsigned int bit) { atomicOr(&g_dev_error, bit); }

// The checked build (compiled with -DSTA_DEBUG=1: libsta_debug.so) tests the
// indices and addresses that come from run-time data before each TMA load,
// TMEM access and global store that uses them: a failed check records
// DEV_ERR_BOUNDS and the access is skipped (a skipped load then ends in a
// bounded pipeline wait, never in a fault). In the product build dbg_ok() is
// the constant true and the checks compile away.
#ifndef STA_DEBUG
#define STA_DEBUG 0
#endif
// Bytes of dynamic shared memory this CTA was launched with.
__device__ __forceinline__ uint32_t dyn_smem_bytes() {
  uint32_t r;
  asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(r));
  return r;
}
__device__ __forceinline__ bool dbg_ok(bool cond) {
#if STA_DEBUG
  if (!cond) record_error(DEV_ERR_BOUNDS);
  return cond;
#else
  (void)cond;
  return true;
#endif
}

// Tile geometry of a T x H x W grid with 1x8x8 tiles.
struct Geo {
  int T, H, W;
  int NH, NW;
  int Nt;      // tiles per head
  long long Lpad;  // rows per head in the tiled layout
};

inline bool make_geo(sta_grid g, Geo *out) {
  if (g.T <= 0 || g.H <= 0 || g.W <= 0) return false;
  long long nh = (g.H + 7) / 8, nw = (g.W + 7) / 8;
  long long nt = (long long)g.T * nh * nw;
  if (nt > (1 << 20)) return false;
  out->T = g.T;
  out->H = g.H;
  out->W = g.W;
  out->NH = (int)nh;
  out->NW = (int)nw;
  out->Nt = (int)nt;
  out->Lpad = 64 * nt;
  return true;
}

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Number of real rows / columns of the tile at tile-row ty, tile-column tx.
__host__ __device__ __forceinline__ int valid_extent(int full, int t8) {
  int v = full - 8 * t8;
  return v < 8 ? v : 8;
}

}  // namespace sta

#define STA_CUDA_TRY(expr)                         \
  do {                                             \
    cudaError_t e_ = (expr);                       \
    if (e_ != cudaSuccess) return STA_ERR_CUDA;    \
  } while (0)
