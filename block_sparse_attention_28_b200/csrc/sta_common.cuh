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
};

__device__ unsigned int g_dev_error;

__device__ __forceinline__ void record_error(unsigned int bit) { atomicOr(&g_dev_error, bit); }

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
