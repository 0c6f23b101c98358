// Tile means of Q and K read straight from the raster layout through TMA:
// the pooling of the mask build's raster form (Rectified SpaAttn abstract,
// pooled queries and keys; tiles of 1 x 8 x 8 tokens).
//
// Persistent CTAs, one per SM, each walking the units u = blockIdx.x +
// i * gridDim.x. A unit is one token tile of one tensor (Q or K) for HB
// consecutive heads: a 5D TMA box (d, head, x, y, frame) of D x HB x 8 x 8 x 1
// bf16 = 64 KB, zero-filled past the grid edge and past the last head.
//   warp 16     TMA producer: boxes into a ring of STAGES buffers
//   warps 0-15  each thread sums two adjacent (head, d) columns of the box
//               over half of the 64 token rows in fp64; the two halves meet
//               in shared memory (exact for bf16 inputs whose magnitudes in a
//               tile span less than 2^39, so the split does not change the
//               result); the sum is divided by the number of real tokens and
//               rounded once to fp32; with qlo / klo given the mean x is stored
//               split for the tensor-core scores, tf32(x) in qbar / kbar and
//               tf32(x - tf32(x)) in qlo / klo
// The ring keeps up to 192 KB of loads in flight per SM without a thread per
// outstanding load.
// Every pipeline wait gives up after wait_limit SM cycles (set by the host);
// on a timeout the kernel records DEV_ERR_TIMEOUT, waits (with a long, fixed
// limit) for its own copies in flight and returns.
#pragma once
#include "sta_mask.cuh"
#include "sta_tc.cuh"

namespace sta {
namespace pool {

constexpr int CONSUMERS = 512;                 // 16 warps: two columns x half the rows per thread
constexpr int NUM_THREADS = CONSUMERS + 32;    // + the producer warp
constexpr int WARP_TMA = CONSUMERS / 32;
constexpr int STAGES = 3;
constexpr long long DRAIN_LIMIT = 200000000LL;  // own copies, after the pipeline

template <int D>
struct Cfg {
  static constexpr int HB = 512 / D;                // heads per box: HB * D = 2 * CONSUMERS columns
  static constexpr int COLS = HB * D;
  static constexpr int BOX_BYTES = 64 * COLS * 2;   // 8 x 8 tokens x HB heads x D bf16
  static constexpr int OFF_PART = STAGES * BOX_BYTES;  // [2][COLS] fp64 partial sums of the upper half
  static constexpr int OFF_BAR = OFF_PART + 2 * COLS * 8;
  static constexpr int SMEM = OFF_BAR + 16 * STAGES + 16 + 1024;  // + alignment slack
  static_assert(COLS == CONSUMERS, "two columns per thread pair");
  static_assert(SMEM <= 227 * 1024, "shared memory");
};

// The consumers of pool_tma_kernel: threads 0 .. CONSUMERS-1.
template <int D>
__device__ __forceinline__ void consume(uint8_t *smem, uint64_t *full, uint64_t *empty,
                                        volatile uint32_t *abort_flag, float *__restrict__ qbar,
                                        float *__restrict__ kbar, float *__restrict__ qlo,
                                        float *__restrict__ klo, const Geo &g, int heads, long long units,
                                        long long wait_limit, int G) {
  using C = Cfg<D>;
  const int tid = threadIdx.x, lane = tid & 31;
  const int pair = tid % (CONSUMERS / 2), half = tid / (CONSUMERS / 2);
  const int col = 2 * pair;  // columns col, col + 1 of the box: head col / D, dims col % D
  const int h_in = col / D, dd = col - h_in * D;
  double *part = reinterpret_cast<double *>(smem + C::OFF_PART);
  long long i = 0;
  for (long long u = blockIdx.x; u < units; u += gridDim.x, ++i) {
    const int s = (int)(i % STAGES);
    const bool got = tc::mbar_wait(full + s, (uint32_t)((i / STAGES) & 1), abort_flag, wait_limit);
    double a0 = 0.0, a1 = 0.0;
    if (got) {
      // box row r = 8 y + x (token of the tile), columns [head][d]; this
      // thread sums rows [32 half, 32 half + 32)
      const __nv_bfloat162 *box = reinterpret_cast<const __nv_bfloat162 *>(smem + s * C::BOX_BYTES) + pair;
#pragma unroll 16
      for (int r = 32 * half; r < 32 * half + 32; ++r) {
        const float2 f = __bfloat1622float2(box[r * (C::COLS / 2)]);
        a0 += (double)f.x;
        a1 += (double)f.y;
      }
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(empty + s);
      if (half == 1) {
        part[(i & 1) * C::COLS + col] = a0;
        part[(i & 1) * C::COLS + col + 1] = a1;
      }
    }
    // the consumers leave the loop together (they share barrier 1), and the
    // barrier also publishes the upper halves' partial sums
    uint32_t all;
    asm volatile("{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.and.pred q, 1, %2, p;\n\t"
                 "selp.u32 %0, 1, 0, q;\n\t}\n"
                 : "=r"(all) : "r"((uint32_t)got), "n"(CONSUMERS) : "memory");
    if (!all) break;
    if (half == 1) continue;
    a0 += part[(i & 1) * C::COLS + col];
    a1 += part[(i & 1) * C::COLS + col + 1];
    long long v = u;
    const int grp = (int)(v % G);
    v /= G;
    const int tensor = (int)(v & 1);
    v >>= 1;
    const int tx = (int)(v % g.NW);
    v /= g.NW;
    const int ty = (int)(v % g.NH);
    const int bt = (int)(v / g.NH);
    const int h = grp * C::HB + h_in;
    // checked build: the row lies in [0, B * heads * Nt) = [0, units / (2G) * heads)
    if (h < heads && dbg_ok((long long)bt * g.NH * g.NW < units / (2 * G))) {
      const int b = bt / g.T, t = bt - b * g.T;
      const double cnt = (double)(valid_extent(g.H, ty) * valid_extent(g.W, tx));
      const long long row = ((long long)b * heads + h) * g.Nt + ((long long)t * g.NH + ty) * g.NW + tx;
      float m0 = (float)(a0 / cnt), m1 = (float)(a1 / cnt);
      float *lo = tensor ? klo : qlo;
      if (lo != nullptr) {
        const float h0 = round_tf32(m0), h1 = round_tf32(m1);
        *reinterpret_cast<float2 *>(lo + row * D + dd) = make_float2(round_tf32(m0 - h0), round_tf32(m1 - h1));
        m0 = h0;
        m1 = h1;
      }
      *reinterpret_cast<float2 *>((tensor ? kbar : qbar) + row * D + dd) = make_float2(m0, m1);
    }
  }
}


// Unit u = ((((b*T + t) * NH + ty) * NW + tx) * 2 + tensor) * G + group,
// G = ceil(heads / HB); consecutive units are neighbouring boxes of memory.
template <int D>
__global__ void __launch_bounds__(NUM_THREADS, 1)
pool_tma_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                float *__restrict__ qbar, float *__restrict__ kbar, float *__restrict__ qlo,
                float *__restrict__ klo, Geo g, int heads, long long units, long long wait_limit) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = tc::smem_u32(smem);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
  uint64_t *empty = full + STAGES;
  volatile uint32_t *abort_flag = reinterpret_cast<volatile uint32_t *>(empty + STAGES);
  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) {
      tc::mbar_init(full + s, 1);
      tc::mbar_init(empty + s, CONSUMERS / 32);  // one arrival per consumer warp
    }
    *abort_flag = 0u;
    tc::fence_barrier_init();
  }
  __syncthreads();
  const int G = (heads + C::HB - 1) / C::HB;

  long long issued = 0;  // boxes the producer has loaded
  if (warp == WARP_TMA) {
    // ---------------------------------------------------------- producer
    if (lane == 0) {
      long long i = 0;
      for (long long u = blockIdx.x; u < units; u += gridDim.x, ++i) {
        const int s = (int)(i % STAGES);
        const long long r = i / STAGES;
        if (r > 0 && !tc::mbar_wait(empty + s, (uint32_t)((r - 1) & 1), abort_flag, wait_limit)) break;
        long long v = u;
        const int grp = (int)(v % G);
        v /= G;
        const int tensor = (int)(v & 1);
        v >>= 1;
        const int tx = (int)(v % g.NW);
        v /= g.NW;
        const int ty = (int)(v % g.NH);
        const int bt = (int)(v / g.NH);
        tc::mbar_expect_tx(full + s, C::BOX_BYTES);
        if (!dbg_ok(grp < G && (long long)bt * g.NH * g.NW < units / (2 * G))) continue;
        tc::tma_load_5d(sbase + s * C::BOX_BYTES, tensor ? &tm_k : &tm_q, full + s, 0, grp * C::HB, tx * 8,
                        ty * 8, bt);
        issued = i + 1;
      }
    }
    __syncwarp();
  } else {
    consume<D>(smem, full, empty, abort_flag, qbar, kbar, qlo, klo, g, heads, units, wait_limit, G);
  }
  // Every thread has left its loop, so a timeout in any of them has raised
  // the abort flag by now; the producer's boxes still in flight (the last use
  // of every ring stage) must land before shared memory is released.
  __syncthreads();
  if (warp == WARP_TMA && lane == 0 && *abort_flag) {
    for (long long j = (issued > STAGES ? issued - STAGES : 0); j < issued; ++j)
      tc::mbar_wait(full + j % STAGES, (uint32_t)((j / STAGES) & 1), nullptr, DRAIN_LIMIT);
  }
}

}  // namespace pool
}  // namespace sta
