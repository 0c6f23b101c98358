// Pooled block scores on the tensor cores (Rectified SpaAttn: block
// importance from pooled queries and keys). Per head, the scores are one
// dense fp32 contraction over d, S = scale * qbar kbar^T [Nt x Nt]; here it
// runs as tcgen05 kind::tf32 MMAs on split operands. Each pooled value x
// (an fp32 mean) is stored as two tf32 parts, hi = tf32(x) and
// lo = tf32(x - hi), so x = hi + lo + r with |r| <= 2^-22 |x|, and each term
// q.k is taken as lo_q hi_k + hi_q lo_k + hi_q hi_k (the dropped lo_q lo_k is
// below 2^-22 |q k|). Within each 32-wide chunk of d the two small
// products go into the accumulator before hi_q hi_k. The pooling kernels
// write the parts.
//
// One CTA per (128 key tiles, range of query tiles, b*heads + h); 192 threads:
//   warp 4     TMA producer: first the CTA's key block (hi and lo parts) into
//              the ring's buffers, then, once it has moved to TMEM, blocks of
//              128 query tiles (the B operand), one 32-wide chunk of d (hi and
//              lo, 32 KB) per ring stage
//   warps 0-3  move the key block from shared memory to TMEM (one key tile
//              per thread = TMEM lane), where it is the A operand of every
//              MMA; then the epilogue of each block, in two halves of 64
//              query tiles: TMEM -> registers -> a transposed tile in shared
//              memory -> rows of S written as 512-byte runs of 16-byte stores
//   warp 5     TMEM allocation and the MMA issue (one thread); accumulators
//              double-buffered in TMEM so the epilogue of block j overlaps
//              the MMAs of block j + 1
// With the key block in TMEM an MMA reads only its query rows from shared
// memory, and with N = 128 it runs at the full tensor-core rate (an N = 64
// MMA takes ~46 cycles for the work of 32). Operands in shared memory are
// K-major with the 128-byte swizzle: a chunk of 32 fp32 along d per 128-byte
// row, 8-row groups 1024 B apart. Every pipeline wait gives up after
// wait_limit SM cycles (set by the host); on a timeout the kernel records
// DEV_ERR_TIMEOUT, waits (with a long, fixed limit) for its own MMAs and
// copies in flight, releases TMEM and returns.
#pragma once
#include "sta_tc.cuh"

namespace sta {
namespace score {

constexpr int M = 128;           // key tiles per CTA (TMEM lanes)
constexpr int N = 128;           // query tiles per MMA block (TMEM columns)
constexpr int NH = 64;           // query tiles per epilogue half
constexpr int NUM_THREADS = 192;
constexpr int WARP_TMA = 4, WARP_MMA = 5;
constexpr long long DRAIN_LIMIT = 200000000LL;  // own copies / MMAs, after the pipeline

template <int D>
struct Cfg {
  static constexpr int CH = D / 32;            // 128-byte chunks along d
  static constexpr int A_CHUNK = M * 128;      // bytes of one chunk of the key block
  static constexpr int A_PART = CH * A_CHUNK;  // one split part of the key block
  static constexpr int B_CHUNK = N * 128;      // bytes of one chunk of a query block
  static constexpr int STAGES = 5;             // ring stages of one chunk (hi part, then lo part)
  static constexpr int STAGE_BYTES = 2 * B_CHUNK;
  static constexpr int OFF_T = STAGES * STAGE_BYTES;  // [NH][M] fp32 epilogue tile
  static constexpr int OFF_BAR = OFF_T + NH * M * 4;
  // a_tma, a_moved, a_full, full[STAGES], empty[STAGES], t_full[2], t_empty[2], mma_done
  static constexpr int NBAR = 3 + 2 * STAGES + 4 + 1;
  static constexpr int OFF_MISC = OFF_BAR + 8 * NBAR;  // tmem address, abort flag
  static constexpr int BYTES = OFF_MISC + 16;
  static constexpr int SMEM = BYTES + 1024;    // slack for the 1024-byte alignment
  // TMEM columns: two accumulators of N, then the key block's hi and lo
  // parts (one fp32 / tf32 element per column, lane = key tile)
  static constexpr uint32_t COL_HI = 2 * N, COL_LO = 2 * N + D;
  static constexpr uint32_t TMEM_COLS = 512;
  static_assert(D % 32 == 0, "d must be a multiple of 32");
  static_assert(2 * A_PART <= STAGES * STAGE_BYTES, "key block staging");
  static_assert(SMEM <= 227 * 1024, "shared memory");
  static_assert(2 * N + 2 * D <= 512, "tensor memory");
};

// instruction descriptor, kind::tf32: tf32 x tf32 -> fp32, B K-major
// (D format bit 4, A / B format 2 = TF32 at bits 7-9 / 10-12, N >> 3 at
// bit 17, M >> 4 at bit 24)
constexpr uint32_t IDESC = (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(N >> 3) << 17) |
                           ((uint32_t)(M >> 4) << 24);

// A from tensor memory (lane = row, one tf32 per column), B from shared memory.
__device__ __forceinline__ void mma_tf32_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b, uint32_t accumulate) {
  // A: K = 8 tf32 columns
  if (!tc::tmem_operand_ok(d_tmem, (uint32_t)N) || !tc::tmem_operand_ok(a_tmem, 8u)) return;
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b), "r"(IDESC), "r"(accumulate)
      : "memory");
}

// AND of `v` over the 128 threads of the epilogue warps (named barrier 1),
// so that they all take the same branch around the barriers that follow.
__device__ __forceinline__ bool all_epilogue(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 1, 128, p;\n\tselp.u32 %0, 1, 0, q;\n\t}\n"
      : "=r"(r)
      : "r"((uint32_t)v)
      : "memory");
  return r != 0u;
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap *map, uint64_t *bar, int x, int y,
                                            int z) {
  if (!tc::tma_args_ok(dst, x)) return;
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(tc::smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// tm_khi / tm_klo / tm_qhi / tm_qlo: the split parts of the pooled keys and
// queries as 3D tensors (d, Nt, b*heads) fp32, boxes of 32 x 128 x 1,
// zero-filled past Nt. S: [b*heads][Nt][Nt] fp32, row = query tile. The query
// tiles of this CTA are [blockIdx.y * q_per_part, ... + q_per_part) clipped to
// Nt, q_per_part a multiple of N.
template <int D>
__global__ void __launch_bounds__(NUM_THREADS, 1)
score_tc_kernel(const __grid_constant__ CUtensorMap tm_khi, const __grid_constant__ CUtensorMap tm_klo,
                const __grid_constant__ CUtensorMap tm_qhi, const __grid_constant__ CUtensorMap tm_qlo,
                float *__restrict__ S, int nt, float scale, int q_per_part, long long wait_limit) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = tc::smem_u32(smem);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int k0 = blockIdx.x * M;
  const int q_begin = blockIdx.y * q_per_part;
  const int q_end = min(nt, q_begin + q_per_part);
  const int bh = blockIdx.z;
  const int nblk = q_end > q_begin ? (q_end - q_begin + N - 1) / N : 0;

  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
  uint64_t *a_tma = bars;         // key block landed in shared memory
  uint64_t *a_moved = bars + 1;   // key block read out of shared memory
  uint64_t *a_full = bars + 2;    // key block in TMEM
  uint64_t *full = bars + 3;
  uint64_t *empty = full + C::STAGES;
  uint64_t *t_full = empty + C::STAGES;
  uint64_t *t_empty = t_full + 2;
  uint64_t *mma_done = t_empty + 2;
  uint32_t *misc = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
  volatile uint32_t *abort_flag = misc + 1;

  if (tid == 0) {
    tc::mbar_init(a_tma, 1);
    tc::mbar_init(a_moved, 4);  // one arrival per epilogue warp
    tc::mbar_init(a_full, 4);
    for (int s = 0; s < C::STAGES; ++s) {
      tc::mbar_init(full + s, 1);
      tc::mbar_init(empty + s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(t_full + b, 1);
      tc::mbar_init(t_empty + b, 4);
    }
    tc::mbar_init(mma_done, 1);
    misc[1] = 0u;
    tc::fence_barrier_init();
  }
  if (warp == WARP_MMA) {
    tc::tmem_alloc(misc, C::TMEM_COLS);
    tc::tmem_relinquish();
  }
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = misc[0];
  const int nchunks = nblk * C::CH;  // ring items: (block j, d-chunk c) = item j * CH + c
  int issued = 0;                    // ring items the producer has loaded

  if (warp == WARP_TMA) {
    // ---------------------------------------------------------- producer
    if (lane == 0 && nblk > 0) {
      tc::mbar_expect_tx(a_tma, 2 * C::A_PART);
#pragma unroll
      for (int c = 0; c < C::CH; ++c) {
        tma_load_3d(sbase + c * C::A_CHUNK, &tm_khi, a_tma, 32 * c, k0, bh);
        tma_load_3d(sbase + C::A_PART + c * C::A_CHUNK, &tm_klo, a_tma, 32 * c, k0, bh);
      }
      // the ring reuses the staging area once the key block is in TMEM (the
      // epilogue warps arrive after a timeout too, with the abort flag raised)
      bool ok = tc::mbar_wait(a_moved, 0, abort_flag, wait_limit) && !*abort_flag;
      for (int it = 0; ok && it < nchunks; ++it) {
        const int s = it % C::STAGES, u = it / C::STAGES;
        if (u > 0 && !tc::mbar_wait(empty + s, (u - 1) & 1, abort_flag, wait_limit)) break;
        const int j = it / C::CH, c = it - j * C::CH;
        const uint32_t dst = sbase + s * C::STAGE_BYTES;
        const int q0 = q_begin + j * N;
        tc::mbar_expect_tx(full + s, C::STAGE_BYTES);
        tma_load_3d(dst, &tm_qhi, full + s, 32 * c, q0, bh);
        tma_load_3d(dst + C::B_CHUNK, &tm_qlo, full + s, 32 * c, q0, bh);
        issued = it + 1;
      }
    }
    __syncwarp();
  } else if (warp == WARP_MMA) {
    // ---------------------------------------------------------- MMA issue
    if (lane == 0 && nblk > 0) {
      bool ok = tc::mbar_wait(a_full, 0, abort_flag, wait_limit);
      tc::fence_after();
      for (int j = 0; ok && j < nblk; ++j) {
        const int buf = j & 1;
        if (j >= 2 && !tc::mbar_wait(t_empty + buf, ((j >> 1) - 1) & 1, abort_flag, wait_limit)) break;
        const uint32_t d_tmem = tmem + (uint32_t)(buf * N);
        for (int c = 0; ok && c < C::CH; ++c) {
          const int it = j * C::CH + c, s = it % C::STAGES;
          if (!tc::mbar_wait(full + s, (it / C::STAGES) & 1, abort_flag, wait_limit)) {
            ok = false;
            break;
          }
          tc::fence_after();
          const uint32_t b_hi = sbase + s * C::STAGE_BYTES, b_lo = b_hi + C::B_CHUNK;
          // lo_k*hi_q, hi_k*lo_q, then hi_k*hi_q over this chunk's four
          // K = 8 steps: 8 TMEM columns of A, 32 bytes of a swizzled B row
#pragma unroll
          for (int part = 0; part < 3; ++part) {
            const uint32_t a = tmem + (part == 0 ? C::COL_LO : C::COL_HI) + (uint32_t)(32 * c);
            const uint32_t b = part == 1 ? b_lo : b_hi;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_tf32_ts(d_tmem, a + (uint32_t)(kk * 8), tc::desc_k_sw128(b + (uint32_t)(kk * 32)),
                          (c > 0 || part > 0 || kk > 0) ? 1u : 0u);
          }
          tc::mma_commit(empty + s);
        }
        if (!ok) break;
        tc::mma_commit(t_full + buf);
      }
      // every issued MMA retires before TMEM is released (a wait on the
      // CTA's own work: the long limit whatever the pipeline limit)
      tc::mma_commit(mma_done);
      tc::mbar_wait(mma_done, 0, nullptr, DRAIN_LIMIT);
    }
    __syncwarp();
  } else {
    // ------------------------------------------- key block into TMEM, epilogue
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    bool ok = nblk > 0;
    if (ok) {
      // row tid of each swizzled chunk: 16-byte granule g sits at g ^ (tid % 8)
      ok = tc::mbar_wait(a_tma, 0, abort_flag, wait_limit);
      if (ok) {
#pragma unroll 1
        for (int part = 0; part < 2; ++part) {
#pragma unroll
          for (int c = 0; c < C::CH; ++c) {
            const uint8_t *row = smem + part * C::A_PART + c * C::A_CHUNK + tid * 128;
            uint32_t r[32];
#pragma unroll
            for (int g = 0; g < 8; ++g) {
              const uint4 v = *reinterpret_cast<const uint4 *>(row + ((g ^ (tid & 7)) << 4));
              r[4 * g] = v.x;
              r[4 * g + 1] = v.y;
              r[4 * g + 2] = v.z;
              r[4 * g + 3] = v.w;
            }
            tc::tmem_st32(tmem + lane_base + (part == 0 ? C::COL_HI : C::COL_LO) + (uint32_t)(32 * c), r);
          }
        }
        tc::tmem_wait_st();
      }
      tc::fence_before();
      __syncwarp();
      if (lane == 0) {
        tc::mbar_arrive(a_moved);
        tc::mbar_arrive(a_full);
      }
    }
    float *T = reinterpret_cast<float *>(smem + C::OFF_T);
    const bool vec = (nt & 3) == 0;  // every row segment of S is 16-byte aligned
    const int kk = k0 + 4 * lane;
    // the four warps leave the loop together (they share barrier 1)
    ok = all_epilogue(ok);
    for (int j = 0; ok && j < nblk; ++j) {
      const int buf = j & 1;
      if (!all_epilogue(tc::mbar_wait(t_full + buf, (j >> 1) & 1, abort_flag, wait_limit))) break;
      tc::fence_after();
#pragma unroll 1
      for (int half = 0; half < 2; ++half) {
        uint32_t v[NH];
        tc::tmem_ld64(tmem + lane_base + (uint32_t)(buf * N + half * NH), v);
        if (half == 1) {
          tc::fence_before();
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(t_empty + buf);
        }
        // transposed tile T[query][key] (consecutive threads, consecutive keys)
#pragma unroll
        for (int c = 0; c < NH; ++c) T[c * M + tid] = __uint_as_float(v[c]) * scale;
        asm volatile("bar.sync 1, 128;" ::: "memory");
        // each warp writes query rows warp, warp + 4, ...: 128 keys per row,
        // four per lane
        const int q0 = q_begin + j * N + half * NH;
        for (int c = warp; c < NH && q0 + c < q_end; c += 4) {
          const float4 val = reinterpret_cast<const float4 *>(T + c * M)[lane];
          float *dst = S + ((long long)bh * nt + q0 + c) * nt + kk;
          if (!dbg_ok(q0 + c < nt && kk >= 0)) continue;
          if (vec && kk + 3 < nt) {
            *reinterpret_cast<float4 *>(dst) = val;
          } else {
            if (kk < nt) dst[0] = val.x;
            if (kk + 1 < nt) dst[1] = val.y;
            if (kk + 2 < nt) dst[2] = val.z;
            if (kk + 3 < nt) dst[3] = val.w;
          }
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");
      }
    }
  }
  // Every role has left its loop, so a timeout in any of them has raised the
  // abort flag by now; the producer's copies still in flight (the key block,
  // the last use of every ring stage) must land before shared memory is
  // released.
  __syncthreads();
  if (warp == WARP_TMA && lane == 0 && nblk > 0 && *abort_flag) {
    tc::mbar_wait(a_tma, 0, nullptr, DRAIN_LIMIT);
    for (int it = (issued > C::STAGES ? issued - C::STAGES : 0); it < issued; ++it)
      tc::mbar_wait(full + it % C::STAGES, (it / C::STAGES) & 1, nullptr, DRAIN_LIMIT);
  }
  tc::fence_before();
  __syncthreads();
  if (warp == WARP_MMA) {
    tc::fence_after();
    tc::tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace score
}  // namespace sta
