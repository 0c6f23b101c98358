// libsta: C ABI entry points (declared in include/sta.h).
// Single translation unit: the kernels live in the included headers.
#include <math.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "sta_attn.cuh"
#include "sta_common.cuh"
#include "sta_host.cuh"
#include "sta_mask.cuh"
#include "sta_pair.cuh"
#include "sta_pool.cuh"
#include "sta_reorder.cuh"
#include "sta_score.cuh"
#include "sta_search.cuh"
#include "sta_select.cuh"

using namespace sta;

namespace {

// SM-cycle limit of every bounded pipeline wait in the kernels launched from
// now on (0: the default of ~1 s); see sta_set_wait_limit.
constexpr long long DEFAULT_WAIT_LIMIT = 2000000000LL;
std::atomic<long long> g_wait_limit{0};

long long wait_limit() {
  const long long v = g_wait_limit.load(std::memory_order_relaxed);
  return v > 0 ? v : DEFAULT_WAIT_LIMIT;
}

bool common_sizes_ok(int32_t B, int32_t heads, int32_t d, sta_grid g, Geo *geo, sta_status *st) {
  if (B <= 0 || heads <= 0 || !make_geo(g, geo)) {
    *st = STA_ERR_INVALID_ARG;
    return false;
  }
  if (d != 64 && d != 128) {
    *st = STA_ERR_UNSUPPORTED;
    return false;
  }
  const long long bh = (long long)B * heads;
  // 2D grids index (b*heads + h) in grid.y; TMA row coordinates and CSR
  // offsets are 32-bit.
  if (bh > 65535 || bh * geo->Lpad >= (1LL << 31) || bh * (long long)geo->Nt * geo->Nt >= (1LL << 31)) {
    *st = STA_ERR_UNSUPPORTED;
    return false;
  }
  return true;
}

// total_min: the fused score/select pass; total: plus the low tf32 parts of
// the pooled Q and K (qlo, klo) and a row buffer [B*heads*Nt, Nt] fp32 for
// the split passes (tensor-core scores, then a select pass with four CTAs
// per SM).
struct MaskWs {
  size_t qbar, kbar, bits, counts, sel, kfloor, pairc, total_min, qlo, klo, prows, total;
};

MaskWs mask_ws_layout(int32_t B, int32_t heads, int32_t d, const Geo &g) {
  const size_t R = (size_t)B * heads * g.Nt;
  const size_t wpr = (size_t)(g.Nt + 31) / 32;
  MaskWs w;
  size_t off = 0;
  w.qbar = off;
  off = align_up(off + R * d * sizeof(float), 256);
  w.kbar = off;
  off = align_up(off + R * d * sizeof(float), 256);
  w.bits = off;
  off = align_up(off + R * wpr * sizeof(uint32_t), 256);
  w.counts = off;
  off = align_up(off + R * sizeof(int32_t), 256);
  w.sel = off;
  off = align_up(off + R * sizeof(int32_t), 256);
  w.kfloor = off;
  off = align_up(off + (size_t)B * heads * sizeof(int32_t), 256);
  w.pairc = off;  // each tile's pairing candidates, in the pairing's order
  off = align_up(off + R * 2 * pairq::NOFF * sizeof(int32_t), 256);
  w.total_min = off;
  w.qlo = off;
  off = align_up(off + R * d * sizeof(float), 256);
  w.klo = off;
  off = align_up(off + R * d * sizeof(float), 256);
  w.prows = off;
  off = align_up(off + R * g.Nt * sizeof(float), 256);
  w.total = off;
  return w;
}

// Dynamic shared memory of score_select_kernel<D, qb, mode>.
size_t select_smem(int d, const Geo &g, bool use_scores, int qb = SEL_QB, int mode = SEL_FUSED) {
  const size_t q = (mode == SEL_FUSED && use_scores) ? (size_t)qb * d : 0;
  const size_t scores = use_scores ? (size_t)(qb * g.Nt + (SEL_THREADS / 32) * 256 * 2) : 0;  // u64 histograms
  // window tables (group of each |dt|, the head's extents) and one row of
  // window bits per warp
  const size_t tables = (size_t)((g.T + 3) & ~3) + 4 * STA_MAX_GROUPS + (SEL_THREADS / 32) * ((g.Nt + 31) / 32);
  return (q + scores + tables) * sizeof(float);
}

constexpr size_t MAX_DYN_SMEM = 227 * 1024;

// Raster [B, L, heads, d] bf16 as the 5D tensor (d, heads, W, H, B*T): a box
// of 64 d-values x 1 head x 8 columns x 8 rows x 1 frame is one token tile
// (zero-filled beyond the grid edge), 128 B swizzle.
bool make_raster_map(CUtensorMap *map, const void *base, const Geo &g, int B, int heads, int d) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t row = (cuuint64_t)heads * d * 2;  // bytes per token
  cuuint64_t dims[5] = {(cuuint64_t)d, (cuuint64_t)heads, (cuuint64_t)g.W, (cuuint64_t)g.H,
                        (cuuint64_t)B * g.T};
  cuuint64_t strides[4] = {(cuuint64_t)d * 2, row, row * g.W, row * g.W * g.H};
  cuuint32_t box[5] = {64, 1, 8, 8, 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void *>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Raster [B, L, heads, d] bf16 as the 5D tensor (d, heads, W, H, B*T) with a
// box of a whole token tile for `hb` heads: d x hb x 8 x 8 x 1 (zero-filled
// beyond the grid edge and the last head), no swizzle.
bool make_raster_pool_map(CUtensorMap *map, const void *base, const Geo &g, int B, int heads, int d, int hb) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t row = (cuuint64_t)heads * d * 2;  // bytes per token
  cuuint64_t dims[5] = {(cuuint64_t)d, (cuuint64_t)heads, (cuuint64_t)g.W, (cuuint64_t)g.H,
                        (cuuint64_t)B * g.T};
  cuuint64_t strides[4] = {(cuuint64_t)d * 2, row, row * g.W, row * g.W * g.H};
  cuuint32_t box[5] = {(cuuint32_t)d, (cuuint32_t)hb, 8, 8, 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void *>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Pooled rows [bh, Nt, d] fp32 as a 3D tensor (d, Nt, bh); a box is 32 d-values
// (128 B) x `rows` tiles x 1 head, zero-filled past Nt, 128 B swizzle.
bool make_pooled_map(CUtensorMap *map, const float *base, long long bh, int nt, int d, int rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)nt, (cuuint64_t)bh};
  cuuint64_t strides[2] = {(cuuint64_t)d * 4, (cuuint64_t)nt * d * 4};
  cuuint32_t box[3] = {32, (cuuint32_t)rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float *>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Tensor-core scores S = scale * qbar kbar^T of every head into rows
// [bh*Nt + qt][kt] of S, from the split pooled parts.
template <int D>
sta_status launch_scores_tc(const float *qhi, const float *qlo, const float *khi, const float *klo, float *S,
                            long long bh, const Geo &g, float scale, cudaStream_t s) {
  CUtensorMap m_khi, m_klo, m_qhi, m_qlo;
  if (!make_pooled_map(&m_khi, khi, bh, g.Nt, D, score::M) || !make_pooled_map(&m_klo, klo, bh, g.Nt, D, score::M) ||
      !make_pooled_map(&m_qhi, qhi, bh, g.Nt, D, score::N) || !make_pooled_map(&m_qlo, qlo, bh, g.Nt, D, score::N))
    return STA_ERR_CUDA;
  auto kern = score::score_tc_kernel<D>;
  const int smem = score::Cfg<D>::SMEM;
  STA_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
  // key blocks x query ranges x heads, with at least two waves of CTAs
  // where the query range can be split
  const int kblocks = (g.Nt + score::M - 1) / score::M;
  const int qblocks = (g.Nt + score::N - 1) / score::N;
  const long long base = (long long)kblocks * bh;
  int parts = (int)((2LL * 148 + base - 1) / base);
  parts = parts < 1 ? 1 : (parts > qblocks ? qblocks : parts);
  const int per_part = (qblocks + parts - 1) / parts;
  parts = (qblocks + per_part - 1) / per_part;  // no empty range
  dim3 grid((unsigned)kblocks, (unsigned)parts, (unsigned)bh);
  kern<<<grid, score::NUM_THREADS, smem, s>>>(m_khi, m_klo, m_qhi, m_qlo, S, g.Nt, scale, per_part * score::N,
                                              wait_limit());
  STA_CUDA_TRY(cudaGetLastError());
  return STA_OK;
}

// One thread waits, with the pipeline's bounded wait, on a barrier that
// expects one arrival that never comes.
__global__ void selftest_wait_kernel(long long limit) {
  __shared__ uint64_t bar;
  __shared__ uint32_t abort_flag;
  if (threadIdx.x == 0) {
    tc::mbar_init(&bar, 1);
    abort_flag = 0u;
    tc::fence_barrier_init();
    tc::mbar_wait(&bar, 0, &abort_flag, limit);
  }
}

// The select pass with the row in registers (sel::select_rows_kernel<NPL>,
// NPL = ceil(Nt / 32) rounded up to a multiple of 8), on rows of scores to be
// softmaxed (P) or window-only rows (P unused). With the per-head floor
// (kfloor != nullptr) it runs twice around head_floor_kernel: first for the
// base counts only (sel_count), then with k_min raised to the floor.
template <int NPL>
sta_status launch_select_regs_npl(const float *P, int logits, float *probs, int B, int heads, const Geo &g,
                                  const sta_mask_params *p, bool use_scores, const int *windows, int G,
                                  const GroupLo &glo, unsigned int *bits, int *counts, int wpr, int *kfloor,
                                  int *sel, cudaStream_t s) {
  auto kern = sel::select_rows_kernel<NPL>;
  const size_t smem = sel::smem_bytes(NPL, wpr, g.T);
  if (smem > MAX_DYN_SMEM) return STA_ERR_UNSUPPORTED;
  STA_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  dim3 grid((unsigned)((g.Nt + sel::WARPS - 1) / sel::WARPS), (unsigned)(B * heads));
  if (kfloor != nullptr) {
    kern<<<grid, sel::THREADS, smem, s>>>(P, nullptr, heads, g, p->top_p, p->k_min, 1, nullptr, 0, glo, bits, counts,
                                          wpr, nullptr, sel);
    STA_CUDA_TRY(cudaGetLastError());
    head_floor_kernel<<<(unsigned)(B * heads), FLOOR_THREADS, 0, s>>>(sel, kfloor, g);
    STA_CUDA_TRY(cudaGetLastError());
  }
  kern<<<grid, sel::THREADS, smem, s>>>(P, probs, heads, g, p->top_p, p->k_min, use_scores ? 1 : 0, windows, G, glo,
                                        bits, counts, wpr, kfloor, nullptr);
  STA_CUDA_TRY(cudaGetLastError());
  return STA_OK;
}

sta_status launch_select_regs(const float *P, int logits, float *probs, int B, int heads, const Geo &g,
                              const sta_mask_params *p, bool use_scores, const int *windows, int G,
                              const GroupLo &glo, unsigned int *bits, int *counts, int wpr, int *kfloor, int *sel,
                              cudaStream_t s) {
  switch ((g.Nt + 255) / 256) {
    case 1: return launch_select_regs_npl<8>(P, logits, probs, B, heads, g, p, use_scores, windows, G, glo, bits, counts, wpr, kfloor, sel, s);
    case 2: return launch_select_regs_npl<16>(P, logits, probs, B, heads, g, p, use_scores, windows, G, glo, bits, counts, wpr, kfloor, sel, s);
    case 3: return launch_select_regs_npl<24>(P, logits, probs, B, heads, g, p, use_scores, windows, G, glo, bits, counts, wpr, kfloor, sel, s);
    case 4: return launch_select_regs_npl<32>(P, logits, probs, B, heads, g, p, use_scores, windows, G, glo, bits, counts, wpr, kfloor, sel, s);
    case 5: return launch_select_regs_npl<40>(P, logits, probs, B, heads, g, p, use_scores, windows, G, glo, bits, counts, wpr, kfloor, sel, s);
    case 6: return launch_select_regs_npl<48>(P, logits, probs, B, heads, g, p, use_scores, windows, G, glo, bits, counts, wpr, kfloor, sel, s);
    case 7: return launch_select_regs_npl<56>(P, logits, probs, B, heads, g, p, use_scores, windows, G, glo, bits, counts, wpr, kfloor, sel, s);
    case 8: return launch_select_regs_npl<64>(P, logits, probs, B, heads, g, p, use_scores, windows, G, glo, bits, counts, wpr, kfloor, sel, s);
  }
  return STA_ERR_UNSUPPORTED;
}

// ws_bytes decides the layout. With the full workspace the scores run on
// the tensor cores into a row buffer (the caller's block_probs when given)
// and a separate, smaller select pass does the softmax and the selection;
// with the minimum workspace one fused pass computes the scores with fp32
// FMA chains. Each layout is deterministic; both are within their stated
// error bounds of the exact scores.
template <int D>
sta_status launch_build(const void *q_tiled, const void *k_tiled, int32_t B, int32_t heads,
                        const Geo &g, const sta_mask_params *p, int32_t *row_ptr, int32_t *col_idx,
                        int64_t *nnz_dev, uint8_t *block_mask, float *block_probs, uint8_t *ws,
                        size_t ws_bytes, cudaStream_t s, bool raster = false) {
  const MaskWs L = mask_ws_layout(B, heads, D, g);
  float *qbar = reinterpret_cast<float *>(ws + L.qbar);
  float *kbar = reinterpret_cast<float *>(ws + L.kbar);
  unsigned int *bits = reinterpret_cast<unsigned int *>(ws + L.bits);
  int *counts = reinterpret_cast<int *>(ws + L.counts);
  const long long R = (long long)B * heads * g.Nt;
  const int wpr = (g.Nt + 31) / 32;
  const bool use_scores = p->use_scores != 0;
  const float scale = p->sm_scale != 0.0f ? p->sm_scale : 1.0f / sqrtf((float)D);
  const bool full_ws = ws_bytes >= L.total;

  const float *P_in = use_scores ? p->block_scores : nullptr;
  const bool tc_scores = use_scores && P_in == nullptr && full_ws;
  float *qlo = tc_scores ? reinterpret_cast<float *>(ws + L.qlo) : nullptr;
  float *klo = tc_scores ? reinterpret_cast<float *>(ws + L.klo) : nullptr;
  if (use_scores && P_in == nullptr) {
    if (raster) {
      // persistent TMA pooling: one CTA per SM over (tile, tensor, head group) boxes
      using PC = pool::Cfg<D>;
      CUtensorMap m_q, m_k;
      if (!make_raster_pool_map(&m_q, q_tiled, g, B, heads, D, PC::HB) ||
          !make_raster_pool_map(&m_k, k_tiled, g, B, heads, D, PC::HB))
        return STA_ERR_CUDA;
      auto kern = pool::pool_tma_kernel<D>;
      STA_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, PC::SMEM));
      const long long units = 2LL * B * g.T * g.NH * g.NW * ((heads + PC::HB - 1) / PC::HB);
      const long long ctas = units < sm_count() ? units : sm_count();
      kern<<<(unsigned)ctas, pool::NUM_THREADS, PC::SMEM, s>>>(m_q, m_k, qbar, kbar, qlo, klo, g, heads, units,
                                                               wait_limit());
    } else {
      const long long warps = 2 * R;
      const unsigned blocks = (unsigned)((warps * 32 + 255) / 256);
      pool_kernel<D><<<blocks, 256, 0, s>>>(static_cast<const uint4 *>(q_tiled), static_cast<const uint4 *>(k_tiled),
                                            qbar, kbar, qlo, klo, R, g);
    }
    STA_CUDA_TRY(cudaGetLastError());
  }
  GroupLo glo;
  for (int i = 0; i < STA_MAX_GROUPS; ++i) glo.v[i] = (i < p->num_groups) ? p->group_lo[i] : 0x7fffffff;
  const bool floor = use_scores && p->head_topk_floor != 0;
  int *sel = reinterpret_cast<int *>(ws + L.sel);
  int *kfloor = reinterpret_cast<int *>(ws + L.kfloor);
  const int *windows = p->windows;
  const int G = p->windows ? p->num_groups : 0;
  const bool split = !use_scores || P_in != nullptr || full_ws;
  if (!split) {
    // fused: scores, softmax, selection and windows per 16-row CTA
    const size_t smem = select_smem(D, g, use_scores, SEL_QB, SEL_FUSED);
    auto kern = score_select_kernel<D, SEL_QB, SEL_FUSED>;
    if (smem > 48 * 1024)
      STA_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    dim3 grid((unsigned)((g.Nt + SEL_QB - 1) / SEL_QB), (unsigned)(B * heads));
    if (floor) {
      // pass 1: base selection counts; per-head floor; pass 2 re-selects with
      // k_min raised to the floor
      kern<<<grid, SEL_THREADS, smem, s>>>(qbar, kbar, heads, g, scale, p->top_p, p->k_min, 1, nullptr, 0, glo,
                                           bits, counts, nullptr, wpr, nullptr, sel, nullptr, 0);
      STA_CUDA_TRY(cudaGetLastError());
      head_floor_kernel<<<(unsigned)(B * heads), FLOOR_THREADS, 0, s>>>(sel, kfloor, g);
      STA_CUDA_TRY(cudaGetLastError());
    }
    kern<<<grid, SEL_THREADS, smem, s>>>(qbar, kbar, heads, g, scale, p->top_p, p->k_min, 1, windows, G, glo,
                                         bits, counts, block_probs, wpr, floor ? kfloor : nullptr, nullptr,
                                         nullptr, 0);
    STA_CUDA_TRY(cudaGetLastError());
  } else {
    const float *P_sel = P_in;  // rows the select pass reads
    int logits = 0;             // whether they are scores still to be softmaxed
    if (tc_scores) {
      // scores into the caller's block_probs when given (the select pass
      // overwrites them with P), else into the workspace's row buffer
      float *rows = block_probs != nullptr ? block_probs : reinterpret_cast<float *>(ws + L.prows);
      const sta_status st = launch_scores_tc<D>(qbar, qlo, kbar, klo, rows, (long long)B * heads, g, scale, s);
      if (st != STA_OK) return st;
      P_sel = rows;
      logits = 1;
    }
    // Rows of up to 2048 key tiles held in registers (scores to softmax, or
    // window-only rows); caller-given block scores, whose rows need not sum
    // to one, and longer rows take the general select pass (64-bit sums).
    const bool in_regs = g.Nt <= 32 * sel::MAX_NPL && (!use_scores || logits);
    if (in_regs) {
      const sta_status st = launch_select_regs(P_sel, logits, block_probs, B, heads, g, p, use_scores, windows, G,
                                               glo, bits, counts, wpr, floor ? kfloor : nullptr, floor ? sel : nullptr,
                                               s);
      if (st != STA_OK) return st;
    } else {
      const size_t smem = select_smem(D, g, use_scores, SEL_QB_SELECT, SEL_SELECT);
      auto kern = score_select_kernel<D, SEL_QB_SELECT, SEL_SELECT>;
      if (smem > 48 * 1024)
        STA_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
      dim3 grid((unsigned)((g.Nt + SEL_QB_SELECT - 1) / SEL_QB_SELECT), (unsigned)(B * heads));
      if (floor) {
        kern<<<grid, SEL_THREADS, smem, s>>>(qbar, kbar, heads, g, scale, p->top_p, p->k_min, 1, nullptr, 0, glo,
                                             bits, counts, nullptr, wpr, nullptr, sel, P_sel, logits);
        STA_CUDA_TRY(cudaGetLastError());
        head_floor_kernel<<<(unsigned)(B * heads), FLOOR_THREADS, 0, s>>>(sel, kfloor, g);
        STA_CUDA_TRY(cudaGetLastError());
      }
      kern<<<grid, SEL_THREADS, smem, s>>>(qbar, kbar, heads, g, scale, p->top_p, p->k_min, use_scores ? 1 : 0,
                                           windows, G, glo, bits, counts, block_probs, wpr,
                                           floor ? kfloor : nullptr, nullptr, P_sel, logits);
      STA_CUDA_TRY(cudaGetLastError());
    }
  }
  scan_kernel<<<1, SCAN_THREADS, 0, s>>>(counts, row_ptr, reinterpret_cast<long long *>(nnz_dev), R);
  STA_CUDA_TRY(cudaGetLastError());
  const unsigned fblocks = (unsigned)((R * 32 + 255) / 256);
  fill_kernel<<<fblocks, 256, 0, s>>>(bits, row_ptr, col_idx, block_mask, R, g.Nt, wpr);
  STA_CUDA_TRY(cudaGetLastError());
  if (p->query_pairs != nullptr) {
    // query-tile pairing by list overlap, from the final row bitsets
    int *pc = reinterpret_cast<int *>(ws + L.pairc);
    pairq::pair_candidates_kernel<<<(unsigned)((R * 32 + 255) / 256), 256, 0, s>>>(bits, pc, R, g, wpr);
    STA_CUDA_TRY(cudaGetLastError());
    const size_t psmem = 2 * (size_t)g.Nt * sizeof(int) + (size_t)g.Nt;
    if (psmem > 48 * 1024)
      STA_CUDA_TRY(cudaFuncSetAttribute(pairq::pair_match_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)psmem));
    pairq::pair_match_kernel<<<(unsigned)(B * heads), pairq::MATCH_THREADS, psmem, s>>>(bits, counts, pc,
                                                                                       p->query_pairs, g, wpr);
    STA_CUDA_TRY(cudaGetLastError());
  }
  if (block_probs != nullptr && !use_scores)
    STA_CUDA_TRY(cudaMemsetAsync(block_probs, 0, (size_t)R * g.Nt * sizeof(float), s));
  return STA_OK;
}

// Pooled key rows per head of the rectified form: Nt rounded up to 64.
inline int pooled_rows(const Geo &g) { return (g.Nt + 63) / 64 * 64; }

template <int D, bool MASS, bool RASTER = false, bool RECT = false>
sta_status launch_attn(const void *q, const void *k, const void *v, void *o, float *lse,
                       const int32_t *row_ptr, const int32_t *col_idx, int32_t B, int32_t heads,
                       const Geo &g, float sm_scale, cudaStream_t s, const float *lse_in = nullptr,
                       float *block_mass = nullptr, const void *kbar = nullptr, const void *vbar = nullptr,
                       const int32_t *query_pairs = nullptr) {
  const unsigned long long rows = (unsigned long long)B * heads * g.Lpad;
  const int ntp = RECT ? pooled_rows(g) : 0;
  CUtensorMap tq, tk, tv, tkb, tvb;
  if (RASTER) {
    if (!make_raster_map(&tq, q, g, B, heads, D) || !make_raster_map(&tk, k, g, B, heads, D) ||
        !make_raster_map(&tv, v, g, B, heads, D))
      return STA_ERR_CUDA;
  } else if (!make_tile_map(&tq, q, rows, D) || !make_tile_map(&tk, k, rows, D) ||
             !make_tile_map(&tv, v, rows, D)) {
    return STA_ERR_CUDA;
  }
  if (RECT) {
    const unsigned long long prow = (unsigned long long)B * heads * ntp;
    if (!make_tile_map(&tkb, kbar, prow, D) || !make_tile_map(&tvb, vbar, prow, D)) return STA_ERR_CUDA;
  } else {
    tkb = tk;  // unused
    tvb = tv;
  }
  const size_t smem = attn::smem_bytes<D>(g.Nt, ntp);
  if (smem > MAX_DYN_SMEM) return STA_ERR_UNSUPPORTED;
  STA_CUDA_TRY(cudaFuncSetAttribute(attn::attn_fwd_kernel<D, MASS, RASTER, RECT>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  if (MASS)
    STA_CUDA_TRY(cudaMemsetAsync(block_mass, 0, (size_t)B * heads * g.Nt * g.Nt * sizeof(float), s));
  const float scale = sm_scale != 0.0f ? sm_scale : 1.0f / sqrtf((float)D);
  const float scale_log2 = scale * 1.4426950408889634f;
  dim3 grid((unsigned)((g.Nt + 1) / 2), (unsigned)(B * heads));
  attn::attn_fwd_kernel<D, MASS, RASTER, RECT><<<grid, attn::NUM_THREADS, smem, s>>>(
      tq, tk, tv, static_cast<__nv_bfloat16 *>(o), lse, row_ptr, col_idx, g, scale_log2, lse_in,
      block_mass, heads, tkb, tvb, ntp, wait_limit(), query_pairs);
  STA_CUDA_TRY(cudaGetLastError());
  return STA_OK;
}

}  // namespace

extern "C" {

int64_t sta_num_tiles(sta_grid g) {
  Geo geo;
  return make_geo(g, &geo) ? (int64_t)geo.Nt : -1;
}

int64_t sta_tiled_len(sta_grid g) {
  Geo geo;
  return make_geo(g, &geo) ? (int64_t)geo.Lpad : -1;
}

sta_status sta_reorder(const void *src, void *dst, int32_t B, int32_t heads, int32_t d, sta_grid g,
                       int32_t inverse, sta_stream_t stream) {
  Geo geo;
  sta_status st = STA_OK;
  if (!common_sizes_ok(B, heads, d, g, &geo, &st)) return st;
  if (src == nullptr || dst == nullptr || !aligned16(src) || !aligned16(dst) || src == dst)
    return STA_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const cudaError_t e = (d == 128) ? launch_reorder<128>(src, dst, B, heads, geo, inverse != 0, s)
                                   : launch_reorder<64>(src, dst, B, heads, geo, inverse != 0, s);
  return e == cudaSuccess ? STA_OK : STA_ERR_CUDA;
}

size_t sta_build_mask_workspace(int32_t B, int32_t heads, int32_t d, sta_grid g) {
  Geo geo;
  sta_status st;
  if (!common_sizes_ok(B, heads, d, g, &geo, &st)) return 0;
  return mask_ws_layout(B, heads, d, geo).total;
}

size_t sta_build_mask_workspace_min(int32_t B, int32_t heads, int32_t d, sta_grid g) {
  Geo geo;
  sta_status st = STA_OK;
  if (!common_sizes_ok(B, heads, d, g, &geo, &st)) return 0;
  return mask_ws_layout(B, heads, d, geo).total_min;
}

sta_status sta_build_mask_pooled_offsets(int32_t B, int32_t heads, int32_t d, sta_grid g, size_t ws_bytes,
                                         size_t offsets[4]) {
  Geo geo;
  sta_status st = STA_OK;
  if (offsets == nullptr) return STA_ERR_INVALID_ARG;
  if (!common_sizes_ok(B, heads, d, g, &geo, &st)) return st;
  const MaskWs L = mask_ws_layout(B, heads, d, geo);
  const bool split = ws_bytes >= L.total;
  offsets[0] = L.qbar;
  offsets[1] = L.kbar;
  offsets[2] = split ? L.qlo : 0;
  offsets[3] = split ? L.klo : 0;
  return STA_OK;
}

static sta_status build_mask_any(const void *q_tiled, const void *k_tiled, int32_t B, int32_t heads,
                                 int32_t d, sta_grid g, const sta_mask_params *p, int32_t *row_ptr,
                                 int32_t *col_idx, int64_t *nnz_dev, uint8_t *block_mask,
                                 float *block_probs, void *workspace, size_t ws_bytes,
                                 sta_stream_t stream, bool raster) {
  Geo geo;
  sta_status st = STA_OK;
  if (!common_sizes_ok(B, heads, d, g, &geo, &st)) return st;
  if (p == nullptr || row_ptr == nullptr || col_idx == nullptr || nnz_dev == nullptr)
    return STA_ERR_INVALID_ARG;
  if (p->use_scores && p->block_scores == nullptr &&
      (q_tiled == nullptr || k_tiled == nullptr || !aligned16(q_tiled) || !aligned16(k_tiled)))
    return STA_ERR_INVALID_ARG;
  if (p->windows != nullptr) {
    if (p->num_groups < 1 || p->num_groups > STA_MAX_GROUPS || p->group_lo[0] != 0) return STA_ERR_INVALID_ARG;
    for (int i = 1; i < p->num_groups; ++i)
      if (p->group_lo[i] <= p->group_lo[i - 1]) return STA_ERR_INVALID_ARG;
  }
  if (p->k_min < 0 || !(p->top_p == p->top_p)) return STA_ERR_INVALID_ARG;
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 ||
      ws_bytes < mask_ws_layout(B, heads, d, geo).total_min)
    return STA_ERR_WORKSPACE;
  if (select_smem(d, geo, p->use_scores != 0) > MAX_DYN_SMEM) return STA_ERR_UNSUPPORTED;
  if (p->query_pairs != nullptr) {
    if ((reinterpret_cast<uintptr_t>(p->query_pairs) & 3u) != 0) return STA_ERR_INVALID_ARG;
    // the pairing keeps two int32 and a byte per tile of a head in shared memory
    if (2 * (size_t)geo.Nt * sizeof(int) + (size_t)geo.Nt > MAX_DYN_SMEM) return STA_ERR_UNSUPPORTED;
  }
  // window tables pack (t, tile row, tile column) into 12 + 10 + 10 bits
  if (p->windows != nullptr && (geo.T >= 4096 || geo.NH >= 1024 || geo.NW >= 1024)) return STA_ERR_UNSUPPORTED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  return (d == 128) ? launch_build<128>(q_tiled, k_tiled, B, heads, geo, p, row_ptr, col_idx, nnz_dev,
                                        block_mask, block_probs, ws, ws_bytes, s, raster)
                    : launch_build<64>(q_tiled, k_tiled, B, heads, geo, p, row_ptr, col_idx, nnz_dev,
                                       block_mask, block_probs, ws, ws_bytes, s, raster);
}

sta_status sta_build_mask(const void *q_tiled, const void *k_tiled, int32_t B, int32_t heads, int32_t d,
                          sta_grid g, const sta_mask_params *p, int32_t *row_ptr, int32_t *col_idx,
                          int64_t *nnz_dev, uint8_t *block_mask, float *block_probs, void *workspace,
                          size_t ws_bytes, sta_stream_t stream) {
  return build_mask_any(q_tiled, k_tiled, B, heads, d, g, p, row_ptr, col_idx, nnz_dev, block_mask,
                        block_probs, workspace, ws_bytes, stream, false);
}

sta_status sta_build_mask_raster(const void *q, const void *k, int32_t B, int32_t heads, int32_t d,
                                 sta_grid g, const sta_mask_params *p, int32_t *row_ptr, int32_t *col_idx,
                                 int64_t *nnz_dev, uint8_t *block_mask, float *block_probs,
                                 void *workspace, size_t ws_bytes, sta_stream_t stream) {
  return build_mask_any(q, k, B, heads, d, g, p, row_ptr, col_idx, nnz_dev, block_mask, block_probs,
                        workspace, ws_bytes, stream, true);
}

static sta_status attn_fwd_any(const void *q, const void *k, const void *v, void *o, float *lse,
                               const int32_t *row_ptr, const int32_t *col_idx, int32_t B, int32_t heads,
                               int32_t d, sta_grid g, float sm_scale, sta_stream_t stream, bool raster,
                               const int32_t *query_pairs = nullptr) {
  Geo geo;
  sta_status st = STA_OK;
  if (!common_sizes_ok(B, heads, d, g, &geo, &st)) return st;
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr || row_ptr == nullptr || col_idx == nullptr)
    return STA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return STA_ERR_INVALID_ARG;
  if (!(sm_scale == sm_scale) || sm_scale < 0.0f) return STA_ERR_INVALID_ARG;
  if (!device_is_sm100()) return STA_ERR_UNSUPPORTED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (raster) {
    // TMA coordinates of the 5D map are 32-bit: B*T frames, W columns, H rows
    if ((long long)B * geo.T >= (1LL << 31)) return STA_ERR_UNSUPPORTED;
    return (d == 128) ? launch_attn<128, false, true>(q, k, v, o, lse, row_ptr, col_idx, B, heads, geo, sm_scale, s,
                                                      nullptr, nullptr, nullptr, nullptr, query_pairs)
                      : launch_attn<64, false, true>(q, k, v, o, lse, row_ptr, col_idx, B, heads, geo, sm_scale, s,
                                                     nullptr, nullptr, nullptr, nullptr, query_pairs);
  }
  return (d == 128) ? launch_attn<128, false>(q, k, v, o, lse, row_ptr, col_idx, B, heads, geo, sm_scale, s, nullptr,
                                              nullptr, nullptr, nullptr, query_pairs)
                    : launch_attn<64, false>(q, k, v, o, lse, row_ptr, col_idx, B, heads, geo, sm_scale, s, nullptr,
                                             nullptr, nullptr, nullptr, query_pairs);
}

sta_status sta_attn_fwd(const void *q, const void *k, const void *v, void *o, float *lse,
                        const int32_t *row_ptr, const int32_t *col_idx, int32_t B, int32_t heads,
                        int32_t d, sta_grid g, float sm_scale, sta_stream_t stream) {
  return attn_fwd_any(q, k, v, o, lse, row_ptr, col_idx, B, heads, d, g, sm_scale, stream, false);
}

sta_status sta_attn_fwd_raster(const void *q, const void *k, const void *v, void *o, float *lse,
                               const int32_t *row_ptr, const int32_t *col_idx, int32_t B, int32_t heads,
                               int32_t d, sta_grid g, float sm_scale, sta_stream_t stream) {
  return attn_fwd_any(q, k, v, o, lse, row_ptr, col_idx, B, heads, d, g, sm_scale, stream, true);
}

sta_status sta_attn_fwd_paired(const void *q, const void *k, const void *v, void *o, float *lse,
                               const int32_t *row_ptr, const int32_t *col_idx, const int32_t *query_pairs,
                               int32_t B, int32_t heads, int32_t d, sta_grid g, float sm_scale,
                               sta_stream_t stream) {
  if (query_pairs == nullptr || (reinterpret_cast<uintptr_t>(query_pairs) & 3u) != 0) return STA_ERR_INVALID_ARG;
  return attn_fwd_any(q, k, v, o, lse, row_ptr, col_idx, B, heads, d, g, sm_scale, stream, false, query_pairs);
}

sta_status sta_attn_fwd_raster_paired(const void *q, const void *k, const void *v, void *o, float *lse,
                                      const int32_t *row_ptr, const int32_t *col_idx,
                                      const int32_t *query_pairs, int32_t B, int32_t heads, int32_t d,
                                      sta_grid g, float sm_scale, sta_stream_t stream) {
  if (query_pairs == nullptr || (reinterpret_cast<uintptr_t>(query_pairs) & 3u) != 0) return STA_ERR_INVALID_ARG;
  return attn_fwd_any(q, k, v, o, lse, row_ptr, col_idx, B, heads, d, g, sm_scale, stream, true, query_pairs);
}

sta_status sta_attn_fwd_block_mass(const void *q, const void *k, const void *v, void *o, float *lse,
                                   const int32_t *row_ptr, const int32_t *col_idx,
                                   const float *lse_cached, float *block_mass, int32_t B,
                                   int32_t heads, int32_t d, sta_grid g, float sm_scale,
                                   sta_stream_t stream) {
  Geo geo;
  sta_status st = STA_OK;
  if (!common_sizes_ok(B, heads, d, g, &geo, &st)) return st;
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr || row_ptr == nullptr ||
      col_idx == nullptr || lse_cached == nullptr || block_mass == nullptr)
    return STA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return STA_ERR_INVALID_ARG;
  if (!(sm_scale == sm_scale) || sm_scale < 0.0f) return STA_ERR_INVALID_ARG;
  if (!device_is_sm100()) return STA_ERR_UNSUPPORTED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  return (d == 128) ? launch_attn<128, true>(q, k, v, o, lse, row_ptr, col_idx, B, heads, geo, sm_scale, s,
                                             lse_cached, block_mass)
                    : launch_attn<64, true>(q, k, v, o, lse, row_ptr, col_idx, B, heads, geo, sm_scale, s,
                                            lse_cached, block_mass);
}

size_t sta_rectified_workspace(int32_t B, int32_t heads, int32_t d, sta_grid g) {
  Geo geo;
  sta_status st = STA_OK;
  if (!common_sizes_ok(B, heads, d, g, &geo, &st)) return 0;
  const size_t one = align_up((size_t)B * heads * pooled_rows(geo) * d * 2, 256);
  return 2 * one;
}

sta_status sta_attn_fwd_rectified(const void *q, const void *k, const void *v, void *o, float *lse,
                                  const int32_t *row_ptr, const int32_t *col_idx, void *workspace,
                                  size_t ws_bytes, int32_t B, int32_t heads, int32_t d, sta_grid g,
                                  float sm_scale, sta_stream_t stream) {
  Geo geo;
  sta_status st = STA_OK;
  if (!common_sizes_ok(B, heads, d, g, &geo, &st)) return st;
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr || row_ptr == nullptr || col_idx == nullptr)
    return STA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return STA_ERR_INVALID_ARG;
  if (!(sm_scale == sm_scale) || sm_scale < 0.0f) return STA_ERR_INVALID_ARG;
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 ||
      ws_bytes < sta_rectified_workspace(B, heads, d, g))
    return STA_ERR_WORKSPACE;
  if (!device_is_sm100()) return STA_ERR_UNSUPPORTED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int ntp = pooled_rows(geo);
  const size_t one = align_up((size_t)B * heads * ntp * d * 2, 256);
  uint8_t *kbar = static_cast<uint8_t *>(workspace);
  uint8_t *vbar = kbar + one;
  const long long bh = (long long)B * heads;
  const unsigned blocks = (unsigned)((2 * bh * ntp * 32 + 255) / 256);
  if (d == 128)
    pool_kv_kernel<128><<<blocks, 256, 0, s>>>(static_cast<const uint4 *>(k), static_cast<const uint4 *>(v),
                                                reinterpret_cast<uint4 *>(kbar), reinterpret_cast<uint4 *>(vbar),
                                                bh, ntp, geo);
  else
    pool_kv_kernel<64><<<blocks, 256, 0, s>>>(static_cast<const uint4 *>(k), static_cast<const uint4 *>(v),
                                               reinterpret_cast<uint4 *>(kbar), reinterpret_cast<uint4 *>(vbar),
                                               bh, ntp, geo);
  STA_CUDA_TRY(cudaGetLastError());
  return (d == 128) ? launch_attn<128, false, false, true>(q, k, v, o, lse, row_ptr, col_idx, B, heads, geo,
                                                           sm_scale, s, nullptr, nullptr, kbar, vbar)
                    : launch_attn<64, false, false, true>(q, k, v, o, lse, row_ptr, col_idx, B, heads, geo,
                                                          sm_scale, s, nullptr, nullptr, kbar, vbar);
}

sta_status sta_search_windows(const float *block_mass, int32_t B, int32_t heads, sta_grid g,
                              int32_t num_groups, const int32_t *group_lo, float tau, float lambda,
                              int32_t *windows, float *stats, sta_stream_t stream) {
  Geo geo;
  if (B <= 0 || heads <= 0 || !make_geo(g, &geo)) return STA_ERR_INVALID_ARG;
  if (block_mass == nullptr || windows == nullptr || group_lo == nullptr) return STA_ERR_INVALID_ARG;
  if (num_groups < 1 || num_groups > STA_MAX_GROUPS || group_lo[0] != 0) return STA_ERR_INVALID_ARG;
  for (int i = 1; i < num_groups; ++i)
    if (group_lo[i] <= group_lo[i - 1]) return STA_ERR_INVALID_ARG;
  if (!(tau >= 0.0f && tau <= 1.0f) || !(lambda >= 0.0f)) return STA_ERR_INVALID_ARG;
  if ((long long)B * heads > 65535 || geo.T >= 4096 || geo.NH >= 1024 || geo.NW >= 1024)
    return STA_ERR_UNSUPPORTED;
  const size_t smem = (size_t)(geo.Nt + geo.T) * sizeof(uint32_t);
  if (smem > 200 * 1024) return STA_ERR_UNSUPPORTED;
  if (smem > 48 * 1024)
    STA_CUDA_TRY(cudaFuncSetAttribute(search_windows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)smem));
  GroupLo glo;
  for (int i = 0; i < STA_MAX_GROUPS; ++i) glo.v[i] = (i < num_groups) ? group_lo[i] : 0x7fffffff;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  search_windows_kernel<<<(unsigned)(B * heads), SEARCH_THREADS, smem, s>>>(block_mass, geo, num_groups, glo,
                                                                           tau, lambda, windows, stats);
  STA_CUDA_TRY(cudaGetLastError());
  return STA_OK;
}

sta_status sta_set_wait_limit(int64_t limit_cycles) {
  if (limit_cycles != 0 && (limit_cycles < 1000 || limit_cycles > DEFAULT_WAIT_LIMIT)) return STA_ERR_INVALID_ARG;
  g_wait_limit.store((long long)limit_cycles, std::memory_order_relaxed);
  return STA_OK;
}

int64_t sta_get_wait_limit(void) { return (int64_t)wait_limit(); }

sta_status sta_selftest_wait_timeout(int64_t limit_cycles, sta_stream_t stream) {
  if (limit_cycles < 1000 || limit_cycles > 2000000000LL) return STA_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  selftest_wait_kernel<<<1, 32, 0, s>>>((long long)limit_cycles);
  STA_CUDA_TRY(cudaGetLastError());
  return STA_OK;
}

sta_status sta_validate_csr(const int32_t *row_ptr, const int32_t *col_idx, int64_t col_capacity, int32_t B,
                            int32_t heads, sta_grid g, sta_stream_t stream) {
  Geo geo;
  if (!make_geo(g, &geo) || B <= 0 || heads <= 0) return STA_ERR_INVALID_ARG;
  if (row_ptr == nullptr || col_idx == nullptr || col_capacity < 0) return STA_ERR_INVALID_ARG;
  if (!device_is_sm100()) return STA_ERR_UNSUPPORTED;
  const long long R = (long long)B * heads * geo.Nt;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  validate_csr_kernel<<<(unsigned)((R * 32 + 255) / 256), 256, 0, s>>>(row_ptr, col_idx, (long long)col_capacity,
                                                                       R, geo.Nt);
  STA_CUDA_TRY(cudaGetLastError());
  return STA_OK;
}

sta_status sta_get_device_error(sta_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  STA_CUDA_TRY(cudaStreamSynchronize(s));
  unsigned int word = 0;
  STA_CUDA_TRY(cudaMemcpyFromSymbol(&word, g_dev_error, sizeof(word)));
  const unsigned int zero = 0;
  STA_CUDA_TRY(cudaMemcpyToSymbol(g_dev_error, &zero, sizeof(zero)));
  if (word & DEV_ERR_BOUNDS) return STA_ERR_BOUNDS;
  if (word & DEV_ERR_TIMEOUT) return STA_ERR_TIMEOUT;
  if (word & DEV_ERR_BAD_MASK) return STA_ERR_BAD_MASK;
  return STA_OK;
}

int32_t sta_debug_build(void) { return STA_DEBUG ? 1 : 0; }

const char *sta_status_string(sta_status s) {
  switch (s) {
    case STA_OK: return "ok";
    case STA_ERR_INVALID_ARG: return "invalid argument";
    case STA_ERR_UNSUPPORTED: return "unsupported size or device";
    case STA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case STA_ERR_CUDA: return "CUDA call failed";
    case STA_ERR_TIMEOUT: return "device pipeline wait timed out";
    case STA_ERR_BAD_MASK: return "CSR column index out of range";
    case STA_ERR_BOUNDS: return "index or address outside its buffer (checked build)";
  }
  return "unknown status";
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free mask build: the workspace is this static device array.
// Host code must not hand the array's name to a kernel (on the host it is only
// a stand-in); its device address is looked up with cudaGetSymbolAddress on
// the first call on a device and cached together with the id of the device's
// current context. A later call that finds another context current (e.g. the
// primary context was reset and re-created, which reloads the module at a new
// address) looks the address up again.
namespace {

constexpr int NOALLOC_MAX_DEVICES = 64;
static __device__ __align__(256) uint8_t g_noalloc_scratch[STA_NOALLOC_SCRATCH_BYTES];
std::mutex g_noalloc_mutex;
void *g_noalloc_addr[NOALLOC_MAX_DEVICES] = {};
unsigned long long g_noalloc_ctx[NOALLOC_MAX_DEVICES] = {};

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long *);

// Unique id of the calling thread's current context, 0 if there is none or
// the driver cannot tell.
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static bool looked_up = false;
  if (!looked_up) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
    looked_up = true;
  }
  CUcontext ctx = nullptr;
  unsigned long long id = 0ull;
  if (get_current == nullptr || get_id == nullptr || get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr ||
      get_id(ctx, &id) != CUDA_SUCCESS)
    return 0ull;
  return id;
}

sta_status noalloc_scratch_address(void **out) {
  int dev = -1;
  STA_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= NOALLOC_MAX_DEVICES) return STA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  const unsigned long long ctx = current_context_id();
  if (g_noalloc_addr[dev] == nullptr || ctx == 0ull || ctx != g_noalloc_ctx[dev]) {
    void *addr = nullptr;
    STA_CUDA_TRY(cudaGetSymbolAddress(&addr, g_noalloc_scratch));
    if (addr == nullptr) return STA_ERR_CUDA;
    g_noalloc_addr[dev] = addr;
    // the lookup makes the device's primary context current if none was
    g_noalloc_ctx[dev] = current_context_id();
  }
  *out = g_noalloc_addr[dev];
  return STA_OK;
}

}  // namespace

extern "C" sta_status sta_build_mask_noalloc(const void *q_tiled, const void *k_tiled, int32_t B,
                                             int32_t heads, int32_t d, sta_grid g,
                                             const sta_mask_params *p, int32_t *row_ptr,
                                             int32_t *col_idx, int64_t *nnz_dev, uint8_t *block_mask,
                                             float *block_probs, sta_stream_t stream) {
  Geo geo;
  sta_status st = STA_OK;
  if (!common_sizes_ok(B, heads, d, g, &geo, &st)) return st;
  if (mask_ws_layout(B, heads, d, geo).total_min > (size_t)STA_NOALLOC_SCRATCH_BYTES) return STA_ERR_WORKSPACE;
  void *scratch = nullptr;
  st = noalloc_scratch_address(&scratch);
  if (st != STA_OK) return st;
  return sta_build_mask(q_tiled, k_tiled, B, heads, d, g, p, row_ptr, col_idx, nnz_dev, block_mask,
                        block_probs, scratch, (size_t)STA_NOALLOC_SCRATCH_BYTES, stream);
}
