/*
 * sta.h -- C ABI of libsta: block-sparse attention over a 3D video token grid
 * with per-head tile masks, for NVIDIA B200 (sm_100a).
 *
 * The method (pages on training-free sparse attention for video diffusion
 * transformers):
 *   - Compact Attention (abstract; Fig. 1(3); Fig. 3; Fig. 4; Table III):
 *     tile-aligned, head-specific masks made of two deformable windows with a
 *     separate extent per temporal-distance group, computed once and loaded
 *     into a block-sparse attention kernel that is reused across steps.
 *   - Rectified SpaAttn (abstract): block importance from pooled query-key.
 *   - SCOPE review (Eqs. (7)-(8) as quoted; abstract): hybrid top-p with a
 *     fixed top-k floor.
 *
 * Conventions shared by every call
 *   - Tiles are 1x8x8 tokens (64). For a T x H x W grid: NH = ceil(H/8),
 *     NW = ceil(W/8), Nt = T*NH*NW tiles per head, Lpad = 64*Nt rows.
 *     Tile n = (t*NH + y/8)*NW + x/8; token row inside the tile = (y%8)*8 + x%8.
 *   - Raster tensors are [B, L, heads, d] bf16, L = T*H*W, token index
 *     (t*H + y)*W + x. Tiled tensors are [B, heads, Lpad, d] bf16.
 *   - Every pointer argument named as a tensor is DEVICE memory owned by the
 *     caller; the library allocates nothing and keeps no pointer after return.
 *   - All calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream). Argument checks are synchronous and return a status
 *     before anything is launched; a launch failure returns STA_ERR_CUDA.
 *     Faults detected on the device (a bounded wait that ran out, an index out
 *     of range) are recorded in a device error word read by
 *     sta_get_device_error().
 *   - d (head dim) must be 64 or 128. Device pointers must be 16-byte aligned.
 */
#ifndef STA_H
#define STA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *sta_stream_t; /* same handle as cudaStream_t */

typedef enum {
  STA_OK = 0,
  STA_ERR_INVALID_ARG = 1, /* NULL pointer, bad size, misaligned pointer */
  STA_ERR_UNSUPPORTED = 2, /* d not in {64,128}, grid too large, wrong GPU */
  STA_ERR_WORKSPACE = 3,   /* workspace NULL or smaller than required */
  STA_ERR_CUDA = 4,        /* a CUDA runtime / driver call failed */
  STA_ERR_TIMEOUT = 5,     /* device: a bounded pipeline wait ran out */
  STA_ERR_BAD_MASK = 6,    /* device: a CSR column index or query pair out of
                              range, or a CSR that sta_validate_csr rejects */
  STA_ERR_BOUNDS = 7       /* device, checked build only: an index or address
                              failed its bounds / alignment check; the access
                              was skipped (see sta_debug_build) */
} sta_status;

typedef struct {
  int32_t T, H, W; /* token grid; the tile is fixed at 1x8x8 */
} sta_grid;

#define STA_MAX_GROUPS 8

/* Mask recipe of sta_build_mask.
 * Selection (Rectified SpaAttn pooled scores; SCOPE hybrid top-p/top-k):
 *   qbar, kbar = mean of Q, K over the real tokens of each tile;
 *   P = softmax over key tiles of sm_scale * qbar . kbar (fp32);
 *   order key tiles by P descending, ties to the lower index; with integer
 *   mass w = floor(P * 2^24) and thr = ceil(double(top_p) * double(sum w)),
 *   keep the shortest prefix reaching thr (all tiles if top_p >= 1, none if
 *   top_p <= 0), extended to at least min(k_min, Nt) tiles.
 * Windows (Compact Attention dual windows per temporal-distance group):
 *   key tile kt is kept for query tile qt of head h iff the group
 *   g = max{g : group_lo[g] <= |t_q - t_k|} exists and
 *   (|dy| <= ry1 && |dx| <= rx1) || (|dy| <= ry2 && |dx| <= rx2)
 *   with (ry1, rx1, ry2, rx2) = windows[(h*num_groups + g)*4 + 0..3], in
 *   tile units; -1 switches a window off. The last group is open-ended.
 * The mask is the union of the two parts. */
typedef struct {
  float top_p;            /* selection mass; >= 1 keeps all; ignored if !use_scores */
  int32_t k_min;          /* floor on the selected count, clipped to Nt */
  int32_t use_scores;     /* 0: window-only mask (no pooling / scoring) */
  float sm_scale;         /* score scale; 0 means 1/sqrt(d) */
  int32_t num_groups;     /* G in [1, STA_MAX_GROUPS] when windows != NULL */
  int32_t group_lo[STA_MAX_GROUPS]; /* ascending, group_lo[0] == 0 */
  const int32_t *windows; /* device int32 [heads][G][4]; NULL = no windows */
  int32_t head_topk_floor; /* 1: raise each row's selection to its head's floor
                              (SCOPE Eqs. (9)-(10) as quoted): with b_c the
                              selected count of query tile c and n_c its real
                              tokens, k_head = ceil(sum n_c b_c / sum n_c), and
                              rows with b_c < k_head keep their first
                              min(k_head, Nt) tiles; ignored if !use_scores */
  const float *block_scores; /* device fp32 [B, heads, Nt, Nt] or NULL. When set
                              (and use_scores), the selection runs on these
                              rows instead of the pooled-score probabilities,
                              e.g. the masses of sta_attn_fwd_block_mass;
                              values are clamped to [0, 1] and q_tiled, k_tiled
                              are not read */
  int32_t *query_pairs;   /* optional output, device int32 [B*heads][2*NP],
                              NP = ceil(Nt/2), 4-byte aligned, or NULL: the
                              query tiles of each head paired into the 128-row
                              tiles of sta_attn_fwd_paired, chosen by list
                              overlap (see sta_attn_fwd_paired); needs
                              9*Nt <= 227 KB (STA_ERR_UNSUPPORTED otherwise) */
} sta_mask_params;

/* Number of tiles per head (Nt) and padded rows per head (Lpad) of a grid;
 * -1 if the grid is invalid. */
int64_t sta_num_tiles(sta_grid g);
int64_t sta_tiled_len(sta_grid g);

/* sta_reorder -- token layout change (Compact Attention: tile-aligned
 * masks; Table III "Cubic" tiles).
 *   inverse == 0: src raster [B, L, heads, d] -> dst tiled [B, heads, Lpad, d];
 *                 rows of partial tiles beyond the grid are written as zero.
 *   inverse != 0: src tiled -> dst raster; pad rows are dropped.
 * bf16 elements are moved bit for bit. src and dst must not overlap. */
sta_status sta_reorder(const void *src, void *dst, int32_t B, int32_t heads, int32_t d,
                       sta_grid g, int32_t inverse, sta_stream_t stream);

/* Bytes of device workspace of sta_build_mask for these sizes. The full size
 * holds the pooled Q and K split into two tf32 parts each and a row buffer
 * [B*heads*Nt, Nt] fp32: the pooled scores then run on the tensor cores
 * (three tf32 products per term, within 2^-22 (3 d/8 + 3) of the sum of
 * |q||k| per score) and a separate select pass does the softmax and the
 * selection (four CTAs per SM). Any workspace of at least the _min size is
 * accepted and runs one fused pass whose scores are fp32 FMA chains. The two
 * layouts agree with the exact scores within their bounds, so a tile whose
 * P sits at the selection threshold may be kept by one and not the other. */
size_t sta_build_mask_workspace(int32_t B, int32_t heads, int32_t d, sta_grid g);
size_t sta_build_mask_workspace_min(int32_t B, int32_t heads, int32_t d, sta_grid g);

/* Where sta_build_mask (and _raster) leaves the pooled means in its
 * workspace, as byte offsets: offsets[0] = qbar, offsets[1] = kbar, each fp32
 * [B*heads*Nt, d] with row (b*heads + h)*Nt + tile. They are written when
 * use_scores is set and block_scores is NULL. With a workspace of at least
 * sta_build_mask_workspace() bytes (the tensor-core layout) each mean x is
 * stored split: tf32(x) at offsets[0] / [1] and tf32(x - tf32(x)) (round to
 * nearest, ties away) at offsets[2] / [3]; with a smaller workspace x itself
 * is stored and offsets[2] = offsets[3] = 0 (nothing written there). x is the
 * mean over the real tokens of the tile, an exact sum rounded once to fp32
 * (Rectified SpaAttn abstract: pooled query-key). Returns STA_ERR_INVALID_ARG
 * or STA_ERR_UNSUPPORTED for sizes sta_build_mask rejects. */
sta_status sta_build_mask_pooled_offsets(int32_t B, int32_t heads, int32_t d, sta_grid g, size_t ws_bytes,
                                         size_t offsets[4]);

/* sta_build_mask -- per-head tile mask as CSR lists (Compact Attention Fig. 3:
 * masks computed online are loaded into the block-sparse kernel; Fig. 4: the
 * result is a binary mask over (query tile, key tile)).
 *   q_tiled, k_tiled : [B, heads, Lpad, d] bf16 (read only if use_scores)
 *   row_ptr          : int32 [B*heads*Nt + 1], written; row r = (b*heads+h)*Nt+qt
 *   col_idx          : int32, capacity >= B*heads*Nt*Nt (worst case, so no
 *                      host synchronisation is ever needed); each row's key
 *                      tiles are written in ascending order
 *   nnz_dev          : device int64 scalar, written with row_ptr[last]
 *   block_mask       : optional uint8 [B, heads, Nt, Nt] (0/1); NULL to skip
 *   block_probs      : optional fp32 [B, heads, Nt, Nt], the P the selection
 *                      used (0 where !use_scores); NULL to skip
 *   workspace        : device, >= sta_build_mask_workspace_min() bytes (the
 *                      full sta_build_mask_workspace() for the fastest
 *                      layout), 256-aligned
 * The call is deterministic: the same inputs and workspace size give
 * bit-identical outputs. */
sta_status sta_build_mask(const void *q_tiled, const void *k_tiled, int32_t B, int32_t heads,
                          int32_t d, sta_grid g, const sta_mask_params *p, int32_t *row_ptr,
                          int32_t *col_idx, int64_t *nnz_dev, uint8_t *block_mask,
                          float *block_probs, void *workspace, size_t ws_bytes,
                          sta_stream_t stream);

/* sta_attn_fwd -- block-sparse attention forward over the listed key tiles
 * (Compact Attention Fig. 3 "block-sparse attention kernels"; Fig. 5 "dense
 * Compact kernel" is the same call with every tile listed).
 * For every real query token of query tile qt in row r = (b*heads+h)*Nt+qt:
 *   o   = sum_j softmax_j(sm_scale * q . k_j) v_j
 *   lse = log(sum_j exp(sm_scale * q . k_j))           (natural log)
 * over the real tokens j of tiles col_idx[row_ptr[r] .. row_ptr[r+1]).
 *   q, k, v : tiled [B, heads, Lpad, d] bf16;  o : tiled [B, heads, Lpad, d] bf16
 *   lse     : optional fp32 [B, heads, Lpad]; NULL to skip
 *   row_ptr, col_idx : CSR as written by sta_build_mask (or the caller's own:
 *             ascending, unique, in [0, Nt) per row; an index out of range is
 *             reported as STA_ERR_BAD_MASK by sta_get_device_error and the
 *             tile is skipped)
 *   sm_scale: 0 means 1/sqrt(d)
 * A row with an empty list gives o = 0 and lse = -inf. Output rows of pad
 * tokens hold unspecified finite values. Accumulation is fp32; P is rounded
 * to bf16 before the P.V product. */
sta_status sta_attn_fwd(const void *q, const void *k, const void *v, void *o, float *lse,
                        const int32_t *row_ptr, const int32_t *col_idx, int32_t B, int32_t heads,
                        int32_t d, sta_grid g, float sm_scale, sta_stream_t stream);

/* Raster-layout forms of sta_build_mask and sta_attn_fwd: the same results
 * (bit for bit) without the layout change of sta_reorder. The token tiles
 * (Compact Attention: tile-aligned masks over 1x8x8 cubes) are gathered by
 * the kernels' loads instead of a separate pass over memory.
 *   q, k, v : raster [B, L, heads, d] bf16
 *   o       : raster [B, L, heads, d] bf16, every real token row written
 *   lse     : optional fp32 [B, heads, Lpad], indexed like the tiled layout
 *             (row 64*qt + (y%8)*8 + x%8 of the head); pad rows unspecified
 * Every other argument, check and error is that of the tiled call. */
sta_status sta_build_mask_raster(const void *q, const void *k, int32_t B, int32_t heads, int32_t d,
                                 sta_grid g, const sta_mask_params *p, int32_t *row_ptr,
                                 int32_t *col_idx, int64_t *nnz_dev, uint8_t *block_mask,
                                 float *block_probs, void *workspace, size_t ws_bytes,
                                 sta_stream_t stream);
sta_status sta_attn_fwd_raster(const void *q, const void *k, const void *v, void *o, float *lse,
                               const int32_t *row_ptr, const int32_t *col_idx, int32_t B,
                               int32_t heads, int32_t d, sta_grid g, float sm_scale,
                               sta_stream_t stream);

/* sta_attn_fwd_paired, sta_attn_fwd_raster_paired -- sta_attn_fwd and
 * sta_attn_fwd_raster with the query tiles paired as the caller says. The
 * kernels run 128 query rows (two 64-token query tiles) per tensor-core tile
 * over the union of the two tiles' key lists; a tile gets P = 0 for the key
 * tiles its own list lacks, so the union steps it does not need are wasted
 * work. The default pairing (frames 2u and 2u+1 of one spatial tile; the last
 * odd frame's tiles with their right-hand neighbour) suits window masks;
 * lists from a top-k selection at low density overlap less between frames.
 * The pages have no counterpart: the results are those of the unpaired calls
 * up to the fp32 summation order of each row.
 *   query_pairs : device int32 [B*heads][2*NP], NP = ceil(Nt/2): pair i of
 *                 head (b, h) is (query_pairs[2i], query_pairs[2i+1]), the
 *                 second -1 for a tile without a partner; every tile of the
 *                 head must appear exactly once. sta_build_mask writes such
 *                 an array when sta_mask_params.query_pairs is set:
 *                 - candidates: tile a = (t, y, x) with b = a + (dt, dy, dx)
 *                   for (dt, dy, dx) in {1} x {-1, 0, 1}^2, (0, 1, -1..1),
 *                   (0, 0, 1) and (2, 0, 0), inside the grid; weight
 *                   |L_a n L_b| of the two final key-tile lists;
 *                 - greedy matching: candidate pairs by weight descending,
 *                   ties to the lower smaller tile, then the lower larger
 *                   tile, each taken if both tiles are free; the tiles left
 *                   over are paired in ascending order (a last one alone if
 *                   their count is odd);
 *                 - per head, if the total union size sum(|L_a u L_b|) of
 *                   this pairing is not below that of the default pairing,
 *                   the default pairing is written instead;
 *                 pairs are written in ascending order of their first tile
 *                 (the default pairing in its own order).
 * A tile index out of range in query_pairs is reported as STA_ERR_BAD_MASK
 * (the pair is skipped). Every other argument, output and error is that of
 * sta_attn_fwd / sta_attn_fwd_raster. */
sta_status sta_attn_fwd_paired(const void *q, const void *k, const void *v, void *o, float *lse,
                               const int32_t *row_ptr, const int32_t *col_idx, const int32_t *query_pairs,
                               int32_t B, int32_t heads, int32_t d, sta_grid g, float sm_scale,
                               sta_stream_t stream);
sta_status sta_attn_fwd_raster_paired(const void *q, const void *k, const void *v, void *o, float *lse,
                                      const int32_t *row_ptr, const int32_t *col_idx,
                                      const int32_t *query_pairs, int32_t B, int32_t heads, int32_t d,
                                      sta_grid g, float sm_scale, sta_stream_t stream);

/* Size in bytes of the static device scratch behind sta_build_mask_noalloc. */
#define STA_NOALLOC_SCRATCH_BYTES (32u << 20)

/* sta_build_mask_noalloc -- sta_build_mask for callers that cannot allocate.
 * The pages have no counterpart to this call: it exists for callers whose
 * device memory is laid out up front by a host framework or a fixed arena
 * (embedded inference runtimes, plug-ins of engines that own every device
 * allocation), so they can neither call cudaMalloc nor lend a workspace.
 * Same arguments as sta_build_mask minus the workspace, and the results of
 * sta_build_mask with a workspace of STA_NOALLOC_SCRATCH_BYTES (the
 * tensor-core layout when sta_build_mask_workspace() fits in it, else the
 * fused one): the workspace is a file-scope static device array of
 * STA_NOALLOC_SCRATCH_BYTES (32 MiB), present on every GPU that loads the
 * library until the process exits. The caller still passes inputs and outputs.
 *   - Sizes whose minimum workspace (sta_build_mask_workspace_min) exceeds
 *     the array are rejected with STA_ERR_WORKSPACE before anything runs
 *     (e.g. 40 heads of a 21x30x52 grid fit; 40 heads of 21x45x80 do not).
 *   - The first call on a device looks up the array's device address with
 *     cudaGetSymbolAddress (the device must be current); make that first call
 *     before any stream capture. Later calls reuse the cached address while
 *     the same context is current; after a device reset (a new primary
 *     context, which reloads the library's device code at a new address) the
 *     next call looks the address up again, and should likewise come before
 *     any stream capture.
 *   - No allocation of any kind (no cudaMalloc / cudaFree, no allocating
 *     library routine). Nothing in the array has to start at zero: every
 *     byte the kernels read is written earlier in the same call.
 *   - All calls share the one array, which keeps the last call's contents:
 *     calls that overlap on the GPU (different streams, or other host threads)
 *     race on it and must be serialised by the caller. */
sta_status sta_build_mask_noalloc(const void *q_tiled, const void *k_tiled, int32_t B, int32_t heads,
                                  int32_t d, sta_grid g, const sta_mask_params *p, int32_t *row_ptr,
                                  int32_t *col_idx, int64_t *nnz_dev, uint8_t *block_mask,
                                  float *block_probs, sta_stream_t stream);

/* sta_attn_fwd_block_mass -- sta_attn_fwd that also measures the exact block
 * importance of every listed pair under a cached log-sum-exp (AdaSpa
 * abstract: block importance computed during a full-attention step with the
 * LSE cached from an earlier step, then reused by the sparse steps):
 *   mass(qt, kt) = (1/n_q) sum_i sum_j exp(sm_scale * q_i . k_j - lse_cached_i)
 * over the real query tokens i of qt (n_q of them) and the real key tokens j
 * of kt; a token whose cached LSE is -inf contributes nothing. With the exact
 * LSE of the same inputs and every tile listed, each row sums to one.
 *   lse_cached : fp32 [B, heads, Lpad] (natural log), e.g. the lse output of
 *                an earlier call on the same layer
 *   block_mass : fp32 [B, heads, Nt, Nt], written: listed pairs get their
 *                mass, every other entry 0
 * All other arguments, outputs and errors are those of sta_attn_fwd. The
 * masses are accumulated in fp32 (per-row sums relative to the running max,
 * one exp2 per row and tile, two adds per pair onto zero: deterministic). */
sta_status sta_attn_fwd_block_mass(const void *q, const void *k, const void *v, void *o, float *lse,
                                   const int32_t *row_ptr, const int32_t *col_idx,
                                   const float *lse_cached, float *block_mass, int32_t B,
                                   int32_t heads, int32_t d, sta_grid g, float sm_scale,
                                   sta_stream_t stream);

/* sta_attn_fwd_rectified -- rectified block-sparse attention (Rectified
 * SpaAttn abstract: dropping tiles inflates the kept weights and loses the
 * dropped ones; the kept weights are reallocated with pooled weights and the
 * dropped ones recovered from the pooled query-key). Reading (the abstract
 * gives no formula): every key tile NOT listed for the row enters the softmax
 * as one pooled key k_bar (mean of its real keys) with value v_bar (mean of
 * its real values) and multiplicity n (its real token count):
 *   o   = (sum_listed e^{s q.k_j} v_j + sum_unlisted n_t e^{s q.k_bar_t} v_bar_t)
 *         / (sum_listed e^{s q.k_j} + sum_unlisted n_t e^{s q.k_bar_t})
 *   lse = ln(denominator), s = sm_scale (0 -> 1/sqrt(d))
 * With every tile listed this is sta_attn_fwd (bit for bit).
 *   q, k, v, o, lse, row_ptr, col_idx : as sta_attn_fwd (tiled layout)
 *   workspace : device, >= sta_rectified_workspace() bytes, 256-aligned;
 *               receives the pooled K and V (bf16) of every head
 * Errors as sta_attn_fwd, plus STA_ERR_WORKSPACE. */
size_t sta_rectified_workspace(int32_t B, int32_t heads, int32_t d, sta_grid g);
sta_status sta_attn_fwd_rectified(const void *q, const void *k, const void *v, void *o, float *lse,
                                  const int32_t *row_ptr, const int32_t *col_idx, void *workspace,
                                  size_t ws_bytes, int32_t B, int32_t heads, int32_t d, sta_grid g,
                                  float sm_scale, sta_stream_t stream);

/* sta_search_windows -- recall-driven offline search of the dual windows
 * (Compact Attention Fig. 3: the windows are shrunk iteratively under the
 * recall (tau) and cost (lambda) constraints, and the configurations are
 * stored for reuse; Fig. 4: starting from full coverage in every
 * temporal-distance group, the dual windows are shrunk while the recall and
 * shrink-penalty constraints hold; Fig. 5(c): recall target vs sparsity).
 * One search per (b, h) on its block importances, e.g. the masses of
 * sta_attn_fwd_block_mass over a dense list with the exact LSE:
 *   masses w = floor(min(max(m, 0), 1) * 2^24); W = sum of w; the recall of a
 *   window set is the covered w over W;
 *   start: (ry1, rx1, ry2, rx2) = (NH-1, NW-1, NH-1, NW-1) in every group;
 *   moves, per group g in order: ry1-1, rx1-1, ry2-1, rx2-1, (ry1-1, ry2-1),
 *   (rx1-1, rx2-1); an extent never goes below -1;
 *   J = removed / Nt^2 - lambda * lost / W for the pairs / mass a move
 *   uncovers; a move is admissible iff covered - lost >= ceil(double(tau) * W)
 *   (recall) and J >= 0 (cost); a move that uncovers nothing (one window
 *   shrunk inside the other) has J = 0, which lets the two windows, equal at
 *   the start, come apart (e.g. into a cross of a row band and a column
 *   band); each step applies the admissible move with the largest J (ties to
 *   the lowest g*6 + m) and the search stops when none is left.
 *   block_mass : device fp32 [B, heads, Nt, Nt]
 *   group_lo   : HOST int32 [num_groups], ascending, group_lo[0] == 0
 *   tau in [0, 1]; lambda >= 0
 *   windows    : device int32 [B*heads][num_groups][4], written (the layout of
 *                sta_mask_params.windows for one batch entry)
 *   stats      : optional device fp32 [B*heads][2] = (recall, density); NULL ok
 * Deterministic: integer sums, one double comparison per move. */
sta_status sta_search_windows(const float *block_mass, int32_t B, int32_t heads, sta_grid g,
                              int32_t num_groups, const int32_t *group_lo, float tau, float lambda,
                              int32_t *windows, float *stats, sta_stream_t stream);

/* sta_set_wait_limit -- how long a stalled pipeline may wait before it is
 * reported. Every pipeline wait of the kernels launched after this call by
 * this process (the attention forms, the tensor-core scores and the raster
 * pooling of the mask build) gives up after limit_cycles SM cycles: the kernel
 * records STA_ERR_TIMEOUT in the device error word, waits (with a fixed limit
 * of 2e8 cycles) for its own MMAs and TMA copies in flight, releases its
 * tensor memory and returns, so the context stays usable; the outputs of that
 * call are unspecified. limit_cycles in [1e3, 2e9], or 0 for the default
 * (2e9 cycles, about a second at the B200's clocks). A limit below the
 * pipeline's ordinary latencies (a few thousand cycles) makes every call time
 * out: it exists to check the timeout path, or to report stalls sooner. The
 * pages have no counterpart. Returns STA_ERR_INVALID_ARG out of range. */
sta_status sta_set_wait_limit(int64_t limit_cycles);

/* The wait limit the next launches will use (SM cycles). */
int64_t sta_get_wait_limit(void);

/* sta_selftest_wait_timeout -- exercises the bounded wait that every pipeline
 * stage of sta_attn_fwd uses, without a fault: one thread initialises a
 * shared-memory mbarrier that nothing will ever complete, waits on it for at
 * most `limit_cycles` SM cycles (1e3 .. 2e9), records STA_ERR_TIMEOUT in the
 * device error word and returns. The pages have no counterpart; it lets a
 * caller check that a stalled pipeline is reported through
 * sta_get_device_error() and leaves the context usable. */
sta_status sta_selftest_wait_timeout(int64_t limit_cycles, sta_stream_t stream);

/* sta_debug_build -- 1 in the checked build of the library
 * (libsta_debug.so, compiled with -DSTA_DEBUG=1), 0 in the product build
 * (libsta.so). The checked build runs the same kernels with the same
 * arithmetic, and in addition tests, before use, every index and address
 * derived from run-time data: TMA box coordinates against the tensor's
 * extents and the 16-byte rule for the innermost coordinate, shared-memory
 * destinations against the CTA's layout, TMEM addresses against the
 * allocation and the warp's lane quarter, and global store indices against
 * their buffers. A failed check records STA_ERR_BOUNDS in the device error
 * word and skips the access (a skipped load then ends in a bounded pipeline
 * wait, reported as well). The pages have no counterpart. */
int32_t sta_debug_build(void);

/* sta_validate_csr -- checks a caller's CSR lists before they are handed to
 * the attention calls (the pages have no counterpart: masks the library
 * builds are valid by construction). One warp per row
 * r < B*heads*Nt reads row_ptr[r], row_ptr[r+1] first and checks
 * row_ptr[0] == 0, row_ptr[r] <= row_ptr[r+1] <= col_capacity and at most Nt
 * entries per row; only then it reads the row's columns, which must be
 * strictly ascending and in [0, Nt). Any violation records STA_ERR_BAD_MASK
 * in the device error word (read it with sta_get_device_error); nothing is
 * written. row_ptr must hold B*heads*Nt + 1 entries; col_capacity is the
 * number of int32 the col_idx array holds, so that no read leaves it.
 * Asynchronous on `stream`; argument errors are returned at once. */
sta_status sta_validate_csr(const int32_t *row_ptr, const int32_t *col_idx, int64_t col_capacity, int32_t B,
                            int32_t heads, sta_grid g, sta_stream_t stream);

/* Reads and clears the device error word of the current device after
 * synchronising `stream`. STA_OK if no device-side fault was recorded;
 * STA_ERR_BOUNDS takes precedence over STA_ERR_TIMEOUT (a skipped access is
 * the cause of the wait that ran out), then STA_ERR_BAD_MASK. */
sta_status sta_get_device_error(sta_stream_t stream);

/* Static description of a status code. */
const char *sta_status_string(sta_status s);

#ifdef __cplusplus
}
#endif
#endif /* STA_H */
