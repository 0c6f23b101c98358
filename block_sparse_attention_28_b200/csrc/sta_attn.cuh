// Block-sparse attention forward over listed key tiles (Compact Attention
// Fig. 3: precomputed masks loaded into a block-sparse attention kernel).
//
// One CTA computes 128 query rows: two query tiles of one head, the same
// spatial tile in two consecutive frames (a 128-row tcgen05 tile; a 64-token
// tile alone would leave half of the MMA rows idle). The two CSR rows are
// merged into one ascending key-tile list with a per-half membership flag; a
// half whose list lacks the key tile gets P = 0 for that tile, so the work is
// |A u B| key tiles of 128 x 64. All roles walk the list from the first key
// tile at or after the CTA's own query tile and wrap around, which spreads
// the requests of neighbouring CTAs over L2.
//
// Warp roles (192 threads):
//   warps 0-3  softmax + correction + epilogue; thread i owns query row i
//              (TMEM lane i): S row -> online softmax (exp2, lazy rescale of
//              O when the running max grows by more than 2^8) -> P (bf16) back
//              into TMEM over S; at the end O / l -> bf16 -> global, and LSE.
//   warp 4     TMA producer: Q once, then K_{j+1} ahead of V_j per listed key
//              tile, each into its own NS-stage ring (128 B swizzle, no
//              multicast); a K slot is freed as soon as its S MMA retires, a V
//              slot when its P.V MMA retires.
//   warp 5     MMA issuer (one thread): S_j = Q K_j^T (SS, M=128 N=64) into
//              one of two TMEM S buffers, O += P_j V_j (A = P from TMEM,
//              B = V MN-major from shared memory, M=128 N=d).
// TMEM columns: S0 [0,64) S1 [64,128) O [128, 128+d). Two CTAs share an SM
// (TMEM 2 x 256 columns, shared memory 2 x 103 KB), so one CTA's softmax runs
// while the other's MMAs do.
// Every pipeline wait gives up after wait_limit SM cycles (set by the host):
// it records DEV_ERR_TIMEOUT and raises the CTA's abort flag, which ends the
// other roles' waits too; the CTA then waits (with a long, fixed limit) for
// its own MMAs and TMA copies in flight, releases TMEM and returns.
#pragma once
#include "sta_common.cuh"
#include "sta_tc.cuh"

namespace sta {
namespace attn {

constexpr int NUM_THREADS = 192;
constexpr int WARP_PRODUCER = 4;
constexpr int WARP_MMA = 5;
// Union-list entry: key tile (bits 0-19; the host keeps Nt <= 2^20), the
// valid extent of a partial key tile (rows - 1 in bits 20-22, columns - 1 in
// bits 23-25, flag bit 26), and the two halves' membership flags.
constexpr uint32_t KT_MASK = (1u << 20) - 1u;
constexpr uint32_t EXT_PARTIAL = 1u << 26;
constexpr uint32_t VIRT = 1u << 27;  // pooled key tile of the rectified form (index in bits 0-19)
constexpr uint32_t FLAG_A = 1u << 30;
constexpr uint32_t FLAG_B = 1u << 31;
constexpr uint32_t TMEM_COLS = 256;
constexpr uint32_t O_COL = 128;
constexpr long long DRAIN_LIMIT = 200000000LL;   // own copies / MMAs, after the pipeline
constexpr float RESCALE_LOG2 = 8.0f;             // lazy O rescale threshold
constexpr int MIN_BLOCKS_PER_SM = 2;             // two CTAs share an SM: one's softmax
                                                 // overlaps the other's MMAs
#ifndef STA_ATTN_NSK
#define STA_ATTN_NSK 2                           // K ring stages at d = 128
#endif
#ifndef STA_ATTN_NSV
#define STA_ATTN_NSV 2                           // V ring stages at d = 128
#endif
#ifndef STA_ATTN_KLEAD
#define STA_ATTN_KLEAD 1                         // K tiles loaded ahead of the V tile
#endif

template <int D>
struct Cfg {
  static constexpr int KB = D / 64;              // 128-byte swizzle atoms along d
  // ring stages: two CTAs per SM fit in shared memory
  static constexpr int NSK = (D == 128) ? STA_ATTN_NSK : 4;
  static constexpr int NSV = (D == 128) ? STA_ATTN_NSV : 4;
  static constexpr int KLEAD = (D == 128) ? STA_ATTN_KLEAD : 1;
  static constexpr int TILE_BYTES = 64 * D * 2;  // one 64-token tile of Q, K or V
  static constexpr int Q_REGION = 128 * 128;     // 128 rows x 128 B per d-atom
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + KB * Q_REGION;
  static constexpr int OFF_V = OFF_K + NSK * TILE_BYTES;
  static constexpr int OFF_BAR = OFF_V + NSV * TILE_BYTES;
  // q_full, k_full[NSK], k_empty[NSK], v_full[NSV], v_empty[NSV], s_full[2], p_full[2],
  // o_done, mma_done
  static constexpr int NUM_BARS = 1 + 2 * NSK + 2 * NSV + 2 + 2 + 1 + 1;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int OFF_LIST = OFF_MISC + 64;
  static constexpr uint32_t IDESC_S = tc::idesc_bf16(128, 64, false);
  static constexpr uint32_t IDESC_O = tc::idesc_bf16(128, D, true);
};

// ntp: pooled key rows of the rectified form (Nt rounded up to 64), 0 otherwise.
template <int D>
inline size_t smem_bytes(int nt, int ntp = 0) {
  const int wpr = (nt + 31) / 32;
  return (size_t)Cfg<D>::OFF_LIST + (size_t)(2 * wpr + nt + ntp / 64 + ntp) * 4 + 16 + 1024;
}

// MASS: also accumulate the LSE-cached exact block importance (AdaSpa) of
// every listed (query tile, key tile) pair into block_mass:
//   mass = (1/n_q) sum_i sum_j 2^(s_ij * scale_log2 - lse_in_i * log2 e),
// which is, per row and tile, the row's softmax sum (relative to its running
// max m_i) times 2^(m_i - lse_in_i * log2 e): one extra exp2 per row and tile.
//
// RASTER: Q, K, V and O stay in the raster layout [B, L, heads, d]. A tile is
// then one box of a 5D tensor map (d, head, x, y, frame), 64 d-values x 1
// head x 8 columns x 8 rows x 1 frame, which TMA writes to shared memory in
// the tile's token order (zeros beyond the grid edge), so the permutation to
// tiles costs no pass over memory; O rows go straight to their raster rows.
//
// RECT (rectified form, Rectified SpaAttn abstract): after the listed tiles
// the CTA walks ntp/64 pooled tiles whose 64 "keys" are the tile means
// k_bar of key tiles 64u .. 64u+63 (and values v_bar), each key carrying its
// tile's real-token count n as a multiplicity: the score of column kt is
// scale * q.k_bar_kt + ln n_kt, and columns of tiles the row lists (or past
// Nt) are masked. The online softmax then weighs listed tokens and pooled
// tiles against one normaliser.
template <int D, bool MASS, bool RASTER, bool RECT = false>
__global__ void __launch_bounds__(NUM_THREADS, MIN_BLOCKS_PER_SM)
attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, __nv_bfloat16 *__restrict__ out,
                float *__restrict__ lse, const int *__restrict__ row_ptr,
                const int *__restrict__ col_idx, Geo g, float scale_log2,
                const float *__restrict__ lse_in, float *__restrict__ block_mass, int heads,
                const __grid_constant__ CUtensorMap tm_kbar, const __grid_constant__ CUtensorMap tm_vbar,
                int ntp, long long wait_limit, const int *__restrict__ query_pairs) {
  static_assert(!(MASS && RECT) && !(RASTER && RECT), "the rectified form is tiled and mass-free");
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sbase = tc::smem_u32(smem);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nt = g.Nt;
  const int bh = blockIdx.y;
  // Query-tile pairing: the caller's (query_pairs: pair blockIdx.x of this
  // head), or by default the same spatial tile in frames 2u and 2u+1 (their
  // lists overlap most when windows dominate: windows and pooled scores change
  // little between neighbouring frames); with an odd frame count the last
  // frame's tiles are paired with their right-hand neighbour.
  int qtA, qtB;
  if (query_pairs != nullptr) {
    const long long at = ((long long)bh * ((nt + 1) / 2) + blockIdx.x) * 2;
    qtA = query_pairs[at];
    qtB = query_pairs[at + 1];
    if ((unsigned)qtA >= (unsigned)nt || (qtB != -1 && (unsigned)qtB >= (unsigned)nt)) {
      // the whole CTA leaves before any shared state exists
      if (threadIdx.x == 0) record_error(DEV_ERR_BAD_MASK);
      return;
    }
  } else {
    const int tpf_q = g.NH * g.NW;
    const int pairs_t = (g.T / 2) * tpf_q;
    if ((int)blockIdx.x < pairs_t) {
      const int u = (int)blockIdx.x / tpf_q, rem = (int)blockIdx.x - u * tpf_q;
      qtA = 2 * u * tpf_q + rem;
      qtB = qtA + tpf_q;
    } else {
      qtA = (g.T - 1) * tpf_q + 2 * ((int)blockIdx.x - pairs_t);
      qtB = qtA + 1;
    }
  }
  const bool hasB = qtB >= 0 && qtB < nt;
  const int wpr = (nt + 31) / 32;

  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
  uint64_t *q_full = bars;
  uint64_t *k_full = bars + 1;
  uint64_t *k_empty = k_full + C::NSK;
  uint64_t *v_full = k_empty + C::NSK;
  uint64_t *v_empty = v_full + C::NSV;
  uint64_t *s_full = v_empty + C::NSV;
  uint64_t *p_full = s_full + 2;
  uint64_t *o_done = p_full + 2;
  uint64_t *mma_done = o_done + 1;
  uint32_t *misc = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);  // tmem, n, abort
  volatile uint32_t *abort_flag = misc + 2;
  uint32_t *bmA = reinterpret_cast<uint32_t *>(smem + C::OFF_LIST);
  uint32_t *bmB = bmA + wpr;
  uint32_t *U = bmB + wpr;

  // ---- set-up: barriers, bitmaps, TMEM
  if (tid == 0) {
    tc::mbar_init(q_full, 1);
    for (int s = 0; s < C::NSK; ++s) {
      tc::mbar_init(k_full + s, 1);
      tc::mbar_init(k_empty + s, 1);
    }
    for (int s = 0; s < C::NSV; ++s) {
      tc::mbar_init(v_full + s, 1);
      tc::mbar_init(v_empty + s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(s_full + b, 1);
      tc::mbar_init(p_full + b, 4);
    }
    tc::mbar_init(o_done, 1);
    tc::mbar_init(mma_done, 1);
    misc[2] = 0u;
    tc::fence_barrier_init();
  }
  for (int i = tid; i < 2 * wpr; i += NUM_THREADS) bmA[i] = 0u;
  if (warp == WARP_MMA) {
    tc::tmem_alloc(misc, TMEM_COLS);
    tc::tmem_relinquish();
  }
  __syncthreads();

  // ---- the two CSR rows as bitmaps, then their ascending union with flags
  {
    const long long rA = (long long)bh * nt + qtA;
    const int a0 = row_ptr[rA], a1 = row_ptr[rA + 1];
    for (int i = a0 + tid; i < a1; i += NUM_THREADS) {
      const int c = col_idx[i];
      if ((unsigned)c < (unsigned)nt)
        atomicOr(bmA + (c >> 5), 1u << (c & 31));
      else
        record_error(DEV_ERR_BAD_MASK);
    }
    if (hasB) {
      const long long rB = (long long)bh * nt + qtB;
      const int b0 = row_ptr[rB], b1 = row_ptr[rB + 1];
      for (int i = b0 + tid; i < b1; i += NUM_THREADS) {
        const int c = col_idx[i];
        if ((unsigned)c < (unsigned)nt)
          atomicOr(bmB + (c >> 5), 1u << (c & 31));
        else
          record_error(DEV_ERR_BAD_MASK);
      }
    }
  }
  __syncthreads();
  if (warp == 0) {
    int base = 0;
    for (int w0 = 0; w0 < wpr; w0 += 32) {
      const int w = w0 + lane;
      const uint32_t a = (w < wpr) ? bmA[w] : 0u, b = (w < wpr) ? bmB[w] : 0u;
      uint32_t u = a | b;
      const int c = __popc(u);
      int incl = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      int pos = base + incl - c;
      while (u) {
        const int bit = __ffs(u) - 1;
        const uint32_t m = 1u << bit;
        U[pos++] = (uint32_t)(w * 32 + bit) | ((a & m) ? FLAG_A : 0u) | ((b & m) ? FLAG_B : 0u);
        u &= u - 1u;
      }
      base += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) misc[1] = (uint32_t)base;
  }
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = misc[0];
  const int n_list = (int)misc[1];
  const int nv = RECT ? ntp / 64 : 0;  // pooled tiles after the listed ones
  const int n = n_list + nv;
  // ln n_kt / scale per pooled key (-inf past Nt), 16-byte aligned for float4 reads
  float *bias = reinterpret_cast<float *>((reinterpret_cast<uintptr_t>(U + nt + nv) + 15u) & ~uintptr_t(15));
  if (RECT) {
    for (int u = tid; u < nv; u += NUM_THREADS) U[n_list + u] = (uint32_t)u | VIRT | FLAG_A | FLAG_B;
    const float ln2_over = 1.0f / scale_log2;  // log2(n) / scale_log2 = ln(n) / scale
    for (int kt = tid; kt < ntp; kt += NUM_THREADS) {
      float b = -INFINITY;
      if (kt < nt) {
        const int rem = kt % (g.NH * g.NW);
        const int ty = rem / g.NW, tx = rem - ty * g.NW;
        b = log2f((float)(valid_extent(g.H, ty) * valid_extent(g.W, tx))) * ln2_over;
      }
      bias[kt] = b;
    }
  }
  // Mark key tiles cut by the grid edge once per entry, so that the softmax
  // loop needs no division to find them.
  for (int i = tid; i < n_list; i += NUM_THREADS) {
    const uint32_t e = U[i];
    const int kt = (int)(e & KT_MASK);
    const int rem = kt % (g.NH * g.NW);
    const int ty = rem / g.NW, tx = rem - ty * g.NW;
    const int vy = valid_extent(g.H, ty), vx = valid_extent(g.W, tx);
    if (vy < 8 || vx < 8) U[i] = e | EXT_PARTIAL | ((uint32_t)(vy - 1) << 20) | ((uint32_t)(vx - 1) << 23);
  }
  __syncthreads();

  // Every role walks the list from the first key tile at or after the CTA's
  // own query tile and wraps around (any order gives the same softmax up to
  // rounding): CTAs that run side by side then start on different key tiles
  // instead of all asking L2 for the same low-numbered ones at once.
  int rot = 0;
  {
    int lo = 0, hi = n_list;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if ((int)(U[mid] & KT_MASK) < qtA) lo = mid + 1; else hi = mid;
    }
    rot = (lo < n) ? lo : 0;
  }
  auto uidx = [&](int j) { const int t = j + rot; return t < n ? t : t - n; };

  int issued_k = 0, issued_v = 0;  // K / V tiles the producer has loaded
  if (warp == WARP_PRODUCER) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0 && n > 0) {
      // all d-atoms of tile `tile` of this (b, h) into dst (+ 8192 per atom
      // for K and V, + Q_REGION for Q)
      auto load_tile_atoms = [&](const CUtensorMap *map, uint64_t *bar, uint32_t dst, uint32_t atom_step,
                                 int tile) {
        if (!dbg_ok(tile >= 0 && tile < nt)) return;
        if (RASTER) {
          const int tpf = g.NH * g.NW;
          const int t = tile / tpf, rem = tile - t * tpf;
          const int ty = rem / g.NW, tx = rem - ty * g.NW;
          const int b = bh / heads, h = bh - b * heads;
#pragma unroll
          for (int kb = 0; kb < C::KB; ++kb)
            tc::tma_load_5d(dst + kb * atom_step, map, bar, kb * 64, h, tx * 8, ty * 8, b * g.T + t);
        } else {
          const int row = (int)(((long long)bh * nt + tile) * 64);
#pragma unroll
          for (int kb = 0; kb < C::KB; ++kb) tc::tma_load_2d(dst + kb * atom_step, map, bar, kb * 64, row);
        }
      };
      tc::mbar_expect_tx(q_full, (hasB ? 2 : 1) * C::TILE_BYTES);
      load_tile_atoms(&tm_q, q_full, sbase + C::OFF_Q, C::Q_REGION, qtA);
      if (hasB) load_tile_atoms(&tm_q, q_full, sbase + C::OFF_Q + 8192, C::Q_REGION, qtB);
      // K runs KLEAD tiles ahead of V: K_{j+1} is needed by S_{j+1}, which the
      // MMA warp issues before P.V_j.
      auto load_tile = [&](const CUtensorMap *map, const CUtensorMap *pooled_map, uint64_t *full,
                           uint64_t *empty, int off, int ns, int j) -> bool {
        const int s = j % ns, u = j / ns;
        if (u > 0 && !tc::mbar_wait(empty + s, (u - 1) & 1, abort_flag, wait_limit)) return false;
        const uint32_t e = U[uidx(j)];
        const int kt = (int)(e & KT_MASK);
        tc::mbar_expect_tx(full + s, C::TILE_BYTES);
        if (RECT && (e & VIRT) != 0u) {
          // 64 pooled rows [64 kt, 64 kt + 64) of this head
          const int row = (int)((long long)bh * ntp + 64LL * kt);
          if (!dbg_ok(kt >= 0 && 64LL * kt + 64 <= ntp)) return true;
#pragma unroll
          for (int kb = 0; kb < C::KB; ++kb)
            tc::tma_load_2d(sbase + off + s * C::TILE_BYTES + kb * 8192, pooled_map, full + s, kb * 64, row);
        } else {
          load_tile_atoms(map, full + s, sbase + off + s * C::TILE_BYTES, 8192u, kt);
        }
        return true;
      };
      bool ok = true;
      for (int j = 0; ok && j < C::KLEAD && j < n; ++j) {
        ok = load_tile(&tm_k, &tm_kbar, k_full, k_empty, C::OFF_K, C::NSK, j);
        if (ok) issued_k = j + 1;
      }
      for (int j = 0; ok && j < n; ++j) {
        if (j + C::KLEAD < n) {
          ok = load_tile(&tm_k, &tm_kbar, k_full, k_empty, C::OFF_K, C::NSK, j + C::KLEAD);
          if (!ok) break;
          issued_k = j + C::KLEAD + 1;
        }
        ok = load_tile(&tm_v, &tm_vbar, v_full, v_empty, C::OFF_V, C::NSV, j);
        if (ok) issued_v = j + 1;
      }
    }
    __syncwarp();
  } else if (warp == WARP_MMA) {
    // ------------------------------------------------------ MMA issuer
    if (lane == 0 && n > 0) {
      bool ok = tc::mbar_wait(q_full, 0, abort_flag, wait_limit);
      tc::fence_after();
      auto issue_s = [&](int j) -> bool {
        const int s = j % C::NSK;
        if (!tc::mbar_wait(k_full + s, (j / C::NSK) & 1, abort_flag, wait_limit)) return false;
        tc::fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)((j & 1) * 64);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t koff = (uint32_t)((kk & 3) * 32);
          const uint64_t a = tc::desc_k_sw128(sbase + C::OFF_Q + (kk >> 2) * C::Q_REGION + koff);
          const uint64_t b =
              tc::desc_k_sw128(sbase + C::OFF_K + s * C::TILE_BYTES + (kk >> 2) * 8192 + koff);
          tc::mma_ss(d_tmem, a, b, C::IDESC_S, kk > 0 ? 1u : 0u);
        }
        tc::mma_commit(s_full + (j & 1));
        tc::mma_commit(k_empty + s);
        return true;
      };
      auto issue_pv = [&](int j) -> bool {
        const int s = j % C::NSV;
        if (!tc::mbar_wait(p_full + (j & 1), (j >> 1) & 1, abort_flag, wait_limit)) return false;
        if (!tc::mbar_wait(v_full + s, (j / C::NSV) & 1, abort_flag, wait_limit)) return false;
        tc::fence_after();
        const uint32_t p_tmem = tmem + (uint32_t)((j & 1) * 64);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t b =
              tc::desc_mn_sw128(sbase + C::OFF_V + s * C::TILE_BYTES + kk * 2048, 8192u);
          tc::mma_ts(tmem + O_COL, p_tmem + (uint32_t)(kk * 8), b, C::IDESC_O,
                     (j > 0 || kk > 0) ? 1u : 0u);
        }
        tc::mma_commit(v_empty + s);
        tc::mma_commit(o_done);
        return true;
      };
      if (ok) ok = issue_s(0);
      for (int j = 1; ok && j < n; ++j) {
        ok = issue_s(j);
        if (ok) ok = issue_pv(j - 1);
      }
      if (ok) ok = issue_pv(n - 1);
      // All issued MMAs must retire before TMEM is released: a wait on the
      // CTA's own work, so the long limit whatever the pipeline limit.
      tc::mma_commit(mma_done);
      tc::mbar_wait(mma_done, 0, nullptr, DRAIN_LIMIT);
    }
    __syncwarp();
  } else {
    // ------------------------------------------- softmax / correction / epilogue
    const bool halfB = warp >= 2;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    float m = -INFINITY, l = 0.0f;
    bool ok = true;
    // cached log-sum-exp of this thread's query token (MASS), in log2 units
    float lin = -INFINITY, inv_nq = 0.0f;
    const int qt_half = halfB ? qtB : qtA;
    if (MASS && (!halfB || hasB)) {
      const int rem = qt_half % (g.NH * g.NW);
      const int ty = rem / g.NW, tx = rem - ty * g.NW;
      const int vy = valid_extent(g.H, ty), vx = valid_extent(g.W, tx);
      const int rr = tid & 63;
      inv_nq = 1.0f / (float)(vy * vx);
      if ((rr >> 3) < vy && (rr & 7) < vx)
        lin = lse_in[(long long)bh * g.Lpad + (long long)qt_half * 64 + rr] * 1.4426950408889634f;
    }
    for (int j = 0; j < n; ++j) {
      const int buf = j & 1;
      const bool got = tc::mbar_wait(s_full + buf, (j >> 1) & 1, abort_flag, wait_limit);
      if (!__all_sync(0xffffffffu, got)) {
        ok = false;
        break;
      }
      tc::fence_after();
      const uint32_t e = U[uidx(j)];
      const bool mine = halfB ? (e & FLAG_B) != 0u : (e & FLAG_A) != 0u;
      const uint32_t sS = tmem + lane_base + (uint32_t)(buf * 64);
      uint32_t pk[32];
      if (!mine) {
#pragma unroll
        for (int c = 0; c < 32; ++c) pk[c] = 0u;
        tc::tmem_st32(sS, pk);
      } else {
        float s[64];
        {
          uint32_t rr[64];
          tc::tmem_ld64(sS, rr);
#pragma unroll
          for (int c = 0; c < 64; ++c) s[c] = __uint_as_float(rr[c]);
        }
        // pooled tiles (rectified form): columns of listed tiles and past Nt
        // are masked; the others get their multiplicity bias ln n / scale
        if (RECT && (e & VIRT) != 0u) {
          const int u = (int)(e & KT_MASK);
          const uint32_t *bm = halfB ? bmB : bmA;
          // columns the row does not list; the bias is -inf past Nt
          const uint32_t a0 = (2 * u < wpr) ? ~bm[2 * u] : ~0u;
          const uint32_t a1 = (2 * u + 1 < wpr) ? ~bm[2 * u + 1] : ~0u;
          const float4 *b4 = reinterpret_cast<const float4 *>(bias + 64 * u);
#pragma unroll
          for (int c4 = 0; c4 < 16; ++c4) {
            const float4 b = b4[c4];
            const float bb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int c = 4 * c4 + q;
              const bool on = (((c < 32) ? (a0 >> c) : (a1 >> (c - 32))) & 1u) != 0u;
              s[c] = on ? s[c] + bb[q] : -INFINITY;
            }
          }
        }
        // keys of partial tiles beyond the grid edge
        const int kt = (int)(e & KT_MASK);
        if (e & EXT_PARTIAL) {
          const int vy = (int)((e >> 20) & 7u) + 1, vx = (int)((e >> 23) & 7u) + 1;
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if ((c >> 3) >= vy || (c & 7) >= vx) s[c] = -INFINITY;
        }
        // row max: a tree of three-input maxima (max is exact in any order)
        float t22[22];
#pragma unroll
        for (int c = 0; c < 21; ++c) t22[c] = tc::fmax3(s[3 * c], s[3 * c + 1], s[3 * c + 2]);
        t22[21] = s[63];
        float t8[8];
#pragma unroll
        for (int c = 0; c < 7; ++c) t8[c] = tc::fmax3(t22[3 * c], t22[3 * c + 1], t22[3 * c + 2]);
        t8[7] = t22[21];
        const float mx = tc::fmax3(tc::fmax3(t8[0], t8[1], t8[2]), tc::fmax3(t8[3], t8[4], t8[5]),
                                   fmaxf(t8[6], t8[7]));
        const float m_new = fmaxf(m, mx * scale_log2);
        const bool rescale = m_new > m + RESCALE_LOG2;
        const float m_use = rescale ? m_new : m;
        const float mref = (m_use == -INFINITY) ? 0.0f : m_use;
        const float alpha = rescale ? tc::ex2(m - m_new) : 1.0f;
        // x = s * scale_log2 - mref two lanes at a time; p = 2^x; pairs summed
        // in four packed accumulators
        const uint64_t scale2 = tc::f2_pack(scale_log2, scale_log2);
        const uint64_t negm2 = tc::f2_pack(-mref, -mref);
        uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          float x0, x1;
          tc::f2_unpack(tc::f2_fma(tc::f2_pack(s[2 * c], s[2 * c + 1]), scale2, negm2), x0, x1);
          const float p0 = tc::ex2(x0), p1 = tc::ex2(x1);
          acc[c & 3] = tc::f2_add(acc[c & 3], tc::f2_pack(p0, p1));
          pk[c] = tc::pack_bf16(p0, p1);
        }
        float sum;
        {
          float a0, a1;
          tc::f2_unpack(tc::f2_add(tc::f2_add(acc[0], acc[1]), tc::f2_add(acc[2], acc[3])), a0, a1);
          sum = a0 + a1;
        }
        tc::tmem_st32(sS, pk);
        l = l * alpha + sum;
        if (MASS) {
          float c = (lin > -INFINITY) ? sum * tc::ex2(mref - lin) : 0.0f;
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
          // two warps (32 rows each) per query tile: two adds onto zero, so the
          // result does not depend on their order
          if (lane == 0 && dbg_ok(qt_half < nt && kt < nt))
            atomicAdd(block_mass + ((long long)bh * nt + qt_half) * nt + kt, c * inv_nq);
        }
        const bool need_o = rescale && (m != -INFINITY);
        if (__any_sync(0xffffffffu, need_o)) {
          // PV_{j-1} must have retired before O is scaled (j >= 1 here). S_j
          // was issued after PV_{j-2}, so its completion proves PV_{j-2}
          // retired: o_done has completed j-1 or j phases and the parity of
          // phase j-1 is unambiguous.
          const bool got_o = tc::mbar_wait(o_done, (j - 1) & 1, abort_flag, wait_limit);
          if (!__all_sync(0xffffffffu, got_o)) {
            ok = false;
            break;
          }
          tc::fence_after();
          const float a = need_o ? alpha : 1.0f;
#pragma unroll
          for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t o[32];
            tc::tmem_ld32(tmem + lane_base + O_COL + cc * 32, o);
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * a);
            tc::tmem_st32(tmem + lane_base + O_COL + cc * 32, o);
          }
        }
        m = m_use;
      }
      tc::tmem_wait_st();
      tc::fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(p_full + buf);
    }
    // a warp that left the loop early may still have its P store in flight
    tc::tmem_wait_st();
    // ---- epilogue
    // Wait on the single-use barrier committed after the last P.V: o_done's
    // parity cannot tell PV_{n-1} from PV_{n-2} here, because the last S MMA
    // was issued before PV_{n-2} and so proves only PV_{n-3} retired.
    if (ok && n > 0) ok = tc::mbar_wait(mma_done, 0, abort_flag, wait_limit);
    ok = __all_sync(0xffffffffu, ok);
    tc::fence_after();
    const bool row_exists = !halfB || hasB;
    if (ok && row_exists) {
      const int qt = halfB ? qtB : qtA;
      const long long orow = (long long)bh * g.Lpad + (long long)qt * 64 + (tid & 63);
      const float inv_l = (l > 0.0f) ? 1.0f / l : 0.0f;
      // destination row: tiled row orow, or the token's raster row (none for
      // the pad rows of a tile cut by the grid edge)
      long long dst_row = orow;
      bool store_row = true;
      if (RASTER) {
        const int tpf = g.NH * g.NW;
        const int t = qt / tpf, rem = qt - t * tpf;
        const int ty = rem / g.NW, tx = rem - ty * g.NW;
        const int r = tid & 63;
        const int y = ty * 8 + (r >> 3), x = tx * 8 + (r & 7);
        const int b = bh / heads, h = bh - b * heads;
        store_row = y < g.H && x < g.W;
        dst_row = (((long long)(b * g.T + t) * g.H + y) * g.W + x) * heads + h;
      }
      const bool rows_ok = dbg_ok(orow < (long long)gridDim.y * g.Lpad &&
                                  (!RASTER || !store_row || dst_row < (long long)gridDim.y * g.T * g.H * g.W));
      if (!rows_ok) store_row = false;
      uint4 *dst = reinterpret_cast<uint4 *>(out + dst_row * D);
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t o[32];
        if (n > 0) {
          tc::tmem_ld32(tmem + lane_base + O_COL + cc * 32, o);
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] = 0u;
        }
        uint32_t pk[16];
#pragma unroll
        for (int c = 0; c < 16; ++c)
          pk[c] = tc::pack_bf16(__uint_as_float(o[2 * c]) * inv_l, __uint_as_float(o[2 * c + 1]) * inv_l);
        if (store_row) {
#pragma unroll
          for (int v = 0; v < 4; ++v)
            dst[cc * 4 + v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
        }
      }
      if (lse != nullptr && rows_ok)
        lse[orow] = (l > 0.0f) ? (m + log2f(l)) * 0.69314718055994530942f : -INFINITY;
    }
  }
  // Every role has left its loop, so a timeout in any of them has raised the
  // abort flag by now. The copies the producer issued must land before the
  // CTA's shared memory is released: after an abort it waits for the last
  // use of every ring slot (an older use was consumed before its slot was
  // refilled) and for Q.
  __syncthreads();
  if (warp == WARP_PRODUCER && lane == 0 && n > 0 && *abort_flag) {
    tc::mbar_wait(q_full, 0, nullptr, DRAIN_LIMIT);
    for (int j = (issued_k > C::NSK ? issued_k - C::NSK : 0); j < issued_k; ++j)
      tc::mbar_wait(k_full + j % C::NSK, (j / C::NSK) & 1, nullptr, DRAIN_LIMIT);
    for (int j = (issued_v > C::NSV ? issued_v - C::NSV : 0); j < issued_v; ++j)
      tc::mbar_wait(v_full + j % C::NSV, (j / C::NSV) & 1, nullptr, DRAIN_LIMIT);
  }
  tc::fence_before();
  __syncthreads();
  if (warp == WARP_MMA) {
    tc::fence_after();
    tc::tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace attn
}  // namespace sta
