// libsta_probe: measurement probes of the hardware paths the attention
// kernel of libsta uses (declared in include/sta_probe.h). They are not part of
// the method and live apart from the product library: the TMA load stream of
// key tiles on its own, and the cost of one tcgen05 MMA shape on its own.
#include "sta_common.cuh"
#include "sta_host.cuh"
#include "sta_tc.cuh"

#include "../../include/sta_probe.h"

using namespace sta;

namespace {

// The attention kernel's load stream without its compute: one thread per CTA
// keeps `slots` 16 KB key-tile loads (two 64x64 bf16 boxes, 128 B swizzle,
// as the kernel issues them) in flight from `tiles` tiles of buf, at
// pseudo-random tile indices, for `iters` loads. Timed by the caller; it
// gives the L2-to-SM rate TMA reaches on this GPU at a given depth.
constexpr int STREAM_MAX_SLOTS = 6;
__global__ void __launch_bounds__(32) tma_stream_kernel(const __grid_constant__ CUtensorMap tm, int tiles,
                                                        int slots, int iters) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t *bar = reinterpret_cast<uint64_t *>(smem + slots * 16384);
  if (threadIdx.x != 0) return;
  for (int sl = 0; sl < slots; ++sl) tc::mbar_init(bar + sl, 1);
  tc::fence_barrier_init();
  uint32_t seed = blockIdx.x * 2654435761u + 12345u;
  auto issue = [&](int sl) {
    seed = seed * 1664525u + 1013904223u;
    const int tile = (int)(seed % (uint32_t)tiles);
    tc::mbar_expect_tx(bar + sl, 16384);
    tc::tma_load_2d(tc::smem_u32(smem + sl * 16384), &tm, bar + sl, 0, tile * 64);
    tc::tma_load_2d(tc::smem_u32(smem + sl * 16384 + 8192), &tm, bar + sl, 64, tile * 64);
  };
  int issued = 0;
  for (; issued < slots && issued < iters; ++issued) issue(issued);
  for (int i = 0; i < iters; ++i) {
    const int sl = i % slots;
    // spin without a suspend hint, so that the wait adds no wake-up delay to
    // the rate being measured; bounded, then recorded like the pipeline waits
    bool ok = false;
    for (long long spin = 0; spin < 100000000LL && !ok; ++spin) ok = tc::mbar_try_wait(bar + sl, (i / slots) & 1);
    if (!ok) {
      record_error(DEV_ERR_TIMEOUT);
      for (int j = i + 1; j < issued; ++j) tc::mbar_wait(bar + j % slots, (j / slots) & 1, nullptr, 200000000LL);
      return;
    }
    if (issued < iters) issue(issued++ % slots);
  }
}

// Back-to-back tcgen05.mma (kind::f16, bf16 x bf16 -> fp32, M = 128, K = 16)
// of one N, A from shared memory (A_TMEM = false) or from TMEM, B from shared
// memory, all into one accumulator; the operands are zeros (their values do
// not change the rate). One thread issues `iters` MMAs and waits for them;
// cycles[blockIdx.x] gets the SM cycles from the first issue to completion.
// One CTA per SM: the dynamic shared memory asked for keeps two off one SM.
constexpr int MMA_RATE_SMEM = 120 * 1024;
template <int N, bool A_TMEM>
__global__ void __launch_bounds__(128, 1) mma_rate_kernel(long long *cycles, int iters) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
  __shared__ uint64_t bar;
  __shared__ uint32_t taddr;
  const int tid = threadIdx.x;
  // A: 128 rows x 128 B; B: N rows x 128 B (K-major, 128-byte swizzle)
  for (int i = tid; i < (16384 + N * 128) / 16; i += 128) reinterpret_cast<uint4 *>(smem)[i] = make_uint4(0, 0, 0, 0);
  if (tid == 0) {
    tc::mbar_init(&bar, 1);
    tc::fence_barrier_init();
  }
  if (tid < 32) {
    tc::tmem_alloc(&taddr, 512);
    tc::tmem_relinquish();
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // zeros visible to the tensor core
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tm = taddr;
  if (tid == 0) {
    const uint32_t sa = tc::smem_u32(smem), sb = sa + 16384;
    constexpr uint32_t idesc = tc::idesc_bf16(128, N, false);
    const long long t0 = clock64();
    for (int i = 0; i < iters; ++i) {
      const uint32_t koff = (uint32_t)((i & 3) * 32);  // the four K = 16 steps of a 128-byte row
      if (A_TMEM)
        tc::mma_ts(tm, tm + 256u + (uint32_t)((i & 3) * 8), tc::desc_k_sw128(sb + koff), idesc, i > 0 ? 1u : 0u);
      else
        tc::mma_ss(tm, tc::desc_k_sw128(sa + koff), tc::desc_k_sw128(sb + koff), idesc, i > 0 ? 1u : 0u);
    }
    tc::mma_commit(&bar);
    const bool ok = tc::mbar_wait(&bar, 0, nullptr, 2000000000LL);
    cycles[blockIdx.x] = ok ? clock64() - t0 : -1;
  }
  tc::fence_before();
  __syncthreads();
  if (tid < 32) {
    tc::fence_after();
    tc::tmem_dealloc(tm, 512);
  }
}

template <int N, bool A_TMEM>
sta_status launch_mma_rate(long long *cycles, int iters, int sms, cudaStream_t s) {
  auto kern = mma_rate_kernel<N, A_TMEM>;
  STA_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, MMA_RATE_SMEM));
  kern<<<(unsigned)sms, 128, MMA_RATE_SMEM, s>>>(cycles, iters);
  STA_CUDA_TRY(cudaGetLastError());
  return STA_OK;
}

}  // namespace

extern "C" {

sta_status sta_probe_tma_stream(const void *buf, size_t bytes, int32_t ctas_per_sm, int32_t slots,
                                int32_t iters, sta_stream_t stream) {
  if (buf == nullptr || (reinterpret_cast<uintptr_t>(buf) & 15u) != 0 || bytes < 16384) return STA_ERR_INVALID_ARG;
  if (ctas_per_sm < 1 || ctas_per_sm > 8 || slots < 1 || slots > STREAM_MAX_SLOTS || iters < 1 ||
      (long long)slots * 16384 * ctas_per_sm > 200 * 1024)
    return STA_ERR_INVALID_ARG;
  if (!device_is_sm100()) return STA_ERR_UNSUPPORTED;
  const long long tiles = (long long)(bytes / 16384);
  if (tiles * 64 >= (1LL << 31)) return STA_ERR_UNSUPPORTED;
  CUtensorMap tm;
  if (!make_tile_map(&tm, buf, (unsigned long long)tiles * 64, 128)) return STA_ERR_CUDA;
  int dev = 0, sms = 0;
  STA_CUDA_TRY(cudaGetDevice(&dev));
  STA_CUDA_TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  const size_t smem = (size_t)slots * 16384 + 64 + 1024;
  STA_CUDA_TRY(cudaFuncSetAttribute(tma_stream_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)((size_t)STREAM_MAX_SLOTS * 16384 + 64 + 1024)));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // ctas_per_sm CTAs per SM through the grid size; they fit on an SM at once
  // (checked above)
  tma_stream_kernel<<<(unsigned)(sms * ctas_per_sm), 32, smem, s>>>(tm, (int)tiles, slots, iters);
  STA_CUDA_TRY(cudaGetLastError());
  return STA_OK;
}

sta_status sta_probe_mma_rate(int32_t n, int32_t a_in_tmem, int32_t iters, int64_t *cycles,
                              sta_stream_t stream) {
  if ((n != 64 && n != 128 && n != 256) || iters < 1 || iters > (1 << 20) || cycles == nullptr)
    return STA_ERR_INVALID_ARG;
  if (!device_is_sm100()) return STA_ERR_UNSUPPORTED;
  const int sms = sm_count();
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  long long *out = reinterpret_cast<long long *>(cycles);
  if (a_in_tmem) {
    if (n == 64) return launch_mma_rate<64, true>(out, iters, sms, s);
    if (n == 128) return launch_mma_rate<128, true>(out, iters, sms, s);
    return launch_mma_rate<256, true>(out, iters, sms, s);
  }
  if (n == 64) return launch_mma_rate<64, false>(out, iters, sms, s);
  if (n == 128) return launch_mma_rate<128, false>(out, iters, sms, s);
  return launch_mma_rate<256, false>(out, iters, sms, s);
}

sta_status sta_probe_get_device_error(sta_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  STA_CUDA_TRY(cudaStreamSynchronize(s));
  unsigned int word = 0;
  STA_CUDA_TRY(cudaMemcpyFromSymbol(&word, g_dev_error, sizeof(word)));
  const unsigned int zero = 0;
  STA_CUDA_TRY(cudaMemcpyToSymbol(g_dev_error, &zero, sizeof(zero)));
  return (word & DEV_ERR_TIMEOUT) ? STA_ERR_TIMEOUT : STA_OK;
}

}  // extern "C"
