/*
 * sta_probe.h -- C ABI of libsta_probe: measurement probes of the two hardware
 * paths the attention kernel of libsta (include/sta.h) is built on, on B200
 * (sm_100a). They compute nothing of the method; they give the denominators
 * the attention kernel is read against: the rate at which TMA brings key
 * tiles from L2 into shared memory, and the cost of one tcgen05 MMA shape.
 * Types and status codes are those of sta.h.
 */
#ifndef STA_PROBE_H
#define STA_PROBE_H

#include "sta.h"

#ifdef __cplusplus
extern "C" {
#endif

/* sta_probe_tma_stream -- the attention kernel's load stream on its own:
 * ctas_per_sm CTAs per SM, each keeping `slots` (1..6) 16 KB key-tile loads
 * in flight (two 64x64 bf16 TMA boxes with 128 B swizzle, as the kernel
 * loads K and V), from pseudo-random tiles of buf (device, bytes >= 16 KB,
 * 16-byte aligned), `iters` loads per CTA; slots x 16 KB x ctas_per_sm must
 * fit in 200 KB. The caller times it; bytes moved = SMs x ctas_per_sm x
 * iters x 16384. It measures the L2-to-SM rate the hardware gives such loads
 * when nothing else runs (a denominator for the attention's load stream). */
sta_status sta_probe_tma_stream(const void *buf, size_t bytes, int32_t ctas_per_sm, int32_t slots,
                                int32_t iters, sta_stream_t stream);

/* sta_probe_mma_rate -- the tensor-core rate of one MMA shape on its own:
 * one CTA per SM of the current device issues `iters` (1..2^20) back-to-back
 * tcgen05.mma of kind::f16 (bf16 x bf16 -> fp32) with M = 128, K = 16 and
 * N = n (64, 128 or 256), A from shared memory (a_in_tmem = 0) or from
 * tensor memory (a_in_tmem != 0), B from shared memory, into one
 * accumulator. cycles: device int64 array with one entry per SM of the
 * current device, written with each CTA's SM cycles from the first issue to
 * completion (-1 if its bounded wait gave up). cycles / iters is the cost
 * of one MMA; 128 * n * 16 / that is the multiply-adds per clock (4096 is
 * the dense bf16 peak of an SM).
 * Arguments out of range give STA_ERR_INVALID_ARG before anything runs. */
sta_status sta_probe_mma_rate(int32_t n, int32_t a_in_tmem, int32_t iters, int64_t *cycles,
                              sta_stream_t stream);

/* Reads and clears this library's device error word (a probe whose bounded
 * wait gave up records STA_ERR_TIMEOUT there) after synchronising `stream`. */
sta_status sta_probe_get_device_error(sta_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* STA_PROBE_H */
