/*
 * qattn_probe.h — measurement aid of the B200 quantized attention library: the
 * tensor-core throughput probe that the attention mainloop's roofline fraction
 * is reported against.  The pages have no counterpart; it measures the machine,
 * not the method.
 */
#ifndef QATTN_PROBE_H_
#define QATTN_PROBE_H_

#include "qattn.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Dense tensor-core peak probe.  Launches n_ctas CTAs (one per SM when n_ctas is
 * the SM count; each CTA takes 116 KB of shared memory); in each, one thread
 * issues `iters` back-to-back tcgen05.mma of shape M128 N256 K32 with both
 * operands in shared memory, accumulating in tensor memory:
 *   kind 0: kind::i8      (s8 x s8 -> s32)
 *   kind 1: kind::f8f6f4  (e4m3 x e4m3 -> f32)
 * One launch performs n_ctas * iters * 2 * 128 * 256 * 32 operations; time it with
 * CUDA events on `stream`.  `cycles` (device, one uint64, caller-owned) receives
 * the largest number of SM clock cycles any CTA spent from its first issue to the
 * completion of its last MMA, so ops per clock per SM = iters * 2*128*256*32 /
 * cycles.  Stream-ordered and asynchronous.
 * Errors: SHAPE (kind not 0/1, iters not in [1, 2^20], n_ctas not in [1, 2^16]),
 * NULL, UNSUPPORTED (not sm_100), CUDA; TIMEOUT via dev_err (not expected: the
 * MMAs of the largest launch take far less than the one-second wait bound). */
qattn_status qattn_tc_probe(int kind, int iters, int n_ctas, unsigned long long* cycles,
                            int* dev_err, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* QATTN_PROBE_H_ */
