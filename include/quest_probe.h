/*
 * quest_probe.h -- measurement aid for the tensor-core roofline of the QuEST
 * integer linear layer on B200 (sm_100a).
 *
 * The pages define no such operation: the entry points below exist only so a
 * benchmark can measure the int8 MMA rate of the part it runs on, the
 * denominator of the linear layer's tensor-core fraction besides the nominal
 * dense figure.
 */
#ifndef QUEST_B200_PROBE_H
#define QUEST_B200_PROBE_H

#include "quest.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Enqueue one launch of back-to-back tcgen05.mma kind::i8 instructions
 * (M = 128, N = 256, K = 32, operands in shared memory, int32 accumulator in
 * TMEM): `iters` instructions per CTA, one CTA per SM, no global memory
 * traffic. `*ctas` receives the number of CTAs launched (host pointer). The
 * caller times the launch on `stream` (CUDA events) and computes
 * 2 * 128 * 256 * 32 * iters * ctas / seconds.
 * Errors: QUEST_EINVAL if iters is outside [1, 2^24] or ctas is NULL;
 * QUEST_ECUDA on a launch error. */
quest_status quest_probe_mma_i8(int iters, int* ctas, void* stream);

/* Synchronise `stream`; QUEST_ETIMEOUT if a probe's bounded completion wait
 * (2 s) gave up since the last call (the flag is then cleared). */
quest_status quest_probe_status(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* QUEST_B200_PROBE_H */
