/*
 * quest_probe.h -- measurement aid for the tensor-core roofline of the QuEST
 * integer linear layer on B200 (sm_100a). Exported by the benchmark's own
 * library, libquest_probe.so, not by the product library libquest_b200.so.
 *
 * The pages define no such operation: the entry points below exist only so a
 * benchmark can measure the int8 and FP4 MMA rates of the part it runs on, the
 * denominators of the linear layers' tensor-core fractions besides the nominal
 * dense figures (and the 2:4-sparse rate of the sparse layer).
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
 * Errors: QUEST_EINVAL if iters is outside [1, 2^16] (so a launch stays far
 * inside the kernel's 2 s completion wait) or ctas is NULL;
 * QUEST_ECUDA on a launch error. */
quest_status quest_probe_mma_i8(int iters, int* ctas, void* stream);

/* The int8 kind as the linear layer issues it: CTA pairs (cluster of two CTAs on
 * two SMs, tcgen05.mma.cta_group::2.kind::i8, M = 256 across the pair, N = 256,
 * K = 32), back to back from shared memory; `*ctas` receives the number of CTAs
 * (an even count, one per SM). The caller computes
 * 2 * 256 * 256 * 32 * iters * (ctas / 2) / seconds. Errors as above. */
quest_status quest_probe_mma_i8_pair(int iters, int* ctas, void* stream);

/* The same for bf16: back-to-back tcgen05.mma kind::f16 (M = 128, N = 256,
 * K = 16, bf16 operands, fp32 accumulator); the caller computes
 * 2 * 128 * 256 * 16 * iters * ctas / seconds. Errors as above. */
quest_status quest_probe_mma_bf16(int iters, int* ctas, void* stream);

/* The same for the block-scaled FP4 kind of the FP4 linear layer: back-to-back
 * tcgen05.mma kind::mxf4 (M = 128, N = 256, K = 64, E2M1 operands in shared
 * memory, unit UE8M0 block scales in TMEM, fp32 accumulator); the caller
 * computes 2 * 128 * 256 * 64 * iters * ctas / seconds. Errors as above. */
quest_status quest_probe_mma_fp4(int iters, int* ctas, void* stream);

/* The same for the 2:4-sparse integer kind of the sparse linear layer:
 * back-to-back tcgen05.mma.sp kind::i8 (M = 128, N = 256, K = 64 logical
 * values, 32 bytes of compressed A per row, metadata in TMEM). With
 * cp_every = c > 0 a tcgen05.cp of four metadata columns from shared memory
 * precedes every c-th MMA, whose group of c MMAs then reads the copied columns;
 * cp_every = 0 keeps the metadata resident. The caller computes the
 * dense-equivalent rate 2 * 128 * 256 * 64 * iters * ctas / seconds.
 * Errors: QUEST_EINVAL if iters is outside [1, 2^16], cp_every outside
 * [0, 64] or ctas is NULL; QUEST_ECUDA on a launch error. */
quest_status quest_probe_mma_sp_i8(int iters, int cp_every, int* ctas, void* stream);

/* Synchronise `stream`; QUEST_ETIMEOUT if a probe's bounded completion wait
 * (2 s) gave up since the last call (the flag is then cleared). */
quest_status quest_probe_status(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* QUEST_B200_PROBE_H */
