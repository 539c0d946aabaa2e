/*
 * pa_timeline.h -- the per-CTA timeline readers of libpa_timeline.so, a build
 * of libpa with globaltimer stamps compiled into the decode and prefill
 * kernels (the compile-time switch PA_TIMELINE).  libpa.so has no stamps and none of
 * these symbols; libpa_timeline.so has these and everything include/pa.h
 * declares, with the same behaviour apart from the stamps' stores.  A
 * profiling aid only: the stamps cost a few stores per CTA.
 *
 * Events (u64 nanoseconds of %globaltimer, 0 = not reached), by kernel:
 *   0  shared-prefix set-up kernel: 0 entry, 1 its wait done, 2 exit
 *   1  tensor-core prefix pass: 0 entry, 1 prologue loads staged, 3 tensor
 *      memory and barriers ready, 4 first scores ready, 2 exit
 *   2  bf16 pass 1: 0 entry, 1 block-table slice staged, 3 first stage
 *      landed, 4 stream done, 2 exit (after the epilogue)
 * Layout of the events array: [3 kernels][65536 CTAs][16 slots], CTA = the
 * linear index x + gridDim.x * (y + gridDim.y * z), slot 15 = the SM id.
 * Per-tile events of the prefix pass, [512 CTAs][16 tiles][8 events]:
 *   0 softmax: scores ready, 1 softmax: P written, 3 P.V issued, 4 S issued,
 *   5 K tile requested, 6 V tile requested.
 * Each launch overwrites the CTAs it runs; pa_timeline_clear zeroes both
 * arrays (and synchronizes the device).
 *
 * The prefill kernel (pa_paged_attention_prefill) has an array of its own,
 * [65536 CTAs][8 slots], CTA = blockIdx.x, slot 7 = the SM id: 0 entry (CTAs
 * with query rows), 1 tensor memory and barriers ready, 2 tile 0's first S
 * MMA issued, 3 tile 0's last P.V issued, 4 tile 1's last P.V issued (0 if
 * the tile has no rows), 5 exit (after the epilogue).
 */
#ifndef PA_TIMELINE_H
#define PA_TIMELINE_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Zero both arrays.  0 or PA_ERR_CUDA. */
int pa_timeline_clear(void);

/* Copy the first `bytes` of the events (which = 0) or the per-tile events
 * (which = 1) to host memory dst; synchronous.  PA_ERR_INVALID_ARG for a bad
 * `which`, a NULL dst or more bytes than the array holds. */
int pa_timeline_read(int which, void* dst, size_t bytes);

/* The prefill kernel's array: zero it (and synchronize the device), or copy
 * its first `bytes` to host memory dst (synchronous; PA_ERR_INVALID_ARG for a
 * NULL dst or more bytes than the array holds).  0 or PA_ERR_CUDA. */
int pa_timeline_clear_prefill(void);
int pa_timeline_read_prefill(void* dst, size_t bytes);

#ifdef __cplusplus
}
#endif

#endif /* PA_TIMELINE_H */
