/*
 * attn_timeline.h -- read-out of the kernel timeline.  Exported only by
 * libattn_timeline.so, a second build of the same sources with -DATTN_TIMELINE
 * (python -m attention_attn_fwd_10_b200.build --timeline); the default
 * libattn.so has neither the symbol nor the instrumentation.
 *
 * In the timeline build, the CTA whose blockIdx.x equals the selected index
 * records clock64() (its SM's cycle counter) at fixed points of its pipeline:
 * event ev of its block i goes to events[ev * 256 + i], for i < 256, and the CTA's
 * start to *t0.  The forward records, per key block j of each tile t (0 = A,
 * 1 = B): 0 + t S_t(j) ready at the softmax, 2 + t row max done, 4 + t P_t(j)
 * published, 6 + t PV_t(j) issued, 8 + t S_t(j) issued (for j >= 1: it follows
 * PV_t(j - 1)), 10 V block j ready at the issuer, 15 V block j's load issued; per
 * work unit u: 11 + t O_t final at the softmax, 13 + t the epilogue done.  The
 * backward main pass (one CTA per key tile) records, per query block:
 * 0 S^T/dP^T issued, 1 S^T ready at the softmax, 2 dS^T published, 3 dS^T seen by
 * the issuer, 4 dV/dK issued, 5 dQ^T issued, 6 dQ^T ready at the staging warps,
 * 7 the dQ tile staged, 8 its reduce-add issued, 9 its source read (in the fixed
 * dQ order: its additions performed and the turn passed on), 10 (fixed dQ order)
 * the turn received, before the reduce-add is issued.  The pair backward records
 * the same events (the issuer's in the even CTA of a pair only) and 11 its dS^T
 * half sent to the other CTA, 12 the issuer holds both CTAs' dS^T halves and the
 * previous dQ^T has been read out, 13 (odd CTA) the even CTA's half landed.
 * Events that
 * did not happen read 0.  The recording changes no result of any kernel.
 */
#ifndef ATTN_TIMELINE_H
#define ATTN_TIMELINE_H

#include "attn.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Synchronises the device, copies the recorded events (16 x 256 int64, host
 * memory of the caller) and the start stamp to `events` and `t0`, clears the
 * events, and selects CTA `next_cta` (-1: none) for the kernels launched after
 * this call.  ATTN_ERR_INVALID_ARG for a null pointer, ATTN_ERR_CUDA if a copy
 * fails. */
attn_status_t attn_timeline_read(long long* events, long long* t0, int next_cta);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_TIMELINE_H */
