/*
 * bsfa_trace.h - cycle trace of the BSFA forward kernel, exported only by the
 * trace build of the library (libbsfa_trace.so, compiled with -DBSFA_TRACE); the
 * regular library (libbsfa.so) contains no trace code. A profiling aid: it
 * shows where each role of the kernel (softmax warpgroups, MMA issuer, TMA
 * producers, S waiter) spends its cycles, step by step.
 */
#ifndef BSFA_TRACE_H_
#define BSFA_TRACE_H_

#include "bsfa.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * bsfa_trace_attach - make every following forward launch on any device stamp
 * the SM clock (clock64) at fixed points of its first `ctas` CTAs into `buf`.
 *
 *   buf   device memory, 8-byte aligned, at least ctas * bsfa_trace_stride()
 *         unsigned 64-bit words, owned by the caller; NULL with ctas = 0 turns
 *         tracing off
 *   ctas  CTAs (in launch order, blockIdx.x) to record
 *
 * Layout of a CTA's words (steps past 64 are not recorded): [0] start, [1] SM
 * id, [2] end; then per slot s and block step j the softmax stamps (S ready,
 * row maxima taken, gate passed, exponentials done, P stored, P announced), the
 * MMA issuer's (P seen, MMAs issued), the S waiter's (S seen), the V producer's
 * (decision seen, load issued), the K producer's (load issued) and the
 * epilogue's (O ready, rows written). threshold_gated_block_b200/trace.py reads it.
 * Returns BSFA_ERR_INVALID_ARG for a negative count or a missing or misaligned buffer.
 */
bsfa_status bsfa_trace_attach(void* buf, int ctas);

/* bsfa_trace_stride - 64-bit words recorded per CTA. */
int bsfa_trace_stride(void);

#ifdef __cplusplus
}
#endif

#endif /* BSFA_TRACE_H_ */
