/*
 * moba_trace.h -- phase traces of libmoba's tensor-core kernels. These entry
 * points exist only in the separate trace build, libmoba_trace.so
 * (python -m long_context_prefill_block_b200.build --trace), which compiles
 * the same sources with MOBA_TRACE defined; the ordinary libmoba.so exports
 * none of them. No counterpart in the paper: this is a measuring aid.
 *
 * While armed, lane 0 of every warp of CTA `cta` of kernel `kernel` records
 * (SM clock64, event id, argument) pairs at the kernel's phase boundaries
 * into buf, one region of `cap` records per warp:
 *   buf    device, unsigned long long [16][cap][2]: [0] = clock64,
 *          [1] = event id | (argument << 32)
 *   counts device, int [16]: records written per warp (may exceed cap; the
 *          surplus was dropped)
 * Kernel ids: 1 the sorting-network gate, 2 history attention, 3 own-block
 * attention, 4 dense causal attention. The event ids of each kernel are
 * listed in long_context_prefill_block_b200/trace.py. The caller owns both
 * buffers and must keep them alive until the traced launches complete.
 */
#ifndef MOBA_TRACE_H_
#define MOBA_TRACE_H_

#include "moba.h"

#ifdef __cplusplus
extern "C" {
#endif

MOBA_API moba_status moba_trace_arm(int kernel, int cta, unsigned long long* buf, int* counts,
                                    int cap);
MOBA_API moba_status moba_trace_disarm(void);

#ifdef __cplusplus
}
#endif

#endif /* MOBA_TRACE_H_ */
