/*
 * pisa_testing.h — test-only hooks of the PISA library.  Not for production callers.
 *
 * The method's description has no counterpart to these calls; they exist so that tests can check
 * the library's failure detection without faulting or hanging a GPU.
 */
#ifndef PISA_TESTING_H_
#define PISA_TESTING_H_

#include "pisa.h"

#ifdef __cplusplus
extern "C" {
#endif

#define PISA_TESTING_FAULT_NONE 0
/* The attention kernel's load warp does not load the query tile, so the MMA warp's bounded wait
 * for it runs out: the kernel must record PISA_DEVERR_WAIT_TIMEOUT, drain its own work, free its
 * tensor memory and return, leaving the context usable. */
#define PISA_TESTING_FAULT_SKIP_Q_LOAD 1

/* The first pass of the bf16 pre-computation does not load the first tile of each CTA's first
 * group of key blocks, so the MMA warp's bounded wait for it runs out: every CTA must record
 * PISA_DEVERR_WAIT_TIMEOUT, give up the rest of its groups, drain its own work, free its tensor
 * memory and return; the H-bar reduction and the second pass, which wait for it, then run to the
 * end on whatever the workspace holds. */
#define PISA_TESTING_FAULT_SKIP_TILE_LOAD 2

/* Sets the fault injected into subsequent bf16 pisa_attention calls of this process and the
 * bounded-wait limit they use (0 = the default of 2 s).  Process-wide, not thread-safe; pass
 * PISA_TESTING_FAULT_NONE and 0 to restore normal behaviour.  Returns PISA_ERR_INVALID_ARG for an
 * unknown fault. */
PISA_API pisa_status pisa_testing_set_attention_fault(int32_t fault, uint64_t wait_limit_ns);

/* The same for subsequent bf16 pisa_precompute calls (and the entry points that run it):
 * PISA_TESTING_FAULT_NONE or PISA_TESTING_FAULT_SKIP_TILE_LOAD, and the bounded-wait limit of the
 * pre-computation kernels (0 = the default of 2 s).  Process-wide, not thread-safe.  Returns
 * PISA_ERR_INVALID_ARG for an unknown fault. */
PISA_API pisa_status pisa_testing_set_precompute_fault(int32_t fault, uint64_t wait_limit_ns);

#ifdef __cplusplus
}
#endif

#endif /* PISA_TESTING_H_ */
