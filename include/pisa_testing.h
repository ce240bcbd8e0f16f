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

/* Sets the fault injected into subsequent bf16 pisa_attention calls of this process and the
 * bounded-wait limit they use (0 = the default of 2 s).  Process-wide, not thread-safe; pass
 * PISA_TESTING_FAULT_NONE and 0 to restore normal behaviour.  Returns PISA_ERR_INVALID_ARG for an
 * unknown fault. */
PISA_API pisa_status pisa_testing_set_attention_fault(int32_t fault, uint64_t wait_limit_ns);

#ifdef __cplusplus
}
#endif

#endif /* PISA_TESTING_H_ */
