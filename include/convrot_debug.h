/*
 * convrot_debug.h — the debug library, libconvrot_debug.so (no counterpart on
 * the pages: a test aid of this library).
 *
 * libconvrot_debug.so is built from the same sources as libconvrot.so with
 * CONVROT_DEBUG=1 and exports everything include/convrot.h declares, with the
 * same behaviour, plus two things:
 *   - every kernel checks the indices of its global stores (and of the
 *     per-token and per-channel scale and bias reads) against the sizes of
 *     the tensors it was given.  An index out of range sets bit 1 of the
 *     device status word and the access is skipped: nothing traps, nothing
 *     writes outside its tensor.  convrot_check_status then returns
 *     CONVROT_ERR_BOUNDS (and clears the word).
 *   - convrot_debug_set_fault() injects a fault from the host into the
 *     kernels launched after it, so that tests can drive the error paths
 *     without a real fault.
 * libconvrot.so exports neither.  Use the debug library for tests only: the
 * checks cost time.
 */
#ifndef CONVROT_DEBUG_H_
#define CONVROT_DEBUG_H_

#include "convrot.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Fault injected into every kernel launched after this call, until it is
 * called again with CONVROT_FAULT_NONE (process-wide; not thread-safe with
 * respect to concurrent launches):
 *   CONVROT_FAULT_SKIP_STAGE  the int8 GEMMs' producers leave the first
 *       stage of their shared-memory ring empty (no expected bytes, no
 *       copies).  The consumer's bounded wait on it runs out after about a
 *       second; the kernel stops issuing work, lets its copies land, frees
 *       its tensor memory and returns; convrot_check_status reports
 *       CONVROT_ERR_TIMEOUT.  The outputs are undefined.
 *   CONVROT_FAULT_SHORT_ROWS  the kernels check their stores against one
 *       row fewer than the output holds (256 elements fewer for the weight
 *       decode and quantization, which see the weight as one flat array):
 *       those stores are caught and skipped, and convrot_check_status
 *       reports CONVROT_ERR_BOUNDS.  Every other output is the normal one.
 * Returns CONVROT_ERR_INVALID_ARG for an unknown code.
 */
#define CONVROT_FAULT_NONE 0
#define CONVROT_FAULT_SKIP_STAGE 1
#define CONVROT_FAULT_SHORT_ROWS 2
convrot_status convrot_debug_set_fault(int fault);

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif /* CONVROT_DEBUG_H_ */
