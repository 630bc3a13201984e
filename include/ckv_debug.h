/*
 * ckv_debug.h -- entry points exported only by libckv_debug.so, the build
 * of libckv with -DCKV_DEBUG_BOUNDS.
 *
 * That build adds range checks to the decode kernels: every community
 * segment a kernel reads or moves (offset and size inside the member pool)
 * and the community an update writes.  A failed check sets CKV_ERR_STATE in
 * the context's error word (read by ckv_last_error) and the kernel skips
 * the access or redirects it in bounds; nothing traps.  Token rows gathered
 * from the K/V cache are checked in both builds.  Every entry point of
 * ckv.h is exported too, with the same behaviour.
 */
#ifndef CKV_DEBUG_H
#define CKV_DEBUG_H

#include "ckv.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Fault injection for the range-check tests: overwrite one int32 of the
 * context's device community state, bypassing every host check.  what 0:
 * member r of community c of graph g (a token id; r below the community's
 * size); what 1: the segment offset of community c of graph g (r unused).
 * c below the communities in use.  Synchronous.  Errors:
 * CKV_ERR_INVALID_ARG (NULL, no state yet, what/g/c/r out of range),
 * CKV_ERR_CUDA. */
ckv_status ckv_debug_poke(ckv_ctx* ctx, int what, int g, int c, int r, int32_t value);

#ifdef __cplusplus
}
#endif
#endif
