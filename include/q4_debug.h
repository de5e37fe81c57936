/*
 * q4_debug.h — host-only diagnostics of libq4_b200.so. None of these touches a
 * GPU: they replay the library's own launch planning and its register unpack on
 * the CPU, so that every copy range, shared-memory offset and workspace offset a
 * kernel would use can be checked before the kernel runs.
 */
#ifndef Q4_B200_DEBUG_H
#define Q4_B200_DEBUG_H

#include <stdint.h>

#include "q4.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Plan one launch for `count` GEMVs (shapes n[i] x k[i], b tokens) exactly as the
 * library would, then replay every unit and warp of it on the host: each bulk
 * copy must stay inside its plane (the d plane counted with its 16-byte padding)
 * and inside its shared-memory slot, be 16-byte aligned and sized, the staged
 * activations must stay inside x and their shared-memory region, every
 * (row, block) must be covered exactly once, and split-K partials and tickets
 * must stay inside the workspace. Returns 0 when every check holds, otherwise
 * the number of the first failed check (see q4_api.cu). */
int q4_debug_check_plan(const int64_t* n, const int64_t* k, int count, int b);

/* Summary of the plan above: out[0] = CTAs (units), out[1] = dynamic shared
 * memory bytes per CTA, out[2] = workspace bytes, out[3 + i] = K splits of GEMV i.
 * Returns Q4_OK or Q4_ERR_INVALID_ARG. */
q4_status q4_debug_plan_info(const int64_t* n, const int64_t* k, int count, int b, int64_t* out);

/* Run the kernels' nibble unpack (compiled for the host from the same source) on
 * `count` pseudo-random code words from `seed` and on all words with one nonzero
 * nibble, comparing with plain nibble extraction. Returns the number of
 * mismatching values (0 when correct). */
int64_t q4_debug_check_unpack(uint64_t seed, int64_t count);

#ifdef __cplusplus
}
#endif

#endif /* Q4_B200_DEBUG_H */
