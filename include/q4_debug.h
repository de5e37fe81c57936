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

/* Plan one batch-1 launch for `count` GEMVs (shapes n[i] x k[i]) exactly as the
 * library would on a device with `num_sms` multiprocessors, then replay every
 * piece and unit of it on the host: the shared-memory layout must fit the
 * budget (two CTAs per SM) with every region aligned, every piece must stay
 * inside its GEMV, its staged activations and per-(row, slice) partial sums
 * inside their regions, every tensor-map box must start at a 16-byte aligned
 * x coordinate inside its plane, every per-row scale copy (planes whose row
 * stride is not a multiple of 16 bytes) must be 16-byte aligned and sized,
 * inside the padded d plane and inside its slot, the scale each lane reads must
 * be its own block's, every (row, slice) must be covered exactly once, and
 * split-K tickets and partial sums must stay inside their workspace regions,
 * disjoint between GEMVs. Returns 0 when every check holds, otherwise the number
 * of the first failed check (see q4_debug.cu). */
int q4_debug_check_b1(const int64_t* n, const int64_t* k, int count, int b, int num_sms);

/* Summary of the CUDA-core plan above for a 148-multiprocessor B200 (1 <= b <= 4):
 * out[0] = CTAs (pieces), out[1] = dynamic shared memory bytes per CTA,
 * out[2] = workspace bytes, out[3] = weight ring slots, out[4 + i] = K splits of
 * GEMV i. Returns Q4_OK or Q4_ERR_INVALID_ARG. */
q4_status q4_debug_plan_info(const int64_t* n, const int64_t* k, int count, int b, int64_t* out);

/* Run the binary32 path's nibble unpack (compiled for the host from the same
 * source) on `count` pseudo-random code words from `seed` and on all words with
 * one nonzero nibble, comparing with plain nibble extraction, and its block dot
 * product on one-hot activations. Returns the number of mismatching values (0
 * when correct). */
int64_t q4_debug_check_unpack(uint64_t seed, int64_t count);

/* Check the batch-1 kernel's activation quantisation and block dot products on
 * the host (the same source compiled for the CPU): every |X| <= 2^30 sampled
 * (boundaries and a stride) splits into two 16-bit digits that add back up; for
 * `blocks` pseudo-random blocks of codes and activations (magnitudes from 2^-100
 * to 2^99, single and paired outliers of 1e4..1e6, subnormal neighbours, exact
 * zeros, all-zero blocks), an unflagged block's integer sum times its scale is
 * within (2^-14 + 2^-23) sum_j |(q_j - 8) x_j| of the exact sum, a flagged
 * block's binary32 sum within 33 * 2^-24 of it, and every block with an outlier
 * is flagged. Returns the number of failures (0 when correct). */
int64_t q4_debug_check_intdot(uint64_t seed, int64_t blocks);

/* The same replay for the batched tensor-core kernel (2 <= b <= 16 tokens):
 * every CTA's range of (tile, block) units and its walk in stages, exactly-once
 * coverage of every (tile, block), every TMA box (16-byte aligned x coordinate,
 * inside the code row), every activation load, the shared-memory operand rows
 * and the MMA descriptor that addresses them, the partial-sum slot of every
 * piece of a tile (slots 0..pieces-1, each once) and its ticket, all inside
 * their workspace regions. Returns 0 when every check holds, otherwise the
 * number of the first failed check (see q4_api.cu). */
int q4_debug_check_tc(const int64_t* n, const int64_t* k, int count, int b);

/* Check the tensor-core kernel's operand preparation on the host (the same
 * source compiled for the CPU): the dequantised A operand of `blocks`
 * pseudo-random code blocks holds q - 8 exactly at every MMA position, and an
 * emulated MMA over the A words and the hi/lo B rows (written at the offsets
 * the kernel uses, read back at the addresses the MMA descriptor gives)
 * reproduces sum_j (q_j - 8) x_j within 2^-16 sum_j |q_j - 8| |x_j|, for both
 * operand layouts (up to 8 tokens, and 9..16). Returns the number of failures. */
int64_t q4_debug_check_tc_operands(uint64_t seed, int64_t blocks);

/* q4_gemv_batched (b = 1: the batch-1 kernel; b >= 2: the tensor-core kernel)
 * with every stage (ring slot) barrier of the launch waiting for 16 bytes more
 * than its copies bring, so that every bounded wait of the kernel runs out: a test of the
 * timeout path without a GPU fault (all copies land; no wait is unbounded). The
 * call returns like q4_gemv_batched; the kernel records Q4_ERR_TIMEOUT in the
 * workspace header (read it with q4_workspace_status, clear it with
 * q4_workspace_init), leaves its copies and MMAs complete and its tensor memory
 * freed, and Y holds no meaningful values. Takes tens to hundreds of
 * milliseconds (20 ms per wait that runs out). */
q4_status q4_debug_gemv_stall(const q4_matrix* m, const float* X, int b, float* Y, void* ws,
                              size_t ws_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* Q4_B200_DEBUG_H */
