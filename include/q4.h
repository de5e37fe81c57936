/*
 * q4.h — C ABI of the B200 Q4_0 decode library (libq4_b200.so).
 *
 * The operation is the decode-phase matrix-vector product y = W x over weights
 * stored at 4 bits per parameter ("MicroLLM Lab", sitech.ge, section "Seven
 * models, all in Q4": 16-bit weights compressed to 4 bits per parameter), with
 * the weights dequantised inside the product, in registers, at decode time
 * ("Llamas on the Web", gist.science technical summary of arXiv 2605.20706,
 * section 3 "Dequantizzazione Integrata"; formats held as flat packed integer
 * buffers, section 3 "Estensibilita'"). The block format is llama.cpp's legacy
 * Q4_0 (the same summary's problem statement names llama.cpp's legacy schemes):
 *
 *   32 consecutive weights of a row form a block; the block stores one IEEE
 *   binary16 scale d and 32 codes q in 0..15; the weight is w = d * (q - 8).
 *   Interchange bytes of a block (18): d little-endian, then qs[16] with
 *   qs[j] = q[j] | q[j + 16] << 4.
 *
 * Device layout ("planes"): the same bytes split in two arrays so that every
 * row of codes starts on a 16-byte boundary for any K:
 *   qs plane : uint8  [n][k/2]   row r, block b at byte (r*(k/32) + b)*16
 *   d  plane : uint16 [n][k/32]  binary16 bits of the scale of (r, b)
 * q4_plane_bytes() gives the sizes to allocate; the d plane is padded to a
 * multiple of 16 bytes because the library reads it in 16-byte pieces.
 *
 * Conventions for every call:
 *   - Ownership: every pointer named "device" is caller-allocated device memory
 *     (allocated, for instance, through PyTorch) and stays owned by the caller.
 *     The library never allocates, frees or synchronises: memory is planned up
 *     front, as "Llamas on the Web" (section 1, "Allocazione Statica della
 *     Memoria") does.
 *   - stream: a cudaStream_t passed as void*; NULL means the legacy default
 *     stream. All work is enqueued on it; calls return before it runs.
 *   - Errors: argument errors are returned before anything is enqueued. A failed
 *     launch returns Q4_ERR_CUDA. Device-side bounded waits that give up record
 *     Q4_ERR_TIMEOUT in the workspace header, read by q4_workspace_status().
 *     Nothing traps, prints or throws across the ABI.
 *   - Sizes and offsets are 64-bit: a stack of weights exceeds 2^31 bytes
 *     (the "WebGPT" README's roadmap splits passes at a binding-size limit;
 *     here offsets are simply int64).
 *   - Determinism: the same inputs and the same arguments give the same bits.
 *   - Architecture: sm_100a (B200) only.
 */
#ifndef Q4_B200_H
#define Q4_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define Q4_QK 32          /* weights per block */
#define Q4_BLOCK_BYTES 18 /* interchange bytes per block */
#define Q4_MAX_BATCH 16   /* tokens per call */
#define Q4_MAX_GROUP 8    /* GEMVs in one dependency group of a stack */

typedef enum {
    Q4_OK = 0,
    Q4_ERR_INVALID_ARG = 1, /* null pointer, k % 32 != 0, n < 1, bad group order */
    Q4_ERR_MISALIGNED = 2,  /* a pointer breaks the alignment rule of its call   */
    Q4_ERR_WORKSPACE = 3,   /* workspace missing or smaller than required        */
    Q4_ERR_UNSUPPORTED = 4, /* b outside 1..16, device is not sm_100             */
    Q4_ERR_CUDA = 5,        /* a CUDA runtime call or launch failed              */
    Q4_ERR_TIMEOUT = 6      /* a bounded device wait gave up (see workspace)     */
} q4_status;

/* A Q4_0 matrix in planes layout. qs and d are device pointers owned by the
 * caller; qs must be 16-byte aligned, d 16-byte aligned. n >= 1, k % 32 == 0. */
typedef struct {
    uint8_t* qs;
    uint16_t* d;
    int64_t n;
    int64_t k;
} q4_matrix;

/* Bytes to allocate for the two planes of an n x k matrix (qs: n*k/2; d: n*k/16
 * rounded up to a multiple of 16). Returns Q4_ERR_INVALID_ARG for bad n or k. */
q4_status q4_plane_bytes(int64_t n, int64_t k, size_t* qs_bytes, size_t* d_bytes);

/* q4_pack — quantise a row-major binary32 matrix to Q4_0 planes on the device.
 * The "Q4 packer" of "MicroLLM Lab" (introduction), run offline before decode.
 * Per block of 32: m = the weight of largest magnitude (lowest index on ties),
 * d = m / -8 in binary32, q_j = min(15, floor(w_j * (1/d) + 8.5)) with 1/d and
 * every step rounded to nearest binary32 and no fused multiply-add (q_j = 8 when
 * d == 0), stored d = binary16(d) rounded to nearest even. Bit-exact by design.
 *   w   : device, binary32 [out->n][out->k], row-major, 16-byte aligned.
 *   out : out->qs, out->d, out->n, out->k filled in by the caller (planes
 *         allocated with q4_plane_bytes). Weights must be finite, with |w| small
 *         enough that d fits binary16 (|w| < 524160); other inputs give
 *         unspecified codes.
 * Errors: Q4_ERR_INVALID_ARG, Q4_ERR_MISALIGNED, Q4_ERR_CUDA. */
q4_status q4_pack(const float* w, const q4_matrix* out, void* stream);

/* q4_dequant — expand Q4_0 planes to binary32: w_out[r][c] = d(r, c/32) *
 * (q(r, c) - 8), exact in binary32. The dequantised tile of the mat-mat path in
 * "Llamas on the Web" section 3, written to memory for inspection; the GEMV
 * calls never write it.
 *   m     : the matrix (device planes).
 *   w_out : device, binary32 [m->n][m->k], row-major, 16-byte aligned.
 * Errors: Q4_ERR_INVALID_ARG, Q4_ERR_MISALIGNED, Q4_ERR_CUDA. */
q4_status q4_dequant(const q4_matrix* m, float* w_out, void* stream);

/* Workspace bytes needed by q4_gemv / q4_gemv_batched for an n x k matrix and b
 * tokens (a 256-byte status header, split-K tickets and partial sums). Returns 0
 * for invalid arguments. */
size_t q4_workspace_bytes(int64_t n, int64_t k, int b);

/* Zero a workspace (header, tickets): required once before its first use. Every
 * call that completes leaves the tickets at zero again, so the workspace can be
 * reused by any later call on the same stream. ws: device, 256-byte aligned. */
q4_status q4_workspace_init(void* ws, size_t ws_bytes, void* stream);

/* Read the status header of a workspace: Q4_OK, or Q4_ERR_TIMEOUT if a bounded
 * device wait of an earlier call gave up. Synchronises the stream (the one call
 * of the library that does), so call it off the hot path. */
q4_status q4_workspace_status(const void* ws, void* stream);

/* q4_gemv — y = W x for one token (batch 1): y[r] = sum_b d(r,b) *
 * sum_{j<32} (q(r,b,j) - 8) * x[32 b + j], binary32 accumulation.
 * The decode-phase mat-vec of "Llamas on the Web" section 3: codes are unpacked
 * in registers, the scale is applied per block, no dequantised weight is written
 * to memory.
 *   m  : the matrix (device planes).
 *   x  : device, binary32 [m->k], 16-byte aligned.
 *   y  : device, binary32 [m->n], 16-byte aligned; fully overwritten.
 *   ws : device workspace of q4_workspace_bytes(n, k, 1) bytes, 256-byte
 *        aligned, zeroed once by q4_workspace_init.
 * Accuracy: |y - y_exact| <= 1e-4 * sum|w x| + 1e-6 per element (tested).
 * Errors: Q4_ERR_INVALID_ARG, Q4_ERR_MISALIGNED, Q4_ERR_WORKSPACE, Q4_ERR_CUDA. */
q4_status q4_gemv(const q4_matrix* m, const float* x, float* y, void* ws, size_t ws_bytes,
                  void* stream);

/* q4_gemv_batched — Y[t] = W X[t] for t < b, 1 <= b <= 16 ("batch 1 to a few
 * tokens"). b = 1 is q4_gemv. Every b reads each weight once per call, in one
 * launch for all tokens:
 *  - 2 <= b <= 4, on the CUDA cores: each code word is unpacked once in
 *    registers into the exact binary32 values q - 8 ("Llamas on the Web"
 *    section 3, mat-vec dequantised in registers) and every token multiplies
 *    them with its own activations; products, block sums and the binary16
 *    scale in binary32: |Y - W X| within binary32 accumulation.
 *  - b >= 5, on the tensor cores: the matrix-matrix form of section 3, the
 *    weights dequantised once into on-chip (tensor) memory and reused for every
 *    token. Each 32-weight block's codes become (q - 8) in bf16 (exact), each
 *    activation x is taken as bf16 parts hi + lo with |x - hi - lo| <= 2^-16 |x|,
 *    every block has its own binary32 accumulator and its binary16 scale is
 *    applied once: |Y - W X| <= 2^-16 sum |w x| plus binary32 accumulation.
 *   X : device, binary32 [b][m->k] row-major, 16-byte aligned.
 *   Y : device, binary32 [b][m->n] row-major, 16-byte aligned.
 *   ws: as for q4_gemv with q4_workspace_bytes(n, k, b).
 * Errors: as q4_gemv, plus Q4_ERR_UNSUPPORTED for b outside 1..16 and
 * Q4_ERR_INVALID_ARG for n or (n / 128) * (k / 32) at or above 2^31 when b >= 5. */
q4_status q4_gemv_batched(const q4_matrix* m, const float* X, int b, float* Y, void* ws,
                          size_t ws_bytes, void* stream);

/* q4_gemv_noalloc — q4_gemv without a caller workspace, for callers that cannot
 * allocate device memory: a plugin inside a host application that owns every
 * device allocation, a runtime whose memory budget is fixed after start-up, or a
 * latency-critical path that must not call cudaMalloc because it can synchronise
 * the whole device. The pages have no counterpart of this call.
 * Same arguments, result and accuracy as q4_gemv, minus ws and ws_bytes; x and y
 * are still the caller's device buffers. Split-K scratch (status header,
 * tickets, partial sums) lives in one fixed device array of 1 MiB
 * (1,048,576 bytes) inside the library, which every GPU that loads the library
 * holds until the process exits. Nothing is allocated or
 * freed by this call.
 *   - A matrix whose scratch need, q4_workspace_bytes(n, k, 1), exceeds that size
 *     is rejected with Q4_ERR_WORKSPACE before anything is enqueued (every matrix
 *     of the 8B-class layer needs at most a few hundred bytes).
 *   - The first call on each device configures the kernels for that device;
 *     make that first call before any stream capture. The array's device
 *     address is looked up on every call (with the device current).
 *   - All calls on a device share the one array, which keeps the last call's
 *     contents; each call clears the tickets it uses before its kernel. Calls
 *     that overlap on the GPU (for instance on two streams) race on the array:
 *     serialise them.
 *   - A bounded device wait that gives up is recorded in the array's status
 *     header; q4_noalloc_status reports (and clears) it.
 * Errors: as q4_gemv. */
q4_status q4_gemv_noalloc(const q4_matrix* m, const float* x, float* y, void* stream);

/* q4_noalloc_status — Q4_ERR_TIMEOUT if a bounded device wait of any
 * q4_gemv_noalloc call on the current device gave up since the last
 * q4_noalloc_status, else Q4_OK; clears the record. Enqueued on `stream` after
 * the calls it reports on, and synchronises that stream (call it off the hot
 * path). The pages have no counterpart of this call. */
q4_status q4_noalloc_status(void* stream);

/* A decode step: `count` GEMVs in dependency groups. group[i] is the group of
 * GEMV i; groups are non-decreasing and run in order; the GEMVs of one group
 * (at most Q4_MAX_GROUP) are independent and run in one launch. x[i] is device
 * binary32 [b][mats[i].k], y[i] device binary32 [b][mats[i].n]. The arrays
 * themselves are host memory, read during the call only. */
typedef struct {
    int count;
    const q4_matrix* mats;
    const float* const* x;
    float* const* y;
    const int* group;
} q4_stack;

/* Workspace bytes for q4_layer_stack / q4_stack_graph_create (the maximum over
 * groups; groups run one after another and share it). 0 for invalid input. */
size_t q4_stack_workspace_bytes(const q4_stack* s, int b);

/* q4_layer_stack — enqueue one decode step: every group as one launch, in order.
 * Kernel submissions are batched ("Llamas on the Web" section 2, "Pianificazione
 * dell'Esecuzione"): after the first launch, each launch may start while the
 * previous one drains, streaming its weights in before it waits for the previous
 * group's results (programmatic dependent launch). The first launch of a call
 * waits for all earlier work on the stream.
 * Errors: as q4_gemv_batched, checked for every GEMV before anything runs. */
q4_status q4_layer_stack(const q4_stack* s, int b, void* ws, size_t ws_bytes, void* stream);

/* A captured decode step ("WebGPT" README roadmap: pipelines initialised every
 * step are inefficient; "Llamas on the Web" section 2: compiled pipelines are
 * cached). q4_stack_graph_create records q4_layer_stack(s, b, ws, ...) into a
 * CUDA graph once (by capturing `stream`, which must not be capturing already
 * and must not be the legacy NULL stream); q4_graph_launch replays the whole
 * step with one call. The graph keeps the pointers given at creation: buffers
 * must outlive it. */
typedef struct q4_graph_s* q4_graph;
q4_status q4_stack_graph_create(const q4_stack* s, int b, void* ws, size_t ws_bytes,
                                void* stream, q4_graph* out);
q4_status q4_graph_launch(q4_graph g, void* stream);
q4_status q4_graph_destroy(q4_graph g);

/* Host-side interchange with llama.cpp-layout blocks (18 bytes each, row-major
 * [n][k/32]). All pointers are host memory. The d plane written has exactly
 * n*k/32 entries (padding is not touched). */
q4_status q4_blocks_to_planes(const uint8_t* blocks, int64_t n, int64_t k, uint8_t* qs,
                              uint16_t* d);
q4_status q4_planes_to_blocks(const uint8_t* qs, const uint16_t* d, int64_t n, int64_t k,
                              uint8_t* blocks);

/* A static, human-readable name for a status code. */
const char* q4_status_string(q4_status s);

/* The CUDA runtime's message for the last CUDA call of this library that failed
 * on the calling thread (what a Q4_ERR_CUDA status came from); "no error" if
 * none has. The string is static. */
const char* q4_last_cuda_error(void);

/* Number of kernels this library has launched in this process (a diagnostic
 * counter; graph replays count the kernels they contain). */
uint64_t q4_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* Q4_B200_H */
