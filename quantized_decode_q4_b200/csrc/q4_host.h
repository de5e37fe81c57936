// Host-side planning and launch of the library's kernels, shared by the C ABI
// (q4_api.cu) and the host-only diagnostics (q4_debug.cu).
#pragma once

#include <cuda_runtime.h>

#include <cstdint>
#include <vector>

#include "../../include/q4.h"
#include "q4_b1_plan.h"
#include "q4_tc_plan.h"

namespace q4k {
cudaError_t launch_pack(const float* w, uint8_t* qs, uint16_t* d, int64_t nblocks, int num_sms,
                        cudaStream_t stream);
cudaError_t launch_dequant(const uint8_t* qs, const uint16_t* d, float* out, int64_t nblocks,
                           int num_sms, cudaStream_t stream);
cudaError_t setup_b1_kernel(int optin_smem);
cudaError_t launch_b1(const q4b::Params& P, bool pdl, cudaStream_t stream);
cudaError_t encode_b1_maps(CUtensorMap* qs_map, CUtensorMap* d_map, int32_t* d_ok, const uint8_t* qs,
                           const uint16_t* d, int64_t n, int64_t k);
cudaError_t setup_tc_kernels(int optin_smem);
cudaError_t launch_tc(const q4t::Params& P, bool pdl, cudaStream_t stream);
cudaError_t encode_tc_maps(q4t::Maps* maps, int32_t* d_box, const uint8_t* qs, const uint16_t* d,
                           const float* x, int64_t n, int64_t k, int b);
int tc_tokens(int b);
}  // namespace q4k

namespace q4h {

constexpr int64_t kHeaderBytes = 256;  // workspace status header (word 0: timeout flag)
constexpr uint32_t kMaxSmem = 226 * 1024;

struct Shape {
    int64_t n, k;
};

struct GemvCall {
    q4_matrix m;
    const float* x;
    float* y;
};

// Record a failed CUDA call for q4_last_cuda_error() and report it.
bool cuda_failed(cudaError_t e);

int64_t ceil_div(int64_t a, int64_t b);
int64_t round_up(int64_t a, int64_t b);
bool aligned(const void* p, uintptr_t a);

q4_status check_shape(int64_t n, int64_t k);
q4_status check_matrix(const q4_matrix* m);

// The current device, checked (sm_100) and configured once; *num_sms is its
// multiprocessor count.
q4_status ensure_device(int* num_sms);

// CUDA-core plan (1 .. q4b::kMaxTokens tokens) of one launch over `count` GEMVs for a device with `num_sms`
// multiprocessors: pieces, splits, shared-memory layout, tickets and partial
// sums (from byte part_base of the workspace). Fills everything except the
// pointers. *tickets = ticket words used, *ws_end = end of the partial sums.
q4_status plan_b1(const Shape* sh, int count, int b, int64_t part_base, int num_sms, q4b::Params* P,
                  int64_t* tickets, int64_t* ws_end);

// Tensor-core plan (q4b::kMaxTokens < b <= 16) of one launch; same outputs.
q4_status plan_tc(const Shape* sh, int count, int b, int64_t part_base, int num_sms,
                  q4t::Params* P, int64_t* tickets, int64_t* ws_end);

// Start of the partial sums for a ticket region of `tickets` words.
int64_t part_base_for(int64_t tickets);

// Tickets and partial-sum bytes (past the ticket region) of one group.
q4_status group_need(const Shape* sh, int count, int b, int num_sms, int64_t* tickets,
                     int64_t* part_bytes);

}  // namespace q4h
