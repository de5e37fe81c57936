// Fused Q4_0 decode mat-vec kernels for sm_100a (CUDA cores).
//
// "Llamas on the Web" (gist.science technical summary of arXiv 2605.20706),
// section 3 "Dequantizzazione Integrata": at decode the mat-vec dequantises in
// registers. Here each warp streams its rows' code bytes and binary16 scales
// from HBM into shared memory with bulk copies on the TMA engine (one mbarrier
// per warp, copies issued before the wait on the previous kernel so that the
// weight stream runs across kernel boundaries), unpacks the nibbles to exact
// binary32 (q - 8) in registers, applies the per-block scale once per 32
// weights, and reduces with warp shuffles ("subgroup operations", same page,
// problem statement). K is split over CTAs when a matrix has too few rows to
// fill the GPU or K exceeds one split; the last CTA of a row tile adds the
// partial sums in split order (deterministic) and resets its ticket.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "q4_device.cuh"
#include "q4_plan.h"

using namespace q4plan;
using namespace q4dev;

namespace q4k {

constexpr uint32_t kTimeoutFlag = 1u;

// Issue the bulk copies of a warp's rows (codes and scales of one K split).
// Lane 0 arms the barrier with the total byte count; lanes r < rows copy code
// row r, lanes 8 + r copy scale row r.
__device__ __forceinline__ void issue_row_copies(const GemvParams& P, const GemvDesc& G, int split,
                                                 int kbs, int64_t row0, int rows, uint8_t* qsw,
                                                 uint16_t* dsw, uint64_t* bar, int lane) {
    if (lane == 0) {
        mbar_init(bar, 1);
        mbar_fence_init();
    }
    __syncwarp();
    if (lane == 0) {
        uint32_t total = (uint32_t)rows * (uint32_t)kbs * 16u;
        for (int r = 0; r < rows; ++r) total += d_range(G, row0 + r, split, kbs).bytes;
        mbar_arrive_expect_tx(bar, total);
    }
    __syncwarp();
    if (lane < rows) {
        bulk_g2s(qsw + (size_t)lane * G.nb_split * 16, G.qs + qs_src_offset(G, row0 + lane, split),
                 (uint32_t)kbs * 16u, bar);
    } else if (lane >= 8 && lane < 8 + rows) {
        const int r = lane - 8;
        const DRange dr = d_range(G, row0 + r, split, kbs);
        bulk_g2s(dsw + (size_t)r * P.d_slot, reinterpret_cast<const uint8_t*>(G.d) + dr.src,
                 dr.bytes, bar);
    }
}

// Wait for the warp's copies; on a timeout record it and wait once more, so that
// no copy is still landing in shared memory when the CTA leaves.
__device__ __forceinline__ bool wait_rows(const GemvParams& P, uint64_t* bar, int lane) {
    if (mbar_wait_bounded(bar, 0)) return true;
    if (lane == 0) atomicOr(P.ws, kTimeoutFlag);
    mbar_wait_bounded(bar, 0);
    return false;
}

// Store one row result (or its split partial). `slot` selects the token.
__device__ __forceinline__ void store_row(const GemvParams& P, const GemvDesc& G, int split, int t,
                                          int64_t row, float v) {
    if (G.splits == 1) {
        G.y[(int64_t)t * G.n + row] = v;
    } else {
        float* part = reinterpret_cast<float*>(P.ws) + G.part_off;
        part[((int64_t)t * G.splits + split) * G.n + row] = v;
        __threadfence();
    }
}

// Split-K completion: the last CTA of a row tile sums the partials in split
// order and resets the tile's ticket.
__device__ __forceinline__ void finish_splits(const GemvParams& P, const GemvDesc& G, int tile,
                                              int batch) {
    __shared__ uint32_t s_last;
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        const uint32_t t = atomicAdd(P.ws + G.ticket_off + tile, 1u);
        s_last = (t == (uint32_t)G.splits - 1u) ? 1u : 0u;
    }
    __syncthreads();
    if (s_last) {
        __threadfence();
        const float* part = reinterpret_cast<const float*>(P.ws) + G.part_off;
        const int64_t t0 = (int64_t)tile * kRowsPerCta;
        const int64_t left = G.n - t0;
        const int tr = left < kRowsPerCta ? (int)left : kRowsPerCta;
        for (int i = threadIdx.x; i < tr * batch; i += kThreads) {
            const int tok = i / tr, r = i % tr;
            float s = 0.0f;
            for (int sp = 0; sp < G.splits; ++sp)
                s += __ldcg(part + ((int64_t)tok * G.splits + sp) * G.n + t0 + r);
            G.y[(int64_t)tok * G.n + t0 + r] = s;
        }
        if (threadIdx.x == 0) P.ws[G.ticket_off + tile] = 0u;
    }
}

// ---------------------------------------------------------------------------
// batch 1: lane j of a warp handles block j of each 32-block iteration
// (16 code bytes, one 128-bit shared load per row), x lives in 32 registers and
// is reused across the warp's kRowsPerWarp rows.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads) gemv_b1_kernel(const __grid_constant__ GemvParams P) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const Unit u = unit_of(P, blockIdx.x);
    const GemvDesc& G = P.g[u.g];
    const int kbs = split_blocks(G, u.split);
    const int rows = warp_rows(G, u.tile, warp);
    const int64_t row0 = (int64_t)u.tile * kRowsPerCta + (int64_t)warp * kRowsPerWarp;
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem) + warp;
    uint8_t* qsw = smem + smem_warp_offset(P, warp);
    uint16_t* dsw = reinterpret_cast<uint16_t*>(qsw + P.smem_qs_warp);

    if (rows > 0) issue_row_copies(P, G, u.split, kbs, row0, rows, qsw, dsw, bar, lane);

    pdl_launch_dependents();
    pdl_wait();

    // stage this split's activations in the lane-interleaved layout
    float4* xs4 = reinterpret_cast<float4*>(smem + smem_x_offset());
    const float4* xg = reinterpret_cast<const float4*>(G.x + (int64_t)u.split * G.nb_split * 32);
    {
        // all loads first, then all stores: one round trip to L2, not one per chunk
        constexpr int kPer = (kMaxBlocksPerSplit * 8 + kThreads - 1) / kThreads;
        float4 t[kPer];
#pragma unroll
        for (int i = 0; i < kPer; ++i) {
            const int c = threadIdx.x + i * kThreads;
            if (c < kbs * 8) t[i] = xg[c];
        }
#pragma unroll
        for (int i = 0; i < kPer; ++i) {
            const int c = threadIdx.x + i * kThreads;
            if (c < kbs * 8) xs4[x_slot_b1(c >> 3, c & 7)] = t[i];
        }
    }
    __syncthreads();

    if (rows > 0 && wait_rows(P, bar, lane)) {
        // Rows past the end of the matrix repeat the last real row (results are
        // not stored), so the inner loop has no per-row branches.
        const uint8_t* qrow[kRowsPerWarp];
        const uint16_t* drow[kRowsPerWarp];
#pragma unroll
        for (int r = 0; r < kRowsPerWarp; ++r) {
            const int rr = r < rows ? r : rows - 1;
            qrow[r] = qsw + (size_t)rr * G.nb_split * 16 + lane * 16;
            drow[r] = dsw + rr * P.d_slot + d_range(G, row0 + rr, u.split, kbs).shift + lane;
        }
        float acc[kRowsPerWarp];
#pragma unroll
        for (int r = 0; r < kRowsPerWarp; ++r) acc[r] = 0.0f;

        const float4* xl = xs4 + lane;
        const int iters = (kbs + 31) >> 5;
        for (int it = 0; it < iters; ++it) {
            if ((it << 5) + lane < kbs) {
                float4 xv[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) xv[i] = xl[((it * 8 + i) << 5)];
#pragma unroll
                for (int r = 0; r < kRowsPerWarp; ++r) {
                    const uint4 q = *reinterpret_cast<const uint4*>(qrow[r] + it * 512);
                    const float dd = __half2float(__ushort_as_half(drow[r][it * 32]));
                    const float2 b = block_dot(q, xv, unpack_consts_default());
                    acc[r] = fmaf(dd, b.x + b.y, acc[r]);
                }
            }
        }
#pragma unroll
        for (int r = 0; r < kRowsPerWarp; ++r) {
            const float s = warp_sum(acc[r]);
            if (lane == r && r < rows) store_row(P, G, u.split, 0, row0 + r, s);
        }
    }
    if (G.splits > 1) finish_splits(P, G, u.tile, 1);
}

// ---------------------------------------------------------------------------
// batch 2..4 on CUDA cores: lane (j, w) handles 32-bit word w of block j of each
// 8-block iteration; each unpacked word is reused for every token.
// ---------------------------------------------------------------------------
template <int B>
__global__ void __launch_bounds__(kThreads) gemv_bs_kernel(const __grid_constant__ GemvParams P) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const Unit u = unit_of(P, blockIdx.x);
    const GemvDesc& G = P.g[u.g];
    const int kbs = split_blocks(G, u.split);
    const int rows = warp_rows(G, u.tile, warp);
    const int64_t row0 = (int64_t)u.tile * kRowsPerCta + (int64_t)warp * kRowsPerWarp;
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem) + warp;
    uint8_t* qsw = smem + smem_warp_offset(P, warp);
    uint16_t* dsw = reinterpret_cast<uint16_t*>(qsw + P.smem_qs_warp);

    if (rows > 0) issue_row_copies(P, G, u.split, kbs, row0, rows, qsw, dsw, bar, lane);

    pdl_launch_dependents();
    pdl_wait();

    float4* xs4 = reinterpret_cast<float4*>(smem + smem_x_offset());
    const int tok_slots = x_token_slots_bs(G.nb_split);
    for (int c = threadIdx.x; c < B * kbs * 8; c += kThreads) {
        const int t = c / (kbs * 8), cc = c % (kbs * 8);
        const float4* xg = reinterpret_cast<const float4*>(G.x + (int64_t)t * G.nb * 32 +
                                                           (int64_t)u.split * G.nb_split * 32);
        xs4[t * tok_slots + x_slot_bs(cc >> 3, cc & 7)] = xg[cc];
    }
    __syncthreads();

    if (rows > 0 && wait_rows(P, bar, lane)) {
        uint32_t shift[kRowsPerWarp];
#pragma unroll
        for (int r = 0; r < kRowsPerWarp; ++r)
            shift[r] = r < rows ? d_range(G, row0 + r, u.split, kbs).shift : 0u;
        float2 acc[kRowsPerWarp][B];
#pragma unroll
        for (int r = 0; r < kRowsPerWarp; ++r)
#pragma unroll
            for (int t = 0; t < B; ++t) acc[r][t] = f2(0.0f, 0.0f);

        const int w = lane & 3;
        const int iters = (kbs + 7) >> 3;
        for (int it = 0; it < iters; ++it) {
            const int j = (it << 3) + (lane >> 2);
            if (j < kbs) {
                float4 xlo[B], xhi[B];
#pragma unroll
                for (int t = 0; t < B; ++t) {
                    xlo[t] = xs4[t * tok_slots + x_slot_bs(j, w)];
                    xhi[t] = xs4[t * tok_slots + x_slot_bs(j, w + 4)];
                }
#pragma unroll
                for (int r = 0; r < kRowsPerWarp; ++r) {
                    if (r < rows) {
                        const uint32_t q = *reinterpret_cast<const uint32_t*>(
                            qsw + ((size_t)r * G.nb_split + j) * 16 + w * 4);
                        const float dd =
                            __half2float(__ushort_as_half(dsw[r * P.d_slot + shift[r] + j]));
                        const Pairs p = unpack_word(q);
#pragma unroll
                        for (int t = 0; t < B; ++t) {
                            float2 s = fma2(p.lo01, f2(xlo[t].x, xlo[t].y), f2(0.0f, 0.0f));
                            s = fma2(p.lo23, f2(xlo[t].z, xlo[t].w), s);
                            s = fma2(p.hi01, f2(xhi[t].x, xhi[t].y), s);
                            s = fma2(p.hi23, f2(xhi[t].z, xhi[t].w), s);
                            acc[r][t] = fma2(s, f2(dd, dd), acc[r][t]);
                        }
                    }
                }
            }
        }
#pragma unroll
        for (int r = 0; r < kRowsPerWarp; ++r)
#pragma unroll
            for (int t = 0; t < B; ++t) {
                const float s = warp_sum(acc[r][t].x + acc[r][t].y);
                if (lane == r && r < rows) store_row(P, G, u.split, t, row0 + r, s);
            }
    }
    if (G.splits > 1) finish_splits(P, G, u.tile, B);
}

// Allow each GEMV kernel the device's opt-in shared memory minus its static
// shared memory (the per-block limit covers both).
template <typename K>
static cudaError_t allow_dynamic_smem(K kernel, int optin) {
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, kernel);
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                optin - (int)fa.sharedSizeBytes);
}

cudaError_t setup_gemv_kernels(int optin_smem) {
    cudaError_t e = allow_dynamic_smem(gemv_b1_kernel, optin_smem);
    if (e == cudaSuccess) e = allow_dynamic_smem(gemv_bs_kernel<2>, optin_smem);
    if (e == cudaSuccess) e = allow_dynamic_smem(gemv_bs_kernel<3>, optin_smem);
    if (e == cudaSuccess) e = allow_dynamic_smem(gemv_bs_kernel<4>, optin_smem);
    return e;
}

cudaError_t launch_gemv(const GemvParams& P, bool pdl, cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)P.total_units, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = P.smem_total;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    switch (P.batch) {
        case 1: return cudaLaunchKernelEx(&cfg, gemv_b1_kernel, P);
        case 2: return cudaLaunchKernelEx(&cfg, gemv_bs_kernel<2>, P);
        case 3: return cudaLaunchKernelEx(&cfg, gemv_bs_kernel<3>, P);
        case 4: return cudaLaunchKernelEx(&cfg, gemv_bs_kernel<4>, P);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace q4k
