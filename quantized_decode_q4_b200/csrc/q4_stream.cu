// Persistent batch-1 Q4_0 decode mat-vec for sm_100a.
//
// "Llamas on the Web" (gist.science technical summary of arXiv 2605.20706),
// section 3 "Dequantizzazione Integrata": the decode mat-vec dequantises in
// registers. One CTA per SM walks a contiguous range of the group's row space
// (rows of (GEMV, K split) segments laid end to end). Each warp streams its
// tiles' code bytes and binary16 scales from HBM through a private ring of
// shared-memory stages filled by bulk copies on the TMA engine (one mbarrier per
// stage; a stage is refilled as soon as the warp has read it), so the weight
// stream never waits for the math. The activations of a (GEMV, split) segment
// are staged once per CTA in 24-bit block fixed point; each block's dot product
// is exact in integers (dp4a over the three digit planes) and its binary16 and
// activation scales are applied once per 32 weights; rows are reduced with warp
// shuffles. Finished rows wait in the lanes and are published 32 at a time; when
// K is split, the last split of a row to arrive adds the partial sums in split
// order (deterministic).
// One dependency group per launch: the first tiles are requested before the
// wait on the previous kernel (programmatic dependent launch), so consecutive
// launches overlap their weight streams.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "q4_device.cuh"
#include "q4_intdot.cuh"
#include "q4_stream_plan.h"

using namespace q4dev;

namespace q4k {

namespace {

constexpr uint32_t kTimeoutFlag = 1u;

// The kernel's source of groups: one dependency group per launch (a whole
// stack in one launch with a software grid barrier between groups measured
// slower on B200 than programmatic dependent launch of one kernel per group).
struct OneGroup {
    const q4s::Params& P;
    __device__ int groups() const { return 1; }
    __device__ q4s::View view(int) const {
        q4s::View v;
        v.g = P.g;
        v.cta_lo = P.cta_lo;
        v.count = P.count;
        v.total_rows = P.total_rows;
        return v;
    }
    __device__ uint32_t* ws() const { return P.ws; }
    __device__ uint32_t tx_extra() const { return P.tx_extra; }
};

// Copy issuer of one warp: walks the warp's tiles in the same order as the math
// loop, group after group (the weights do not wait for the barrier between
// groups), and issues each tile's copies (two requests when K is not split: all
// codes, all scales) into the next stage.
template <class Src>
struct Issuer {
    q4s::Walk wk;
    q4s::View v;                 // the current group
    int64_t row0;                // first row of the next tile to issue
    int gi, ngroups, warp;
    bool has;                    // a tile is pending

    __device__ bool done() const { return !has; }

    __device__ void start(const Src& S) {
        for (; gi < ngroups; ++gi) {
            v = S.view(gi);
            int64_t lo, hi;
            q4s::cta_range(v, blockIdx.x, &lo, &hi);
            wk.begin(lo, hi, warp);
            has = wk.next_piece(v);
            if (has) {
                row0 = wk.wr;
                return;
            }
        }
        has = false;
    }

    __device__ void begin(const Src& S, int w) {
        warp = w;
        gi = 0;
        ngroups = S.groups();
        start(S);
    }

    // issue the pending tile into `stage` (whole warp), then advance
    __device__ void issue(const Src& S, uint8_t* stage_base, uint64_t* bar, int lane) {
        const q4s::Desc& G = v.g[wk.g];
        const int64_t left = wk.wend - row0;
        const int rows = left < q4s::kRows ? (int)left : q4s::kRows;
        const q4s::LaneCopy c = q4s::lane_copy(G, wk.split, row0, rows, lane);
        const uint32_t bytes = c.active ? c.bytes : 0u;
        const uint32_t total = __reduce_add_sync(0xffffffffu, bytes);
        if (lane == 0) mbar_arrive_expect_tx(bar, total + S.tx_extra());
        __syncwarp();
        if (c.active)
            bulk_g2s(stage_base + c.dst,
                     (c.scales ? reinterpret_cast<const uint8_t*>(G.d) : G.qs) + c.src_off, bytes,
                     bar);
        row0 += q4s::kRows;
        if (row0 >= wk.wend) {
            has = wk.next_piece(v);
            if (has) {
                row0 = wk.wr;
            } else {
                ++gi;
                start(S);
            }
        }
    }
};

__device__ __forceinline__ void wait_stage(uint32_t* ws, uint64_t* bar, uint32_t parity, int lane) {
    if (!mbar_wait_bounded(bar, parity)) {
        if (lane == 0) atomicOr(ws, kTimeoutFlag);
        mbar_wait_bounded(bar, parity);
    }
}

// Stage the activations of split `split` of GEMV `G` in 24-bit block fixed
// point (all threads of the CTA). Eight lanes share a block: lane l of a warp
// takes block (pass * 4 + l / 8) of the warp's blocks and its elements
// 4 g .. 4 g + 3, g = l % 8 (one 16-byte load, from L2: the activations may have
// been written by another CTA or kernel). The block's largest |x| and its digit
// sums are reduced over the eight lanes with shuffles; each lane stores its four
// elements' digits as one 32-bit word per digit plane (word g % 4 of entry
// 2 p + g / 4), lane g = 0 the block constants.
__device__ __forceinline__ void stage_x(const q4s::Desc& G, int split, uint4* xq, int warp,
                                        int lane) {
    constexpr int kBlocksPerWarp = (q4s::kMaxSplitBlocks + q4s::kWarps - 1) / q4s::kWarps;
    constexpr int kPasses = (kBlocksPerWarp + 3) / 4;
    const int kbs = q4s::split_blocks(G, split);
    const float* xg = G.x + (int64_t)split * G.nb_split * 32;
    const int g = lane & 7;
    float4 v[kPasses];
#pragma unroll
    for (int p = 0; p < kPasses; ++p) {
        // warp w quantises blocks w, w + kWarps, ... (four per pass)
        const int j = warp + (p * 4 + (lane >> 3)) * q4s::kWarps;
        v[p] = j < kbs ? __ldcg(reinterpret_cast<const float4*>(xg + j * 32 + 4 * g))
                       : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    }
    uint32_t* xw = reinterpret_cast<uint32_t*>(xq);
#pragma unroll
    for (int p = 0; p < kPasses; ++p) {
        const int j = warp + (p * 4 + (lane >> 3)) * q4s::kWarps;
        // |x| of non-negative binary32 values orders like their bit patterns
        uint32_t m = max(max(__float_as_uint(fabsf(v[p].x)), __float_as_uint(fabsf(v[p].y))),
                         max(__float_as_uint(fabsf(v[p].z)), __float_as_uint(fabsf(v[p].w))));
#pragma unroll
        for (int off = 4; off > 0; off >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, off));
        const float inv = q4dev::xq_inv(__uint_as_float(m));
        const float e[4] = {v[p].x, v[p].y, v[p].z, v[p].w};
        uint32_t wa = 0, wb = 0, wc = 0;
        int32_t sa = 0, sb = 0, sc = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            int32_t a, b, c;
            q4dev::x_digits(q4dev::xq_int(e[i], inv), &a, &b, &c);
            wa |= ((uint32_t)a & 0xFFu) << (8 * i);
            wb |= ((uint32_t)b & 0xFFu) << (8 * i);
            wc |= ((uint32_t)c & 0xFFu) << (8 * i);
            sa += a;
            sb += b;
            sc += c;
        }
#pragma unroll
        for (int off = 4; off > 0; off >>= 1) {
            sa += __shfl_xor_sync(0xffffffffu, sa, off);
            sb += __shfl_xor_sync(0xffffffffu, sb, off);
            sc += __shfl_xor_sync(0xffffffffu, sc, off);
        }
        if (j < kbs) {
            const int half = g >> 2, word = g & 3;
            xw[q4s::xq_slot(j, 0 + half) * 4 + word] = wa;
            xw[q4s::xq_slot(j, 2 + half) * 4 + word] = wb;
            xw[q4s::xq_slot(j, 4 + half) * 4 + word] = wc;
            if (g == 0)
                xq[q4s::xq_slot(j, 6)] = make_uint4((uint32_t)(-8 * sa), (uint32_t)(-8 * sb),
                                                    (uint32_t)(-8 * sc),
                                                    __float_as_uint(q4dev::xq_scale(__uint_as_float(m))));
        }
    }
}

// Sum each of a tile's rows over the lanes (butterflies interleaved); every
// lane gets every row's total.
__device__ __forceinline__ void reduce_tile(float (&v)[q4s::kRows]) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
#pragma unroll
        for (int r = 0; r < q4s::kRows; ++r) v[r] += __shfl_xor_sync(0xffffffffu, v[r], off);
}

// Publish up to 32 consecutive rows of one (GEMV, split) piece, row
// brow0 + l held by lane l: store y, or, with a split K, store the partial
// sums, fence once, take each row's ticket, and let the last split of a row to
// arrive add the partials in split order and reset the ticket.
__device__ __forceinline__ void flush_rows(uint32_t* ws, const q4s::Desc& G, int split, int64_t brow0,
                                           int nbuf, float mine, int lane) {
    const bool act = lane < nbuf;
    const int64_t row = brow0 + lane;
    if (G.splits == 1) {
        if (act) G.y[row] = mine;
        return;
    }
    float* part = reinterpret_cast<float*>(ws) + G.part_off;
    if (act) part[(int64_t)split * G.n + row] = mine;
    __threadfence();
    bool last = false;
    if (act) last = atomicAdd(ws + G.ticket_off + row, 1u) == (uint32_t)G.splits - 1u;
    if (__any_sync(0xffffffffu, last)) {
        __threadfence();
        if (last) {
            float sum = 0.0f;
            for (int sp = 0; sp < G.splits; ++sp) sum += __ldcg(part + (int64_t)sp * G.n + row);
            G.y[row] = sum;
            ws[G.ticket_off + row] = 0u;
        }
    }
}

template <class Src>
__device__ __forceinline__ void stream_body(const Src& S) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem_raw) + warp * q4s::kStages;
    uint4* xq = reinterpret_cast<uint4*>(smem_raw + q4s::kBarBytes);
    uint8_t* ring = smem_raw + q4s::stage_offset(warp, 0);
    uint32_t* ws = S.ws();

    if (lane == 0) {
        for (int s = 0; s < q4s::kStages; ++s) mbar_init(bars + s, 1);
        mbar_fence_init();
    }
    __syncwarp();

    // the copy issuer runs kStages tiles ahead of the math
    Issuer<Src> is;
    is.begin(S, warp);
    for (int s = 0; s < q4s::kStages && !is.done(); ++s)
        is.issue(S, ring + s * q4s::kStageBytes, bars + s, lane);

    // warm L2 with the activations of the first piece (a hint only: the reads
    // that use them come after the wait on the previous kernel)
    {
        const q4s::View v0 = S.view(0);
        int64_t lo0, hi0;
        q4s::cta_range(v0, blockIdx.x, &lo0, &hi0);
        if (lo0 < hi0 && warp == 0 && lane == 0) {
            const q4s::Where w0 = q4s::locate(v0, lo0);
            const q4s::Desc& G0 = v0.g[w0.g];
            bulk_prefetch_l2(G0.x + (int64_t)w0.split * G0.nb_split * 32,
                             (uint32_t)q4s::split_blocks(G0, w0.split) * 128u);
        }
    }

    pdl_launch_dependents();
    pdl_wait();

    uint32_t stage = 0, parity = 0;
    for (int gi = 0; gi < S.groups(); ++gi) {
        const q4s::View V = S.view(gi);
        int64_t lo, hi;
        q4s::cta_range(V, blockIdx.x, &lo, &hi);
        int64_t pos = lo;
        while (pos < hi) {
            const q4s::Where w = q4s::locate(V, pos);
            const int64_t p1 = w.seg_end < hi ? w.seg_end : hi;
            const int64_t seg_row0 = pos - w.row;
            const q4s::Desc& G = V.g[w.g];
            __syncthreads();  // every warp is done with the previous activations
            stage_x(G, w.split, xq, warp, lane);
            __syncthreads();
            const int kbs = q4s::split_blocks(G, w.split);
            const int nsub = (kbs + 31) >> 5;
            const uint4* xl = xq + lane;
            int64_t ra, rb;
            q4s::warp_rows(pos, p1, warp, &ra, &rb);
            // finished rows wait in the lanes (row brow0 + l in lane l) and are
            // published 32 at a time
            int64_t brow0 = ra - seg_row0;
            int nbuf = 0;
            float mine = 0.0f;
            for (int64_t row0 = ra - seg_row0; row0 < rb - seg_row0; row0 += q4s::kRows) {
                const int64_t left = rb - seg_row0 - row0;
                const int rows = left < q4s::kRows ? (int)left : q4s::kRows;
                uint8_t* st = ring + stage * q4s::kStageBytes;
                const uint8_t* qrow[q4s::kRows];
                const uint8_t* drow[q4s::kRows];
#pragma unroll
                for (int r = 0; r < q4s::kRows; ++r) {
                    uint32_t qo, dof;
                    q4s::row_read_offsets(G, w.split, row0, rows, r, &qo, &dof);
                    qrow[r] = st + qo + lane * 16;
                    drow[r] = st + dof + lane * 2;
                }
                float acc[q4s::kRows];
#pragma unroll
                for (int r = 0; r < q4s::kRows; ++r) acc[r] = 0.0f;
                wait_stage(ws, bars + stage, parity, lane);
                for (int sub = 0; sub < nsub; ++sub) {
                    if ((sub << 5) + lane < kbs) {
                        const uint4* xe = xl + ((sub * q4s::kXEntries) << 5);
                        q4dev::XDigits xd;
                        const uint4 a0 = xe[0 << 5], a1 = xe[1 << 5], b0 = xe[2 << 5],
                                    b1 = xe[3 << 5], c0 = xe[4 << 5], c1 = xe[5 << 5],
                                    k = xe[6 << 5];
                        xd.a[0] = a0.x; xd.a[1] = a0.y; xd.a[2] = a0.z; xd.a[3] = a0.w;
                        xd.a[4] = a1.x; xd.a[5] = a1.y; xd.a[6] = a1.z; xd.a[7] = a1.w;
                        xd.b[0] = b0.x; xd.b[1] = b0.y; xd.b[2] = b0.z; xd.b[3] = b0.w;
                        xd.b[4] = b1.x; xd.b[5] = b1.y; xd.b[6] = b1.z; xd.b[7] = b1.w;
                        xd.c[0] = c0.x; xd.c[1] = c0.y; xd.c[2] = c0.z; xd.c[3] = c0.w;
                        xd.c[4] = c1.x; xd.c[5] = c1.y; xd.c[6] = c1.z; xd.c[7] = c1.w;
                        const float sx = __uint_as_float(k.w);
#pragma unroll
                        for (int r = 0; r < q4s::kRows; ++r) {
                            const uint4 q = *reinterpret_cast<const uint4*>(qrow[r] + sub * 512);
                            const float dd = __half2float(
                                *reinterpret_cast<const __half*>(drow[r] + sub * 64));
                            const float v = q4dev::block_dot_int(q, xd, (int32_t)k.x,
                                                                 (int32_t)k.y, (int32_t)k.z);
                            acc[r] = fmaf(dd * sx, v, acc[r]);
                        }
                    }
                }
                __syncwarp();
                // (under the stall test hook a stage's phase never completes, so it is
                // never armed twice)
                if (!is.done() && S.tx_extra() == 0) {
                    // the stage is free: refill it kStages tiles ahead (the proxy fence
                    // orders this warp's reads before the async writes)
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    is.issue(S, st, bars + stage, lane);
                }
                if (++stage == q4s::kStages) {
                    stage = 0;
                    parity ^= 1u;
                }
                reduce_tile(acc);
                if (nbuf + rows > 32) {
                    flush_rows(ws, G, w.split, brow0, nbuf, mine, lane);
                    brow0 = row0;
                    nbuf = 0;
                }
#pragma unroll
                for (int r = 0; r < q4s::kRows; ++r)
                    if (r < rows && lane == nbuf + r) mine = acc[r];
                nbuf += rows;
            }
            if (nbuf > 0) flush_rows(ws, G, w.split, brow0, nbuf, mine, lane);
            pos = p1;
        }
    }
}

}  // namespace

__global__ void __launch_bounds__(q4s::kThreads, Q4_STREAM_MINB)
    gemv_stream_kernel(const __grid_constant__ q4s::Params P) {
    stream_body(OneGroup{P});
}

cudaError_t setup_stream_kernel(int optin_smem) {
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, gemv_stream_kernel);
    if (e != cudaSuccess) return e;
    if (q4s::kSmemBytes + (int)fa.sharedSizeBytes > optin_smem) return cudaErrorInvalidValue;
    return cudaFuncSetAttribute(gemv_stream_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                q4s::kSmemBytes);
}

cudaError_t launch_stream(const q4s::Params& P, int grid, bool pdl, cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid, 1, 1);
    cfg.blockDim = dim3(q4s::kThreads, 1, 1);
    cfg.dynamicSmemBytes = q4s::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, gemv_stream_kernel, P);
}

}  // namespace q4k
