// Batched (5..16 tokens) Q4_0 decode GEMV on the sm_100a tensor cores.
//
// "Llamas on the Web" (gist.science technical summary of arXiv 2605.20706),
// section 3 "Dequantizzazione Integrata": for a matrix-matrix product the
// weights are dequantised into fast on-chip memory and reused there. Here the
// on-chip memory is tensor memory: each 32-weight block of a 128-row tile is
// dequantised once to (q - 8) as bf16 (exact) and written with tcgen05.st into
// tensor memory, and tcgen05.mma multiplies it with the tokens' activations held
// in shared memory as bf16 hi + lo parts (x = hi + lo to 2^-16 relative; both
// parts are columns of one N = 16 or 32 operand). Every block has its own
// binary32 accumulator, so its binary16 scale is applied exactly once, by the
// epilogue: y[t][r] += d[r][b] * (D_b[r][t] + D_b[r][N/2 + t]).
//
// Measured on B200 (M = 128, K = 16, bf16): one thread issues an MMA about
// every 50 cycles for any N up to 64; two issuing threads reach about 25; an
// N = 256 MMA takes 128 cycles (the tensor core's peak). With N = 16 or 32 the
// tensor core is bound by issue, so two threads issue alternate quads; the
// dequant fills the A ring quad by quad (4 blocks) as soon as a quad's earlier
// MMAs are done, and the accumulators live in a separate D ring read by the
// epilogue.
//
// Roles of the 15 warps of a CTA (one CTA per SM, persistent over a contiguous
// range of (tile, block) units, walked in stages of up to 8 blocks):
//   producer warp         per stage, on one barrier: the codes (one 2-D TMA box,
//                         128-byte swizzle), the activations (one box, binary32)
//                         and the scales (one box, or one bulk copy per row)
//   operand warps (8)     activations -> bf16 hi/lo B operands (shared -> shared),
//                         then codes -> (q - 8) bf16 A operands in tensor memory
//                         (two warps per tensor-memory lane quarter)
//   MMA issuers (2)       tcgen05.mma M = 128, N = 16 or 32, K = 16, one thread
//                         each, quads alternating; per quad all blocks chunk by
//                         chunk (consecutive MMAs accumulate into different
//                         blocks), two commits per quad
//   epilogue warps (4)    tcgen05.ld of the blocks' accumulators, scale, sum
// Shared-memory stages and tensor-memory quads are handed over with mbarriers;
// every wait is bounded and a wait that gives up records Q4_ERR_TIMEOUT, makes
// every role leave its loop, and the kernel still waits for its own copies and
// MMAs before it frees tensor memory and returns.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "q4_device.cuh"
#include "q4_maps.h"
#include "q4_tc_math.cuh"
#include "q4_tc_plan.h"

using namespace q4dev;

namespace q4k {

namespace {

constexpr uint32_t kTimeoutFlag = 1u;

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int32_t x,
                                            int32_t y, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void tc_alloc(uint32_t dst_smem, uint32_t cols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
                 "r"(cols)
                 : "memory");
}
__device__ __forceinline__ void tc_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tc_dealloc(uint32_t taddr, uint32_t cols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(cols)
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Arrive once on `bar` when every tcgen05.mma this thread issued so far is done.
__device__ __forceinline__ void tc_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     bar)
                 : "memory");
}
// D[128 x N] (+)= A[128 x 16] (tensor memory) * B[N x 16]^T (shared memory)
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %3, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %4, {%5, %5, %5, %5}, p;\n}\n" ::"r"(
            d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(accumulate), "r"(idesc), "r"(0u)
        : "memory");
}
// No memory clobber: the store writes tensor memory only, and as a volatile asm
// it stays ordered with the wait, fence and barrier asm that publish it, while
// shared-memory loads of later blocks may move above it.
__device__ __forceinline__ void tc_st16(uint32_t taddr, const uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15, %16};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
        "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
        "r"(v[15]));
}
__device__ __forceinline__ void tc_wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tc_ld16(uint32_t taddr, uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15}, [%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
          "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]),
          "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(taddr)
        : "memory");
}
__device__ __forceinline__ void tc_wait_ld() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

struct Ctx {
    uint8_t* smem;
    uint32_t sbase;  // shared-memory address of smem
    uint32_t tmem;   // tensor-memory base (lane 0, first column)
    int* abort_flag;
    int64_t lo, hi;

    __device__ uint32_t bar(int i) const { return sbase + 8u * (uint32_t)i; }
    __device__ bool aborted() const { return *reinterpret_cast<volatile int*>(abort_flag) != 0; }
    __device__ void abort(const q4t::Params& P) const {
        *reinterpret_cast<volatile int*>(abort_flag) = 1;
        atomicOr(P.ws, kTimeoutFlag);
    }
};

// Bounded wait of a single thread.
__device__ __forceinline__ bool wait1(const Ctx& C, const q4t::Params& P, int b, uint32_t parity) {
    if (mbar_wait_short_bounded(reinterpret_cast<uint64_t*>(C.smem + 8 * b), parity)) return true;
    C.abort(P);
    return false;
}

// Bounded wait of a whole warp; the outcome is the same for every lane.
__device__ __forceinline__ bool waitw(const Ctx& C, const q4t::Params& P, int b, uint32_t parity) {
    const bool ok = __all_sync(0xffffffffu,
                               mbar_wait_short_bounded(reinterpret_cast<uint64_t*>(C.smem + 8 * b), parity));
    if (!ok && (threadIdx.x & 31) == 0) C.abort(P);
    return ok;
}

__device__ __forceinline__ bool warp_aborted(const Ctx& C) {
    return __shfl_sync(0xffffffffu, C.aborted() ? 1 : 0, 0) != 0;
}

// ---- producer warp: every TMA byte of a stage, on one barrier ----
// Lane 0 issues the boxes (codes, activations, scales); with per-row scale
// copies every lane issues the copies of rows lane, lane + 32, ... The
// activations come from the previous kernel: the first kStages stages are
// requested without them (weights only), then, after the wait on the previous
// kernel, their activation boxes follow on the same barriers.
template <int BT>
__device__ void run_producer(const Ctx& C, const q4t::Params& P, int lane) {
    constexpr uint32_t kXBox = (uint32_t)BT * q4t::kS * 32 * 4;
    q4t::Walk wk;
    wk.begin(C.lo, C.hi);
    q4t::Walk wx = wk;
    q4t::Stage s;
    uint32_t q = 0;
    bool x_started = false;
    while (!warp_aborted(C)) {
        const bool has = wk.next(P, &s);
        if (!x_started && (!has || q == (uint32_t)q4t::kStages)) {
            pdl_wait();
            if (lane == 0) {
                for (uint32_t qq = 0; qq < q; ++qq) {
                    q4t::Stage sx;
                    wx.next(P, &sx);
                    const int st = (int)(qq % q4t::kStages);
                    tma_load_2d(C.sbase + q4t::stage_xraw(st), &P.maps[sx.g].x,
                                32 * q4t::window_of(sx.kb0), 0, C.bar(q4t::kBarFull + st));
                }
            }
            x_started = true;
        }
        if (!has) break;
        const int st = (int)(q % q4t::kStages);
        const uint32_t v = q / q4t::kStages;
        if (!waitw(C, P, q4t::kBarStageEmpty + st, (v & 1u) ^ 1u)) break;
        const q4t::Desc& G = P.g[s.g];
        const int32_t w0 = q4t::window_of(s.kb0);
        const uint32_t full = C.bar(q4t::kBarFull + st);
        uint32_t dbytes = 2048u;
        q4t::DCopy dc[4];
        if (!G.d_box) {
            uint32_t mine = 0;
#pragma unroll
            for (int rr = 0; rr < 4; ++rr) {
                const int r = lane + 32 * rr;
                dc[rr] = q4t::d_copy(G, s.tile, s.kb0, s.nblk, r);
                if ((int64_t)s.tile * q4t::kM + r < G.n) mine += dc[rr].bytes;
            }
            dbytes = __reduce_add_sync(0xffffffffu, mine);
        }
        if (lane == 0) {
            mbar_arrive_expect_tx(reinterpret_cast<uint64_t*>(C.smem + 8 * (q4t::kBarFull + st)),
                                  (uint32_t)q4t::kCodesBytes + kXBox + dbytes + P.tx_extra);
        }
        __syncwarp();
        if (lane == 0) {
            tma_load_2d(C.sbase + q4t::stage_codes(st), &P.maps[s.g].codes, 16 * w0,
                        s.tile * q4t::kM, full);
            if (G.d_box)
                tma_load_2d(C.sbase + q4t::stage_d(st), &P.maps[s.g].d, w0, s.tile * q4t::kM, full);
            if (x_started)
                tma_load_2d(C.sbase + q4t::stage_xraw(st), &P.maps[s.g].x, 32 * w0, 0, full);
        }
        if (!G.d_box) {
#pragma unroll
            for (int rr = 0; rr < 4; ++rr) {
                const int r = lane + 32 * rr;
                if ((int64_t)s.tile * q4t::kM + r < G.n)
                    bulk_g2s(C.smem + q4t::stage_d(st) + r * q4t::kDSlot,
                             reinterpret_cast<const uint8_t*>(G.d) + dc[rr].src_off, dc[rr].bytes,
                             reinterpret_cast<uint64_t*>(C.smem + 8 * (q4t::kBarFull + st)));
            }
        }
        ++q;
    }
    // every copy issued lands before the kernel may exit: wait for the latest
    // phase of each stage that was filled
    if (lane == 0) {
        const uint32_t n = q < (uint32_t)q4t::kStages ? q : (uint32_t)q4t::kStages;
        for (uint32_t k = 0; k < n; ++k) {
            const uint32_t qq = q - 1 - k;
            mbar_wait_bounded(
                reinterpret_cast<uint64_t*>(C.smem + 8 * (q4t::kBarFull + (int)(qq % q4t::kStages))),
                (qq / q4t::kStages) & 1u);
        }
    }
    __syncwarp();
}

// ---- operand warps: activations -> hi/lo B operands, codes -> A operands ----
// Eight warps (two per tensor-memory lane quarter) per stage: first the
// stage's activations (shared binary32 -> bf16 hi/lo, items split over the 256
// threads), then quad by quad the (q - 8) bf16 A operands of their blocks (warp
// half h takes the blocks of a quad with block % 2 == h).
template <int BT>
__device__ void run_prep(const Ctx& C, const q4t::Params& P, int warp, int lane) {
    constexpr int kN = q4t::mma_n(BT);
    constexpr int kThreadsX = q4t::kPrepWarps * 32;
    constexpr int kMaxItems = (BT * q4t::kS * 4 + kThreadsX - 1) / kThreadsX;
    const int quarter = warp & 3, half = warp >> 3;
    const int r = quarter * 32 + lane;  // tensor-memory lane = tile row
    const int tid = half * 128 + r;     // 0..255
    const uint32_t tlane = C.tmem + ((uint32_t)(quarter * 32) << 16);
    pdl_wait();  // every stage barrier also waits for the activations
    q4t::Walk wk;
    wk.begin(C.lo, C.hi);
    q4t::Stage s;
    uint32_t q = 0, j = 0;
    bool ok = true;
    while (ok && !warp_aborted(C) && wk.next(P, &s)) {
        const int st = (int)(q % q4t::kStages);
        const uint32_t v = q / q4t::kStages;
        if (!waitw(C, P, q4t::kBarFull + st, v & 1u)) break;
        const int c0 = s.kb0 - q4t::window_of(s.kb0);
        // activations
        {
            const int per_t = s.nblk * 4;
            const int items = P.b * per_t;
            const uint8_t* raw = C.smem + q4t::stage_xraw(st);
            uint8_t* xs = C.smem + q4t::stage_xop(st);
#pragma unroll
            for (int m = 0; m < kMaxItems; ++m) {
                const int it = tid + kThreadsX * m;
                if (it < items) {
                    const int t = it / per_t, rem = it - t * per_t;
                    const int i = rem >> 2, c2 = (rem >> 1) & 1, hh = rem & 1;
                    const float4* src = reinterpret_cast<const float4*>(
                        raw + t * (q4t::kS * 128) + (c0 + i) * 128 + c2 * 64 + hh * 32);
                    const float4 xa = src[0], xb = src[1];
                    const float e[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
                    uint4 H, L;
                    q4tm::split_row(e, &H, &L);
                    *reinterpret_cast<uint4*>(xs + q4t::x_row_off(kN, i, c2, hh, t, 0)) = H;
                    *reinterpret_cast<uint4*>(xs + q4t::x_row_off(kN, i, c2, hh, t, 1)) = L;
                }
            }
            // the MMA reads these operands through the async proxy
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if (lane == 0) mbar_arrive(C.bar(q4t::kBarXOpFull + st));
        }
        // A operands, quad by quad
        const uint8_t* codes = C.smem + q4t::stage_codes(st);
        for (int i0 = 0; i0 < s.nblk; i0 += q4t::kQ, ++j) {
            const int sa = (int)(j % q4t::kRingA);
            const uint32_t ua = j / q4t::kRingA;
            if (!waitw(C, P, q4t::kBarAEmpty + sa, (ua & 1u) ^ 1u)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const int nq = s.nblk - i0 < q4t::kQ ? s.nblk - i0 : q4t::kQ;
            uint4 qv[q4t::kQ / 2];
#pragma unroll
            for (int k = 0; k < q4t::kQ / 2; ++k) {
                const int ii = 2 * k + half;
                qv[k] = ii < nq ? *reinterpret_cast<const uint4*>(codes + q4t::code_off(r, c0 + i0 + ii))
                                : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int k = 0; k < q4t::kQ / 2; ++k) {
                const int ii = 2 * k + half;
                if (ii < nq) {
                    uint32_t a[16];
                    q4tm::dequant_block(qv[k], a);
                    tc_st16(tlane + q4t::a_col(sa, ii), a);
                }
            }
            tc_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(C.bar(q4t::kBarAFull + sa));
        }
        if (!ok) break;
        if (lane == 0) mbar_arrive(C.bar(q4t::kBarStageEmpty + st));
        ++q;
    }
}

// ---- MMA issuers ----
// Issuer e takes the quads j with j % 2 == e. Per quad: for each 16-value chunk
// the MMAs of the quad's blocks in turn (consecutive MMAs accumulate into
// different blocks), then one commit frees the quad's A columns and another
// hands its accumulators to the epilogue. Every issuer arrives once per stage
// on the stage's empty barrier: by commit when it read the stage's operands,
// else directly. One thread issues an MMA about every 50 cycles; two issuers
// keep the tensor core ahead of the weight stream.
template <int BT>
__device__ void run_mma(const Ctx& C, const q4t::Params& P, int e) {
    constexpr int kN = q4t::mma_n(BT);
    constexpr int kRD = q4t::ring_d(BT);
    constexpr uint32_t kIdesc = q4t::instr_desc(kN);
    constexpr uint32_t kOpStep = (uint32_t)kN * 32u >> 4;  // descriptor step between operands
    pdl_wait();  // the activations come after the previous kernel
    q4t::Walk wk;
    wk.begin(C.lo, C.hi);
    q4t::Stage s;
    uint32_t q = 0, j = 0;
    bool ok = true;
    while (ok && !C.aborted() && wk.next(P, &s)) {
        const int st = (int)(q % q4t::kStages);
        const uint32_t v = q / q4t::kStages;
        bool used = false;
        const uint64_t desc0 = q4t::smem_desc(C.sbase + q4t::stage_xop(st), kN);
        for (int i0 = 0; i0 < s.nblk; i0 += q4t::kQ, ++j) {
            if ((int)(j & 1u) != e) continue;
            if (!used) {
                if (!wait1(C, P, q4t::kBarXOpFull + st, v & 1u)) {
                    ok = false;
                    break;
                }
                used = true;
            }
            const int sa = (int)(j % q4t::kRingA), sd = (int)(j % kRD);
            const uint32_t ua = j / q4t::kRingA, ud = j / kRD;
            if (!wait1(C, P, q4t::kBarAFull + sa, ua & 1u) ||
                !wait1(C, P, q4t::kBarDEmpty + sd, (ud & 1u) ^ 1u)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const int nq = s.nblk - i0 < q4t::kQ ? s.nblk - i0 : q4t::kQ;
            const uint32_t a0 = C.tmem + q4t::a_col(sa, 0);
            const uint32_t d0 = C.tmem + q4t::d_col(BT, sd, 0);
            // operand of block i0 + ii, chunk c2: desc0 + (2 (i0 + ii) + c2) * kOpStep
            const uint64_t dq = desc0 + (uint64_t)(2 * i0) * kOpStep;
#pragma unroll
            for (int c2 = 0; c2 < 2; ++c2)
#pragma unroll
                for (int ii = 0; ii < q4t::kQ; ++ii)
                    if (ii < nq)
                        tc_mma(d0 + (uint32_t)(ii * kN), a0 + (uint32_t)(ii * q4t::kACols + 8 * c2),
                               dq + (uint64_t)(2 * ii + c2) * kOpStep, kIdesc, c2);
            tc_commit(C.bar(q4t::kBarAEmpty + sa));
            tc_commit(C.bar(q4t::kBarDFull + sd));
        }
        if (!ok) break;
        if (used)
            tc_commit(C.bar(q4t::kBarStageEmpty + st));
        else
            mbar_arrive(C.bar(q4t::kBarStageEmpty + st));
        ++q;
    }
    // every MMA issued completes before tensor memory is freed
    tc_commit(C.bar(q4t::kBarDone));
    mbar_wait_bounded(reinterpret_cast<uint64_t*>(C.smem + 8 * q4t::kBarDone), 0);
}

// ---- epilogue warps ----
template <int BT>
__device__ __forceinline__ void finish_piece(const q4t::Params& P, const q4t::Stage& s, int ew,
                                             int lane, const float (&acc)[BT]) {
    const q4t::Desc& G = P.g[s.g];
    const int r = ew * 32 + lane;
    const int64_t row = (int64_t)s.tile * q4t::kM + r;
    int np, slot;
    q4t::tile_pieces(P, G, s.tile, blockIdx.x, &np, &slot);
    if (np == 1) {
        if (row < G.n) {
#pragma unroll
            for (int t = 0; t < BT; ++t)
                if (t < P.b) G.y[t * G.n + row] = acc[t];
        }
        return;
    }
    float* part = reinterpret_cast<float*>(P.ws) + G.part_off;
    float* mine = part + ((int64_t)s.tile * G.maxp + slot) * P.b * q4t::kM + r;
#pragma unroll
    for (int t = 0; t < BT; ++t)
        if (t < P.b) mine[t * q4t::kM] = acc[t];
    __threadfence();
    __syncwarp();
    uint32_t tk = 0;
    uint32_t* ticket = P.ws + G.ticket_off + (int64_t)s.tile * 4 + ew;
    if (lane == 0) tk = atomicAdd(ticket, 1u);
    tk = __shfl_sync(0xffffffffu, tk, 0);
    if (tk != (uint32_t)np - 1u) return;
    __threadfence();
    const float* base = part + (int64_t)s.tile * G.maxp * P.b * q4t::kM + r;
#pragma unroll
    for (int t = 0; t < BT; ++t) {
        if (t < P.b) {
            float sum = 0.0f;
            for (int sl = 0; sl < np; ++sl) sum += __ldcg(base + ((int64_t)sl * P.b + t) * q4t::kM);
            if (row < G.n) G.y[t * G.n + row] = sum;
        }
    }
    if (lane == 0) *ticket = 0u;
}

// acc[t] += d * (hi + lo) of one block's accumulator columns: hi parts of
// token t in column t, lo parts in column N / 2 + t.
template <int BT>
__device__ __forceinline__ void accumulate(float (&acc)[BT], float dd, const uint32_t (&Dh)[16],
                                           const uint32_t (&Dl)[16]) {
    constexpr int kHalf = q4t::mma_n(BT) / 2;
#pragma unroll
    for (int t = 0; t < BT; ++t) {
        const float hi = __uint_as_float(Dh[t]);
        const float lo = kHalf == 8 ? __uint_as_float(Dh[8 + t]) : __uint_as_float(Dl[t]);
        acc[t] = fmaf(dd, hi + lo, acc[t]);
    }
}

template <int BT>
__device__ void run_epilogue(const Ctx& C, const q4t::Params& P, int ew, int lane) {
    constexpr int kN = q4t::mma_n(BT);
    constexpr int kRD = q4t::ring_d(BT);
    const int r = ew * 32 + lane;
    const uint32_t tlane = C.tmem + ((uint32_t)(ew * 32) << 16);
    pdl_wait();  // partial sums, tickets and y are written below
    q4t::Walk wk;
    wk.begin(C.lo, C.hi);
    q4t::Stage s;
    uint32_t q = 0, j = 0;
    bool ok = true;
    float acc[BT];
#pragma unroll
    for (int t = 0; t < BT; ++t) acc[t] = 0.0f;
    while (ok && !warp_aborted(C) && wk.next(P, &s)) {
        const int st = (int)(q % q4t::kStages);
        const uint32_t v = q / q4t::kStages;
        if (s.first) {
#pragma unroll
            for (int t = 0; t < BT; ++t) acc[t] = 0.0f;
        }
        if (!waitw(C, P, q4t::kBarFull + st, v & 1u)) break;  // the stage's scales
        const q4t::Desc& G = P.g[s.g];
        const int c0 = s.kb0 - q4t::window_of(s.kb0);
        const bool live = (int64_t)s.tile * q4t::kM + r < G.n;
        const uint8_t* dsm = C.smem + q4t::stage_d(st);
        const uint16_t* drow =
            G.d_box ? reinterpret_cast<const uint16_t*>(dsm + r * 16) + c0
                    : reinterpret_cast<const uint16_t*>(
                          dsm + r * q4t::kDSlot + q4t::d_copy(G, s.tile, s.kb0, s.nblk, r).lead);
        for (int i0 = 0; i0 < s.nblk; i0 += q4t::kQ, ++j) {
            const int sd = (int)(j % kRD);
            const uint32_t ud = j / kRD;
            if (!waitw(C, P, q4t::kBarDFull + sd, ud & 1u)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const int nq = s.nblk - i0 < q4t::kQ ? s.nblk - i0 : q4t::kQ;
            // two blocks per round: their columns, one wait, then the math
            for (int ii = 0; ii < nq; ii += 2) {
                uint32_t H0[16], L0[16], H1[16], L1[16];
                const uint32_t c = tlane + q4t::d_col(BT, sd, ii);
                tc_ld16(c, H0);
                if (kN == 32) tc_ld16(c + 16u, L0);
                if (ii + 1 < nq) {
                    tc_ld16(c + (uint32_t)kN, H1);
                    if (kN == 32) tc_ld16(c + (uint32_t)kN + 16u, L1);
                }
                tc_wait_ld();
                const int i = i0 + ii;
                accumulate<BT>(acc, live ? __half2float(__ushort_as_half(drow[i])) : 0.0f, H0, L0);
                if (ii + 1 < nq)
                    accumulate<BT>(acc, live ? __half2float(__ushort_as_half(drow[i + 1])) : 0.0f, H1,
                                   L1);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(C.bar(q4t::kBarDEmpty + sd));
        }
        if (!ok) break;
        __syncwarp();
        if (lane == 0) mbar_arrive(C.bar(q4t::kBarStageEmpty + st));
        ++q;
        if (s.last) finish_piece<BT>(P, s, ew, lane, acc);
    }
}

}  // namespace

template <int BT>
__global__ void __launch_bounds__(q4t::kThreads, 1) gemv_tc_kernel(const __grid_constant__ q4t::Params P) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    Ctx C;
    C.smem = smem_raw;
    C.sbase = smem_addr(smem_raw);
    C.abort_flag = reinterpret_cast<int*>(smem_raw + q4t::kAbortOff);
    q4t::cta_range(P.total, blockIdx.x, P.grid, &C.lo, &C.hi);

    if (threadIdx.x == 0) {
        uint64_t* b = reinterpret_cast<uint64_t*>(smem_raw);
        for (int st = 0; st < q4t::kStages; ++st) {
            mbar_init(b + q4t::kBarFull + st, 1);
            mbar_init(b + q4t::kBarXOpFull + st, q4t::kArrivalsXOpFull);
            mbar_init(b + q4t::kBarStageEmpty + st, q4t::kArrivalsStageEmpty);
        }
        for (int k = 0; k < q4t::kRingA; ++k) {
            mbar_init(b + q4t::kBarAFull + k, q4t::kArrivalsAFull);
            mbar_init(b + q4t::kBarAEmpty + k, 1);
        }
        for (int k = 0; k < q4t::kMaxRingD; ++k) {
            mbar_init(b + q4t::kBarDFull + k, 1);
            mbar_init(b + q4t::kBarDEmpty + k, q4t::kArrivalsDEmpty);
        }
        mbar_init(b + q4t::kBarDone, q4t::kMmaIssuers);
        // the swizzled code box needs a 1024-byte aligned destination
        *C.abort_flag = (C.sbase & 1023u) ? 1 : 0;
        if (C.sbase & 1023u) atomicOr(P.ws, kTimeoutFlag);
        mbar_fence_init();
    }
    // operand rows of absent tokens stay zero for the whole launch
    for (int st = 0; st < q4t::kStages; ++st)
        for (int off = threadIdx.x * 16; off < q4t::kXOpBytes; off += q4t::kThreads * 16)
            *reinterpret_cast<uint4*>(smem_raw + q4t::stage_xop(st) + off) = make_uint4(0, 0, 0, 0);
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    if (warp == 0) {
        tc_alloc(C.sbase + q4t::kTmemAddrOff, q4t::kTmemCols);
        tc_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    C.tmem = *reinterpret_cast<volatile uint32_t*>(smem_raw + q4t::kTmemAddrOff);

    pdl_launch_dependents();

    if (warp < q4t::kEpiWarp0 || (warp >= q4t::kEpiWarp0 + 4 && warp < q4t::kProdWarp)) {
        run_prep<BT>(C, P, warp, lane);
    } else if (warp < q4t::kEpiWarp0 + 4) {
        run_epilogue<BT>(C, P, warp - q4t::kEpiWarp0, lane);
    } else if (warp == q4t::kProdWarp) {
        run_producer<BT>(C, P, lane);
    } else {
        if (lane == 0) run_mma<BT>(C, P, warp - q4t::kMmaWarp0);
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tc_dealloc(C.tmem, q4t::kTmemCols);
    }
}

namespace {

template <int BT>
cudaError_t setup_one(int optin_smem) {
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, gemv_tc_kernel<BT>);
    if (e != cudaSuccess) return e;
    if (q4t::kSmemBytes + (int)fa.sharedSizeBytes > optin_smem) return cudaErrorInvalidValue;
    return cudaFuncSetAttribute(gemv_tc_kernel<BT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                q4t::kSmemBytes);
}

template <int BT>
cudaError_t launch_one(const q4t::Params& P, bool pdl, cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)P.grid, 1, 1);
    cfg.blockDim = dim3(q4t::kThreads, 1, 1);
    cfg.dynamicSmemBytes = q4t::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, gemv_tc_kernel<BT>, P);
}

}  // namespace

// Token count a launch is compiled for: the smallest of 2, 4, 8, 16 >= b.
// Token columns of the compiled kernels (up to four tokens take the CUDA-core kernel).
int tc_tokens(int b) { return b <= 8 ? 8 : 16; }

// Tensor maps of one GEMV for b tokens (rows and columns past the ends read as
// zero): code plane uint8 [n][k/2], box 128 B x 128 rows with the 128-byte
// swizzle; activations binary32 [b][k], box 256 x (b rounded up to the compiled
// token count); scale plane uint16 [n][k/32], box 8 x 128 rows, when its row
// stride is a multiple of 16 bytes (*d_box = 1).
cudaError_t encode_tc_maps(q4t::Maps* maps, int32_t* d_box, const uint8_t* qs, const uint16_t* d,
                           const float* x, int64_t n, int64_t k, int b) {
    cudaError_t e = encode_2d(&maps->codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, qs, (uint64_t)(k / 2),
                           (uint64_t)n, (uint64_t)(k / 2), 128u, (uint32_t)q4t::kM,
                           CU_TENSOR_MAP_SWIZZLE_128B);
    if (e != cudaSuccess) return e;
    e = encode_2d(&maps->x, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, x, (uint64_t)k, (uint64_t)b,
               (uint64_t)(k * 4), (uint32_t)(q4t::kS * 32), (uint32_t)tc_tokens(b),
               CU_TENSOR_MAP_SWIZZLE_NONE);
    if (e != cudaSuccess) return e;
    const int64_t nb = k / 32;
    *d_box = nb % 8 == 0 ? 1 : 0;
    if (*d_box)
        e = encode_2d(&maps->d, CU_TENSOR_MAP_DATA_TYPE_UINT16, d, (uint64_t)nb, (uint64_t)n,
                   (uint64_t)(nb * 2), (uint32_t)q4t::kS, (uint32_t)q4t::kM,
                   CU_TENSOR_MAP_SWIZZLE_NONE);
    return e;
}


cudaError_t setup_tc_kernels(int optin_smem) {
    cudaError_t e;
    if ((e = setup_one<8>(optin_smem)) != cudaSuccess) return e;
    return setup_one<16>(optin_smem);
}

cudaError_t launch_tc(const q4t::Params& P, bool pdl, cudaStream_t stream) {
    switch (tc_tokens(P.b)) {
        case 8: return launch_one<8>(P, pdl, stream);
        default: return launch_one<16>(P, pdl, stream);
    }
}

}  // namespace q4k
