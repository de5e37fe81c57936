// Batch-1 Q4_0 decode mat-vec for sm_100a.
//
// "Llamas on the Web" (gist.science technical summary of arXiv 2605.20706),
// section 3 "Dequantizzazione Integrata": the decode mat-vec dequantises in
// registers; no dequantised weight is ever written to memory. The work split is
// described in q4_b1_plan.h. Per CTA (8 warps; two CTAs fit one SM):
//  * the piece's units (8 rows x 32 blocks: 4 KB of codes and their binary16
//    scales) stream from HBM into a ring of shared-memory slots as 2-D tensor
//    loads on the TMA engine, each completing on its slot's mbarrier. The first
//    units are requested before the wait on the previous kernel (programmatic
//    dependent launch): weights never depend on an earlier kernel, so
//    consecutive launches overlap their weight streams. A warp that has read a
//    unit requests the unit `slots` further into the slot it just freed; the
//    issuing lane rotates with the unit, so no thread has many copies in flight;
//  * the warps quantise the piece's activations once into shared memory (31-bit
//    block fixed point as two 16-bit digit planes, q4_intdot.cuh), then take
//    units round-robin. Lane l owns block l of the unit's slice: its activation
//    digits stay in registers while the slice does not change, and for each of
//    the unit's rows it reads the block's 16 code bytes with one 128-bit shared
//    load, forms sum_j (q_j - 8) X_j with 16 dp2a instructions, and applies the
//    block's binary16 scale and power-of-two activation scale once. A slice
//    holding a flagged block (an element the fixed point cannot carry within
//    2^-14 of itself) is multiplied in binary32 instead;
//  * the 8 rows of a unit are summed over the lanes with shuffles and written to
//    per-(row, slice) shared slots; after the last unit each row's slices are
//    added in slice order (deterministic) and y is stored, or, for a K split
//    across CTAs, a partial sum that the last split of the row to arrive adds up
//    in split order.
// Every wait is bounded (%globaltimer): a wait that gives up records
// Q4_ERR_TIMEOUT in the workspace header and the CTA stops its work.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "q4_b1_plan.h"
#include "q4_device.cuh"
#include "q4_intdot.cuh"
#include "q4_maps.h"

using namespace q4dev;

namespace q4k {

namespace {

constexpr uint32_t kTimeoutFlag = 1u;
constexpr int kConsumerBar = 1;  // named barrier of the CTA's warps

__device__ __forceinline__ void consumer_sync() {
    asm volatile("bar.sync %0, %1;" ::"n"(kConsumerBar), "n"(q4b::kThreads) : "memory");
}


__device__ __forceinline__ float half_bits_f32(uint32_t h) {
    return __half2float(__ushort_as_half((unsigned short)h));
}

// Quantise the piece's activations (all consumer threads): item i of
// S * 32 * 8 is float4 g = i % 8 of block i / 8 (local slice (i / 8) / 32), and
// thread `tid` takes items tid + 256 m, m < S. All of a thread's loads are issued
// before any is used (one latency instead of S). Eight consecutive lanes share a
// block; the block's largest |x|, digit sums and flag are reduced over them with
// shuffles.
__device__ __forceinline__ void stage_x(const q4b::Desc& G, int s0, int S, uint8_t* xs, int tid) {
    float4 v[q4b::kPieceSlices];
#pragma unroll
    for (int m = 0; m < q4b::kPieceSlices; ++m) {
        const int i = m * q4b::kWarps * 32 + tid;
        const int jl = i >> 3, g = i & 7;
        const int s = jl >> 5, jb = jl & 31;
        const int64_t b = (int64_t)(s0 + s) * q4b::kSliceBlocks + jb;
        v[m] = (m < S && jb < q4b::slice_blocks(G, s0 + s))
                   ? __ldcg(reinterpret_cast<const float4*>(G.x + b * 32) + g)
                   : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    }
#pragma unroll
    for (int m = 0; m < q4b::kPieceSlices; ++m) {
        if (m >= S) break;
        const int i = m * q4b::kWarps * 32 + tid;
        const int jl = i >> 3, g = i & 7;
        const int s = jl >> 5, jb = jl & 31;
        uint32_t mx = max(max(__float_as_uint(v[m].x) & 0x7FFFFFFFu, __float_as_uint(v[m].y) & 0x7FFFFFFFu),
                          max(__float_as_uint(v[m].z) & 0x7FFFFFFFu, __float_as_uint(v[m].w) & 0x7FFFFFFFu));
#pragma unroll
        for (int off = 4; off > 0; off >>= 1) mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        float sc, inv;
        bool ok = xq_scale(mx, &sc, &inv);
        const float e[4] = {v[m].x, v[m].y, v[m].z, v[m].w};
        int32_t d0[4], d1[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            bool ek = true;
            const int32_t X = ok ? xq_int(e[k], inv, &ek) : 0;
            ok = ok && ek;
            x_digits16(X, &d0[k], &d1[k]);
        }
        int32_t sum0 = d0[0] + d0[1] + d0[2] + d0[3], sum1 = d1[0] + d1[1] + d1[2] + d1[3];
        uint32_t flag = ok ? 0u : 1u;
#pragma unroll
        for (int off = 4; off > 0; off >>= 1) {
            sum0 += __shfl_xor_sync(0xffffffffu, sum0, off);
            sum1 += __shfl_xor_sync(0xffffffffu, sum1, off);
            flag |= __shfl_xor_sync(0xffffffffu, flag, off);
        }
        const uint32_t half = (uint32_t)(g & 1) * 8u;
        *reinterpret_cast<uint2*>(xs + q4b::xchunk_offset(s, g >> 1, jb) + half) =
            make_uint2(pack16(d0[0], d0[1]), pack16(d0[2], d0[3]));
        *reinterpret_cast<uint2*>(xs + q4b::xchunk_offset(s, 4 + (g >> 1), jb) + half) =
            make_uint2(pack16(d1[0], d1[1]), pack16(d1[2], d1[3]));
        if (g == 0)
            *reinterpret_cast<uint4*>(xs + q4b::xchunk_offset(s, 8, jb)) =
                make_uint4((uint32_t)(-8 * sum0), (uint32_t)(-8 * sum1), __float_as_uint(sc * 0.0625f), flag);
    }
}

// Copy the piece's activations of B tokens (2..4) into shared memory, binary32:
// chunk c (values 4c .. 4c+3) of block j of local slice s of token t goes to
// xfchunk_offset(s, t, B, c, j). Item i of a (slice, token) pair is chunk
// 2 (w % 4) + (l % 2) of block 16 (w / 4) + l / 2 for i = 32 w + l, so two
// neighbouring lanes read the two halves of one 32-byte sector; blocks past K are
// staged as zeros. Loads go out eight rounds at a time before their stores.
template <int B>
__device__ __forceinline__ void stage_xf(const q4b::Desc& G, int s0, int S, uint8_t* xs, int tid) {
    static_assert(q4b::kThreads == 256, "one (slice, token) pair of 256 chunks per round");
    const int64_t k = (int64_t)G.nb * 32;
    const int rounds = S * B;  // one (slice, token) pair of 256 chunks per round
    for (int m0 = 0; m0 < rounds; m0 += 8) {
        float4 v[8];
#pragma unroll
        for (int m = 0; m < 8; ++m) {
            const int st = m0 + m, s = st / B, t = st - s * B;
            const int w = tid >> 5, l = tid & 31;
            const int c = ((w & 3) << 1) | (l & 1), jb = ((w >> 2) << 4) | (l >> 1);
            v[m] = (st < rounds && jb < q4b::slice_blocks(G, s0 + s))
                       ? __ldcg(reinterpret_cast<const float4*>(G.x + t * k +
                                                                ((int64_t)(s0 + s) * q4b::kSliceBlocks + jb) * 32) + c)
                       : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        }
#pragma unroll
        for (int m = 0; m < 8; ++m) {
            const int st = m0 + m, s = st / B, t = st - s * B;
            if (st >= rounds) break;
            const int w = tid >> 5, l = tid & 31;
            const int c = ((w & 3) << 1) | (l & 1), jb = ((w >> 2) << 4) | (l >> 1);
            *reinterpret_cast<float4*>(xs + q4b::xfchunk_offset(s, t, B, c, jb)) = v[m];
        }
    }
}

// Sum each of 8 rows over the 32 lanes: afterwards lane l holds the total of
// row l / 4 (lanes 4r .. 4r + 3 all hold row r).
__device__ __forceinline__ float reduce8(float (&v)[8], int lane) {
    const bool b4 = lane & 16, b3 = lane & 8, b2 = lane & 4;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float send = b4 ? v[i] : v[i + 4], keep = b4 ? v[i + 4] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const float send = b3 ? v[i] : v[i + 2], keep = b3 ? v[i + 2] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
    }
    {
        const float send = b2 ? v[0] : v[1], keep = b2 ? v[1] : v[0];
        v[0] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
    }
    v[0] += __shfl_xor_sync(0xffffffffu, v[0], 2);
    v[0] += __shfl_xor_sync(0xffffffffu, v[0], 1);
    return v[0];
}

__device__ __forceinline__ bool wait_bounded(uint64_t* bar, uint32_t parity, uint32_t* ws,
                                             volatile int* abort_flag, int lane) {
    if (mbar_wait_short_bounded(bar, parity)) return true;
    if (lane == 0) {
        atomicOr(ws, kTimeoutFlag);
        *abort_flag = 1;
    }
    return false;
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int32_t x, int32_t y,
                                            uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_addr(bar))
        : "memory");
}

// Issue the loads of unit (tile t, local slice s) of a piece into ring slot
// `slot` (whole warp): lane `lane_issue` loads the codes (and, with the scale
// map, the scales) as 2-D boxes; without the scale map lanes 8..15 copy one row's
// scales each. Spreading the issuing lane over units and warps keeps few copies
// in flight per thread.
template <bool kDMap>
__device__ __forceinline__ void issue_unit(const q4b::Params& P, const q4b::Desc& G, const q4b::Piece& pc,
                                           int gsl, int t, int slot, uint8_t* ring, uint64_t* full,
                                           int lane, int lane_issue) {
    const int32_t row0 = pc.r0 + t * q4b::kTileRows;
    uint8_t* dst = ring + (size_t)slot * q4b::kSlotBytes;
    if (kDMap) {
        if (lane == lane_issue) {
            mbar_arrive_expect_tx(full + slot, q4b::kMapCodeBytes + q4b::kMapScaleBytes + P.tx_extra);
            tma_load_2d(dst, &P.qs_map[pc.g], gsl * (q4b::kSliceBlocks * 4), row0, full + slot);
            tma_load_2d(dst + q4b::kSlotQs, &P.d_map[pc.g], gsl * q4b::kSliceBlocks, row0, full + slot);
        }
        return;
    }
    q4b::LaneCopy c = q4b::lane_copy(G, pc, t, gsl, lane);
    c.active = c.active && c.scales;
    const uint32_t bytes = c.active ? c.bytes : 0u;
    const uint32_t total = __reduce_add_sync(0xffffffffu, bytes) + q4b::kMapCodeBytes;
    if (lane == lane_issue) {
        mbar_arrive_expect_tx(full + slot, total + P.tx_extra);
        tma_load_2d(dst, &P.qs_map[pc.g], gsl * (q4b::kSliceBlocks * 4), row0, full + slot);
    }
    __syncwarp();
    if (c.active)
        bulk_g2s(dst + c.dst, reinterpret_cast<const uint8_t*>(G.d) + c.src_off, c.bytes, full + slot);
}

// Position of a warp in its piece's unit sequence (unit u = t * S + s), moved
// 8 units at a time without division.
struct Cursor {
    int t, s;
    __device__ void set(int u, int S) {
        t = u / S;
        s = u - t * S;
    }
    __device__ void advance(int dt, int ds, int S) {
        t += dt;
        s += ds;
        if (s >= S) {
            s -= S;
            ++t;
        }
    }
};

// Activation data of lane `lane` for local slice s.
struct LaneX {
    XPlanes p;
    float scale;
    bool flagged;  // some block of the slice takes the binary32 path
};

__device__ __forceinline__ void load_lane_x(const uint8_t* xs, int s, int lane, LaneX* lx) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const uint4 a = *reinterpret_cast<const uint4*>(xs + q4b::xchunk_offset(s, q, lane));
        const uint4 b = *reinterpret_cast<const uint4*>(xs + q4b::xchunk_offset(s, 4 + q, lane));
        lx->p.a0[4 * q] = a.x;
        lx->p.a0[4 * q + 1] = a.y;
        lx->p.a0[4 * q + 2] = a.z;
        lx->p.a0[4 * q + 3] = a.w;
        lx->p.a1[4 * q] = b.x;
        lx->p.a1[4 * q + 1] = b.y;
        lx->p.a1[4 * q + 2] = b.z;
        lx->p.a1[4 * q + 3] = b.w;
    }
    const uint4 k = *reinterpret_cast<const uint4*>(xs + q4b::xchunk_offset(s, 8, lane));
    lx->p.c0 = (int32_t)k.x;
    lx->p.c1 = (int32_t)k.y;
    lx->scale = __uint_as_float(k.z);
    lx->flagged = __any_sync(0xffffffffu, k.w != 0u);
}

}  // namespace

template <int B, bool kDMap>
__global__ void __launch_bounds__(q4b::kThreads, q4b::ctas_per_sm(B))
    gemv_b1_kernel(const __grid_constant__ q4b::Params P) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const q4b::Piece pc = q4b::piece_of(P, blockIdx.x);
    const q4b::Desc& G = P.g[pc.g];
    int s0, S;
    q4b::piece_slices(G, pc.split, &s0, &S);
    const int T = q4b::piece_tiles(pc);
    const int U = T * S;
    const int slots = P.slots;
    const int nb = G.nb;
    const float* const xg_base = G.x;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    float* red = reinterpret_cast<float*>(smem + q4b::red_offset());
    uint8_t* xs = smem + q4b::x_offset(P);
    uint8_t* ring = smem + q4b::ring_offset(P);
    __shared__ int abort_flag;

    if (threadIdx.x == 0) {
        for (int i = 0; i < slots; ++i) mbar_init(full + i, 1);
        abort_flag = 0;
        mbar_fence_init();
    }
    __syncthreads();
    pdl_launch_dependents();

    // the warp's units are u = warp + 8 k; cursors step 8 units at a time
    const int dt8 = q4b::kWarps / S, ds8 = q4b::kWarps - dt8 * S;  // one step: kWarps units
    // weights never depend on an earlier kernel: the first `slots` units are
    // requested before the wait on the previous kernel (unit u by warp u % 8,
    // into slot u)
    {
        Cursor c;
        c.set(warp, S);
        for (int u = warp, k = 0; u < U && u < slots; u += q4b::kWarps, ++k) {
            issue_unit<kDMap>(P, G, pc, s0 + c.s, c.t, u, ring, full, lane, k & 31);
            c.advance(dt8, ds8, S);
        }
    }

    // warm L2 with the piece's activations (a hint: they are read only after
    // the wait, and L2 holds whatever the previous kernel wrote)
    if (threadIdx.x == 32) {
        const int64_t e0 = (int64_t)s0 * q4b::kSliceBlocks * 32;
        const int64_t e1 = min((int64_t)(s0 + S) * q4b::kSliceBlocks * 32, (int64_t)nb * 32);
#pragma unroll
        for (int tk = 0; tk < B; ++tk)
            bulk_prefetch_l2(xg_base + (int64_t)tk * nb * 32 + e0, (uint32_t)((e1 - e0) * 4));
    }
    pdl_wait();
    const int tid = threadIdx.x;
    if constexpr (B == 1)
        stage_x(G, s0, S, xs, tid);
    else
        stage_xf<B>(G, s0, S, xs, tid);
    consumer_sync();

    volatile int* abort_v = &abort_flag;
    int cur = -1;
    LaneX lx;                  // one token: digit planes
    uint64_t xp[B][16];        // 2..4 tokens: binary32 pairs, chunk c as pairs 2c, 2c + 1
    const UnpackConsts kc = unpack_consts_default();
    // refills: unit u + slots goes to the slot unit u leaves (the same warp's)
    Cursor cu, cr;
    cu.set(warp, S);
    cr.set(warp + slots, S);
    int slot = warp;
    uint32_t phase = 0;
    int issued_end = min(U, slots);
    int u = warp, k = 0;
    for (; u < U; u += q4b::kWarps, ++k) {
        if (*abort_v) break;
        const int t = cu.t, s = cu.s;
        if (s != cur) {
            if constexpr (B == 1) {
                load_lane_x(xs, s, lane, &lx);
            } else {
#pragma unroll
                for (int tk = 0; tk < B; ++tk)
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const float4 f =
                            *reinterpret_cast<const float4*>(xs + q4b::xfchunk_offset(s, tk, B, c, lane));
                        xp[tk][2 * c] = pack2(f.x, f.y);
                        xp[tk][2 * c + 1] = pack2(f.z, f.w);
                    }
            }
            cur = s;
        }
        const bool ok = wait_bounded(full + slot, phase, P.ws, &abort_flag, lane);
        if (!__all_sync(0xffffffffu, ok)) break;
        const int gs = s0 + s;
        const int bs = min(q4b::kSliceBlocks, nb - gs * q4b::kSliceBlocks);
        const int nr = min(q4b::kTileRows, pc.r1 - pc.r0 - t * q4b::kTileRows);
        const uint8_t* sb = ring + (size_t)slot * q4b::kSlotBytes;
        float v[B][8];
        if constexpr (B > 1) {
            // each code word unpacked once into exact (q - 8) pairs, reused by
            // every token with f32x2 fused multiply-adds
            const bool whole = kDMap && bs == q4b::kSliceBlocks && nr == q4b::kTileRows;
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                const uint4 q = *reinterpret_cast<const uint4*>(sb + r * (q4b::kSliceBlocks * 16) + lane * 16);
                const uint32_t dh = *reinterpret_cast<const uint16_t*>(
                    sb + (kDMap ? q4b::kSlotQs + r * q4b::kDMapRow + 2 * lane
                                : q4b::scale_offset(G, pc, t, gs, r, lane)));
                const uint32_t words[4] = {q.x, q.y, q.z, q.w};
                uint64_t acc[B][2];  // two chains per token: even and odd words
#pragma unroll
                for (int tk = 0; tk < B; ++tk) acc[tk][0] = acc[tk][1] = 0ull;
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    uint64_t pr[4];
                    code_pairs(words[w], kc, pr);
#pragma unroll
                    for (int tk = 0; tk < B; ++tk) {
                        uint64_t a = acc[tk][w & 1];
                        a = ffma2(pr[0], xp[tk][2 * w], a);
                        a = ffma2(pr[1], xp[tk][2 * w + 1], a);
                        a = ffma2(pr[2], xp[tk][2 * w + 8], a);
                        a = ffma2(pr[3], xp[tk][2 * w + 9], a);
                        acc[tk][w & 1] = a;
                    }
                }
                const float d = half_bits_f32(dh);
                const bool live = whole || (lane < bs && r < nr);
#pragma unroll
                for (int tk = 0; tk < B; ++tk) v[tk][r] = live ? d * sum_pairs(acc[tk][0], acc[tk][1]) : 0.0f;
            }
        } else if (!lx.flagged) {
            const float ls = lx.scale;
            if (kDMap && bs == q4b::kSliceBlocks && nr == q4b::kTileRows) {
#pragma unroll
                for (int r = 0; r < 8; ++r) {
                    const uint4 q = *reinterpret_cast<const uint4*>(sb + r * (q4b::kSliceBlocks * 16) + lane * 16);
                    const uint32_t dh =
                        *reinterpret_cast<const uint16_t*>(sb + q4b::kSlotQs + r * q4b::kDMapRow + 2 * lane);
                    v[0][r] = half_bits_f32(dh) * ls * block_dot16(q, lx.p);
                }
            } else {
#pragma unroll
                for (int r = 0; r < 8; ++r) {
                    const uint4 q = *reinterpret_cast<const uint4*>(sb + r * (q4b::kSliceBlocks * 16) + lane * 16);
                    const uint32_t dh = *reinterpret_cast<const uint16_t*>(
                        sb + (kDMap ? q4b::kSlotQs + r * q4b::kDMapRow + 2 * lane
                                    : q4b::scale_offset(G, pc, t, gs, r, lane)));
                    const float dot = block_dot16(q, lx.p);
                    v[0][r] = (lane < bs && r < nr) ? half_bits_f32(dh) * ls * dot : 0.0f;
                }
            }
        } else {
            // exact path: binary32 products with the activations themselves
            float4 xf[8];
            const float4* xg = reinterpret_cast<const float4*>(xg_base + ((int64_t)gs * q4b::kSliceBlocks + lane) * 32);
#pragma unroll
            for (int c = 0; c < 8; ++c) xf[c] = lane < bs ? __ldcg(xg + c) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                const uint4 q = *reinterpret_cast<const uint4*>(sb + r * (q4b::kSliceBlocks * 16) + lane * 16);
                const uint32_t dh = *reinterpret_cast<const uint16_t*>(
                    sb + (kDMap ? q4b::kSlotQs + r * q4b::kDMapRow + 2 * lane
                                : q4b::scale_offset(G, pc, t, gs, r, lane)));
                const float2 d2 = block_dot(q, xf, kc);
                v[0][r] = (lane < bs && r < nr) ? half_bits_f32(dh) * (d2.x + d2.y) : 0.0f;
            }
        }
        // the slot is read: refill it with unit u + slots (the proxy fence orders
        // this warp's shared-memory reads before the copies' writes)
        __syncwarp();
        if (u + slots < U) {
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            issue_unit<kDMap>(P, G, pc, s0 + cr.s, cr.t, slot, ring, full, lane, (k + slots / q4b::kWarps) & 31);
            issued_end = u + slots + 1;
        }
        const int r = lane >> 2;
#pragma unroll
        for (int tk = 0; tk < B; ++tk) {
            const float row_sum = reduce8(v[tk], lane);
            if ((lane & 3) == 0 && r < nr) red[((tk * T + t) * q4b::kTileRows + r) * S + s] = row_sum;
        }
        cu.advance(dt8, ds8, S);
        cr.advance(dt8, ds8, S);
        slot += q4b::kWarps;
        if (slot >= slots) {
            slot -= slots;
            phase ^= 1u;
        }
    }
    if (*abort_v) {
        // leave no copy in flight: wait (bounded) for the units this warp
        // requested and did not read
        for (; u < issued_end; u += q4b::kWarps) {
            mbar_wait_short_bounded(full + slot, phase);
            slot += q4b::kWarps;
            if (slot >= slots) {
                slot -= slots;
                phase ^= 1u;
            }
        }
    }
    consumer_sync();
    if (*abort_v) return;

    // each (token, row)'s slices in slice order; y is [b][n]
    const int rows = pc.r1 - pc.r0;
    const int T8 = T * q4b::kTileRows;
    if (G.splits == 1) {
        for (int i = tid; i < rows * B; i += q4b::kThreads) {
            const int tk = i / rows, rl = i - tk * rows;
            float sum = 0.0f;
            for (int s = 0; s < S; ++s) sum += red[(tk * T8 + rl) * S + s];
            G.y[(int64_t)tk * G.n + pc.r0 + rl] = sum;
        }
        return;
    }
    // K split: this piece's partial sums, then one ticket per row range (pieces
    // j of every split cover the same rows); the CTA that arrives last adds the
    // range's partials in split order and resets the ticket
    float* part = reinterpret_cast<float*>(P.ws) + G.part_off;
    uint32_t* ticket = P.ws + G.ticket_off + pc.j;
    for (int i = tid; i < rows * B; i += q4b::kThreads) {
        const int tk = i / rows, rl = i - tk * rows;
        float sum = 0.0f;
        for (int s = 0; s < S; ++s) sum += red[(tk * T8 + rl) * S + s];
        part[((int64_t)pc.split * B + tk) * G.n + pc.r0 + rl] = sum;
    }
    __threadfence();
    consumer_sync();
    __shared__ int last_split;
    if (tid == 0) last_split = atomicAdd(ticket, 1u) == (uint32_t)G.splits - 1u;
    consumer_sync();
    if (!last_split) return;
    __threadfence();
    for (int i = tid; i < rows * B; i += q4b::kThreads) {
        const int tk = i / rows;
        const int64_t row = pc.r0 + (i - tk * rows);
        float sum = 0.0f;
        for (int sp = 0; sp < G.splits; ++sp) sum += __ldcg(part + ((int64_t)sp * B + tk) * G.n + row);
        G.y[(int64_t)tk * G.n + row] = sum;
    }
    if (tid == 0) *ticket = 0u;
}

namespace {
template <int B>
cudaError_t setup_b1_tokens(int optin_smem) {
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, gemv_b1_kernel<B, true>);
    if (e != cudaSuccess) return e;
    const int budget = q4b::smem_budget(B);
    if (budget + (int)fa.sharedSizeBytes > optin_smem) return cudaErrorInvalidValue;
    e = cudaFuncSetAttribute(gemv_b1_kernel<B, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, budget);
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(gemv_b1_kernel<B, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, budget);
}
}  // namespace

cudaError_t setup_b1_kernel(int optin_smem) {
    cudaError_t e = setup_b1_tokens<1>(optin_smem);
    if (e == cudaSuccess) e = setup_b1_tokens<2>(optin_smem);
    if (e == cudaSuccess) e = setup_b1_tokens<3>(optin_smem);
    if (e == cudaSuccess) e = setup_b1_tokens<4>(optin_smem);
    return e;
}

// Tensor maps of one GEMV: the code plane as uint32 [n][k/8] in boxes of 128 x 8
// (one unit: 8 rows x 512 bytes), and, when its row stride is a multiple of 16
// bytes, the scale plane uint16 [n][k/32] in boxes of 32 x 8 (*d_map = 1).
cudaError_t encode_b1_maps(CUtensorMap* qs_map, CUtensorMap* d_map, int32_t* d_ok, const uint8_t* qs,
                           const uint16_t* d, int64_t n, int64_t k) {
    cudaError_t e = encode_2d(qs_map, CU_TENSOR_MAP_DATA_TYPE_UINT32, qs, (uint64_t)(k / 8), (uint64_t)n,
                              (uint64_t)(k / 2), (uint32_t)(q4b::kSliceBlocks * 4), (uint32_t)q4b::kTileRows,
                              CU_TENSOR_MAP_SWIZZLE_NONE);
    if (e != cudaSuccess) return e;
    const int64_t nb = k / 32;
    *d_ok = nb % 8 == 0 ? 1 : 0;
    if (*d_ok)
        e = encode_2d(d_map, CU_TENSOR_MAP_DATA_TYPE_UINT16, d, (uint64_t)nb, (uint64_t)n, (uint64_t)(nb * 2),
                      (uint32_t)q4b::kSliceBlocks, (uint32_t)q4b::kTileRows, CU_TENSOR_MAP_SWIZZLE_NONE);
    return e;
}

cudaError_t launch_b1(const q4b::Params& P, bool pdl, cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)P.npieces, 1, 1);
    cfg.blockDim = dim3(q4b::kThreads, 1, 1);
    cfg.dynamicSmemBytes = q4b::smem_bytes(P);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    // the scale-map instantiation when every GEMV of the group has a scale map
    bool all_maps = true;
    for (int i = 0; i < P.count; ++i) all_maps = all_maps && P.g[i].d_map;
    switch (P.b) {
        case 1:
            return all_maps ? cudaLaunchKernelEx(&cfg, gemv_b1_kernel<1, true>, P)
                            : cudaLaunchKernelEx(&cfg, gemv_b1_kernel<1, false>, P);
        case 2:
            return all_maps ? cudaLaunchKernelEx(&cfg, gemv_b1_kernel<2, true>, P)
                            : cudaLaunchKernelEx(&cfg, gemv_b1_kernel<2, false>, P);
        case 3:
            return all_maps ? cudaLaunchKernelEx(&cfg, gemv_b1_kernel<3, true>, P)
                            : cudaLaunchKernelEx(&cfg, gemv_b1_kernel<3, false>, P);
        case 4:
            return all_maps ? cudaLaunchKernelEx(&cfg, gemv_b1_kernel<4, true>, P)
                            : cudaLaunchKernelEx(&cfg, gemv_b1_kernel<4, false>, P);
        default:
            return cudaErrorInvalidValue;
    }
}

}  // namespace q4k
