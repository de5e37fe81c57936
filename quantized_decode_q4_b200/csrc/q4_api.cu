// C ABI of the Q4_0 decode library: argument checks (before any CUDA call),
// launch planning, the layer stack with programmatic dependent launch, CUDA
// graph capture, host interchange helpers and the host-side plan validator.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <atomic>
#include <climits>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include "../../include/q4.h"
#include "../../include/q4_debug.h"
#include "q4_device.cuh"
#include "q4_intdot.cuh"
#include "q4_plan.h"
#include "q4_stream_plan.h"
#include "q4_tc_math.cuh"
#include "q4_tc_plan.h"

namespace q4k {
cudaError_t launch_pack(const float* w, uint8_t* qs, uint16_t* d, int64_t nblocks,
                        cudaStream_t stream);
cudaError_t launch_dequant(const uint8_t* qs, const uint16_t* d, float* out, int64_t nblocks,
                           cudaStream_t stream);
cudaError_t setup_gemv_kernels(int optin_smem);
cudaError_t launch_gemv(const q4plan::GemvParams& P, bool pdl, cudaStream_t stream);
cudaError_t setup_stream_kernel(int optin_smem);
cudaError_t launch_stream(const q4s::Params& P, int grid, bool pdl, cudaStream_t stream);
cudaError_t setup_tc_kernels(int optin_smem);
cudaError_t launch_tc(const q4t::Params& P, bool pdl, cudaStream_t stream);
cudaError_t encode_tc_maps(q4t::Maps* maps, int32_t* d_box, const uint8_t* qs, const uint16_t* d,
                           const float* x, int64_t n, int64_t k, int b);
int tc_tokens(int b);
}  // namespace q4k

using q4plan::GemvDesc;
using q4plan::GemvParams;

namespace {

std::atomic<uint64_t> g_launches{0};
thread_local cudaError_t g_last_cuda_error = cudaSuccess;

// Record a failed CUDA call for q4_last_cuda_error() and map it to Q4_ERR_CUDA.
bool cuda_failed(cudaError_t e) {
    if (e == cudaSuccess) return false;
    g_last_cuda_error = e;
    return true;
}

// CTAs a launch aims for before K is split further: two per SM of a B200.
constexpr int64_t kTargetUnits = 2 * 148;
constexpr int kMaxCudaCoreBatch = 4;
// Batches of at least this many tokens run on the tensor-core kernel; smaller
// ones (above 1) on the CUDA-core kernel.
#ifndef Q4_TC_MIN_BATCH
#define Q4_TC_MIN_BATCH 2
#endif
constexpr int kTcMinBatch = Q4_TC_MIN_BATCH;
constexpr uint32_t kMaxSmem = 226 * 1024;  // below the opt-in limit minus static smem

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
int64_t round_up(int64_t a, int64_t b) { return ceil_div(a, b) * b; }

q4_status check_shape(int64_t n, int64_t k) {
    if (n < 1 || k < Q4_QK || k % Q4_QK != 0) return Q4_ERR_INVALID_ARG;
    if (n > (int64_t(1) << 34) || k > (int64_t(1) << 34)) return Q4_ERR_INVALID_ARG;
    return Q4_OK;
}

q4_status check_matrix(const q4_matrix* m) {
    if (!m || !m->qs || !m->d) return Q4_ERR_INVALID_ARG;
    q4_status s = check_shape(m->n, m->k);
    if (s != Q4_OK) return s;
    if (!aligned(m->qs, 16) || !aligned(m->d, 16)) return Q4_ERR_MISALIGNED;
    return Q4_OK;
}

struct Shape {
    int64_t n, k;
};

// Plan one launch over `count` GEMVs of the given shapes. Fills everything in P
// except the pointers. Workspace layout of a call: [256-byte status header]
// [split-K tickets, one uint32 per row tile of every split GEMV][partial sums].
// Tickets start right after the header; partial sums start at `part_base` bytes,
// which a stack sets past the largest ticket region of all its groups so that no
// partial sum of any group overlaps any ticket. Every call zeroes its ticket
// region before its first kernel. Returns the tickets used (*tickets) and the
// end of the partial sums (*ws_end, bytes).
q4_status plan_shapes(const Shape* sh, int count, int batch, int64_t part_base, GemvParams* P,
                      int64_t* tickets, int64_t* ws_end) {
    if (count < 1 || count > Q4_MAX_GROUP || batch < 1 || batch > kMaxCudaCoreBatch)
        return Q4_ERR_INVALID_ARG;
    std::memset(P, 0, sizeof *P);
    const int maxb = q4plan::max_blocks_per_split(batch);
    int64_t base_units = 0;
    for (int i = 0; i < count; ++i) {
        q4_status s = check_shape(sh[i].n, sh[i].k);
        if (s != Q4_OK) return s;
        base_units += ceil_div(sh[i].n, q4plan::kRowsPerCta) * ceil_div(sh[i].k / Q4_QK, maxb);
    }
    const int64_t factor = base_units >= kTargetUnits ? 1 : ceil_div(kTargetUnits, base_units);
    int64_t units = 0;
    int64_t tick = 0;
    int64_t part = part_base;
    int nbs_max = 1;
    for (int i = 0; i < count; ++i) {
        GemvDesc& G = P->g[i];
        const int64_t nb = sh[i].k / Q4_QK;
        const int64_t tiles = ceil_div(sh[i].n, q4plan::kRowsPerCta);
        const int64_t smin = ceil_div(nb, maxb);
        int64_t S = smin * factor;
        S = std::min(S, std::max(smin, nb / 8));  // splits keep at least 8 blocks
        int64_t nbs = ceil_div(nb, S);
        if (nbs > 8) nbs = std::min<int64_t>(round_up(nbs, 8), maxb);
        S = ceil_div(nb, nbs);
        G.n = sh[i].n;
        G.nb = (int32_t)nb;
        G.splits = (int32_t)S;
        G.nb_split = (int32_t)nbs;
        G.row_tiles = (int32_t)tiles;
        G.unit_begin = (int32_t)units;
        if (S > 1) {
            G.ticket_off = q4plan::kHeaderBytes / 4 + tick;
            tick += tiles;
            G.part_off = part / 4;
            part += round_up((int64_t)batch * S * sh[i].n * 4, 256);
        }
        units += tiles * S;
        nbs_max = std::max<int>(nbs_max, (int)nbs);
        if (units > INT_MAX / 2) return Q4_ERR_INVALID_ARG;
    }
    if (q4plan::kHeaderBytes + 4 * tick > part_base) return Q4_ERR_INVALID_ARG;
    P->count = count;
    P->total_units = (int32_t)units;
    P->batch = batch;
    if (batch == 1)
        P->smem_x = (uint32_t)ceil_div(nbs_max, 32) * 32 * 8 * 16;
    else
        P->smem_x = (uint32_t)(batch * q4plan::x_token_slots_bs(nbs_max) * 16);
    P->smem_qs_warp = (uint32_t)(q4plan::kRowsPerWarp * nbs_max * 16);
    P->d_slot = (uint32_t)round_up(nbs_max + 14, 8);
    P->smem_d_warp = (uint32_t)(q4plan::kRowsPerWarp * P->d_slot * 2);
    P->smem_total = q4plan::kBarrierBytes + P->smem_x +
                    q4plan::kWarps * (P->smem_qs_warp + P->smem_d_warp);
    if (P->smem_total > kMaxSmem) return Q4_ERR_UNSUPPORTED;
    *tickets = tick;
    *ws_end = part;
    return Q4_OK;
}

// Tickets of one launch, found by planning with room for any ticket count.
q4_status count_tickets(const Shape* sh, int count, int batch, int64_t* tickets) {
    GemvParams P;
    int64_t end = 0;
    return plan_shapes(sh, count, batch, INT64_MAX / 4, &P, tickets, &end);
}

int64_t part_base_for(int64_t tickets) {
    return q4plan::kHeaderBytes + round_up(4 * tickets, 256);
}

// Streaming (batch 1) plan over `count` GEMVs: splits, units, grid, tickets and
// partial sums laid out as for plan_shapes.
constexpr int kNumSMs = 148;
static_assert(kNumSMs * Q4_STREAM_CTAS_PER_SM <= q4s::kMaxGrid, "CTA range table too small");

// CTA ranges of a streaming launch over the row space of P (segments already
// laid out). With at least as many CTAs as segments, each segment gets whole
// CTAs: one each, then one at a time to the segment whose CTAs carry the most
// weight bytes (rows x blocks of the split), never more CTAs than rows; a
// segment's rows are cut into equal ranges (to within one). A CTA then stages
// one piece's activations, where a range across a segment boundary would stage
// two and finish last. With more segments than CTAs the row space is cut into
// `grid` equal ranges.
void stream_cta_ranges(q4s::Params* P, int grid) {
    struct Seg {
        int64_t begin, rows, weight;
        int ctas;
    };
    std::vector<Seg> seg;
    for (int i = 0; i < P->count; ++i) {
        const q4s::Desc& G = P->g[i];
        for (int sp = 0; sp < G.splits; ++sp)
            seg.push_back({G.row_begin + sp * G.n, G.n, G.n * q4s::split_blocks(G, sp), 1});
    }
    const int nseg = (int)seg.size();
    if (nseg > grid) {
        const uint64_t R = (uint64_t)P->total_rows;  // < 2^31
        for (int c = 0; c <= grid; ++c) P->cta_lo[c] = (int32_t)(R * (uint32_t)c / (uint32_t)grid);
        return;
    }
    // grid <= total rows, so a segment with a CTA to spare is always left
    for (int left = grid - nseg; left > 0; --left) {
        int best = -1;
        for (int s = 0; s < nseg; ++s) {
            if (seg[s].ctas >= seg[s].rows) continue;
            if (best < 0 || seg[s].weight * seg[best].ctas > seg[best].weight * seg[s].ctas) best = s;
        }
        ++seg[best].ctas;
    }
    int c = 0;
    for (const Seg& s : seg)
        for (int j = 0; j < s.ctas; ++j) P->cta_lo[c++] = (int32_t)(s.begin + s.rows * j / s.ctas);
    P->cta_lo[grid] = (int32_t)P->total_rows;
}

q4_status plan_stream(const Shape* sh, int count, int64_t part_base, q4s::Params* P, int* grid,
                      int64_t* tickets, int64_t* ws_end) {
    if (count < 1 || count > Q4_MAX_GROUP) return Q4_ERR_INVALID_ARG;
    std::memset(P, 0, sizeof *P);
    int64_t base_rows = 0;
    for (int i = 0; i < count; ++i) {
        q4_status s = check_shape(sh[i].n, sh[i].k);
        if (s != Q4_OK) return s;
        base_rows += sh[i].n * ceil_div(sh[i].k / Q4_QK, q4s::kMaxSplitBlocks);
    }
    // enough rows for one row per warp of the grid, splitting K (in whole
    // sub-steps of 32 blocks) when the matrices are shorter (splitting further, to
    // a full tile per warp, measured slower on the 8B-class stack: the split-K
    // finish costs more than the idle lanes)
    const int64_t target = (int64_t)kNumSMs * Q4_STREAM_CTAS_PER_SM * q4s::kWarps;
    const int64_t factor = base_rows >= target ? 1 : ceil_div(target, base_rows);
    int64_t rows = 0, tick = 0, part = part_base;
    for (int i = 0; i < count; ++i) {
        q4s::Desc& G = P->g[i];
        const int64_t nb = sh[i].k / Q4_QK;
        const int64_t smin = ceil_div(nb, q4s::kMaxSplitBlocks);
        const int64_t smax = std::max<int64_t>(smin, nb / 32);
        const int64_t S0 = std::min(smin * factor, smax);
        int64_t nbs = ceil_div(nb, S0);
        if (S0 > 1) nbs = std::min<int64_t>(round_up(nbs, 32), q4s::kMaxSplitBlocks);
        const int64_t S = ceil_div(nb, nbs);
        G.n = sh[i].n;
        G.nb = (int32_t)nb;
        G.splits = (int32_t)S;
        G.nb_split = (int32_t)nbs;
        G.row_begin = rows;
        if (S > 1) {
            G.ticket_off = q4plan::kHeaderBytes / 4 + tick;
            tick += sh[i].n;
            G.part_off = part / 4;
            part += round_up(S * sh[i].n * 4, 256);
        }
        rows += sh[i].n * S;
        if (rows >= (int64_t(1) << 31)) return Q4_ERR_INVALID_ARG;  // 32-bit row space
    }
    if (q4plan::kHeaderBytes + 4 * tick > part_base) return Q4_ERR_INVALID_ARG;
    P->count = count;
    P->total_rows = rows;
    *grid = (int)std::min<int64_t>((int64_t)kNumSMs * Q4_STREAM_CTAS_PER_SM, rows);
    stream_cta_ranges(P, *grid);
    *tickets = tick;
    *ws_end = part;
    return Q4_OK;
}

// Tensor-core plan over `count` GEMVs for b tokens: the flat (tile, block)
// space, the grid, and per GEMV its partial-sum slots per tile, tickets (four
// per tile: one per epilogue warp) and partial sums [tiles][slots][b][128].
q4_status plan_tc(const Shape* sh, int count, int b, int64_t part_base, q4t::Params* P,
                  int64_t* tickets, int64_t* ws_end) {
    if (count < 1 || count > Q4_MAX_GROUP || b < 2 || b > Q4_MAX_BATCH) return Q4_ERR_INVALID_ARG;
    std::memset(P, 0, sizeof *P);
    int64_t F = 0;
    for (int i = 0; i < count; ++i) {
        q4_status s = check_shape(sh[i].n, sh[i].k);
        if (s != Q4_OK) return s;
        q4t::Desc& G = P->g[i];
        G.n = sh[i].n;
        G.nb = (int32_t)(sh[i].k / Q4_QK);
        G.tiles = (int32_t)ceil_div(sh[i].n, q4t::kM);
        G.d_box = G.nb % 8 == 0 ? 1 : 0;
        G.flat_begin = F;
        F += (int64_t)G.tiles * G.nb;
        if (F >= (int64_t(1) << 31) || sh[i].k / 2 >= (int64_t(1) << 31) ||
            sh[i].n >= (int64_t(1) << 31))
            return Q4_ERR_INVALID_ARG;  // 32-bit unit space and TMA coordinates
    }
    P->count = count;
    P->b = b;
    P->total = F;
    P->grid = (int32_t)std::min<int64_t>(kNumSMs, F);
    int64_t tick = 0, part = part_base;
    for (int i = 0; i < count; ++i) {
        q4t::Desc& G = P->g[i];
        int maxp = 1;
        for (int32_t t = 0; t < G.tiles; ++t) {
            int np = 0, slot = 0;
            q4t::tile_pieces(*P, G, t, 0, &np, &slot);
            maxp = std::max(maxp, np);
        }
        G.maxp = maxp;
        if (maxp > 1) {
            G.ticket_off = q4plan::kHeaderBytes / 4 + tick;
            tick += 4 * (int64_t)G.tiles;
            G.part_off = part / 4;
            part += round_up((int64_t)G.tiles * maxp * b * q4t::kM * 4, 256);
        }
    }
    if (q4plan::kHeaderBytes + 4 * tick > part_base) return Q4_ERR_INVALID_ARG;
    *tickets = tick;
    *ws_end = part;
    return Q4_OK;
}

// Token chunks: batches above the CUDA-core kernel's width run as several
// launches of at most kMaxCudaCoreBatch tokens.
int chunk_tokens(int b, int c0) { return std::min(kMaxCudaCoreBatch, b - c0); }

std::mutex g_dev_mu;
bool g_dev_ready[64];

q4_status ensure_device() {
    int dev = 0;
    if (cuda_failed(cudaGetDevice(&dev))) return Q4_ERR_CUDA;
    if (dev < 0 || dev >= 64) return Q4_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_dev_mu);
    if (g_dev_ready[dev]) return Q4_OK;
    int major = 0, minor = 0, optin = 0;
    if (cuda_failed(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) ||
        cuda_failed(cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) ||
        cuda_failed(cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)))
        return Q4_ERR_CUDA;
    if (major != 10 || minor != 0) return Q4_ERR_UNSUPPORTED;
    if (cuda_failed(q4k::setup_gemv_kernels(optin))) return Q4_ERR_CUDA;
    if (cuda_failed(q4k::setup_stream_kernel(optin))) return Q4_ERR_CUDA;
    if (cuda_failed(q4k::setup_tc_kernels(optin))) return Q4_ERR_CUDA;
    g_dev_ready[dev] = true;
    return Q4_OK;
}

struct GemvCall {
    q4_matrix m;
    const float* x;
    float* y;
};

// Tickets and partial-sum bytes (past the ticket region) of one launch group
// of the given shapes for `b` tokens, planned exactly as the launch will be.
q4_status group_need(const Shape* sh, int count, int b, int64_t* tickets, int64_t* part_bytes) {
    if (count < 1 || count > Q4_MAX_GROUP) return Q4_ERR_INVALID_ARG;
    if (b < 1 || b > Q4_MAX_BATCH) return Q4_ERR_UNSUPPORTED;
    constexpr int64_t kBase = 0x40000000LL;
    int64_t tmax = 0, pmax = 0;
    if (b == 1) {
        q4s::Params P;
        int grid = 0;
        int64_t t = 0, end = 0;
        q4_status s = plan_stream(sh, count, kBase, &P, &grid, &t, &end);
        if (s != Q4_OK) return s;
        tmax = t;
        pmax = end - kBase;
    } else if (b >= kTcMinBatch) {
        q4t::Params P;
        int64_t t = 0, end = 0;
        q4_status s = plan_tc(sh, count, b, kBase, &P, &t, &end);
        if (s != Q4_OK) return s;
        tmax = t;
        pmax = end - kBase;
    } else {
        for (int c0 = 0; c0 < b; c0 += kMaxCudaCoreBatch) {
            GemvParams P;
            int64_t t = 0, end = 0;
            q4_status s = plan_shapes(sh, count, chunk_tokens(b, c0), kBase, &P, &t, &end);
            if (s != Q4_OK) return s;
            tmax = std::max(tmax, t);
            pmax = std::max(pmax, end - kBase);
        }
    }
    *tickets = tmax;
    *part_bytes = pmax;
    return Q4_OK;
}

// Validate one group for `b` tokens; returns its ticket count and the
// partial-sum bytes it needs past the ticket region.
q4_status check_group(const GemvCall* calls, int count, int b, int64_t* tickets,
                      int64_t* part_bytes) {
    if (count < 1 || count > Q4_MAX_GROUP) return Q4_ERR_INVALID_ARG;
    if (b < 1 || b > Q4_MAX_BATCH) return Q4_ERR_UNSUPPORTED;
    Shape sh[Q4_MAX_GROUP];
    for (int i = 0; i < count; ++i) {
        q4_status s = check_matrix(&calls[i].m);
        if (s != Q4_OK) return s;
        if (!calls[i].x || !calls[i].y) return Q4_ERR_INVALID_ARG;
        if (!aligned(calls[i].x, 16) || !aligned(calls[i].y, 16)) return Q4_ERR_MISALIGNED;
        sh[i] = {calls[i].m.n, calls[i].m.k};
    }
    return group_need(sh, count, b, tickets, part_bytes);
}

q4_status check_ws(void* ws, size_t ws_bytes, size_t need) {
    if (!ws || ws_bytes < need) return Q4_ERR_WORKSPACE;
    if (!aligned(ws, 256)) return Q4_ERR_MISALIGNED;
    return Q4_OK;
}

// Enqueue one group (all token chunks) with partial sums from `part_base`. The
// first launch may use PDL only if `pdl_first` is set.
q4_status launch_group(const GemvCall* calls, int count, int b, void* ws, int64_t part_base,
                       bool pdl_first, cudaStream_t stream, uint32_t tx_extra = 0) {
    Shape sh[Q4_MAX_GROUP];
    for (int i = 0; i < count; ++i) sh[i] = {calls[i].m.n, calls[i].m.k};
    if (b == 1) {
        q4s::Params P;
        int grid = 0;
        int64_t t = 0, end = 0;
        q4_status s = plan_stream(sh, count, part_base, &P, &grid, &t, &end);
        if (s != Q4_OK) return s;
        for (int i = 0; i < count; ++i) {
            P.g[i].qs = calls[i].m.qs;
            P.g[i].d = calls[i].m.d;
            P.g[i].x = calls[i].x;
            P.g[i].y = calls[i].y;
        }
        P.ws = static_cast<uint32_t*>(ws);
        P.tx_extra = tx_extra;
        if (cuda_failed(q4k::launch_stream(P, grid, pdl_first, stream))) return Q4_ERR_CUDA;
        g_launches.fetch_add(1, std::memory_order_relaxed);
        return Q4_OK;
    }
    if (b >= kTcMinBatch) {
        q4t::Params P;
        int64_t t = 0, end = 0;
        q4_status s = plan_tc(sh, count, b, part_base, &P, &t, &end);
        if (s != Q4_OK) return s;
        for (int i = 0; i < count; ++i) {
            P.g[i].qs = calls[i].m.qs;
            P.g[i].d = calls[i].m.d;
            P.g[i].x = calls[i].x;
            P.g[i].y = calls[i].y;
            if (cuda_failed(q4k::encode_tc_maps(&P.maps[i], &P.g[i].d_box, calls[i].m.qs,
                                                calls[i].m.d, calls[i].x, calls[i].m.n,
                                                calls[i].m.k, b)))
                return Q4_ERR_CUDA;
        }
        P.ws = static_cast<uint32_t*>(ws);
        P.tx_extra = tx_extra;
        if (cuda_failed(q4k::launch_tc(P, pdl_first, stream))) return Q4_ERR_CUDA;
        g_launches.fetch_add(1, std::memory_order_relaxed);
        return Q4_OK;
    }
    bool pdl = pdl_first;
    for (int c0 = 0; c0 < b; c0 += kMaxCudaCoreBatch) {
        const int bt = chunk_tokens(b, c0);
        GemvParams P;
        int64_t t = 0, end = 0;
        q4_status s = plan_shapes(sh, count, bt, part_base, &P, &t, &end);
        if (s != Q4_OK) return s;
        for (int i = 0; i < count; ++i) {
            P.g[i].qs = calls[i].m.qs;
            P.g[i].d = calls[i].m.d;
            P.g[i].x = calls[i].x + (int64_t)c0 * calls[i].m.k;
            P.g[i].y = calls[i].y + (int64_t)c0 * calls[i].m.n;
        }
        P.ws = static_cast<uint32_t*>(ws);
        if (cuda_failed(q4k::launch_gemv(P, pdl, stream))) return Q4_ERR_CUDA;
        g_launches.fetch_add(1, std::memory_order_relaxed);
        pdl = true;
    }
    return Q4_OK;
}

// Zero the ticket region of a call before its first kernel.
q4_status clear_tickets(void* ws, int64_t tickets, cudaStream_t stream) {
    if (tickets == 0) return Q4_OK;
    if (cuda_failed(cudaMemsetAsync(static_cast<uint8_t*>(ws) + q4plan::kHeaderBytes, 0,
                                    (size_t)(4 * tickets), stream)))
        return Q4_ERR_CUDA;
    return Q4_OK;
}

// Split a stack into groups: [begin, end) index ranges.
q4_status stack_groups(const q4_stack* s, std::vector<std::pair<int, int>>* out) {
    if (!s || s->count < 1 || !s->mats || !s->x || !s->y || !s->group) return Q4_ERR_INVALID_ARG;
    out->clear();
    int begin = 0;
    for (int i = 1; i <= s->count; ++i) {
        if (i < s->count && s->group[i] < s->group[i - 1]) return Q4_ERR_INVALID_ARG;
        if (i == s->count || s->group[i] != s->group[i - 1]) {
            if (i - begin > Q4_MAX_GROUP) return Q4_ERR_INVALID_ARG;
            out->push_back({begin, i});
            begin = i;
        }
    }
    return Q4_OK;
}

// Validate a stack; returns the ticket region shared by all groups and the
// workspace bytes needed.
// Validate a stack; returns the ticket region shared by all groups and the
// workspace bytes needed.
q4_status stack_check(const q4_stack* s, int b, std::vector<std::pair<int, int>>* groups,
                      int64_t* tickets, size_t* need) {
    q4_status st = stack_groups(s, groups);
    if (st != Q4_OK) return st;
    int64_t tmax = 0, pmax = 0;
    for (auto& g : *groups) {
        GemvCall calls[Q4_MAX_GROUP];
        for (int i = g.first; i < g.second; ++i)
            calls[i - g.first] = {s->mats[i], s->x[i], s->y[i]};
        int64_t t = 0, p = 0;
        st = check_group(calls, g.second - g.first, b, &t, &p);
        if (st != Q4_OK) return st;
        tmax = std::max(tmax, t);
        pmax = std::max(pmax, p);
    }
    *tickets = tmax;
    *need = (size_t)(part_base_for(tmax) + pmax);
    return Q4_OK;
}

uint64_t stack_kernel_count(const std::vector<std::pair<int, int>>& groups, int b) {
    if (b == 1 || b >= kTcMinBatch) return (uint64_t)groups.size();
    return (uint64_t)groups.size() * (uint64_t)ceil_div(b, kMaxCudaCoreBatch);
}

}  // namespace

struct q4_graph_s {
    cudaGraph_t graph;
    cudaGraphExec_t exec;
    uint64_t kernels;
};

extern "C" {

q4_status q4_plane_bytes(int64_t n, int64_t k, size_t* qs_bytes, size_t* d_bytes) {
    if (check_shape(n, k) != Q4_OK || !qs_bytes || !d_bytes) return Q4_ERR_INVALID_ARG;
    *qs_bytes = (size_t)(n * (k / 2));
    *d_bytes = (size_t)round_up(n * (k / Q4_QK) * 2, 16);
    return Q4_OK;
}

q4_status q4_pack(const float* w, const q4_matrix* out, void* stream) {
    q4_status s = check_matrix(out);
    if (s != Q4_OK) return s;
    if (!w) return Q4_ERR_INVALID_ARG;
    if (!aligned(w, 16)) return Q4_ERR_MISALIGNED;
    if ((s = ensure_device()) != Q4_OK) return s;
    const int64_t nblocks = out->n * (out->k / Q4_QK);
    if (q4k::launch_pack(w, out->qs, out->d, nblocks, static_cast<cudaStream_t>(stream)) !=
        cudaSuccess)
        return Q4_ERR_CUDA;
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return Q4_OK;
}

q4_status q4_dequant(const q4_matrix* m, float* w_out, void* stream) {
    q4_status s = check_matrix(m);
    if (s != Q4_OK) return s;
    if (!w_out) return Q4_ERR_INVALID_ARG;
    if (!aligned(w_out, 16)) return Q4_ERR_MISALIGNED;
    if ((s = ensure_device()) != Q4_OK) return s;
    const int64_t nblocks = m->n * (m->k / Q4_QK);
    if (q4k::launch_dequant(m->qs, m->d, w_out, nblocks, static_cast<cudaStream_t>(stream)) !=
        cudaSuccess)
        return Q4_ERR_CUDA;
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return Q4_OK;
}

size_t q4_workspace_bytes(int64_t n, int64_t k, int b) {
    if (check_shape(n, k) != Q4_OK || b < 1 || b > Q4_MAX_BATCH) return 0;
    const Shape sh = {n, k};
    int64_t t = 0, p = 0;
    if (group_need(&sh, 1, b, &t, &p) != Q4_OK) return 0;
    return (size_t)(part_base_for(t) + p);
}

q4_status q4_workspace_init(void* ws, size_t ws_bytes, void* stream) {
    if (!ws || ws_bytes < (size_t)q4plan::kHeaderBytes) return Q4_ERR_WORKSPACE;
    if (!aligned(ws, 256)) return Q4_ERR_MISALIGNED;
    if (cuda_failed(cudaMemsetAsync(ws, 0, ws_bytes, static_cast<cudaStream_t>(stream))))
        return Q4_ERR_CUDA;
    return Q4_OK;
}

q4_status q4_workspace_status(const void* ws, void* stream) {
    if (!ws) return Q4_ERR_WORKSPACE;
    uint32_t flag = 0;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cuda_failed(cudaMemcpyAsync(&flag, ws, sizeof flag, cudaMemcpyDeviceToHost, st)))
        return Q4_ERR_CUDA;
    if (cuda_failed(cudaStreamSynchronize(st))) return Q4_ERR_CUDA;
    return flag ? Q4_ERR_TIMEOUT : Q4_OK;
}

q4_status q4_gemv_batched(const q4_matrix* m, const float* X, int b, float* Y, void* ws,
                          size_t ws_bytes, void* stream) {
    if (!m) return Q4_ERR_INVALID_ARG;
    GemvCall call = {*m, X, Y};
    int64_t tickets = 0, part = 0;
    q4_status s = check_group(&call, 1, b, &tickets, &part);
    if (s != Q4_OK) return s;
    const int64_t base = part_base_for(tickets);
    if ((s = check_ws(ws, ws_bytes, (size_t)(base + part))) != Q4_OK) return s;
    if ((s = ensure_device()) != Q4_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if ((s = clear_tickets(ws, tickets, st)) != Q4_OK) return s;
    return launch_group(&call, 1, b, ws, base, false, st);
}

q4_status q4_gemv(const q4_matrix* m, const float* x, float* y, void* ws, size_t ws_bytes,
                  void* stream) {
    return q4_gemv_batched(m, x, 1, y, ws, ws_bytes, stream);
}

size_t q4_stack_workspace_bytes(const q4_stack* s, int b) {
    std::vector<std::pair<int, int>> groups;
    int64_t tickets = 0;
    size_t need = 0;
    if (stack_check(s, b, &groups, &tickets, &need) != Q4_OK) return 0;
    return need;
}

q4_status q4_layer_stack(const q4_stack* s, int b, void* ws, size_t ws_bytes, void* stream) {
    std::vector<std::pair<int, int>> groups;
    int64_t tickets = 0;
    size_t need = 0;
    q4_status st = stack_check(s, b, &groups, &tickets, &need);
    if (st != Q4_OK) return st;
    if ((st = check_ws(ws, ws_bytes, need)) != Q4_OK) return st;
    if ((st = ensure_device()) != Q4_OK) return st;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    if ((st = clear_tickets(ws, tickets, cs)) != Q4_OK) return st;
    const int64_t base = part_base_for(tickets);
    bool first = true;
    for (auto& g : groups) {
        GemvCall calls[Q4_MAX_GROUP];
        for (int i = g.first; i < g.second; ++i)
            calls[i - g.first] = {s->mats[i], s->x[i], s->y[i]};
        st = launch_group(calls, g.second - g.first, b, ws, base, !first, cs);
        if (st != Q4_OK) return st;
        first = false;
    }
    return Q4_OK;
}

q4_status q4_stack_graph_create(const q4_stack* s, int b, void* ws, size_t ws_bytes, void* stream,
                                q4_graph* out) {
    if (!out || !stream) return Q4_ERR_INVALID_ARG;
    *out = nullptr;
    std::vector<std::pair<int, int>> groups;
    int64_t tickets = 0;
    size_t need = 0;
    q4_status st = stack_check(s, b, &groups, &tickets, &need);
    if (st != Q4_OK) return st;
    if ((st = check_ws(ws, ws_bytes, need)) != Q4_OK) return st;
    if ((st = ensure_device()) != Q4_OK) return st;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cuda_failed(cudaStreamIsCapturing(cs, &cap))) return Q4_ERR_CUDA;
    if (cap != cudaStreamCaptureStatusNone) return Q4_ERR_INVALID_ARG;
    if (cuda_failed(cudaStreamBeginCapture(cs, cudaStreamCaptureModeThreadLocal)))
        return Q4_ERR_CUDA;
    const uint64_t before = g_launches.load();
    q4_status run = q4_layer_stack(s, b, ws, ws_bytes, stream);
    g_launches.store(before);  // captured launches do not run now
    cudaGraph_t graph = nullptr;
    cudaError_t e = cudaStreamEndCapture(cs, &graph);
    cuda_failed(e);
    if (run != Q4_OK || e != cudaSuccess) {
        if (graph) cudaGraphDestroy(graph);
        return run != Q4_OK ? run : Q4_ERR_CUDA;
    }
    cudaGraphExec_t exec = nullptr;
    if (cuda_failed(cudaGraphInstantiate(&exec, graph, 0))) {
        cudaGraphDestroy(graph);
        return Q4_ERR_CUDA;
    }
    q4_graph g = new (std::nothrow) q4_graph_s;
    if (!g) {
        cudaGraphExecDestroy(exec);
        cudaGraphDestroy(graph);
        return Q4_ERR_INVALID_ARG;
    }
    g->graph = graph;
    g->exec = exec;
    g->kernels = stack_kernel_count(groups, b);
    *out = g;
    return Q4_OK;
}

q4_status q4_graph_launch(q4_graph g, void* stream) {
    if (!g) return Q4_ERR_INVALID_ARG;
    if (cuda_failed(cudaGraphLaunch(g->exec, static_cast<cudaStream_t>(stream))))
        return Q4_ERR_CUDA;
    g_launches.fetch_add(g->kernels, std::memory_order_relaxed);
    return Q4_OK;
}

q4_status q4_graph_destroy(q4_graph g) {
    if (!g) return Q4_ERR_INVALID_ARG;
    cudaError_t e1 = cudaGraphExecDestroy(g->exec);
    cudaError_t e2 = cudaGraphDestroy(g->graph);
    delete g;
    return (e1 == cudaSuccess && e2 == cudaSuccess) ? Q4_OK : Q4_ERR_CUDA;
}

q4_status q4_blocks_to_planes(const uint8_t* blocks, int64_t n, int64_t k, uint8_t* qs,
                              uint16_t* d) {
    if (!blocks || !qs || !d || check_shape(n, k) != Q4_OK) return Q4_ERR_INVALID_ARG;
    const int64_t nblocks = n * (k / Q4_QK);
    for (int64_t i = 0; i < nblocks; ++i) {
        const uint8_t* b = blocks + i * Q4_BLOCK_BYTES;
        d[i] = (uint16_t)(b[0] | (b[1] << 8));
        std::memcpy(qs + i * 16, b + 2, 16);
    }
    return Q4_OK;
}

q4_status q4_planes_to_blocks(const uint8_t* qs, const uint16_t* d, int64_t n, int64_t k,
                              uint8_t* blocks) {
    if (!blocks || !qs || !d || check_shape(n, k) != Q4_OK) return Q4_ERR_INVALID_ARG;
    const int64_t nblocks = n * (k / Q4_QK);
    for (int64_t i = 0; i < nblocks; ++i) {
        uint8_t* b = blocks + i * Q4_BLOCK_BYTES;
        b[0] = (uint8_t)(d[i] & 0xFF);
        b[1] = (uint8_t)(d[i] >> 8);
        std::memcpy(b + 2, qs + i * 16, 16);
    }
    return Q4_OK;
}

// ---------------------------------------------------------------------------
// q4_gemv_noalloc: the batch-1 GEMV with its split-K scratch in a fixed device
// array instead of a caller workspace.
//
// Some callers cannot hand the library a workspace: a plugin inside a host
// application that owns every device allocation, a runtime with a fixed memory
// budget that forbids allocating after start-up, or a latency-critical path that
// must not call cudaMalloc because it can synchronise the whole device. For
// them the scratch lives in the array below, which every GPU that loads this
// library holds until the process exits.
// ---------------------------------------------------------------------------

constexpr size_t kNoAllocScratchBytes = size_t(1) << 20;  // 1 MiB per GPU

// Header, split-K tickets and partial sums of q4_gemv_noalloc. In host code this
// name is only a stand-in for the symbol, never a device address: the address
// comes from cudaGetSymbolAddress, looked up once per device.
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[64];

// Device address of the scratch array on the current device (looked up on the
// first call made while that device is current).
q4_status noalloc_scratch(void** out) {
    int dev = 0;
    if (cuda_failed(cudaGetDevice(&dev))) return Q4_ERR_CUDA;
    if (dev < 0 || dev >= 64) return Q4_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void* p = nullptr;
        if (cuda_failed(cudaGetSymbolAddress(&p, g_noalloc_scratch))) return Q4_ERR_CUDA;
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return Q4_OK;
}
}  // namespace

q4_status q4_gemv_noalloc(const q4_matrix* m, const float* x, float* y, void* stream) {
    if (!m) return Q4_ERR_INVALID_ARG;
    GemvCall call = {*m, x, y};
    int64_t tickets = 0, part = 0;
    q4_status s = check_group(&call, 1, 1, &tickets, &part);
    if (s != Q4_OK) return s;
    const int64_t base = part_base_for(tickets);
    if ((size_t)(base + part) > kNoAllocScratchBytes) return Q4_ERR_WORKSPACE;
    if ((s = ensure_device()) != Q4_OK) return s;
    void* scratch = nullptr;
    if ((s = noalloc_scratch(&scratch)) != Q4_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if ((s = clear_tickets(scratch, tickets, st)) != Q4_OK) return s;
    return launch_group(&call, 1, 1, scratch, base, false, st);
}

const char* q4_status_string(q4_status s) {
    switch (s) {
        case Q4_OK: return "ok";
        case Q4_ERR_INVALID_ARG: return "invalid argument";
        case Q4_ERR_MISALIGNED: return "misaligned pointer";
        case Q4_ERR_WORKSPACE: return "workspace missing or too small";
        case Q4_ERR_UNSUPPORTED: return "unsupported (batch or device)";
        case Q4_ERR_CUDA: return "CUDA error";
        case Q4_ERR_TIMEOUT: return "device wait timed out";
    }
    return "unknown status";
}

uint64_t q4_launch_count(void) { return g_launches.load(); }

const char* q4_last_cuda_error(void) { return cudaGetErrorString(g_last_cuda_error); }

// ---------------------------------------------------------------------------
// host-side diagnostics
// ---------------------------------------------------------------------------

q4_status q4_debug_plan_info(const int64_t* n, const int64_t* k, int count, int b, int64_t* out) {
    if (!n || !k || !out || count < 1 || count > Q4_MAX_GROUP || b < 1 || b > kMaxCudaCoreBatch)
        return Q4_ERR_INVALID_ARG;
    Shape sh[Q4_MAX_GROUP];
    for (int i = 0; i < count; ++i) sh[i] = {n[i], k[i]};
    int64_t tickets = 0, end = 0;
    q4_status s = count_tickets(sh, count, b, &tickets);
    if (s != Q4_OK) return s;
    GemvParams P;
    s = plan_shapes(sh, count, b, part_base_for(tickets), &P, &tickets, &end);
    if (s != Q4_OK) return s;
    out[0] = P.total_units;
    out[1] = P.smem_total;
    out[2] = end;
    for (int i = 0; i < count; ++i) out[3 + i] = P.g[i].splits;
    return Q4_OK;
}

int q4_debug_check_plan(const int64_t* n, const int64_t* k, int count, int b) {
    using namespace q4plan;
    if (!n || !k || count < 1 || count > Q4_MAX_GROUP || b < 1 || b > kMaxCudaCoreBatch) return 1;
    Shape sh[Q4_MAX_GROUP];
    for (int i = 0; i < count; ++i) sh[i] = {n[i], k[i]};
    GemvParams P;
    int64_t tickets = 0, end = 0;
    if (count_tickets(sh, count, b, &tickets) != Q4_OK) return 2;
    const int64_t base = part_base_for(tickets);
    if (plan_shapes(sh, count, b, base, &P, &tickets, &end) != Q4_OK) return 2;
    const size_t ws_bytes = (size_t)end;
    if (P.smem_total > kMaxSmem) return 3;
    if (P.smem_x % 16 || P.smem_qs_warp % 16 || P.smem_d_warp % 16) return 4;
    if ((int64_t)kBarrierBytes < (int64_t)kWarps * 8) return 5;
    std::vector<std::vector<uint8_t>> cover(count);
    for (int i = 0; i < count; ++i) cover[i].assign((size_t)(sh[i].n * (sh[i].k / Q4_QK)), 0);
    int64_t units_seen = 0;
    for (int unit = 0; unit < P.total_units; ++unit) {
        const Unit u = unit_of(P, unit);
        if (u.g < 0 || u.g >= count) return 10;
        const GemvDesc& G = P.g[u.g];
        if (u.tile < 0 || u.tile >= G.row_tiles || u.split < 0 || u.split >= G.splits) return 11;
        const int kbs = split_blocks(G, u.split);
        if (kbs < 1 || kbs > G.nb_split) return 12;
        const int64_t qs_plane = sh[u.g].n * (sh[u.g].k / 2);
        const int64_t d_plane = round_up(sh[u.g].n * G.nb * 2, 16);
        // activations of the split
        const int64_t x0 = (int64_t)u.split * G.nb_split * 32;
        if (x0 + (int64_t)kbs * 32 > sh[u.g].k) return 13;
        if (b == 1) {
            for (int j = 0; j < kbs; ++j)
                for (int c = 0; c < 8; ++c)
                    if ((int64_t)(x_slot_b1(j, c) + 1) * 16 > P.smem_x) return 14;
        } else {
            const int slots = x_token_slots_bs(G.nb_split);
            for (int j = 0; j < kbs; ++j)
                for (int c = 0; c < 8; ++c)
                    if (x_slot_bs(j, c) >= slots || (int64_t)(b * slots) * 16 > P.smem_x) return 15;
        }
        for (int warp = 0; warp < kWarps; ++warp) {
            const int rows = warp_rows(G, u.tile, warp);
            const int64_t row0 = (int64_t)u.tile * kRowsPerCta + (int64_t)warp * kRowsPerWarp;
            const int64_t wbase = smem_warp_offset(P, warp);
            if (wbase % 16) return 16;
            if (wbase + P.smem_qs_warp + P.smem_d_warp > P.smem_total) return 17;
            int64_t tx = 0;
            for (int r = 0; r < rows; ++r) {
                const int64_t row = row0 + r;
                if (row >= sh[u.g].n) return 18;
                const int64_t qsrc = qs_src_offset(G, row, u.split);
                if (qsrc < 0 || qsrc % 16 || qsrc + (int64_t)kbs * 16 > qs_plane) return 19;
                const int64_t qdst = (int64_t)r * G.nb_split * 16;
                if (qdst + (int64_t)kbs * 16 > P.smem_qs_warp) return 20;
                const DRange dr = d_range(G, row, u.split, kbs);
                if (dr.src < 0 || dr.src % 16 || dr.bytes % 16 || dr.bytes == 0) return 21;
                if (dr.src + dr.bytes > d_plane) return 22;
                if ((int64_t)r * P.d_slot * 2 + dr.bytes > P.smem_d_warp) return 23;
                if (dr.shift + (uint32_t)kbs > P.d_slot) return 24;
                if ((int64_t)dr.shift * 2 + (int64_t)kbs * 2 > dr.bytes) return 25;
                tx += (int64_t)kbs * 16 + dr.bytes;
                for (int j = 0; j < kbs; ++j) {
                    uint8_t& c = cover[u.g][(size_t)(row * G.nb + (int64_t)u.split * G.nb_split + j)];
                    if (c) return 26;
                    c = 1;
                }
            }
            if (tx >= (int64_t(1) << 20)) return 27;
        }
        if (G.splits > 1) {
            if ((G.ticket_off + G.row_tiles) * 4 > (int64_t)ws_bytes) return 28;
            if ((G.part_off + (int64_t)b * G.splits * G.n) * 4 > (int64_t)ws_bytes) return 29;
            if (G.ticket_off * 4 < kHeaderBytes || G.part_off * 4 < base) return 30;
            if ((G.ticket_off + G.row_tiles) * 4 > base) return 34;  // tickets before partials
        }
        ++units_seen;
    }
    for (int i = 0; i < count; ++i)
        for (uint8_t c : cover[i])
            if (!c) return 31;
    // ticket ranges of different GEMVs are disjoint, and so are partial-sum ranges
    for (int i = 0; i < count; ++i)
        for (int j = i + 1; j < count; ++j) {
            const GemvDesc &A = P.g[i], &B = P.g[j];
            if (A.splits < 2 || B.splits < 2) continue;
            if (A.ticket_off < B.ticket_off + B.row_tiles && B.ticket_off < A.ticket_off + A.row_tiles)
                return 32;
            const int64_t a1 = A.part_off + (int64_t)b * A.splits * A.n;
            const int64_t b1 = B.part_off + (int64_t)b * B.splits * B.n;
            if (A.part_off < b1 && B.part_off < a1) return 35;
        }
    return units_seen == P.total_units ? 0 : 33;
}

int q4_debug_check_stream(const int64_t* n, const int64_t* k, int count) {
    using namespace q4s;
    if (!n || !k || count < 1 || count > Q4_MAX_GROUP) return 1;
    Shape sh[Q4_MAX_GROUP];
    for (int i = 0; i < count; ++i) sh[i] = {n[i], k[i]};
    Params P;
    int grid = 0;
    int64_t tickets = 0, end = 0;
    if (plan_stream(sh, count, INT64_MAX / 4, &P, &grid, &tickets, &end) != Q4_OK) return 2;
    const int64_t base = part_base_for(tickets);
    if (plan_stream(sh, count, base, &P, &grid, &tickets, &end) != Q4_OK) return 2;
    if (kSmemBytes > (int)kMaxSmem) return 3;
    if (grid < 1 || grid > kNumSMs * Q4_STREAM_CTAS_PER_SM) return 4;
    for (int i = 0; i < count; ++i) {
        const Desc& G = P.g[i];
        for (int sp = 0; sp < G.splits; ++sp)
            if (split_blocks(G, sp) < 1 || split_blocks(G, sp) > kMaxSplitBlocks) return 5;
    }
    struct Tile {
        int g, split;
        int64_t row0;
        int rows;
    };
    std::vector<std::vector<uint8_t>> cover(count);
    for (int i = 0; i < count; ++i) cover[i].assign((size_t)(sh[i].n * (sh[i].k / Q4_QK)), 0);
    int64_t nseg = 0;
    for (int i = 0; i < count; ++i) nseg += P.g[i].splits;
    int64_t prev_hi = 0;
    for (int cta = 0; cta < grid; ++cta) {
        int64_t lo, hi;
        cta_range(P, cta, &lo, &hi);
        if (lo != prev_hi || hi <= lo) return 6;
        prev_hi = hi;
        // with a CTA per segment at least, no range crosses a segment boundary
        if (nseg <= grid && locate(P, hi - 1).seg_end < hi) return 24;
        for (int warp = 0; warp < kWarps; ++warp) {
            // the math loop's order: pieces, this warp's rows, tiles
            std::vector<Tile> consumer;
            for (int64_t pos = lo; pos < hi;) {
                const Where w = locate(P, pos);
                const int64_t p1 = w.seg_end < hi ? w.seg_end : hi;
                if (p1 <= pos || w.row < 0 || w.row >= P.g[w.g].n) return 7;
                const int64_t seg_row0 = pos - w.row;
                int64_t ra, rb;
                warp_rows(pos, p1, warp, &ra, &rb);
                for (int64_t row0 = ra - seg_row0; row0 < rb - seg_row0; row0 += kRows) {
                    const int64_t left = rb - seg_row0 - row0;
                    consumer.push_back({w.g, w.split, row0, left < kRows ? (int)left : kRows});
                }
                pos = p1;
            }
            // the copy issuer's walk visits the same tiles in the same order
            Walk wk;
            wk.begin(lo, hi, warp);
            size_t idx = 0;
            for (bool has = wk.next_piece(P); has; has = wk.next_piece(P))
                for (int64_t row0 = wk.wr; row0 < wk.wend; row0 += kRows, ++idx) {
                    const int64_t left = wk.wend - row0;
                    const int rows = left < kRows ? (int)left : kRows;
                    if (idx >= consumer.size()) return 8;
                    const Tile& t = consumer[idx];
                    if (t.g != wk.g || t.split != wk.split || t.row0 != row0 || t.rows != rows) return 8;
                }
            if (idx != consumer.size()) return 9;
            for (const Tile& t : consumer) {
                const Desc& G = P.g[t.g];
                const int kbs = split_blocks(G, t.split);
                if (t.rows < 1 || t.rows > kRows || kbs < 1 || kbs > kMaxSplitBlocks) return 10;
                const int64_t qs_plane = sh[t.g].n * (sh[t.g].k / 2);
                const int64_t d_plane = round_up(sh[t.g].n * G.nb * 2, 16);
                int64_t tx = 0;
                // copied[b] marks the stage bytes a copy wrote, src[b] their source
                std::vector<int64_t> src_of(kStageBytes, -1);
                for (int lane = 0; lane < 32; ++lane) {
                    const LaneCopy lc = lane_copy(G, t.split, t.row0, t.rows, lane);
                    if (!lc.active) continue;
                    const int64_t plane = lc.scales ? d_plane : qs_plane;
                    if (lc.src_off < 0 || lc.src_off % 16 || lc.bytes % 16 || lc.bytes == 0 ||
                        lc.src_off + lc.bytes > plane)
                        return 11;
                    if (lc.dst % 16 || lc.dst + lc.bytes > (uint32_t)kStageBytes) return 12;
                    if (!lc.scales && lc.dst + lc.bytes > (uint32_t)kStageQs) return 12;
                    if (lc.scales && lc.dst < (uint32_t)kStageQs) return 13;
                    for (uint32_t b = 0; b < lc.bytes; ++b) {
                        if (src_of[lc.dst + b] != -1) return 13;  // two copies overlap
                        src_of[lc.dst + b] = (lc.scales ? (int64_t(1) << 60) : 0) + lc.src_off + b;
                    }
                    tx += lc.bytes;
                }
                if (tx >= (int64_t(1) << 20)) return 14;
                // every byte the math reads was copied from the right place
                for (int r = 0; r < kRows; ++r) {
                    uint32_t qoff, doff;
                    row_read_offsets(G, t.split, t.row0, t.rows, r, &qoff, &doff);
                    const int rr = r < t.rows ? r : t.rows - 1;
                    const int64_t e = (t.row0 + rr) * G.nb + (int64_t)t.split * G.nb_split;
                    for (int j = 0; j < kbs; ++j) {
                        for (int b = 0; b < 16; ++b)
                            if (qoff + 16 * j + b >= (uint32_t)kStageBytes ||
                                src_of[qoff + 16 * j + b] != (e + j) * 16 + b)
                                return 15;
                        for (int b = 0; b < 2; ++b)
                            if (doff + 2 * j + b >= (uint32_t)kStageBytes ||
                                src_of[doff + 2 * j + b] != (int64_t(1) << 60) + (e + j) * 2 + b)
                                return 15;
                    }
                }
                for (int r = 0; r < t.rows; ++r)
                    for (int j = 0; j < kbs; ++j) {
                        uint8_t& cv = cover[t.g][(size_t)((t.row0 + r) * G.nb +
                                                          (int64_t)t.split * G.nb_split + j)];
                        if (cv) return 16;
                        cv = 1;
                    }
            }
        }
        for (int w = 0; w < kWarps; ++w)
            for (int s = 0; s < kStages; ++s)
                if (stage_offset(w, s) % 16 || stage_offset(w, s) + kStageBytes > (uint32_t)kSmemBytes)
                    return 17;
    }
    if (prev_hi != P.total_rows) return 18;
    for (int i = 0; i < count; ++i)
        for (uint8_t cv : cover[i])
            if (!cv) return 19;
    for (int i = 0; i < count; ++i) {
        const Desc& G = P.g[i];
        if (G.splits < 2) continue;
        if (G.ticket_off * 4 < q4plan::kHeaderBytes || (G.ticket_off + G.n) * 4 > base) return 20;
        if (G.part_off * 4 < base || (G.part_off + (int64_t)G.splits * G.n) * 4 > end) return 21;
        for (int j = i + 1; j < count; ++j) {
            const Desc& H = P.g[j];
            if (H.splits < 2) continue;
            if (G.ticket_off < H.ticket_off + H.n && H.ticket_off < G.ticket_off + G.n) return 22;
            if (G.part_off < H.part_off + (int64_t)H.splits * H.n &&
                H.part_off < G.part_off + (int64_t)G.splits * G.n)
                return 23;
        }
    }
    return 0;
}

q4_status q4_debug_gemv_stall(const q4_matrix* m, const float* X, int b, float* Y, void* ws,
                              size_t ws_bytes, void* stream) {
    if (!m) return Q4_ERR_INVALID_ARG;
    GemvCall call = {*m, X, Y};
    int64_t tickets = 0, part = 0;
    q4_status s = check_group(&call, 1, b, &tickets, &part);
    if (s != Q4_OK) return s;
    if (b > 1 && b < kTcMinBatch) return Q4_ERR_UNSUPPORTED;  // CUDA-core batched kernel
    const int64_t base = part_base_for(tickets);
    if ((s = check_ws(ws, ws_bytes, (size_t)(base + part))) != Q4_OK) return s;
    if ((s = ensure_device()) != Q4_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if ((s = clear_tickets(ws, tickets, st)) != Q4_OK) return s;
    return launch_group(&call, 1, b, ws, base, false, st, 16u);
}

int q4_debug_check_tc(const int64_t* n, const int64_t* k, int count, int b) {
    using namespace q4t;
    if (!n || !k || count < 1 || count > Q4_MAX_GROUP || b < 2 || b > Q4_MAX_BATCH) return 1;
    Shape sh[Q4_MAX_GROUP];
    for (int i = 0; i < count; ++i) sh[i] = {n[i], k[i]};
    Params P;
    int64_t tickets = 0, end = 0;
    if (plan_tc(sh, count, b, INT64_MAX / 4, &P, &tickets, &end) != Q4_OK) return 2;
    const int64_t base = part_base_for(tickets);
    if (plan_tc(sh, count, b, base, &P, &tickets, &end) != Q4_OK) return 2;
    if (kSmemBytes > (int)kMaxSmem || 2 * kSmemBytes <= 228 * 1024) return 3;  // one CTA per SM
    if (P.grid < 1 || P.grid > kNumSMs || P.grid > P.total) return 4;
    const int bt = q4k::tc_tokens(b);
    const int nn = mma_n(bt);
    // operand layout: every (block, chunk, K half, MMA row) has its own 16-byte
    // row inside the stage's activation region, the MMA descriptor of each
    // operand addresses exactly those rows, and every token's hi and lo rows
    // are the operand's rows t and N / 2 + t
    {
        std::vector<int> used(kXOpBytes / 16, 0);
        for (int i = 0; i < kS; ++i)
            for (int c2 = 0; c2 < 2; ++c2) {
                const uint32_t op = x_operand_off(nn, i, c2);
                for (int rho = 0; rho < nn; ++rho)
                    for (int hh = 0; hh < 2; ++hh) {
                        const uint32_t a = op + hh * lbo(nn) + (rho >> 3) * kSBO + (rho & 7) * 16;
                        if (a % 16 || a + 16 > (uint32_t)kXOpBytes) return 30;
                        if (used[a / 16]++) return 31;
                    }
                for (int t = 0; t < bt; ++t)
                    for (int hh = 0; hh < 2; ++hh)
                        for (int hl = 0; hl < 2; ++hl) {
                            const int rho = hl ? nn / 2 + t : t;
                            const uint32_t want =
                                op + hh * lbo(nn) + (rho >> 3) * kSBO + (rho & 7) * 16;
                            if (x_row_off(nn, i, c2, hh, t, hl) != want) return 32;
                        }
            }
        if (bt > nn / 2) return 32;
        const uint64_t dsc = smem_desc(0x1230u, nn);
        if ((dsc & 0x3FFF) != (0x1230u >> 4) || ((dsc >> 16) & 0x3FFF) != lbo(nn) / 16 ||
            ((dsc >> 32) & 0x3FFF) != kSBO / 16 || ((dsc >> 46) & 3) != 1 || (dsc >> 61) != 0)
            return 33;
        // descriptors advance by adding (offset >> 4) to the 14-bit start address
        if ((kSmemBytes >> 4) >= (1 << 14)) return 33;
        for (int i = 0; i < kS; ++i)
            for (int c2 = 0; c2 < 2; ++c2)
                if (smem_desc(0x400u, nn) + (uint64_t)((2 * i + c2) * nn * 32 >> 4) !=
                    smem_desc(0x400u + x_operand_off(nn, i, c2), nn))
                    return 33;
        const uint32_t id = instr_desc(nn);
        if (((id >> 17) & 63) != (uint32_t)nn / 8 || ((id >> 24) & 31) != 8 || ((id >> 4) & 3) != 1 ||
            ((id >> 7) & 7) != 1 || ((id >> 10) & 7) != 1)
            return 33;
        for (int st = 0; st < kStages; ++st)
            if (stage_base(st) % 1024 || stage_d(st) + kDBytes > (uint32_t)kSmemBytes ||
                stage_codes(st) + kCodesBytes != stage_xraw(st) ||
                stage_xraw(st) + kXRawBytes != stage_xop(st) || stage_xop(st) + kXOpBytes != stage_d(st))
                return 34;
        // tensor memory: the A ring and the D ring are disjoint and inside 512 columns
        std::vector<int> cols(kTmemCols, 0);
        for (int sa = 0; sa < kRingA; ++sa)
            for (int i = 0; i < kQ; ++i)
                for (int c = 0; c < kACols; ++c) {
                    const uint32_t col = a_col(sa, i) + c;
                    if (col >= (uint32_t)kTmemCols || cols[col]++) return 35;
                }
        if (ring_d(bt) > kMaxRingD || ring_d(bt) < 2) return 35;
        for (int sd = 0; sd < ring_d(bt); ++sd)
            for (int i = 0; i < kQ; ++i)
                for (int c = 0; c < nn; ++c) {
                    const uint32_t col = d_col(bt, sd, i) + c;
                    if (col >= (uint32_t)kTmemCols || cols[col]++) return 35;
                }
        for (int r = 0; r < kM; ++r)
            for (int c = 0; c < kS; ++c)
                if (code_off(r, c) % 16 || code_off(r, c) + 16 > (uint32_t)kCodesBytes) return 36;
    }
    std::vector<std::vector<uint8_t>> cover(count);
    for (int i = 0; i < count; ++i)
        cover[i].assign((size_t)P.g[i].tiles * P.g[i].nb, 0);
    // slots seen per (GEMV, tile)
    std::vector<std::vector<std::vector<int>>> slots(count);
    for (int i = 0; i < count; ++i) slots[i].resize(P.g[i].tiles);
    int64_t prev_hi = 0;
    for (int cta = 0; cta < P.grid; ++cta) {
        int64_t lo, hi;
        cta_range(P.total, cta, P.grid, &lo, &hi);
        if (lo != prev_hi || hi <= lo) return 6;
        prev_hi = hi;
        Walk wk;
        wk.begin(lo, hi);
        Stage s;
        int64_t pos = lo;
        bool expect_first = true;
        int cur_g = -1;
        int32_t cur_tile = -1, next_kb = -1;
        while (wk.next(P, &s)) {
            const Desc& G = P.g[s.g];
            if (s.nblk < 1 || s.nblk > kS || s.kb0 < 0 || s.kb0 + s.nblk > G.nb) return 7;
            if (s.tile < 0 || s.tile >= G.tiles) return 7;
            if (G.flat_begin + (int64_t)s.tile * G.nb + s.kb0 != pos) return 8;  // contiguous
            if (s.first != expect_first) return 9;
            if (!s.first && (s.g != cur_g || s.tile != cur_tile || s.kb0 != next_kb)) return 9;
            cur_g = s.g;
            cur_tile = s.tile;
            next_kb = s.kb0 + s.nblk;
            pos += s.nblk;
            const int32_t w0 = window_of(s.kb0);
            const int c0 = s.kb0 - w0;
            if (w0 % kS || c0 + s.nblk > kS) return 7;  // inside one window
            // TMA boxes: 16-byte aligned x, inside the row; first row inside
            if ((16 * (int64_t)w0) % 16 || 16 * (int64_t)w0 >= sh[s.g].k / 2 ||
                (int64_t)s.tile * kM >= sh[s.g].n)
                return 11;
            if (32 * (int64_t)w0 >= sh[s.g].k || (32 * (int64_t)w0 * 4) % 16) return 12;
            if (G.d_box != (G.nb % 8 == 0 ? 1 : 0)) return 24;
            if (G.d_box && ((2 * (int64_t)w0) % 16 || w0 >= G.nb || (G.nb * 2) % 16)) return 25;
            if (!G.d_box) {
                const int64_t dplane = round_up(sh[s.g].n * G.nb * 2, 16);
                for (int r = 0; r < kM; ++r) {
                    if ((int64_t)s.tile * kM + r >= sh[s.g].n) break;
                    const DCopy dc = d_copy(G, s.tile, s.kb0, s.nblk, r);
                    if (dc.src_off % 16 || dc.src_off < 0 || (dc.bytes != 16 && dc.bytes != 32) ||
                        dc.src_off + dc.bytes > dplane || dc.lead + 2 * s.nblk > dc.bytes ||
                        dc.bytes > (uint32_t)kDSlot)
                        return 26;
                }
            }
            for (int i = 0; i < s.nblk; ++i) {
                uint8_t& cv = cover[s.g][(size_t)s.tile * G.nb + s.kb0 + i];
                if (cv) return 10;
                cv = 1;
                // activation rows read by the x warps stay inside the raw box
                if ((c0 + i) * 128 + 64 + 32 + 32 > kS * 128) return 12;
            }
            if (s.last) {
                if (pos != hi && G.flat_begin + (int64_t)(s.tile + 1) * G.nb != pos) return 13;
                int np = 0, slot = 0;
                tile_pieces(P, G, s.tile, cta, &np, &slot);
                if (np < 1 || np > G.maxp || slot < 0 || slot >= np) return 14;
                if (np > 1) {
                    const int64_t p0 = G.part_off + ((int64_t)s.tile * G.maxp + slot) * b * kM;
                    if (p0 * 4 < base || (p0 + (int64_t)b * kM) * 4 > end) return 15;
                    const int64_t t0 = G.ticket_off + (int64_t)s.tile * 4;
                    if (t0 * 4 < q4plan::kHeaderBytes || (t0 + 4) * 4 > base) return 16;
                }
                slots[s.g][s.tile].push_back(slot);
                expect_first = true;
            } else {
                expect_first = false;
            }
        }
        if (pos != hi || !expect_first) return 17;
    }
    if (prev_hi != P.total) return 18;
    for (int i = 0; i < count; ++i) {
        for (uint8_t cv : cover[i])
            if (!cv) return 19;
        for (int32_t t = 0; t < P.g[i].tiles; ++t) {
            std::vector<int>& v = slots[i][t];
            std::sort(v.begin(), v.end());
            int np = 0, slot = 0;
            tile_pieces(P, P.g[i], t, 0, &np, &slot);
            if ((int)v.size() != np) return 20;
            for (int j = 0; j < np; ++j)
                if (v[j] != j) return 20;
        }
    }
    for (int i = 0; i < count; ++i) {
        const Desc& G = P.g[i];
        if (G.maxp < 2) continue;
        for (int j = i + 1; j < count; ++j) {
            const Desc& H = P.g[j];
            if (H.maxp < 2) continue;
            if (G.ticket_off < H.ticket_off + 4 * H.tiles && H.ticket_off < G.ticket_off + 4 * G.tiles)
                return 22;
            const int64_t gs = (int64_t)G.tiles * G.maxp * b * kM;
            const int64_t hs = (int64_t)H.tiles * H.maxp * b * kM;
            if (G.part_off < H.part_off + hs && H.part_off < G.part_off + gs) return 23;
        }
    }
    return 0;
}

int64_t q4_debug_check_tc_operands(uint64_t seed, int64_t blocks) {
    using namespace q4t;
    int64_t bad = 0;
    uint64_t st = seed ? seed : 1;
    auto next = [&st]() {
        st ^= st << 13;
        st ^= st >> 7;
        st ^= st << 17;
        return st;
    };
    // element map: a bijection of 0..31
    {
        int seen[32] = {0};
        for (int kap = 0; kap < 32; ++kap) {
            const int e = element_at(kap);
            if (e < 0 || e > 31 || seen[e]++) ++bad;
        }
    }
    std::vector<uint8_t> mem(kXOpBytes);
    for (int64_t it = 0; it < blocks; ++it) {
        uint8_t codes[16];
        for (int j = 0; j < 16; ++j) codes[j] = (uint8_t)next();
        int q[32];
        for (int j = 0; j < 16; ++j) {
            q[j] = codes[j] & 15;
            q[j + 16] = codes[j] >> 4;
        }
        const int mag = (int)(next() % 5);
        const float scale = mag == 0 ? 1.0f : mag == 1 ? 1e-3f : mag == 2 ? 37.0f : mag == 3 ? 1e-20f : 3e20f;
        float x[32];
        for (int j = 0; j < 32; ++j) {
            const double u = (double)(next() >> 11) * (1.0 / 9007199254740992.0);
            x[j] = (float)((2.0 * u - 1.0) * scale);
        }
        uint4 qv;
        std::memcpy(&qv, codes, 16);
        uint32_t a[16];
        q4tm::dequant_block(qv, a);
        // A value at MMA position kappa: column kappa/2, half kappa%2
        double aval[32];
        for (int kap = 0; kap < 32; ++kap) {
            const uint32_t bits = (a[kap >> 1] >> (16 * (kap & 1))) & 0xFFFFu;
            aval[kap] = (double)q4tm::bf16_value(bits);
            if (aval[kap] != (double)(q[element_at(kap)] - 8)) ++bad;
        }
        for (int mode = 0; mode < 2; ++mode) {
            const int nn = mode == 0 ? 16 : 32;
            const int t = mode == 0 ? 5 : 13;  // a token of each layout
            std::fill(mem.begin(), mem.end(), 0);
            // token t of block 0 in the layout the x warps write
            for (int c2 = 0; c2 < 2; ++c2)
                for (int hh = 0; hh < 2; ++hh) {
                    float e[8];
                    for (int m = 0; m < 8; ++m) e[m] = x[16 * c2 + 8 * hh + m];
                    uint4 H, L;
                    q4tm::split_row(e, &H, &L);
                    std::memcpy(&mem[x_row_off(nn, 0, c2, hh, t, 0)], &H, 16);
                    std::memcpy(&mem[x_row_off(nn, 0, c2, hh, t, 1)], &L, 16);
                }
            // the MMA: D[row 0][col] = sum_kappa A[kappa] B[col][kappa] over both
            // chunks, at the addresses the descriptor gives; the epilogue adds
            // columns t (hi) and N / 2 + t (lo)
            double dsum = 0.0;
            for (int hl = 0; hl < 2; ++hl) {
                const int col = hl ? nn / 2 + t : t;
                for (int kap = 0; kap < 32; ++kap) {
                    const int c2 = kap >> 4, kk = kap & 15;
                    const uint32_t addr = x_operand_off(nn, 0, c2) + (kk >> 3) * lbo(nn) +
                                          (col >> 3) * kSBO + (col & 7) * 16 + (kk & 7) * 2;
                    uint16_t bits;
                    std::memcpy(&bits, &mem[addr], 2);
                    dsum += aval[kap] * (double)q4tm::bf16_value(bits);
                }
            }
            double exact = 0.0, bound = 0.0;
            for (int j = 0; j < 32; ++j) {
                exact += (double)(q[j] - 8) * (double)x[j];
                bound += std::fabs((double)(q[j] - 8)) * std::fabs((double)x[j]);
            }
            if (!(std::fabs(dsum - exact) <= bound * std::ldexp(1.0, -16) + 1e-300)) ++bad;
        }
    }
    return bad;
}

int64_t q4_debug_check_intdot(uint64_t seed, int64_t blocks) {
    using namespace q4dev;
    int64_t bad = 0;
    // every integer in range splits into three in-range digits that add back up
    for (int32_t X = -kXMax; X <= kXMax; ++X) {
        int32_t a, b, c;
        x_digits(X, &a, &b, &c);
        if (a < -128 || a > 127 || b < -128 || b > 127 || c < -128 || c > 127 ||
            65536 * a + 256 * b + c != X)
            ++bad;
    }
    uint64_t z = seed;
    auto next = [&]() {
        z += 0x9E3779B97F4A7C15ull;
        uint64_t t = z;
        t = (t ^ (t >> 30)) * 0xBF58476D1CE4E5B9ull;
        t = (t ^ (t >> 27)) * 0x94D049BB133111EBull;
        return t ^ (t >> 31);
    };
    for (int64_t n = 0; n < blocks; ++n) {
        float x[32];
        uint32_t codes[32];
        const int kind = (int)(n % 5);
        for (int j = 0; j < 32; ++j) {
            const uint64_t r = next();
            const double u = ((r >> 11) & ((1ull << 40) - 1)) / double(1ull << 40) * 2.0 - 1.0;
            double v = u;
            if (kind == 1) v = u * ((n % 10 == 1) ? 1e-31 : 1e-20);  // tiny; below 1e-30: dropped
            if (kind == 2) v = u * 1e30;                         // huge
            if (kind == 3) v = (j == 7) ? 1e4 : u * 1e-3;        // one dominant element
            if (kind == 4) v = (j % 3 == 0) ? 0.0 : u;           // exact zeros
            x[j] = (float)v;
            codes[j] = (uint32_t)(r >> 60);
        }
        if (n % 97 == 0)
            for (int j = 0; j < 32; ++j) x[j] = 0.0f;
        float m = 0.0f;
        for (int j = 0; j < 32; ++j) m = fmaxf(m, fabsf(x[j]));
        const float sc = xq_scale(m), inv = xq_inv(m);
        XDigits xd;
        int32_t sa = 0, sb = 0, sc3 = 0;
        int32_t dig[3][32];
        for (int j = 0; j < 32; ++j) {
            int32_t a, b, c;
            x_digits(xq_int(x[j], inv), &a, &b, &c);
            dig[0][j] = a;
            dig[1][j] = b;
            dig[2][j] = c;
            sa += a;
            sb += b;
            sc3 += c;
        }
        for (int w = 0; w < 8; ++w) {
            xd.a[w] = xd.b[w] = xd.c[w] = 0u;
            for (int m2 = 0; m2 < 4; ++m2) {
                xd.a[w] |= (uint32_t)(uint8_t)dig[0][4 * w + m2] << (8 * m2);
                xd.b[w] |= (uint32_t)(uint8_t)dig[1][4 * w + m2] << (8 * m2);
                xd.c[w] |= (uint32_t)(uint8_t)dig[2][4 * w + m2] << (8 * m2);
            }
        }
        // code bytes: byte j holds code j (low nibble) and code j + 16 (high nibble)
        uint32_t qw[4] = {0u, 0u, 0u, 0u};
        for (int j = 0; j < 16; ++j) qw[j / 4] |= (codes[j] | (codes[j + 16] << 4)) << (8 * (j % 4));
        const float v = block_dot_int(make_uint4(qw[0], qw[1], qw[2], qw[3]), xd, -8 * sa, -8 * sb,
                                      -8 * sc3);
        double exact = 0.0, bound = 0.0;
        for (int j = 0; j < 32; ++j) {
            const double w8 = (double)codes[j] - 8.0;
            exact += w8 * (double)x[j];
            // half a step of s per element, plus two binary32 roundings in x * inv;
            // a block below kXTiny is dropped whole
            bound += fabs(w8) * (m < kXTiny ? fabs((double)x[j])
                                            : (double)sc * 0.5000001 + fabs((double)x[j]) * 2.4e-7);
        }
        bound += fabs(exact) * 2.4e-7 + 1e-300;  // the binary32 result and its scaling
        if (!(fabs((double)v * (double)sc - exact) <= bound)) ++bad;
    }
    return bad;
}

int64_t q4_debug_check_unpack(uint64_t seed, int64_t count) {
    int64_t bad = 0;
    auto check = [&](uint32_t word) {
        const q4dev::Pairs p = q4dev::unpack_word(word);
        auto code = [&](int bit) { return (float)((int)((word >> bit) & 0xFu) - 8); };
        // byte m: low nibble at bit 8m -> weight 4w+m, high nibble at 8m+4 -> 16+4w+m
        bad += p.lo01.x != code(0);
        bad += p.lo01.y != code(8);
        bad += p.lo23.x != code(16);
        bad += p.lo23.y != code(24);
        bad += p.hi01.x != code(4);
        bad += p.hi01.y != code(12);
        bad += p.hi23.x != code(20);
        bad += p.hi23.y != code(28);
    };
    for (int nib = 0; nib < 8; ++nib)
        for (uint32_t v = 0; v < 16; ++v) check(v << (4 * nib));
    uint64_t z = seed;
    for (int64_t i = 0; i < count; ++i) {
        z += 0x9E3779B97F4A7C15ull;
        uint64_t t = z;
        t = (t ^ (t >> 30)) * 0xBF58476D1CE4E5B9ull;
        t = (t ^ (t >> 27)) * 0x94D049BB133111EBull;
        t ^= t >> 31;
        check((uint32_t)t);
        check((uint32_t)(t >> 32));
    }
    // one block through block_dot with x = one-hot: each weight comes out alone
    for (int pos = 0; pos < 32; ++pos) {
        uint32_t words[4];
        for (int w = 0; w < 4; ++w) words[w] = 0x9C2E4A71u * (uint32_t)(w + 3 + pos);
        const uint4 q = make_uint4(words[0], words[1], words[2], words[3]);
        float4 x[8];
        for (int i = 0; i < 8; ++i) x[i] = make_float4(0.f, 0.f, 0.f, 0.f);
        float* xf = reinterpret_cast<float*>(x);
        xf[pos] = 1.0f;
        const float2 r = q4dev::block_dot(q, x, q4dev::unpack_consts_default());
        const int byte = (pos % 16), hi = pos >= 16;
        const uint32_t bv = (words[byte / 4] >> (8 * (byte % 4))) & 0xFFu;
        const float want = (float)((int)(hi ? (bv >> 4) : (bv & 0xFu)) - 8);
        bad += (r.x + r.y) != want;
    }
    return bad;
}

}  // extern "C"
