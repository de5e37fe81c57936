// C ABI of the Q4_0 decode library: argument checks (before any CUDA call),
// launch planning, the layer stack with programmatic dependent launch, CUDA
// graph capture, host interchange helpers, and the allocation-free GEMV.
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <climits>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include "../../include/q4.h"
#include "q4_host.h"

namespace q4h {

namespace {
std::atomic<uint64_t> g_launches{0};
thread_local cudaError_t g_last_cuda_error = cudaSuccess;

// Pieces the K-split rule for narrow groups aims at (two per multiprocessor of a
// B200). A constant, not the device's count, so that workspace sizes do not
// depend on the device.
constexpr int64_t kSplitPieces = 296;
// Shared-memory bytes a piece's per-(row, slice) partial sums may take: more
// rows per piece give it more pieces (CTAs).
constexpr int64_t kRedPref = 8192;
}  // namespace

bool cuda_failed(cudaError_t e) {
    if (e == cudaSuccess) return false;
    g_last_cuda_error = e;
    return true;
}

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
int64_t round_up(int64_t a, int64_t b) { return ceil_div(a, b) * b; }
bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

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

// ---------------------------------------------------------------------------
// batch-1 plan
// ---------------------------------------------------------------------------

q4_status plan_b1(const Shape* sh, int count, int b, int64_t part_base, int num_sms, q4b::Params* P,
                  int64_t* tickets, int64_t* ws_end) {
    if (count < 1 || count > Q4_MAX_GROUP || num_sms < 1 || b < 1 || b > q4b::kMaxTokens)
        return Q4_ERR_INVALID_ARG;
    std::memset(P, 0, sizeof *P);
    int64_t R = 0;
    for (int i = 0; i < count; ++i) {
        q4_status s = check_shape(sh[i].n, sh[i].k);
        if (s != Q4_OK) return s;
        if (sh[i].n >= (int64_t(1) << 31) || sh[i].k / Q4_QK >= (int64_t(1) << 31))
            return Q4_ERR_INVALID_ARG;  // 32-bit rows and blocks
        R += sh[i].n;
    }
    // a group with fewer rows than kSplitPieces splits K further, for parallelism
    const int64_t want = ceil_div(kSplitPieces, R);
    int64_t tick = 0, part = part_base;
    int64_t cps[Q4_MAX_GROUP], wsplit[Q4_MAX_GROUP];
    int max_slices = 1;
    for (int i = 0; i < count; ++i) {
        q4b::Desc& G = P->g[i];
        const int64_t nb = sh[i].k / Q4_QK;
        const int64_t nsl = ceil_div(nb, q4b::kSliceBlocks);
        // K in splits of q4b::kPieceSlices slices: a piece stages only the activations
        // of its own slices (read by every piece of the split), so short K-ranges
        // keep that traffic small next to the piece's weights
        const int64_t s0 = std::max(ceil_div(nsl, q4b::kPieceSlices), std::min(nsl, want));
        const int64_t sps = ceil_div(nsl, s0);
        const int64_t splits = ceil_div(nsl, sps);
        G.n = sh[i].n;
        G.nb = (int32_t)nb;
        G.nslices = (int32_t)nsl;
        G.splits = (int32_t)splits;
        G.slices_per_split = (int32_t)ceil_div(nsl, splits);
        G.d_map = nb % 8 == 0 ? 1 : 0;
        if (splits > 1) {
            G.ticket_off = kHeaderBytes / 4 + tick;
            tick += sh[i].n;
            G.part_off = part / 4;
            part += round_up(splits * b * sh[i].n * 4, 256);  // [splits][b][n]
        }
        max_slices = std::max<int>(max_slices, G.slices_per_split);
        // rows of one piece: its per-(token, row, slice) partial sums stay within kRedPref
        const int64_t max_rows = std::max<int64_t>(
            q4b::kTileRows, kRedPref / 4 / sps / b / q4b::kTileRows * q4b::kTileRows);
        cps[i] = std::min<int64_t>(sh[i].n, ceil_div(sh[i].n, max_rows));
        wsplit[i] = std::min<int64_t>(nb, G.slices_per_split * q4b::kSliceBlocks);  // blocks of a split
    }
    if (kHeaderBytes + 4 * tick > part_base) return Q4_ERR_INVALID_ARG;
    // spare CTAs (up to q4b::pieces_per_sm(b) per multiprocessor): to the GEMV whose
    // pieces carry the most weight bytes, a split's worth of pieces at a time
    const int64_t target = (int64_t)num_sms * q4b::pieces_per_sm(b);
    int64_t total = 0;
    for (int i = 0; i < count; ++i) total += P->g[i].splits * cps[i];
    while (true) {
        int best = -1;
        for (int i = 0; i < count; ++i) {
            if (cps[i] >= sh[i].n || total + P->g[i].splits > target) continue;
            if (best < 0 || sh[i].n * wsplit[i] * cps[best] > sh[best].n * wsplit[best] * cps[i]) best = i;
        }
        if (best < 0) break;
        ++cps[best];
        total += P->g[best].splits;
    }
    if (total >= (int64_t(1) << 31)) return Q4_ERR_UNSUPPORTED;
    int64_t pb = 0, red_floats = 0;
    for (int i = 0; i < count; ++i) {
        q4b::Desc& G = P->g[i];
        G.piece_begin = (int32_t)pb;
        G.cps = (int32_t)cps[i];
        pb += G.splits * cps[i];
        int64_t rows_max = 0;  // the first (widest) row range
        for (int64_t j = 0; j < cps[i]; ++j)
            rows_max = std::max(rows_max, q4b::range_start(sh[i].n, cps[i], j + 1) - q4b::range_start(sh[i].n, cps[i], j));
        red_floats = std::max<int64_t>(red_floats,
                                       ceil_div(rows_max, q4b::kTileRows) * q4b::kTileRows * G.slices_per_split * b);
    }
    P->count = count;
    P->npieces = (int32_t)total;
    P->red_bytes = (uint32_t)round_up(red_floats * 4, 128);
    P->b = b;
    P->max_slices = max_slices;
    P->x_bytes = (uint32_t)(max_slices * (b == 1 ? q4b::kXSliceBytes : b * q4b::kXFSliceBytes));
    const int64_t room = (int64_t)q4b::smem_budget(b) - q4b::kBarBytes - P->red_bytes - P->x_bytes;
    // a multiple of the CTA's warps: each slot is requested and read by one warp
    const int64_t slots =
        std::min<int64_t>(room / q4b::kSlotBytes, q4b::max_slots(b)) / q4b::kWarps * q4b::kWarps;
    if (slots < q4b::kMinSlots) return Q4_ERR_UNSUPPORTED;
    P->slots = (int32_t)slots;
    *tickets = tick;
    *ws_end = part;
    return Q4_OK;
}

// ---------------------------------------------------------------------------
// tensor-core plan (2..16 tokens)
// ---------------------------------------------------------------------------

q4_status plan_tc(const Shape* sh, int count, int b, int64_t part_base, int num_sms, q4t::Params* P,
                  int64_t* tickets, int64_t* ws_end) {
    if (count < 1 || count > Q4_MAX_GROUP || b < 2 || b > Q4_MAX_BATCH || num_sms < 1)
        return Q4_ERR_INVALID_ARG;
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
    P->grid = (int32_t)std::min<int64_t>(num_sms, F);
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
            G.ticket_off = kHeaderBytes / 4 + tick;
            tick += 4 * (int64_t)G.tiles;
            G.part_off = part / 4;
            part += round_up((int64_t)G.tiles * maxp * b * q4t::kM * 4, 256);
        }
    }
    if (kHeaderBytes + 4 * tick > part_base) return Q4_ERR_INVALID_ARG;
    *tickets = tick;
    *ws_end = part;
    return Q4_OK;
}

int64_t part_base_for(int64_t tickets) { return kHeaderBytes + round_up(4 * tickets, 256); }

q4_status group_need(const Shape* sh, int count, int b, int num_sms, int64_t* tickets,
                     int64_t* part_bytes) {
    if (count < 1 || count > Q4_MAX_GROUP) return Q4_ERR_INVALID_ARG;
    if (b < 1 || b > Q4_MAX_BATCH) return Q4_ERR_UNSUPPORTED;
    constexpr int64_t kBase = 0x40000000LL;
    int64_t t = 0, end = 0;
    q4_status s;
    if (b <= q4b::kMaxTokens) {
        q4b::Params P;
        s = plan_b1(sh, count, b, kBase, num_sms, &P, &t, &end);
    } else {
        q4t::Params P;
        s = plan_tc(sh, count, b, kBase, num_sms, &P, &t, &end);
    }
    if (s != Q4_OK) return s;
    *tickets = t;
    *part_bytes = end - kBase;
    return Q4_OK;
}

// ---------------------------------------------------------------------------
// devices
// ---------------------------------------------------------------------------

namespace {
std::mutex g_dev_mu;
bool g_dev_ready[64];
int g_dev_sms[64];

// Multiprocessors of the current device for workspace sizing: the device's own
// count when a device is there, else the B200's 148.
int sizing_sms() {
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1) {
        cudaGetLastError();  // clear a no-device error
        return 148;
    }
    return sms;
}
}  // namespace

q4_status ensure_device(int* num_sms) {
    int dev = 0;
    if (cuda_failed(cudaGetDevice(&dev))) return Q4_ERR_CUDA;
    if (dev < 0 || dev >= 64) return Q4_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_dev_mu);
    if (!g_dev_ready[dev]) {
        int major = 0, minor = 0, optin = 0, sms = 0;
        if (cuda_failed(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) ||
            cuda_failed(cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) ||
            cuda_failed(cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) ||
            cuda_failed(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)))
            return Q4_ERR_CUDA;
        if (major != 10 || minor != 0 || sms < 1) return Q4_ERR_UNSUPPORTED;
        if (cuda_failed(q4k::setup_b1_kernel(optin))) return Q4_ERR_CUDA;
        if (cuda_failed(q4k::setup_tc_kernels(optin))) return Q4_ERR_CUDA;
        g_dev_sms[dev] = sms;
        g_dev_ready[dev] = true;
    }
    *num_sms = g_dev_sms[dev];
    return Q4_OK;
}

}  // namespace q4h

using namespace q4h;

namespace {

// Argument checks of one group for `b` tokens (no CUDA call).
q4_status check_args(const GemvCall* calls, int count, int b) {
    if (count < 1 || count > Q4_MAX_GROUP) return Q4_ERR_INVALID_ARG;
    if (b < 1 || b > Q4_MAX_BATCH) return Q4_ERR_UNSUPPORTED;
    for (int i = 0; i < count; ++i) {
        q4_status s = check_matrix(&calls[i].m);
        if (s != Q4_OK) return s;
        if (!calls[i].x || !calls[i].y) return Q4_ERR_INVALID_ARG;
        if (!aligned(calls[i].x, 16) || !aligned(calls[i].y, 16)) return Q4_ERR_MISALIGNED;
    }
    return Q4_OK;
}

// Validate one group for `b` tokens; returns its ticket count and the
// partial-sum bytes it needs past the ticket region.
q4_status check_group(const GemvCall* calls, int count, int b, int num_sms, int64_t* tickets,
                      int64_t* part_bytes) {
    q4_status s = check_args(calls, count, b);
    if (s != Q4_OK) return s;
    Shape sh[Q4_MAX_GROUP];
    for (int i = 0; i < count; ++i) sh[i] = {calls[i].m.n, calls[i].m.k};
    return group_need(sh, count, b, num_sms, tickets, part_bytes);
}

// Argument checks of a whole stack (no CUDA call).
q4_status stack_args(const q4_stack* s, int b, std::vector<std::pair<int, int>>* groups);

q4_status check_ws(void* ws, size_t ws_bytes, size_t need) {
    if (!ws || ws_bytes < need) return Q4_ERR_WORKSPACE;
    if (!aligned(ws, 256)) return Q4_ERR_MISALIGNED;
    return Q4_OK;
}

// Enqueue one group as one launch, with partial sums from `part_base`. The
// launch may overlap the previous kernel of the stream (programmatic dependent
// launch) only if `pdl` is set.
q4_status launch_group(const GemvCall* calls, int count, int b, void* ws, int64_t part_base,
                       int num_sms, bool pdl, cudaStream_t stream, uint32_t tx_extra = 0) {
    Shape sh[Q4_MAX_GROUP];
    for (int i = 0; i < count; ++i) sh[i] = {calls[i].m.n, calls[i].m.k};
    int64_t t = 0, end = 0;
    if (b <= q4b::kMaxTokens) {
        q4b::Params P;
        q4_status s = plan_b1(sh, count, b, part_base, num_sms, &P, &t, &end);
        if (s != Q4_OK) return s;
        for (int i = 0; i < count; ++i) {
            P.g[i].qs = calls[i].m.qs;
            P.g[i].d = calls[i].m.d;
            P.g[i].x = calls[i].x;
            P.g[i].y = calls[i].y;
            if (cuda_failed(q4k::encode_b1_maps(&P.qs_map[i], &P.d_map[i], &P.g[i].d_map, calls[i].m.qs,
                                                calls[i].m.d, calls[i].m.n, calls[i].m.k)))
                return Q4_ERR_CUDA;
        }
        P.ws = static_cast<uint32_t*>(ws);
        P.tx_extra = tx_extra;
        if (cuda_failed(q4k::launch_b1(P, pdl, stream))) return Q4_ERR_CUDA;
        g_launches.fetch_add(1, std::memory_order_relaxed);
        return Q4_OK;
    }
    q4t::Params P;
    q4_status s = plan_tc(sh, count, b, part_base, num_sms, &P, &t, &end);
    if (s != Q4_OK) return s;
    for (int i = 0; i < count; ++i) {
        P.g[i].qs = calls[i].m.qs;
        P.g[i].d = calls[i].m.d;
        P.g[i].x = calls[i].x;
        P.g[i].y = calls[i].y;
        if (cuda_failed(q4k::encode_tc_maps(&P.maps[i], &P.g[i].d_box, calls[i].m.qs, calls[i].m.d,
                                            calls[i].x, calls[i].m.n, calls[i].m.k, b)))
            return Q4_ERR_CUDA;
    }
    P.ws = static_cast<uint32_t*>(ws);
    P.tx_extra = tx_extra;
    if (cuda_failed(q4k::launch_tc(P, pdl, stream))) return Q4_ERR_CUDA;
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return Q4_OK;
}

// Zero the ticket region of a call before its first kernel.
q4_status clear_tickets(void* ws, int64_t tickets, cudaStream_t stream) {
    if (tickets == 0) return Q4_OK;
    if (cuda_failed(cudaMemsetAsync(static_cast<uint8_t*>(ws) + kHeaderBytes, 0, (size_t)(4 * tickets),
                                    stream)))
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

q4_status stack_args(const q4_stack* s, int b, std::vector<std::pair<int, int>>* groups) {
    q4_status st = stack_groups(s, groups);
    if (st != Q4_OK) return st;
    for (auto& g : *groups) {
        GemvCall calls[Q4_MAX_GROUP];
        for (int i = g.first; i < g.second; ++i) calls[i - g.first] = {s->mats[i], s->x[i], s->y[i]};
        if ((st = check_args(calls, g.second - g.first, b)) != Q4_OK) return st;
    }
    return Q4_OK;
}

// Validate a stack; returns the ticket region shared by all groups and the
// workspace bytes needed.
q4_status stack_check(const q4_stack* s, int b, int num_sms, std::vector<std::pair<int, int>>* groups,
                      int64_t* tickets, size_t* need) {
    q4_status st = stack_groups(s, groups);
    if (st != Q4_OK) return st;
    int64_t tmax = 0, pmax = 0;
    for (auto& g : *groups) {
        GemvCall calls[Q4_MAX_GROUP];
        for (int i = g.first; i < g.second; ++i) calls[i - g.first] = {s->mats[i], s->x[i], s->y[i]};
        int64_t t = 0, p = 0;
        st = check_group(calls, g.second - g.first, b, num_sms, &t, &p);
        if (st != Q4_OK) return st;
        tmax = std::max(tmax, t);
        pmax = std::max(pmax, p);
    }
    *tickets = tmax;
    *need = (size_t)(part_base_for(tmax) + pmax);
    return Q4_OK;
}

}  // namespace

struct q4_graph_s {
    cudaGraph_t graph;
    cudaGraphExec_t exec;
    uint64_t kernels;
};

// Entry points shared with the diagnostics in q4_debug.cu.
namespace q4h {
q4_status gemv_call(const q4_matrix* m, const float* X, int b, float* Y, void* ws, size_t ws_bytes,
                    void* stream, uint32_t tx_extra) {
    if (!m) return Q4_ERR_INVALID_ARG;
    GemvCall call = {*m, X, Y};
    q4_status s = check_args(&call, 1, b);
    if (s != Q4_OK) return s;
    if (!ws || ws_bytes < (size_t)kHeaderBytes) return Q4_ERR_WORKSPACE;
    if (!aligned(ws, 256)) return Q4_ERR_MISALIGNED;
    if (b <= q4b::kMaxTokens) {  // the CUDA-core need does not depend on the device
        int64_t t = 0, p = 0;
        if ((s = check_group(&call, 1, b, 148, &t, &p)) != Q4_OK) return s;
        if ((s = check_ws(ws, ws_bytes, (size_t)(part_base_for(t) + p))) != Q4_OK) return s;
    }
    int num_sms = 0;
    if ((s = ensure_device(&num_sms)) != Q4_OK) return s;
    int64_t tickets = 0, part = 0;
    if ((s = check_group(&call, 1, b, num_sms, &tickets, &part)) != Q4_OK) return s;
    const int64_t base = part_base_for(tickets);
    if ((s = check_ws(ws, ws_bytes, (size_t)(base + part))) != Q4_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if ((s = clear_tickets(ws, tickets, st)) != Q4_OK) return s;
    return launch_group(&call, 1, b, ws, base, num_sms, false, st, tx_extra);
}
}  // namespace q4h

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
    int num_sms = 0;
    if ((s = ensure_device(&num_sms)) != Q4_OK) return s;
    const int64_t nblocks = out->n * (out->k / Q4_QK);
    if (cuda_failed(q4k::launch_pack(w, out->qs, out->d, nblocks, num_sms, static_cast<cudaStream_t>(stream))))
        return Q4_ERR_CUDA;
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return Q4_OK;
}

q4_status q4_dequant(const q4_matrix* m, float* w_out, void* stream) {
    q4_status s = check_matrix(m);
    if (s != Q4_OK) return s;
    if (!w_out) return Q4_ERR_INVALID_ARG;
    if (!aligned(w_out, 16)) return Q4_ERR_MISALIGNED;
    int num_sms = 0;
    if ((s = ensure_device(&num_sms)) != Q4_OK) return s;
    const int64_t nblocks = m->n * (m->k / Q4_QK);
    if (cuda_failed(q4k::launch_dequant(m->qs, m->d, w_out, nblocks, num_sms,
                                        static_cast<cudaStream_t>(stream))))
        return Q4_ERR_CUDA;
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return Q4_OK;
}

size_t q4_workspace_bytes(int64_t n, int64_t k, int b) {
    if (check_shape(n, k) != Q4_OK || b < 1 || b > Q4_MAX_BATCH) return 0;
    const Shape sh = {n, k};
    int64_t t = 0, p = 0;
    if (group_need(&sh, 1, b, sizing_sms(), &t, &p) != Q4_OK) return 0;
    return (size_t)(part_base_for(t) + p);
}

q4_status q4_workspace_init(void* ws, size_t ws_bytes, void* stream) {
    if (!ws || ws_bytes < (size_t)kHeaderBytes) return Q4_ERR_WORKSPACE;
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
    return gemv_call(m, X, b, Y, ws, ws_bytes, stream, 0u);
}

q4_status q4_gemv(const q4_matrix* m, const float* x, float* y, void* ws, size_t ws_bytes,
                  void* stream) {
    return q4_gemv_batched(m, x, 1, y, ws, ws_bytes, stream);
}

size_t q4_stack_workspace_bytes(const q4_stack* s, int b) {
    std::vector<std::pair<int, int>> groups;
    int64_t tickets = 0;
    size_t need = 0;
    if (stack_check(s, b, sizing_sms(), &groups, &tickets, &need) != Q4_OK) return 0;
    return need;
}

q4_status q4_layer_stack(const q4_stack* s, int b, void* ws, size_t ws_bytes, void* stream) {
    std::vector<std::pair<int, int>> groups;
    q4_status st = stack_args(s, b, &groups);
    if (st != Q4_OK) return st;
    if (!ws || ws_bytes < (size_t)kHeaderBytes) return Q4_ERR_WORKSPACE;
    if (!aligned(ws, 256)) return Q4_ERR_MISALIGNED;
    int num_sms = 0;
    if ((st = ensure_device(&num_sms)) != Q4_OK) return st;
    int64_t tickets = 0;
    size_t need = 0;
    if ((st = stack_check(s, b, num_sms, &groups, &tickets, &need)) != Q4_OK) return st;
    if ((st = check_ws(ws, ws_bytes, need)) != Q4_OK) return st;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    if ((st = clear_tickets(ws, tickets, cs)) != Q4_OK) return st;
    const int64_t base = part_base_for(tickets);
    bool first = true;
    for (auto& g : groups) {
        GemvCall calls[Q4_MAX_GROUP];
        for (int i = g.first; i < g.second; ++i) calls[i - g.first] = {s->mats[i], s->x[i], s->y[i]};
        st = launch_group(calls, g.second - g.first, b, ws, base, num_sms, !first, cs);
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
    q4_status st = stack_args(s, b, &groups);
    if (st != Q4_OK) return st;
    if (!ws || ws_bytes < (size_t)kHeaderBytes) return Q4_ERR_WORKSPACE;
    if (!aligned(ws, 256)) return Q4_ERR_MISALIGNED;
    int num_sms = 0;
    if ((st = ensure_device(&num_sms)) != Q4_OK) return st;
    int64_t tickets = 0;
    size_t need = 0;
    if ((st = stack_check(s, b, num_sms, &groups, &tickets, &need)) != Q4_OK) return st;
    if ((st = check_ws(ws, ws_bytes, need)) != Q4_OK) return st;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cuda_failed(cudaStreamIsCapturing(cs, &cap))) return Q4_ERR_CUDA;
    if (cap != cudaStreamCaptureStatusNone) return Q4_ERR_INVALID_ARG;
    if (cuda_failed(cudaStreamBeginCapture(cs, cudaStreamCaptureModeThreadLocal))) return Q4_ERR_CUDA;
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
    g->kernels = (uint64_t)groups.size();
    *out = g;
    return Q4_OK;
}

q4_status q4_graph_launch(q4_graph g, void* stream) {
    if (!g) return Q4_ERR_INVALID_ARG;
    if (cuda_failed(cudaGraphLaunch(g->exec, static_cast<cudaStream_t>(stream)))) return Q4_ERR_CUDA;
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

q4_status q4_blocks_to_planes(const uint8_t* blocks, int64_t n, int64_t k, uint8_t* qs, uint16_t* d) {
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
// comes from cudaGetSymbolAddress, looked up on every call with the device
// current (cheap, and still right after the device's context has been reset).
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
q4_status noalloc_scratch(void** out) {
    void* p = nullptr;
    if (cuda_failed(cudaGetSymbolAddress(&p, g_noalloc_scratch))) return Q4_ERR_CUDA;
    *out = p;
    return Q4_OK;
}
}  // namespace

q4_status q4_gemv_noalloc(const q4_matrix* m, const float* x, float* y, void* stream) {
    if (!m) return Q4_ERR_INVALID_ARG;
    GemvCall call = {*m, x, y};
    q4_status s = check_args(&call, 1, 1);
    if (s != Q4_OK) return s;
    // the scratch need does not depend on the device: checked before any CUDA call
    int64_t tickets = 0, part = 0;
    if ((s = check_group(&call, 1, 1, 148, &tickets, &part)) != Q4_OK) return s;
    if ((size_t)(part_base_for(tickets) + part) > kNoAllocScratchBytes) return Q4_ERR_WORKSPACE;
    int num_sms = 0;
    if ((s = ensure_device(&num_sms)) != Q4_OK) return s;
    if ((s = check_group(&call, 1, 1, num_sms, &tickets, &part)) != Q4_OK) return s;
    const int64_t base = part_base_for(tickets);
    if ((size_t)(base + part) > kNoAllocScratchBytes) return Q4_ERR_WORKSPACE;
    void* scratch = nullptr;
    if ((s = noalloc_scratch(&scratch)) != Q4_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // the status header is not cleared here: a timeout stays recorded until
    // q4_noalloc_status reads (and clears) it
    if ((s = clear_tickets(scratch, tickets, st)) != Q4_OK) return s;
    return launch_group(&call, 1, 1, scratch, base, num_sms, false, st);
}

q4_status q4_noalloc_status(void* stream) {
    void* scratch = nullptr;
    q4_status s = noalloc_scratch(&scratch);
    if (s != Q4_OK) return s;
    uint32_t flag = 0;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cuda_failed(cudaMemcpyAsync(&flag, scratch, sizeof flag, cudaMemcpyDeviceToHost, st)))
        return Q4_ERR_CUDA;
    if (cuda_failed(cudaMemsetAsync(scratch, 0, sizeof flag, st))) return Q4_ERR_CUDA;
    if (cuda_failed(cudaStreamSynchronize(st))) return Q4_ERR_CUDA;
    return flag ? Q4_ERR_TIMEOUT : Q4_OK;
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

}  // extern "C"
