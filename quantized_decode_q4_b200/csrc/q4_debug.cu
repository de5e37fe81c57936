// Host-only diagnostics of the library (include/q4_debug.h): replays of the
// launch plans and of the register-level arithmetic on the CPU, plus the stall
// hook that exercises the bounded-wait timeout path on a GPU without a fault.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

#include "../../include/q4.h"
#include "../../include/q4_debug.h"
#include "q4_b1_plan.h"
#include "q4_device.cuh"
#include "q4_host.h"
#include "q4_intdot.cuh"
#include "q4_tc_math.cuh"
#include "q4_tc_plan.h"

using namespace q4h;

namespace q4h {
q4_status gemv_call(const q4_matrix* m, const float* X, int b, float* Y, void* ws, size_t ws_bytes,
                    void* stream, uint32_t tx_extra);
}

namespace {

constexpr int kRefSms = 148;  // B200

uint64_t splitmix(uint64_t* z) {
    *z += 0x9E3779B97F4A7C15ull;
    uint64_t t = *z;
    t = (t ^ (t >> 30)) * 0xBF58476D1CE4E5B9ull;
    t = (t ^ (t >> 27)) * 0x94D049BB133111EBull;
    return t ^ (t >> 31);
}

}  // namespace

extern "C" {

int q4_debug_check_b1(const int64_t* n, const int64_t* k, int count, int b, int num_sms) {
    using namespace q4b;
    if (!n || !k || count < 1 || count > Q4_MAX_GROUP || num_sms < 1 || b < 1 || b > kMaxTokens) return 1;
    Shape sh[Q4_MAX_GROUP];
    for (int i = 0; i < count; ++i) sh[i] = {n[i], k[i]};
    Params P;
    int64_t tickets = 0, end = 0;
    if (plan_b1(sh, count, b, INT64_MAX / 4, num_sms, &P, &tickets, &end) != Q4_OK) return 2;
    const int64_t base = part_base_for(tickets);
    if (plan_b1(sh, count, b, base, num_sms, &P, &tickets, &end) != Q4_OK) return 2;
    if (P.b != b) return 2;
    // shared memory: inside the budget, regions aligned, ring within its bounds
    if (smem_bytes(P) > (uint32_t)smem_budget(b)) return 3;
    if (P.slots < kMinSlots || P.slots > max_slots(b) || P.slots % kWarps) return 3;
    if (ring_offset(P) % 128 || x_offset(P) % 16 || red_offset() % 16) return 4;
    if (P.npieces < 1) return 5;
    {
        // pieces of each GEMV laid end to end, and no multiprocessor left idle
        // while a GEMV could still take a split's worth of pieces
        int64_t pb = 0;
        for (int i = 0; i < count; ++i) {
            if (P.g[i].piece_begin != pb || P.g[i].cps < 1 || P.g[i].cps > P.g[i].n) return 5;
            pb += (int64_t)P.g[i].splits * P.g[i].cps;
        }
        if (pb != P.npieces) return 5;
        for (int i = 0; i < count; ++i)
            if (P.g[i].cps < P.g[i].n && P.npieces + P.g[i].splits <= pieces_per_sm(b) * num_sms) return 5;
    }
    // coverage of every (row, global slice) and the copies of every unit
    std::vector<std::vector<uint8_t>> cover(count);
    for (int i = 0; i < count; ++i) cover[i].assign((size_t)(sh[i].n * P.g[i].nslices), 0);
    for (int c = 0; c < P.npieces; ++c) {
        const Piece pc = piece_of(P, c);
        if (pc.g < 0 || pc.g >= count) return 6;
        const Desc& G = P.g[pc.g];
        if (pc.r0 < 0 || pc.r1 <= pc.r0 || pc.r1 > G.n) return 7;
        if (pc.split < 0 || pc.split >= G.splits) return 8;
        // the ticket of the piece's row range: inside the GEMV's ticket words, and
        // shared only with the pieces of the same rows in the other splits
        if (pc.j < 0 || pc.j >= G.cps || pc.j >= G.n) return 8;
        if (G.splits > 1) {
            const Piece q0 = piece_of(P, G.piece_begin + pc.j * G.splits);
            if (q0.split != 0 || q0.j != pc.j || q0.r0 != pc.r0 || q0.r1 != pc.r1) return 8;
        }
        int s0 = 0, S = 0;
        piece_slices(G, pc.split, &s0, &S);
        if (S < 1 || S > kPieceSlices || s0 + S > G.nslices) return 9;  // staging holds kPieceSlices
        if (b == 1) {
            if ((uint32_t)S * kXSliceBytes > P.x_bytes) return 10;
            if (xchunk_offset(S - 1, kXChunks - 1, kSliceBlocks - 1) + 16 > P.x_bytes) return 10;
        } else {
            if ((uint32_t)(S * b * kXFSliceBytes) > P.x_bytes) return 10;
            if (xfchunk_offset(S - 1, b - 1, b, 7, kSliceBlocks - 1) + 16 > P.x_bytes) return 10;
            // the staging rounds: one (slice, token) pair per 256 threads
            if (kThreads != 256) return 10;
        }
        const int T = piece_tiles(pc);
        if ((int64_t)T * kTileRows * S * b * 4 > (int64_t)P.red_bytes) return 11;
        const int64_t qs_plane = sh[pc.g].n * (sh[pc.g].k / 2);
        const int64_t d_plane = round_up(sh[pc.g].n * G.nb * 2, 16);
        for (int t = 0; t < T; ++t)
            for (int s = 0; s < S; ++s) {
                const int gs = s0 + s;
                const int bs = slice_blocks(G, gs);
                if (bs < 1 || bs > kSliceBlocks) return 12;
                // codes: one box of 128 uint32 x 8 rows at (gs * 128, row0): its
                // x coordinate is 16-byte aligned and it covers the unit's blocks
                const int64_t row0 = (int64_t)pc.r0 + (int64_t)t * kTileRows;
                if (((int64_t)gs * kSliceBlocks * 16) % 16 || row0 >= (int64_t(1) << 31)) return 14;
                if ((int64_t)gs * kSliceBlocks * 16 >= sh[pc.g].k / 2) return 15;
                if (kMapCodeBytes != (uint32_t)(kTileRows * kSliceBlocks * 16) || kMapCodeBytes > (uint32_t)kSlotQs)
                    return 16;
                int64_t tx = kMapCodeBytes;
                if (G.d_map) {
                    // scales: one box of 32 uint16 x 8 rows at (gs * 32, row0); the
                    // plane's row stride must be a multiple of 16 bytes
                    if ((G.nb * 2) % 16 || ((int64_t)gs * kSliceBlocks * 2) % 16) return 17;
                    if (kMapScaleBytes > (uint32_t)(kTileRows * kDRow)) return 19;
                    for (int r = 0; r < kTileRows; ++r)
                        for (int j = 0; j < kSliceBlocks; ++j) {
                            const uint32_t off = scale_offset(G, pc, t, gs, r, j);
                            if (off != (uint32_t)(kSlotQs + (r * kSliceBlocks + j) * 2)) return 20;
                        }
                    tx += kMapScaleBytes;
                } else {
                    for (int lane = 8; lane < 16; ++lane) {
                        const LaneCopy lc = lane_copy(G, pc, t, gs, lane);
                        const int r = lane & 7;
                        const int64_t row = row0 + r;
                        if (row >= pc.r1) {
                            if (lc.active) return 13;
                            continue;
                        }
                        if (!lc.active || !lc.scales) return 13;
                        if (lc.src_off < 0 || lc.src_off % 16 || lc.bytes % 16 || lc.bytes == 0 || lc.dst % 16)
                            return 14;
                        if (lc.src_off + lc.bytes > d_plane) return 18;
                        if (lc.dst < (uint32_t)kSlotQs || lc.dst + lc.bytes > (uint32_t)(kSlotQs + (r + 1) * kDRow))
                            return 19;
                        // the scale the math lane reads is the one of its block
                        for (int j = 0; j < bs; ++j) {
                            const uint32_t off = scale_offset(G, pc, t, gs, r, j);
                            const int64_t want = (row * G.nb + (int64_t)gs * kSliceBlocks + j) * 2;
                            if (off < lc.dst || off + 2 > lc.dst + lc.bytes) return 20;
                            if ((int64_t)(off - lc.dst) + lc.src_off != want) return 20;
                        }
                        tx += lc.bytes;
                    }
                }
                (void)qs_plane;
                if (tx >= (int64_t(1) << 20)) return 21;
                for (int r = 0; r < kTileRows; ++r) {
                    const int64_t row = (int64_t)pc.r0 + (int64_t)t * kTileRows + r;
                    if (row >= pc.r1) break;
                    uint8_t& cv = cover[pc.g][(size_t)(row * G.nslices + gs)];
                    if (cv) return 22;
                    cv = 1;
                }
            }
    }
    for (int i = 0; i < count; ++i)
        for (uint8_t cv : cover[i])
            if (!cv) return 23;
    // split-K tickets and partial sums inside the workspace, and disjoint
    for (int i = 0; i < count; ++i) {
        const Desc& G = P.g[i];
        if (G.splits < 1 || (int64_t)G.splits * G.slices_per_split < G.nslices) return 24;
        if (G.splits == 1) continue;
        if (G.ticket_off * 4 < kHeaderBytes || (G.ticket_off + G.n) * 4 > base) return 25;
        if (G.part_off * 4 < base || (G.part_off + (int64_t)G.splits * b * G.n) * 4 > end) return 26;
        for (int j = i + 1; j < count; ++j) {
            const Desc& H = P.g[j];
            if (H.splits == 1) continue;
            if (G.ticket_off < H.ticket_off + H.n && H.ticket_off < G.ticket_off + G.n) return 27;
            if (G.part_off < H.part_off + (int64_t)H.splits * b * H.n &&
                H.part_off < G.part_off + (int64_t)G.splits * b * G.n)
                return 27;
        }
    }
    return 0;
}

q4_status q4_debug_plan_info(const int64_t* n, const int64_t* k, int count, int b, int64_t* out) {
    if (!n || !k || !out || count < 1 || count > Q4_MAX_GROUP || b < 1 || b > q4b::kMaxTokens)
        return Q4_ERR_INVALID_ARG;
    Shape sh[Q4_MAX_GROUP];
    for (int i = 0; i < count; ++i) sh[i] = {n[i], k[i]};
    q4b::Params P;
    int64_t tickets = 0, end = 0;
    q4_status s = plan_b1(sh, count, b, INT64_MAX / 4, kRefSms, &P, &tickets, &end);
    if (s != Q4_OK) return s;
    const int64_t base = part_base_for(tickets);
    if ((s = plan_b1(sh, count, b, base, kRefSms, &P, &tickets, &end)) != Q4_OK) return s;
    out[0] = P.npieces;
    out[1] = q4b::smem_bytes(P);
    out[2] = end;
    out[3] = P.slots;
    for (int i = 0; i < count; ++i) out[4 + i] = P.g[i].splits;
    return Q4_OK;
}

q4_status q4_debug_gemv_stall(const q4_matrix* m, const float* X, int b, float* Y, void* ws,
                              size_t ws_bytes, void* stream) {
    return gemv_call(m, X, b, Y, ws, ws_bytes, stream, 16u);
}

int64_t q4_debug_check_intdot(uint64_t seed, int64_t blocks) {
    using namespace q4dev;
    int64_t bad = 0;
    // digit split: every boundary and a stride through the range add back up
    auto digits_ok = [](int32_t X) {
        int32_t d0, d1;
        x_digits16(X, &d0, &d1);
        return d0 >= -32768 && d0 <= 32767 && d1 >= -16384 && d1 <= 16384 &&
               (int64_t)d1 * 65536 + d0 == (int64_t)X;
    };
    for (int64_t X = -(int64_t(1) << 30); X <= (int64_t(1) << 30); X += 65521)
        bad += !digits_ok((int32_t)X);
    for (int32_t e = -3; e <= 3; ++e)
        for (int32_t c : {0, 32767, 32768, 65535, 65536, (1 << 30) - 1, 1 << 30})
            for (int sgn : {-1, 1}) {
                const int64_t X = (int64_t)sgn * c + e;
                if (X >= -(int64_t(1) << 30) && X <= (int64_t(1) << 30)) bad += !digits_ok((int32_t)X);
            }
    // blocks over many magnitudes, with outliers, subnormals and zeros: a block
    // that is not flagged is within 2^-14 of each element; a flagged one goes
    // through the binary32 path and is within binary32 rounding
    uint64_t z = seed;
    const q4dev::UnpackConsts kc = q4dev::unpack_consts_default();
    int64_t flagged = 0;
    for (int64_t it = 0; it < blocks; ++it) {
        float x[32];
        uint32_t codes[32];
        const int kind = (int)(it % 8);
        const uint64_t rb = splitmix(&z);
        const double mag = std::ldexp(1.0, (int)(rb % 200) - 100);
        const int pos = (int)((rb >> 32) % 32);
        for (int j = 0; j < 32; ++j) {
            const uint64_t r = splitmix(&z);
            const double u = ((r >> 11) & ((1ull << 40) - 1)) / double(1ull << 40) * 2.0 - 1.0;
            double v = u;
            if (kind == 1) v = u * mag;                                   // any magnitude
            if (kind == 2) v = (j == pos) ? 1e6 * (u < 0 ? -1 : 1) : u;  // one outlier
            if (kind == 3) v = (j % 11 == 0) ? 1e5 : u * 1e-40;           // subnormal rest
            if (kind == 4) v = (j % 3 == 0) ? 0.0 : u;                    // exact zeros
            if (kind == 5) v = u * 1e-5;                                  // small normal
            if (kind == 6) v = (j < 2) ? (j ? -1e4 : 1e4) : u;            // two mixed-sign outliers
            x[j] = (float)v;
            codes[j] = (uint32_t)(r >> 60);
        }
        const bool zeros = it % 97 == 0;
        if (zeros)
            for (int j = 0; j < 32; ++j) x[j] = 0.0f;
        XPlanes xp;
        float sc = 0.0f;
        const bool flag = xq_block(x, &xp, &sc);
        uint32_t qw[4] = {0u, 0u, 0u, 0u};
        for (int j = 0; j < 16; ++j) qw[j / 4] |= (codes[j] | (codes[j + 16] << 4)) << (8 * (j % 4));
        const uint4 q = make_uint4(qw[0], qw[1], qw[2], qw[3]);
        double exact = 0.0, abs_sum = 0.0;
        for (int j = 0; j < 32; ++j) {
            const double w8 = (double)codes[j] - 8.0;
            exact += w8 * (double)x[j];
            abs_sum += std::fabs(w8 * (double)x[j]);
        }
        double got;
        if (!flag) {
            got = (double)block_dot16(q, xp) * (double)sc / 16.0;
            // per element 2^-14 of itself, plus the binary32 rounding of the block sum
            if (!(std::fabs(got - exact) <= abs_sum * (std::ldexp(1.0, -14) + std::ldexp(1.0, -23)) + 1e-300))
                ++bad;
        } else {
            ++flagged;
            float4 xv[8];
            std::memcpy(xv, x, sizeof x);
            const float2 r2 = block_dot(q, xv, kc);
            got = (double)r2.x + (double)r2.y;
            // binary32 products and sums of 32 terms
            if (!(std::fabs(got - exact) <= abs_sum * 33.0 * std::ldexp(1.0, -24) + 1e-44)) ++bad;
        }
        // an outlier forces the block onto the binary32 path
        if ((kind == 2 || kind == 3) && !zeros && !flag) ++bad;
    }
    if (blocks > 100 && flagged == 0) ++bad;
    return bad;
}

int q4_debug_check_tc(const int64_t* n, const int64_t* k, int count, int b) {
    using namespace q4t;
    if (!n || !k || count < 1 || count > Q4_MAX_GROUP || b < 2 || b > Q4_MAX_BATCH) return 1;
    Shape sh[Q4_MAX_GROUP];
    for (int i = 0; i < count; ++i) sh[i] = {n[i], k[i]};
    Params P;
    int64_t tickets = 0, end = 0;
    if (plan_tc(sh, count, b, INT64_MAX / 4, kRefSms, &P, &tickets, &end) != Q4_OK) return 2;
    const int64_t base = part_base_for(tickets);
    if (plan_tc(sh, count, b, base, kRefSms, &P, &tickets, &end) != Q4_OK) return 2;
    if (kSmemBytes > (int)q4h::kMaxSmem || 2 * kSmemBytes <= 228 * 1024) return 3;  // one CTA per SM
    if (P.grid < 1 || P.grid > kRefSms || P.grid > P.total) return 4;
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
                    if (t0 * 4 < q4h::kHeaderBytes || (t0 + 4) * 4 > base) return 16;
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
