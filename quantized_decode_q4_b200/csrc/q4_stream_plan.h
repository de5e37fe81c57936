// Work decomposition of the persistent batch-1 streaming GEMV kernel, shared by
// the device code and by the host replay in q4_debug_check_stream.
//
// A launch covers one dependency group (up to Q4_MAX_GROUP GEMVs). Its work is
// counted in rows of segments: segment (g, split) is K split `split` of every row
// of GEMV g. Segments are ordered (g, split) and their rows laid end to end in
// one "row space" of total_rows rows. CTA c owns rows [cta_lo[c], cta_lo[c + 1])
// of that space. The planner gives every segment whole CTAs when there are at
// least as many CTAs as segments (so no CTA stages the activations of two
// segments: such a CTA finishes last and the next launch waits for it), else
// cuts the row space into equal ranges. The part of a CTA's range inside one
// segment is a piece, and warp w of the CTA takes rows
// [len w / W, len (w + 1) / W) of each piece, so every warp of a CTA gets the
// same number of rows to within one. A warp walks its rows in tiles of up to
// kRows rows (x reuse) and streams each tile's code and scale bytes (every block
// of the split) through a private ring of kStages shared-memory stages.
#pragma once

#include <cstdint>

#include "../../include/q4.h"

#if defined(__CUDACC__)
#define Q4S_HD __host__ __device__ __forceinline__
#else
#define Q4S_HD inline
#endif

namespace q4s {

#ifndef Q4_STREAM_WARPS
#define Q4_STREAM_WARPS 16
#endif
#ifndef Q4_STREAM_MINB
#define Q4_STREAM_MINB 1  // CTAs per SM the registers must allow
#endif
#ifndef Q4_STREAM_STAGES
#define Q4_STREAM_STAGES 2
#endif
#ifndef Q4_STREAM_CTAS_PER_SM
#define Q4_STREAM_CTAS_PER_SM 1  // CTAs of one launch per SM
#endif
#ifndef Q4_STREAM_ROWS
#define Q4_STREAM_ROWS 2  // rows per tile
#endif

constexpr int kWarps = Q4_STREAM_WARPS;        // warps per CTA
constexpr int kThreads = kWarps * 32;
constexpr int kRows = Q4_STREAM_ROWS;           // rows per tile (x reuse per warp)
constexpr int kStages = Q4_STREAM_STAGES;       // ring depth per warp (one tile per stage)
constexpr int kMaxGrid = 148 * Q4_STREAM_CTAS_PER_SM;  // B200 SMs x CTAs of a launch per SM
constexpr int kMaxSplitBlocks = 128;            // K per split <= 4096
constexpr int kDSlot = kMaxSplitBlocks + 16;    // uint16 per scale row (per-row copies)
constexpr int kStageQs = kRows * kMaxSplitBlocks * 16;
constexpr int kStageD = kRows * kDSlot * 2 + 32;
constexpr int kStageBytes = kStageQs + kStageD;
constexpr int kBarBytes = ((kWarps * kStages * 8 + 127) / 128) * 128;
constexpr int kXBytes = kMaxSplitBlocks * 7 * 16;
constexpr int kSmemBytes = kBarBytes + kXBytes + kWarps * kStages * kStageBytes;

static_assert(kStageBytes % 16 == 0, "stages must keep 16-byte alignment");
static_assert(kMaxSplitBlocks % 32 == 0, "split size");

struct Desc {
    const uint8_t* qs;
    const uint16_t* d;
    const float* x;
    float* y;
    int64_t n;
    int32_t nb;           // k / 32
    int32_t splits;
    int32_t nb_split;     // blocks per split (the last split may be shorter)
    int32_t pad_;
    int64_t row_begin;    // first row of this GEMV's segments in the row space
    int64_t part_off;     // floats: partial sums [splits][n]
    int64_t ticket_off;   // uint32: one ticket per row
};

struct Params {
    Desc g[Q4_MAX_GROUP];
    int32_t count;
    uint32_t tx_extra;  // 0; test hook: bytes every stage waits for beyond its copies
    int64_t total_rows;
    uint32_t* ws;
    int32_t cta_lo[kMaxGrid + 1];  // CTA c owns rows [cta_lo[c], cta_lo[c + 1]) (< 2^31)
};

// One dependency group as the walks see it (Params has the same members).
struct View {
    const Desc* g;
    const int32_t* cta_lo;
    int32_t count;
    int64_t total_rows;
};

// Segment of a row-space index: GEMV g, split, row within the GEMV, and the end
// (exclusive, in row space) of the segment.
struct Where {
    int g, split;
    int64_t row, seg_end;
};

// The row space stays below 2^31 rows (checked by the planner), so this uses
// 32-bit division.
template <class PV>
Q4S_HD Where locate(const PV& P, int64_t r) {
    int g = 0;
    while (g + 1 < P.count && r >= P.g[g + 1].row_begin) ++g;
    const Desc& G = P.g[g];
    const uint32_t local = (uint32_t)(r - G.row_begin);
    const uint32_t n = (uint32_t)G.n;
    Where w;
    w.g = g;
    w.split = (int)(local / n);
    w.row = (int64_t)(local - (uint32_t)w.split * n);
    w.seg_end = G.row_begin + (int64_t)(w.split + 1) * G.n;
    return w;
}

Q4S_HD int split_blocks(const Desc& G, int split) {
    const int rest = G.nb - split * G.nb_split;
    return rest < G.nb_split ? rest : G.nb_split;
}

template <class PV>
Q4S_HD void cta_range(const PV& P, int cta, int64_t* lo, int64_t* hi) {
    *lo = P.cta_lo[cta];
    *hi = P.cta_lo[cta + 1];
}

// Rows [*a, *b) of a piece [p0, p1) that warp w takes.
Q4S_HD void warp_rows(int64_t p0, int64_t p1, int warp, int64_t* a, int64_t* b) {
    const uint32_t len = (uint32_t)(p1 - p0);
    *a = p0 + (int64_t)(len * (uint32_t)warp / (uint32_t)kWarps);
    *b = p0 + (int64_t)(len * (uint32_t)(warp + 1) / (uint32_t)kWarps);
}

// The copy lane `lane` issues for a tile of `rows` rows starting at row `row0`
// of GEMV G, split `split` (every block of the split). With one split the rows
// are contiguous in both planes: lane 0 copies all code bytes in one request and
// lane 8 the 16-byte aligned superset of all scales in another. With a split K,
// lane r copies the codes of row r and lane 8 + r the superset of its scales
// (into a slot of kDSlot entries). The d plane is padded to 16 bytes, so no
// superset leaves it.
struct LaneCopy {
    int64_t src_off;  // byte offset in the qs plane (lanes 0-7) or d plane (8-15)
    uint32_t dst;     // byte offset inside a stage
    uint32_t bytes;
    bool active;
    bool scales;      // true for a scale copy
};

Q4S_HD LaneCopy lane_copy(const Desc& G, int split, int64_t row0, int rows, int lane) {
    LaneCopy c;
    const int kbs = split_blocks(G, split);
    c.scales = lane >= 8;
    const int r = lane & 7;
    if (G.splits == 1) {
        c.active = lane == 0 || lane == 8;
        const int64_t e = row0 * G.nb;
        if (lane < 8) {
            c.src_off = e * 16;
            c.dst = 0;
            c.bytes = (uint32_t)rows * (uint32_t)kbs * 16u;
        } else {
            const int64_t a = e * 2, a0 = a & ~(int64_t)15;
            c.src_off = a0;
            c.dst = kStageQs;
            c.bytes = (uint32_t)(((a + 2 * (int64_t)rows * kbs + 15) & ~(int64_t)15) - a0);
        }
        return c;
    }
    c.active = lane < 16 && r < rows;
    const int64_t e = (row0 + r) * G.nb + (int64_t)split * G.nb_split;
    if (lane < 8) {
        c.src_off = e * 16;
        c.dst = (uint32_t)(r * kMaxSplitBlocks * 16);
        c.bytes = (uint32_t)kbs * 16u;
    } else {
        const int64_t a = e * 2, a0 = a & ~(int64_t)15;
        c.src_off = a0;
        c.dst = (uint32_t)(kStageQs + r * kDSlot * 2);
        c.bytes = (uint32_t)(((a + 2 * (int64_t)kbs + 15) & ~(int64_t)15) - a0);
    }
    return c;
}

// Where the math reads row r of the tile inside a stage: block j of the split is
// at qoff + 16 j (codes) and doff + 2 j (scale). Rows past the tile's end read
// its last row; their results are not stored.
Q4S_HD void row_read_offsets(const Desc& G, int split, int64_t row0, int rows, int r,
                             uint32_t* qoff, uint32_t* doff) {
    const int rr = r < rows ? r : rows - 1;
    const int kbs = split_blocks(G, split);
    if (G.splits == 1) {
        const int64_t a = row0 * G.nb * 2;
        *qoff = (uint32_t)(rr * kbs * 16);
        *doff = (uint32_t)(kStageQs + (a & 15) + rr * kbs * 2);
        return;
    }
    const int64_t e = (row0 + rr) * G.nb + (int64_t)split * G.nb_split;
    *qoff = (uint32_t)(rr * kMaxSplitBlocks * 16);
    *doff = (uint32_t)(kStageQs + (rr * kDSlot + (int)(e & 7)) * 2);
}

Q4S_HD uint32_t stage_offset(int warp, int stage) {
    return kBarBytes + kXBytes + (uint32_t)(warp * kStages + stage) * kStageBytes;
}

// Staged activations, in 24-bit block fixed point: for block j of the split,
// seven 16-byte entries t = 0..6: digit words 0-3 and 4-7 of digit planes a, b,
// c (t = 2 p + half) and the block constants (-8 sum a, -8 sum b, -8 sum c,
// scale). Entry (j, t) sits at uint4 index [j/32][t][j%32], so that the 32
// lanes of a warp read 32 consecutive entries for a given t.
constexpr int kXEntries = 7;
Q4S_HD int xq_slot(int j, int t) { return (((j >> 5) * kXEntries + t) << 5) + (j & 31); }

// Walk of one warp over its rows, shared by the copy issuer and the math loop:
// the pieces of the CTA range in order, and in each piece this warp's rows.
struct Walk {
    int64_t pos, hi;          // next row-space index of the CTA range, range end
    int64_t wr, wend;         // this warp's rows [wr, wend) of the current segment
    int g, split;             // current segment
    int warp;

    Q4S_HD void begin(int64_t lo, int64_t hi_, int w) {
        pos = lo;
        hi = hi_;
        wr = wend = 0;
        warp = w;
        g = split = 0;
    }

    // advance to the next piece that gives this warp at least one row
    template <class PV>
    Q4S_HD bool next_piece(const PV& P) {
        while (pos < hi) {
            const Where w = locate(P, pos);
            const int64_t p1 = w.seg_end < hi ? w.seg_end : hi;
            const int64_t seg_row0 = pos - w.row;
            g = w.g;
            split = w.split;
            int64_t a, b;
            warp_rows(pos, p1, warp, &a, &b);
            pos = p1;
            if (a < b) {
                wr = a - seg_row0;
                wend = b - seg_row0;
                return true;
            }
        }
        return false;
    }
};

}  // namespace q4s
