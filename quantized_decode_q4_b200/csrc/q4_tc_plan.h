// Work decomposition and shared-memory / tensor-memory layout of the batched
// (2..16 tokens) tensor-core GEMV, shared by the device code and by the host
// replay in q4_debug_check_tc.
//
// A launch covers one dependency group (up to Q4_MAX_GROUP GEMVs). The unit of
// work is one K block (32 weights) of one M tile (128 rows) of one GEMV. Units
// are ordered (GEMV, tile, block) and laid end to end in one "flat" space of F
// units; CTA c of G owns units [F c / G, F (c + 1) / G). The part of a CTA's
// range inside one tile is a piece; a piece is walked in stages that never
// cross a multiple of kS blocks, so that every stage lies inside one aligned
// group of kS blocks (the "window" [w0, w0 + kS), w0 = kb0 - kb0 % kS) and
// every TMA box of a stage starts at a 16-byte aligned coordinate. A tile
// covered by several pieces (several CTAs) is finished by the last one to
// arrive: each piece stores its 128 x b partial sums in its own slot (slot =
// CTA index - first CTA of the tile), and the last arriver adds the slots in
// order (deterministic).
//
// Per stage, shared memory holds:
//   codes   the window's code bytes, one TMA box of 128 B x 128 rows with the
//           128-byte swizzle: block c of the window, row r at
//           r * 128 + ((c ^ (r % 8)) * 16)
//   xraw    the window's activations, one TMA box of 256 binary32 x 16 tokens
//           (token t at t * 1024 bytes; absent tokens read as zero)
//   xop     the stage's activations as the MMA's B operand: bf16 hi and lo parts
//           in the canonical K-major layout without swizzle (8 x 16-byte core
//           matrices), written by the x warps from xraw
//   d       the window's binary16 scales: one TMA box of 8 x 128 rows
//           ([r][8]) when the row stride of the scale plane is a multiple of 16
//           bytes, else one 16-byte aligned bulk copy per row into a 32-byte
//           slot per row (the stage's scales at an offset inside it)
//
// Tensor memory (512 columns x 128 lanes) holds two rings, both in quads of
// kQ = 4 blocks (a stage is one or two quads): the A ring, kRingA quads of
// 4 x 16 columns (row r = lane r, a block's 32 values (q - 8) as bf16 pairs),
// freed as soon as the quad's MMAs complete; and the D ring, ring_d quads of
// 4 x N columns (each block's accumulator, 128 x N binary32), freed when the
// epilogue has read it. N = 16 up to 8 tokens (hi parts of token t in column
// t, lo parts in 8 + t), N = 32 above (hi in t, lo in 16 + t): one MMA per
// 16-value chunk and block either way, since an MMA's cost does not grow with
// N up to 256.
#pragma once

#include <cuda.h>
#include <cstdint>

#include "../../include/q4.h"

#if defined(__CUDACC__)
#define Q4T_HD __host__ __device__ __forceinline__
#else
#define Q4T_HD inline
#endif

namespace q4t {

constexpr int kM = 128;        // rows per tile (MMA M)
constexpr int kS = 8;          // K blocks per window (and at most per stage)
constexpr int kQ = 4;          // blocks per tensor-memory quad
constexpr int kStages = 4;     // shared-memory ring depth
constexpr int kACols = 16;     // tensor-memory columns of one block's A operand
constexpr int kRingA = 4;      // A quads
constexpr int kTmemCols = 512;
constexpr int kMaxTokens = 16;
constexpr int kCodesBytes = kM * 128;               // 16 KB
constexpr int kXRawBytes = kMaxTokens * kS * 32 * 4;  // 16 KB
constexpr int kBlockXBytes = 2048;                  // 2 chunks x 32 rows x 32 B
constexpr int kXOpBytes = kS * kBlockXBytes;        // 16 KB
constexpr int kDSlot = 32;                          // bytes per row (per-row copies)
constexpr int kDBytes = kM * kDSlot;                // 4 KB
constexpr int kStageBytes = kCodesBytes + kXRawBytes + kXOpBytes + kDBytes;
constexpr int kHeaderBytes = 1024;  // barriers, tensor-memory address, abort flag
constexpr int kSmemBytes = kHeaderBytes + kStages * kStageBytes;

// warp roles: warps 0-3 and 8-11 prepare the operands (two per tensor-memory lane
// quarter: warp w reaches lanes 32 (w % 4) .. 32 (w % 4) + 31; the warps of half
// w / 8 dequantise the blocks of a quad with block % 2 == w / 8, and all eight
// share the stage's activations)
constexpr int kPrepWarps = 8;
constexpr int kEpiWarp0 = 4;      // 4 warps: accumulators x scale, partial sums, y
constexpr int kProdWarp = 12;     // TMA loads (lane 0) and per-row scale copies (all lanes)
constexpr int kMmaWarp0 = 13;     // 2 warps, one thread each: tcgen05.mma issue, quads
                                  // alternating between them
constexpr int kMmaIssuers = 2;
constexpr int kWarps = 15;
constexpr int kThreads = kWarps * 32;

static_assert(kStageBytes % 1024 == 0, "stages keep the 1024-byte alignment of the swizzled box");
static_assert(kS == 2 * kQ, "a stage is one or two quads");

// MMA N, D quads, and tensor-memory columns for a launch compiled for BT tokens.
Q4T_HD constexpr int mma_n(int bt) { return bt <= 8 ? 16 : 32; }
Q4T_HD constexpr int ring_d(int bt) { return (kTmemCols - kRingA * kQ * kACols) / (kQ * mma_n(bt)); }
Q4T_HD constexpr uint32_t a_col(int slot, int i) { return (uint32_t)((slot * kQ + i) * kACols); }
Q4T_HD constexpr uint32_t d_col(int bt, int slot, int i) {
    return (uint32_t)(kRingA * kQ * kACols + (slot * kQ + i) * mma_n(bt));
}
static_assert(ring_d(2) == 4 && ring_d(16) == 2, "tensor-memory rings");

// barrier indices (uint64 words at the start of shared memory)
constexpr int kMaxRingD = 4;
constexpr int kBarFull = 0;                          // [kStages] every TMA byte of the stage
constexpr int kBarXOpFull = kBarFull + kStages;      // [kStages] B operands written
constexpr int kBarStageEmpty = kBarXOpFull + kStages;  // [kStages]
constexpr int kBarAFull = kBarStageEmpty + kStages;  // [kRingA] A quad written
constexpr int kBarAEmpty = kBarAFull + kRingA;       // [kRingA] A quad's MMAs done
constexpr int kBarDFull = kBarAEmpty + kRingA;       // [kMaxRingD] D quad's MMAs done
constexpr int kBarDEmpty = kBarDFull + kMaxRingD;    // [kMaxRingD] D quad read
constexpr int kBarDone = kBarDEmpty + kMaxRingD;     // 1
constexpr int kNumBars = kBarDone + 1;
constexpr int kTmemAddrOff = 8 * kNumBars;  // uint32 written by tcgen05.alloc
constexpr int kAbortOff = kTmemAddrOff + 4;  // int32 abort flag
static_assert(kAbortOff + 4 <= kHeaderBytes, "header");

// arrivals per barrier phase
constexpr uint32_t kArrivalsStageEmpty = kPrepWarps + 4 + kMmaIssuers;  // operand and
                                                                       // epilogue warps,
                                                                       // MMA issuers
constexpr uint32_t kArrivalsXOpFull = kPrepWarps;
constexpr uint32_t kArrivalsAFull = kPrepWarps;
constexpr uint32_t kArrivalsDEmpty = 4;

Q4T_HD uint32_t stage_base(int st) { return (uint32_t)(kHeaderBytes + st * kStageBytes); }
Q4T_HD uint32_t stage_codes(int st) { return stage_base(st); }
Q4T_HD uint32_t stage_xraw(int st) { return stage_base(st) + kCodesBytes; }
Q4T_HD uint32_t stage_xop(int st) { return stage_base(st) + kCodesBytes + kXRawBytes; }
Q4T_HD uint32_t stage_d(int st) { return stage_base(st) + kCodesBytes + kXRawBytes + kXOpBytes; }

// Code bytes of block c (0..kS-1) of the window, row r, inside the swizzled box.
Q4T_HD uint32_t code_off(int r, int c) { return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4)); }

// Byte offset, inside a stage's operand region, of the N x 16 bf16 B operand
// of chunk c2 (16 K values) of stage block i, and of the 16-byte row holding
// its MMA positions [8 hh, 8 hh + 8) for token t, part hl (0 = hi, 1 = lo):
// operand row t (hi) or N / 2 + t (lo). Inside an operand: core matrix (row
// group g = row / 8, K half hh) at hh * LBO + g * 128 with LBO = N * 16, row
// r % 8 at 16 (r % 8).
constexpr uint32_t kSBO = 128;  // between 8-row groups
Q4T_HD uint32_t lbo(int n) { return (uint32_t)(n * 16); }
Q4T_HD uint32_t x_operand_off(int n, int i, int c2) { return (uint32_t)((2 * i + c2) * n * 32); }
Q4T_HD uint32_t x_row_off(int n, int i, int c2, int hh, int t, int hl) {
    const int row = hl ? n / 2 + t : t;
    return x_operand_off(n, i, c2) + (uint32_t)hh * lbo(n) + (uint32_t)((row >> 3) * kSBO) +
           (uint32_t)((row & 7) * 16);
}

// Element of a block (0..31) at MMA position kappa (0..31) of the A and B
// operands. The dequant writes tensor-memory column c = kappa / 2 (half
// kappa % 2) of a block from its code bytes as: column 2 i + s of chunk h2
// (= columns 8 h2 + 2 i + s) holds the nibble h2 (low / high) of bytes
// 4 i + s (low half) and 4 i + s + 2 (high half). So element
// 16 h2 + 4 i + s + 2 h sits at position 16 h2 + 4 i + 2 s + h.
Q4T_HD int element_at(int kappa) {
    const int h2 = kappa >> 4, i = (kappa >> 2) & 3, s = (kappa >> 1) & 1, h = kappa & 1;
    return 16 * h2 + 4 * i + s + 2 * h;
}

// tcgen05.mma instruction descriptor: kind::f16, A and B bf16, D binary32,
// both K-major, M = 128, N = n.
Q4T_HD constexpr uint32_t instr_desc(int n) {
    return (1u << 4)      // D format F32
           | (1u << 7)    // A format BF16
           | (1u << 10)   // B format BF16
           | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(kM >> 4) << 24);
}

// Shared-memory matrix descriptor of one n x 16 bf16 B operand at byte address
// `addr` (canonical K-major layout, no swizzle).
Q4T_HD uint64_t smem_desc(uint32_t addr, int n) {
    return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo(n) >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((kSBO >> 4) & 0x3FFFu) << 32) | ((uint64_t)1 << 46);
}

struct Desc {
    const uint8_t* qs;
    const uint16_t* d;
    const float* x;
    float* y;
    int64_t n;
    int32_t nb;          // k / 32
    int32_t tiles;       // ceil(n / 128)
    int64_t flat_begin;  // first unit of this GEMV in the flat space
    int64_t part_off;    // floats: partial sums [tiles][maxp][b][128]
    int64_t ticket_off;  // uint32: four tickets per tile (one per epilogue warp)
    int32_t maxp;        // partial slots per tile (1: no split tiles)
    int32_t d_box;       // 1: scales by one TMA box per stage (nb % 8 == 0)
};

// Tensor maps of GEMV g: codes uint8 [n][k/2] (box 128 x 128, 128-byte swizzle),
// activations binary32 [b][k] (box 256 x 16), scales uint16 [n][nb] (box 8 x 128,
// only when d_box).
struct Maps {
    CUtensorMap codes, x, d;
};

struct Params {
    Maps maps[Q4_MAX_GROUP];
    Desc g[Q4_MAX_GROUP];
    int32_t count;
    int32_t b;      // tokens
    int64_t total;  // F, < 2^31
    int32_t grid;   // G
    uint32_t tx_extra;  // 0; test hook: bytes every stage waits for beyond its copies
    uint32_t* ws;
};

// CTA owning flat unit f.
Q4T_HD int owner(int64_t f, int64_t F, int G) { return (int)(((f + 1) * G - 1) / F); }

Q4T_HD void cta_range(int64_t F, int c, int G, int64_t* lo, int64_t* hi) {
    *lo = F * c / G;
    *hi = F * (c + 1) / G;
}

// One stage of a CTA's walk.
struct Stage {
    int g;
    int32_t tile;
    int32_t kb0;    // first block
    int32_t nblk;   // blocks (1..kS), all inside the window of kb0
    bool first;     // first stage of a piece
    bool last;      // last stage of a piece
};

Q4T_HD int32_t window_of(int32_t kb0) { return kb0 - kb0 % kS; }

struct Walk {
    int64_t pos, hi;
    bool fresh;

    Q4T_HD void begin(int64_t lo, int64_t hi_) {
        pos = lo;
        hi = hi_;
        fresh = true;
    }

    Q4T_HD bool next(const Params& P, Stage* s) {
        if (pos >= hi) return false;
        int g = 0;
        while (g + 1 < P.count && pos >= P.g[g + 1].flat_begin) ++g;
        const Desc& G = P.g[g];
        const uint32_t local = (uint32_t)(pos - G.flat_begin);
        const uint32_t nb = (uint32_t)G.nb;
        const uint32_t tile = local / nb;
        const int32_t kb = (int32_t)(local - tile * nb);
        const int64_t tile_end = G.flat_begin + (int64_t)(tile + 1) * nb;
        const int64_t pend = tile_end < hi ? tile_end : hi;
        const int64_t left = pend - pos;
        const int32_t room = kS - kb % kS;
        s->g = g;
        s->tile = (int32_t)tile;
        s->kb0 = kb;
        s->nblk = (int32_t)(left < room ? left : room);
        s->first = fresh;
        s->last = pos + s->nblk == pend;
        pos += s->nblk;
        fresh = s->last;
        return true;
    }
};

// Pieces of tile `tile` of GEMV G and the slot of CTA c among them.
Q4T_HD void tile_pieces(const Params& P, const Desc& G, int32_t tile, int c, int* np, int* slot) {
    const int64_t f0 = G.flat_begin + (int64_t)tile * G.nb;
    const int64_t f1 = f0 + G.nb - 1;
    const int c0 = owner(f0, P.total, P.grid), c1 = owner(f1, P.total, P.grid);
    *np = c1 - c0 + 1;
    *slot = c - c0;
}

// Per-row scale copy of row r of a stage (when the scales are not one box):
// the 16-byte aligned superset of the stage's scales, and where the scale of
// stage block i lands: slot r, byte (src_off % 16) + 2 i.
struct DCopy {
    int64_t src_off;  // byte offset in the scale plane (16-byte aligned)
    uint32_t bytes;   // 16 or 32
    uint32_t lead;    // (first scale's byte offset) % 16
};
Q4T_HD DCopy d_copy(const Desc& G, int32_t tile, int32_t kb0, int32_t nblk, int r) {
    const int64_t a = (((int64_t)tile * kM + r) * G.nb + kb0) * 2;
    const int64_t a0 = a & ~(int64_t)15;
    DCopy c;
    c.src_off = a0;
    c.lead = (uint32_t)(a - a0);
    c.bytes = (uint32_t)(((a + 2 * nblk + 15) & ~(int64_t)15) - a0);
    return c;
}

}  // namespace q4t
