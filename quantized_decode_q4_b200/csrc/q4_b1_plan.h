// Work decomposition of the batch-1 decode mat-vec kernel, shared by the device
// code and by the host replay in q4_debug_check_b1.
//
// A launch covers one dependency group (up to Q4_MAX_GROUP GEMVs). Its work is
// cut into pieces, one per CTA: GEMV g owns pieces [piece_begin, piece_begin +
// splits * cps), piece piece_begin + j * splits + split being row range j of
// the cps ranges of K split `split` (see piece_of). K is split into ranges of at
// most a few slices of 32 blocks (1024 weights, one block per lane), so that the
// activations a piece stages stay small next to its weights. Within a piece, K
// is walked in slices and rows in tiles of 8: unit
// u = t * S + s is tile t, slice s of the piece's S slices (tile-major, so a
// consumer warp that takes every 8th unit keeps one slice when S divides 8).
//
// Per CTA: eight warps take units round-robin (unit u by warp u % 8). Every
// unit's code bytes and binary16 scales come from HBM into ring slot u % slots
// on the TMA engine, two 2-D tensor loads per unit (8 rows x 512 code bytes; 8
// rows x 32 scales) completing on the slot's mbarrier (a scale plane whose row
// stride is not a multiple of 16 bytes is copied row by row instead); the first
// `slots` units are requested at kernel entry, and each warp, once it has read
// unit u, requests unit u + slots into the slot it just freed. Warps multiply
// units with the piece's activations (staged once per piece in shared memory)
// and write per-(row, slice) partial sums to shared memory; after the last unit
// the CTA adds each row's slices in slice order and stores y (or a split-K
// partial; the last piece of a row range to arrive adds the range's partials up
// in split order). For 1 and 2 tokens a launch has one piece per SM although two
// CTAs fit: the SM's other CTA slot takes the next launch's CTA, which streams
// its first units in while this one computes (measured 6% faster than two pieces
// per SM for one token).
#pragma once

#include <cuda.h>

#include <cstdint>

#include "../../include/q4.h"

#if defined(__CUDACC__)
#define Q4B_HD __host__ __device__ __forceinline__
#define Q4B_HD_CONST __host__ __device__ constexpr
#else
#define Q4B_HD inline
#define Q4B_HD_CONST constexpr
#endif

namespace q4b {

#ifndef Q4B_WARPS
#define Q4B_WARPS 8  // warps per CTA
#endif
#ifndef Q4B_CTAS_PER_SM
#define Q4B_CTAS_PER_SM 2  // CTAs of consecutive launches sharing an SM (1 and 2 tokens)
#endif
constexpr int kWarps = Q4B_WARPS;
constexpr int kThreads = kWarps * 32;
constexpr int kCtasPerSm = Q4B_CTAS_PER_SM;
// Tokens one launch of this kernel multiplies, at most (one pass over the weights).
#ifndef Q4B_MAX_TOKENS
#define Q4B_MAX_TOKENS 4
#endif
constexpr int kMaxTokens = Q4B_MAX_TOKENS;
// CTAs per SM for b tokens: three and four tokens keep 32 b activation values per
// lane in registers, which takes the register file of a whole SM.
Q4B_HD_CONST int ctas_per_sm(int b) { return b <= 2 ? kCtasPerSm : 1; }
constexpr int kTileRows = 8;                  // rows per unit
constexpr int kSliceBlocks = 32;              // blocks per unit (one per lane)
constexpr int kSlotQs = kTileRows * kSliceBlocks * 16;  // code bytes of a unit
constexpr int kDRow = 80;                     // scale bytes per row in a slot (64 + alignment slack)
constexpr int kDMapRow = 64;                  // scale bytes per row when loaded by the tensor map
constexpr int kSlotBytes = kSlotQs + kTileRows * kDRow;
constexpr int kXBlockBytes = 144;             // staged activation block (1 token): 32 digit words + 4 words
constexpr int kXChunks = kXBlockBytes / 16;   // 16-byte chunks per staged block
constexpr int kXSliceBytes = kSliceBlocks * kXBlockBytes;
constexpr int kXFSliceBytes = kSliceBlocks * 128;  // one token's slice in binary32 (2..4 tokens)
// Slices of one piece, at most (its activations are staged whole, and must leave
// room for the weight ring). Fewer slices mean less activation staging per piece
// but a split-K reduction at the end; four measured fastest.
#ifndef Q4B_PIECE_SLICES
#define Q4B_PIECE_SLICES 4
#endif
constexpr int kPieceSlices = Q4B_PIECE_SLICES;
constexpr int kMaxSlices = 14;
static_assert(kPieceSlices >= 1 && kPieceSlices <= kMaxSlices, "slices per piece");
// Ring slots: a multiple of kWarps, so that every unit routed to a slot
// (u = slot mod slots) belongs to the same warp, which both requests and waits
// for it: the warp is never more than one phase ahead of the slot's barrier,
// which a parity wait requires.
// Pieces (CTAs) of one launch per multiprocessor (at most as many as fit at once).
#ifndef Q4B_PIECES_PER_SM
#define Q4B_PIECES_PER_SM 1
#endif
Q4B_HD_CONST int pieces_per_sm(int b) { return ctas_per_sm(b) == 2 ? Q4B_PIECES_PER_SM : 1; }
Q4B_HD_CONST int max_slots(int b) { return 48 / ctas_per_sm(b) / kWarps * kWarps; }
constexpr int kMaxSlots = 48 / kWarps * kWarps;  // over every token count
constexpr int kMinSlots = kWarps;
constexpr int kBarBytes = (kMaxSlots * 8 + 127) / 128 * 128;  // full[] barriers, padded
// Shared memory of one CTA: two CTAs of consecutive launches share an SM.
Q4B_HD_CONST int smem_budget(int b) { return (ctas_per_sm(b) == 2 ? 113 : 226) * 1024; }

static_assert(kSlotBytes % 128 == 0, "slots keep 128-byte alignment");
static_assert(kMaxSlots * 8 <= kBarBytes && kBarBytes % 128 == 0, "barrier region");
static_assert(kMaxSlots % kWarps == 0 && kMinSlots % kWarps == 0, "slots per warp");
static_assert(kXSliceBytes % 16 == 0, "staged slices keep 16-byte alignment");
static_assert(kCtasPerSm == 1 || kCtasPerSm == 2, "one or two CTAs per SM");

struct Desc {
    const uint8_t* qs;
    const uint16_t* d;
    const float* x;
    float* y;
    int64_t n;
    int32_t nb;                // k / 32
    int32_t nslices;           // ceil(nb / 32)
    int32_t splits;            // K splits across CTAs
    int32_t slices_per_split;  // slices of the widest split
    int32_t piece_begin;       // first piece (CTA) of this GEMV
    int32_t cps;               // pieces (CTAs) per split
    int32_t d_map;             // 1: scales loaded by the tensor map (row stride % 16 == 0)
    int32_t pad_;
    int64_t part_off;          // floats: split-K partial sums [splits][n]
    int64_t ticket_off;        // uint32: n words reserved; row range j (piece j of each split) uses word j
};

struct Piece {
    int32_t g, split;
    int32_t j;                 // index within the split: pieces j of all splits share rows
    int32_t r0, r1;            // rows of GEMV g (< 2^31)
};

struct Params {
    // code plane as uint32 [n][k/8], box 128 x 8 rows; scale plane uint16
    // [n][k/32], box 32 x 8 rows (used when Desc::d_map is set)
    CUtensorMap qs_map[Q4_MAX_GROUP];
    CUtensorMap d_map[Q4_MAX_GROUP];
    Desc g[Q4_MAX_GROUP];
    int32_t count;
    int32_t slots;             // ring slots of this launch
    uint32_t red_bytes;        // shared memory for per-(row, slice) partial sums
    uint32_t x_bytes;          // shared memory for the staged activations
    uint32_t tx_extra;         // 0; test hook: bytes every slot waits for beyond its copies
    int32_t npieces;
    int32_t b;                 // tokens (1 .. kMaxTokens); x [b][k], y [b][n]
    int32_t max_slices;        // slices of the largest piece (staging stride of a token)
    uint32_t* ws;
};

// First row of row range j of the cps equal ranges of n rows.
Q4B_HD int64_t range_start(int64_t n, int64_t cps, int64_t j) { return n * j / cps; }

// Piece c of a launch. A GEMV's pieces are ordered row range first: piece
// piece_begin + j * splits + split covers row range j of K split `split`, so the
// pieces of one row range (one ticket) start together.
template <class PP>
Q4B_HD Piece piece_of(const PP& P, int c) {
    int g = 0;
    while (g + 1 < P.count && c >= P.g[g + 1].piece_begin) ++g;
    const Desc& G = P.g[g];
    const int local = c - G.piece_begin;
    Piece p;
    p.g = g;
    const int j = local / G.splits;
    p.split = local - j * G.splits;
    p.j = j;
    p.r0 = (int32_t)range_start(G.n, G.cps, j);
    p.r1 = (int32_t)range_start(G.n, G.cps, j + 1);
    return p;
}

Q4B_HD uint32_t smem_bytes(const Params& P) {
    return (uint32_t)kBarBytes + P.red_bytes + P.x_bytes + (uint32_t)P.slots * kSlotBytes;
}
Q4B_HD uint32_t red_offset() { return (uint32_t)kBarBytes; }
Q4B_HD uint32_t x_offset(const Params& P) { return (uint32_t)kBarBytes + P.red_bytes; }
Q4B_HD uint32_t ring_offset(const Params& P) { return (uint32_t)kBarBytes + P.red_bytes + P.x_bytes; }

// Slices of a piece: first global slice and count.
// Splits cover nslices * split / splits .. nslices * (split + 1) / splits: as
// even as whole slices allow (at most slices_per_split = ceil(nslices / splits)).
Q4B_HD void piece_slices(const Desc& G, int split, int* s0, int* S) {
    *s0 = (int)((int64_t)G.nslices * split / G.splits);
    *S = (int)((int64_t)G.nslices * (split + 1) / G.splits) - *s0;
}

// Blocks of global slice gs (32, or fewer in the last slice).
Q4B_HD int slice_blocks(const Desc& G, int gs) {
    const int rest = G.nb - gs * kSliceBlocks;
    return rest < kSliceBlocks ? rest : kSliceBlocks;
}

Q4B_HD int piece_tiles(const Piece& p) { return (p.r1 - p.r0 + kTileRows - 1) / kTileRows; }

// Bytes one unit brings into its slot through the tensor maps: all 8 rows of the
// box, rows and blocks past the ends read as zero.
constexpr uint32_t kMapCodeBytes = kSlotQs;
constexpr uint32_t kMapScaleBytes = kTileRows * kDMapRow;

// The per-row copy lane `lane` of the producer issues for unit (tile t, global
// slice gs) of a piece when the scales cannot use the tensor map: lanes 8..15 the
// 16-byte aligned superset of row r = lane - 8's scales (the d plane is padded
// to 16 bytes, so a superset never leaves it). Lanes 0..7 describe the code
// bytes of row r = lane (loaded by the tensor map; the replay checks them).
struct LaneCopy {
    int64_t src_off;  // byte offset in the qs plane (code copy) or the d plane
    uint32_t dst;     // byte offset inside a slot
    uint32_t bytes;
    bool active;
    bool scales;
};

Q4B_HD LaneCopy lane_copy(const Desc& G, const Piece& p, int t, int gs, int lane) {
    LaneCopy c;
    const int r = lane & 7;
    const int64_t row = (int64_t)p.r0 + (int64_t)t * kTileRows + r;
    const int bs = slice_blocks(G, gs);
    c.scales = lane >= 8;
    c.active = lane < 16 && row < p.r1;
    const int64_t e = row * G.nb + (int64_t)gs * kSliceBlocks;  // first block of the copy
    if (!c.scales) {
        c.src_off = e * 16;
        c.dst = (uint32_t)(r * kSliceBlocks * 16);
        c.bytes = (uint32_t)bs * 16u;
    } else {
        const int64_t a = e * 2, a0 = a & ~(int64_t)15;
        c.src_off = a0;
        c.dst = (uint32_t)(kSlotQs + r * kDRow);
        c.bytes = (uint32_t)(((a + 2 * (int64_t)bs + 15) & ~(int64_t)15) - a0);
    }
    return c;
}

// Byte offset, inside a slot, of the scale of block `lane` of row r of the unit.
Q4B_HD uint32_t scale_offset(const Desc& G, const Piece& p, int t, int gs, int r, int lane) {
    if (G.d_map) return (uint32_t)(kSlotQs + r * kDMapRow + 2 * lane);
    const int64_t row = (int64_t)p.r0 + (int64_t)t * kTileRows + r;
    const int64_t a = (row * G.nb + (int64_t)gs * kSliceBlocks) * 2;
    return (uint32_t)(kSlotQs + r * kDRow + (int)(a & 15) + 2 * lane);
}

// Staged activations of tokens 2..4: chunk c (values 4c .. 4c+3) of block j of
// local slice s of token t, binary32, at x_offset + (((s * b + t) * 8 + c) * 32 +
// j) * 16 (the 32 lanes of a warp read 32 consecutive chunks).
Q4B_HD uint32_t xfchunk_offset(int s, int t, int b, int c, int j) {
    return (uint32_t)((((s * b + t) * 8 + c) * kSliceBlocks + j) * 16);
}

// Staged activation block j of local slice s: chunk q (0..8) of 16 bytes at
// x_offset + ((s * 9 + q) * 32 + j) * 16, so that the 32 lanes of a warp read 32
// consecutive chunks. Chunks 0-3: digit plane 0 words 0-15; chunks 4-7: plane 1;
// chunk 8: (c0, c1, scale bits, flag).
Q4B_HD uint32_t xchunk_offset(int s, int q, int j) {
    return (uint32_t)(((s * kXChunks + q) * kSliceBlocks + j) * 16);
}

}  // namespace q4b
