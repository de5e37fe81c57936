// Work decomposition of the Q4_0 GEMV kernels, shared by the device code and by
// the host-side validator that replays every copy and shared-memory offset of a
// launch on the CPU (q4_debug_check_plan) before the kernels ever run.
//
// A launch covers one dependency group: up to Q4_MAX_GROUP independent GEMVs.
// Each CTA processes one unit = (GEMV, row tile, K split). A row tile is
// kRowsPerCta consecutive rows; warp w of the CTA owns rows w*kRowsPerWarp ..
// +kRowsPerWarp-1 of it. A K split is nb_split consecutive blocks of 32.
// Every warp streams its rows' codes and scales into shared memory with bulk
// copies, then computes its rows' dot products over the split.
#pragma once

#include <cstdint>

#include "../../include/q4.h"

#if defined(__CUDACC__)
#define Q4_HD __host__ __device__ __forceinline__
#else
#define Q4_HD inline
#endif

namespace q4plan {

constexpr int kWarps = 4;                         // warps per CTA
constexpr int kThreads = kWarps * 32;
constexpr int kRowsPerWarp = 4;                   // rows per warp (x reuse)
constexpr int kRowsPerCta = kWarps * kRowsPerWarp;
#ifndef Q4_MAX_BLOCKS_PER_SPLIT
#define Q4_MAX_BLOCKS_PER_SPLIT 128
#endif
constexpr int kMaxBlocksPerSplit = Q4_MAX_BLOCKS_PER_SPLIT;  // K per split (blocks of 32)
constexpr int kHeaderBytes = 256;                 // workspace status header
constexpr int kBarrierBytes = 128;                // mbarriers at the start of smem

struct GemvDesc {
    const uint8_t* qs;
    const uint16_t* d;
    const float* x;      // [batch][k]
    float* y;            // [batch][n]
    int64_t n;
    int32_t nb;          // k / 32
    int32_t splits;      // K splits
    int32_t nb_split;    // blocks per split (the last split may be shorter)
    int32_t row_tiles;   // ceil(n / kRowsPerCta)
    int32_t unit_begin;  // first unit of this GEMV in the launch
    int32_t pad_;
    int64_t part_off;    // floats: partial sums [batch][splits][n] in the workspace
    int64_t ticket_off;  // uint32: split-K tickets [row_tiles] in the workspace
};

struct GemvParams {
    GemvDesc g[Q4_MAX_GROUP];
    int32_t count;
    int32_t total_units;
    int32_t batch;
    uint32_t smem_x;        // bytes of staged activations
    uint32_t smem_qs_warp;  // bytes of code rows per warp
    uint32_t smem_d_warp;   // bytes of scale rows per warp
    uint32_t d_slot;        // uint16 entries per scale row slot
    uint32_t smem_total;
    uint32_t* ws;           // workspace base (256-byte aligned)
};

struct Unit {
    int g;       // GEMV index in the launch
    int tile;    // row tile
    int split;   // K split
};

Q4_HD Unit unit_of(const GemvParams& P, int unit) {
    int g = 0;
    while (g + 1 < P.count && unit >= P.g[g + 1].unit_begin) ++g;
    const int local = unit - P.g[g].unit_begin;
    Unit u;
    u.g = g;
    u.tile = local / P.g[g].splits;
    u.split = local % P.g[g].splits;
    return u;
}

Q4_HD int split_blocks(const GemvDesc& G, int split) {
    const int kb0 = split * G.nb_split;
    const int rest = G.nb - kb0;
    return rest < G.nb_split ? rest : G.nb_split;
}

// Rows of the warp that exist (0 .. kRowsPerWarp).
Q4_HD int warp_rows(const GemvDesc& G, int tile, int warp) {
    const int64_t row0 = (int64_t)tile * kRowsPerCta + (int64_t)warp * kRowsPerWarp;
    const int64_t left = G.n - row0;
    return left <= 0 ? 0 : (left < kRowsPerWarp ? (int)left : kRowsPerWarp);
}

// Code bytes of (row, split): a contiguous, 16-byte aligned range of the qs plane.
Q4_HD int64_t qs_src_offset(const GemvDesc& G, int64_t row, int split) {
    return (row * G.nb + (int64_t)split * G.nb_split) * 16;
}

// Scale bytes of (row, split) are [a, a + 2*blocks). The copy takes the 16-byte
// aligned superset [a & ~15, (a + 2*blocks + 15) & ~15); the d plane is padded
// to a multiple of 16 bytes, so the superset never leaves it. `shift` is the
// index of the first wanted scale inside the copied range.
struct DRange {
    int64_t src;     // byte offset in the d plane
    uint32_t bytes;  // multiple of 16
    uint32_t shift;  // uint16 entries
};

Q4_HD DRange d_range(const GemvDesc& G, int64_t row, int split, int blocks) {
    const int64_t a = (row * G.nb + (int64_t)split * G.nb_split) * 2;
    const int64_t b = a + 2 * (int64_t)blocks;
    DRange r;
    r.src = a & ~(int64_t)15;
    r.bytes = (uint32_t)(((b + 15) & ~(int64_t)15) - r.src);
    r.shift = (uint32_t)((a - r.src) / 2);
    return r;
}

// Shared memory layout of a CTA: [barriers][x staging][warp 0 codes|scales]...
Q4_HD uint32_t smem_x_offset() { return kBarrierBytes; }
Q4_HD uint32_t smem_warp_offset(const GemvParams& P, int warp) {
    return kBarrierBytes + P.smem_x + (uint32_t)warp * (P.smem_qs_warp + P.smem_d_warp);
}

// Position (in float4 units) of chunk i (x[4i..4i+3] of block j of the split)
// in the batch-1 staging layout: [iteration j/32][chunk i][lane j%32], so that the
// 32 lanes of a warp read 32 consecutive float4 for a given chunk.
Q4_HD int x_slot_b1(int j, int i) { return (((j >> 5) * 8 + i) << 5) + (j & 31); }

// Batched staging layout (per token): lane (j % 8) * 4 + w of an 8-block
// iteration handles code word w of block j and reads chunks w and w + 4, so the
// layout is [iteration j/8][half i/4][block j%8][word i%4]: for a given half,
// the 32 lanes read 32 consecutive float4.
Q4_HD int x_slot_bs(int j, int i) {
    return ((((j >> 3) << 1) + (i >> 2)) << 5) + ((j & 7) << 2) + (i & 3);
}
// float4 slots per token in the batched layout.
Q4_HD int x_token_slots_bs(int nb_split) { return ((nb_split + 7) >> 3) * 64; }

// Largest K split (in blocks) for a batch: the staged activations stay at
// 16 KB per CTA.
Q4_HD int max_blocks_per_split(int batch) {
    return batch <= 1 ? kMaxBlocksPerSplit : (batch == 2 ? 64 : 32);
}

}  // namespace q4plan
