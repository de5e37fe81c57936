// Work decomposition of the persistent batch-1 layer-stack kernel, shared by the
// device code and by the host replay in q4_debug_check_stack.
//
// One launch runs a run of consecutive dependency groups of a decode step. Each
// group is planned exactly as a launch of the one-group kernel would be
// (q4_b1_plan.h: pieces of rows x K-split, one piece per SM), and CTA c takes
// piece c of every group that has one. A CTA is resident for the whole launch
// (one per SM, 16 warps), so its shared-memory ring of weight units never
// drains between groups: the warps walk one sequence of units through all the
// CTA's pieces, unit v of the sequence being read by warp v % kSWarps from slot
// v % slots, and a warp that has read unit v requests unit v + slots, which may
// lie in a later group. Weights never depend on earlier results, so the loads
// of the next group stream in while the CTA waits for the group before it.
//
// Dependencies: group i of a step starts its multiplications only after every
// piece of group i - 1 has finished. A piece that has written its outputs (or
// its split-K partial sums, or, arriving last on a ticket, the sums of them)
// adds one to the group's completion count in the workspace, after a
// device-scope fence; a CTA entering group i waits (bounded) until the count of
// group i - 1 reaches that group's number of pieces. As group i - 1's pieces
// themselves waited for group i - 2, the wait covers every earlier group. The
// first group of a launch waits for the previous kernel instead (programmatic
// dependent launch).
#pragma once

#include "q4_b1_plan.h"

namespace q4s {

#ifndef Q4S_WARPS
#define Q4S_WARPS 16  // warps of the persistent CTA
#endif
constexpr int kSWarps = Q4S_WARPS;
constexpr int kSThreads = kSWarps * 32;
// GEMVs and groups one launch carries in its parameters (32 KB at most).
constexpr int kStackGemvs = 80;
constexpr int kStackGroups = 64;
// Dynamic shared memory of the persistent CTA.
constexpr int kSmemBudget = 226 * 1024;
constexpr int kMaxSlots = 64 / kSWarps * kSWarps;
constexpr int kBarBytes = (kMaxSlots * 8 + 127) / 128 * 128;
static_assert(kSThreads % 256 == 0, "activation staging covers a slice per 256 threads");
static_assert(kMaxSlots % kSWarps == 0, "slots per warp");

struct alignas(64) Gemv {
    CUtensorMap qs_map;  // code plane as uint32 [n][k/8], box 128 x 8 rows
    CUtensorMap d_map;   // scale plane uint16 [n][k/32], box 32 x 8 (when desc.d_map)
    q4b::Desc desc;      // piece_begin counts from the group's first piece
};

struct Group {
    int32_t first;    // first GEMV (index into Params::gemv)
    int32_t count;    // GEMVs of the group
    int32_t npieces;  // pieces (CTAs with work) of the group
    int32_t counter;  // workspace word of the group's completion count
};

struct Params {
    Gemv gemv[kStackGemvs];
    Group grp[kStackGroups];
    int32_t ngroups;
    int32_t slots;           // ring slots (a multiple of kSWarps)
    uint32_t red_bytes;      // per-(row, slice) partial sums of the largest piece
    uint32_t x_bytes;        // staged activations of the largest piece
    uint32_t* ws;            // workspace (header, tickets, counts, partial sums)
    uint32_t count_extra;    // 0; test hook: pieces every count wait expects beyond the group's
    int32_t pad_;
};
static_assert(sizeof(Params) <= 32764, "kernel parameter space");

Q4B_HD uint32_t smem_bytes(const Params& P) {
    return (uint32_t)kBarBytes + P.red_bytes + P.x_bytes + (uint32_t)P.slots * q4b::kSlotBytes;
}
Q4B_HD uint32_t red_offset() { return (uint32_t)kBarBytes; }
Q4B_HD uint32_t x_offset(const Params& P) { return (uint32_t)kBarBytes + P.red_bytes; }
Q4B_HD uint32_t ring_offset(const Params& P) { return (uint32_t)kBarBytes + P.red_bytes + P.x_bytes; }

// The piece of CTA c in group gi.
struct Piece {
    int32_t gemv;         // index into Params::gemv
    int32_t split, j;     // K split; row range (ticket) within the split
    int32_t r0, r1;       // rows
    int32_t s0, S;        // first global slice, slices
    int32_t T, U;         // 8-row tiles, units (T * S)
};

// False when group gi has no piece for CTA c.
Q4B_HD bool piece_of(const Params& P, int gi, int c, Piece* p) {
    const Group& G = P.grp[gi];
    if (c >= G.npieces) return false;
    int i = G.first;
    while (i + 1 < G.first + G.count && c >= P.gemv[i + 1].desc.piece_begin) ++i;
    const q4b::Desc& D = P.gemv[i].desc;
    const int local = c - D.piece_begin;
    p->gemv = i;
    p->j = local / D.splits;
    p->split = local - p->j * D.splits;
    p->r0 = (int32_t)q4b::range_start(D.n, D.cps, p->j);
    p->r1 = (int32_t)q4b::range_start(D.n, D.cps, p->j + 1);
    q4b::piece_slices(D, p->split, &p->s0, &p->S);
    p->T = (p->r1 - p->r0 + q4b::kTileRows - 1) / q4b::kTileRows;
    p->U = p->T * p->S;
    return true;
}

// A warp's place in its CTA's unit sequence: unit lu (= t * S + s) of the piece
// of group gi; gi == ngroups past the end. Moves kSWarps units at a time.
struct Seq {
    int32_t gi, lu, t, s;
    int32_t dt, ds;  // one step of kSWarps units inside the piece
    Piece p;

    // Move to the first unit at or after (gi, lu) that exists, skipping
    // groups without a piece for CTA c.
    Q4B_HD void settle(const Params& P, int c) {
        bool have = gi < P.ngroups && piece_of(P, gi, c, &p);
        while (gi < P.ngroups) {
            if (have && lu < p.U) break;
            if (have) lu -= p.U;
            ++gi;
            have = gi < P.ngroups && piece_of(P, gi, c, &p);
        }
        if (gi >= P.ngroups) return;
        t = lu / p.S;
        s = lu - t * p.S;
        dt = kSWarps / p.S;
        ds = kSWarps - dt * p.S;
    }
    Q4B_HD void start(const Params& P, int c, int warp) {
        gi = 0;
        lu = warp;
        settle(P, c);
    }
    Q4B_HD void advance(const Params& P, int c) {
        lu += kSWarps;
        if (lu < p.U) {
            t += dt;
            s += ds;
            if (s >= p.S) {
                s -= p.S;
                ++t;
            }
            return;
        }
        settle(P, c);
    }
    Q4B_HD bool valid(const Params& P) const { return gi < P.ngroups; }
};

}  // namespace q4s
