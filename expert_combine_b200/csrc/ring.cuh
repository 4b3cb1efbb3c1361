// ring.cuh -- the row-streaming skeleton shared by the norm-quant and the
// post-expert combine kernels.
//
// A persistent CTA holds NTEAM "teams" of TW consumer warps plus one producer
// warp.  Each team owns a ring of NSLOT shared-memory row slots; lane `team`
// of the producer warp fills the team's slots with 1-D bulk copies
// (cp.async.bulk, completion counted on the slot's "full" mbarrier) while the
// team consumes them in order and hands each slot back on its "empty"
// mbarrier.  Rows therefore stream through shared memory with no registers
// held in flight, and the producer runs up to NSLOT rows ahead.
//
// Thread t of a team owns B consecutive 16-element blocks of every row
// (elements [16 B t, 16 B (t + 1))).  Its sum-of-squares partial is reduced by
// a lane butterfly and then a pairwise tree over the team's warps, which
// together form the balanced pairwise tree over the row's block partials (with
// zero partials past the row end; adding +0 to a non-negative partial is
// exact, so the padded tree equals the tree that carries an odd tail).
//
// Every wait is bounded (2 s); a team whose wait runs out stops as a whole
// (the abort flag travels with the reduction), the producer stops issuing,
// drains the copies it has in flight and the kernel returns; the host sees
// the flag through mb_device_status().
#pragma once

#include "common.cuh"

namespace mb {

constexpr int kConsumerThreads = 512;     // per CTA, split into teams
constexpr int kRingBytes = 196 * 1024;    // row slots per CTA (all teams)

// Shared-memory carve-up of one CTA (dynamic shared memory, 128-byte aligned
// base).  Slots first (16-byte aligned for the bulk copies), then barriers,
// then the reduction scratch.
struct RingLayout {
    int nteam, nslot, slot_bytes, tw;
    __host__ __device__ size_t slots_bytes() const {
        return static_cast<size_t>(nteam) * nslot * slot_bytes;
    }
    __host__ __device__ size_t bars_offset() const { return (slots_bytes() + 15) & ~size_t(15); }
    __host__ __device__ size_t red_offset() const {
        return bars_offset() + static_cast<size_t>(nteam) * nslot * 2 * sizeof(uint64_t);
    }
    __host__ __device__ size_t total_bytes() const {
        // per team: [2][tw] float partials + [2][tw] int abort flags
        return red_offset() + static_cast<size_t>(nteam) * 2 * tw * (sizeof(float) + sizeof(int));
    }
};

// Team-wide sum of one float per thread, in the canonical tree order.  One
// named barrier per call when the team spans several warps.
template <int TW>
struct TeamSum {
    float* red;        // [2][TW]
    int* flags;        // [2][TW]
    int bar_id;
    int warp_in_team;
    int lane;
    int buf;

    // Returns the sum; `abort` becomes true on every thread of the team when
    // any thread passed fail = true.
    __device__ __forceinline__ float operator()(float v, bool fail, bool& abort) {
        v = warp_tree_sum(v);
        const bool any_fail = __any_sync(0xffffffffu, fail);
        if constexpr (TW == 1) {
            __syncwarp();
            abort = any_fail;
            return v;
        } else {
            if (lane == 0) {
                red[buf * TW + warp_in_team] = v;
                flags[buf * TW + warp_in_team] = any_fail ? 1 : 0;
            }
            named_bar_sync(bar_id, TW * 32);
            float p[TW];
            int f = 0;
#pragma unroll
            for (int i = 0; i < TW; ++i) {
                p[i] = red[buf * TW + i];
                f |= flags[buf * TW + i];
            }
            buf ^= 1;
            abort = f != 0;
            return tree_sum_array<TW>(p);
        }
    }
};

// Reads this thread's B blocks (16 B * B bf16 values, 32 B per block) of a
// row slot into 8 B 32-bit words (two BF16 each).  The 16-byte chunks are
// visited in a lane-rotated order so that each quarter-warp touches all 32
// banks once; the rotation is undone with selects (no dynamic register
// indexing).
template <int B>
__device__ __forceinline__ void read_slot_blocks(const uint8_t* slot, int tid_in_team, int nvalid_blocks,
                                                 uint32_t (&w)[8 * B]) {
    constexpr int NCH = 2 * B;                      // 16-byte chunks per thread
    const int shift = (B == 1) ? ((tid_in_team >> 2) & 1) : ((tid_in_team >> 1) & 3);
    const uint8_t* base = slot + static_cast<size_t>(tid_in_team) * (32 * B);
    uint4 r[NCH];
#pragma unroll
    for (int i = 0; i < NCH; ++i) {
        const int c = (i + shift) & (NCH - 1);
        // chunk c belongs to block c / 2 of this thread
        if (c / 2 < nvalid_blocks)
            r[i] = *reinterpret_cast<const uint4*>(base + 16 * c);
        else
            r[i] = make_uint4(0u, 0u, 0u, 0u);
    }
    // undo the rotation: chunk c was read at step (c - shift) mod NCH
#pragma unroll
    for (int bit = 1; bit < NCH; bit <<= 1) {
        if (shift & bit) {
            uint4 t[NCH];
#pragma unroll
            for (int c = 0; c < NCH; ++c) t[c] = r[(c + NCH - bit) & (NCH - 1)];
#pragma unroll
            for (int c = 0; c < NCH; ++c) r[c] = t[c];
        }
    }
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
        w[4 * c + 0] = r[c].x;
        w[4 * c + 1] = r[c].y;
        w[4 * c + 2] = r[c].z;
        w[4 * c + 3] = r[c].w;
    }
}

}  // namespace mb
