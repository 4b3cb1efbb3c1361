// ring.cuh -- the row-streaming skeleton shared by the norm-quant and the
// post-expert combine kernels.
//
// A persistent CTA of 16 warps is split into NTEAM "teams" of TW warps.  Each
// team owns a ring of NSLOT shared-memory row slots, filled by TMA copies whose
// completion is counted on the slot's "full" mbarrier.  The team's leader
// (its thread 0) keeps a cursor over the rows the team will consume, issues
// the first NSLOT copies up front and, each time the team has finished
// reading a slot (after the team barrier of that row), refills it with the
// row NSLOT places ahead.  Rows therefore stream through shared memory with no
// registers held in flight and no producer warp (all 16 warps compute, and
// each thread may use up to 128 registers).
//
// Thread t of a team owns the 32 consecutive elements [32 t, 32 t + 32) of
// every row (two 16-element blocks).  Its sum-of-squares partial
// b_{2t} + b_{2t+1} is reduced by a lane butterfly and then a pairwise tree
// over the team's warps: together the balanced pairwise tree over the row's
// block partials, with zero partials past the row end (adding +0 to a
// non-negative partial is exact, so the padded tree equals the tree that
// carries an odd tail up unchanged).
//
// Two copy paths fill a slot:
//  - SWZ: H % 64 == 0.  The row is one 2-D tensor tile of 128-byte lines
//    copied with SWIZZLE_128B, so the eight 16-byte chunks of each line land
//    XOR-permuted by (line % 8); the consumer's 16-byte reads are then
//    bank-conflict free with static register destinations.
//  - plain: any H % 16 == 0.  1-D bulk copies; the consumer visits its four
//    chunks in a lane-rotated order and undoes the rotation with selects.
//
// Every wait is bounded (2 s); a team whose wait runs out stops as a whole
// (the abort word is read after the team barrier), its leader drains the
// copies it has in flight and the kernel returns; the host sees the flag
// through mb_device_status().
#pragma once

#include "common.cuh"
#include "tmem.cuh"

namespace mb {

constexpr int kConsumerThreads = 512;     // per CTA (16 warps), split into teams
constexpr int kRingBytes = 192 * 1024;    // row slots per CTA (all teams)
constexpr int kSlotAlign = 1024;          // swizzle atom of SWIZZLE_128B

// The leader's copy cursor (kept in shared memory so that it costs the other
// threads no registers): the next (token, slot) to examine, the next slot to
// fill, and the counts of rows copied and consumed.
struct RingCursor {
    int ct, cj, wslot, issued, consumed, pad0, pad1, pad2;
};

// Shared-memory carve-up of one CTA.  The dynamic shared-memory base is
// rounded up to kSlotAlign in the kernel (the launch asks for that much more).
struct RingLayout {
    int nteam, nslot, slot_bytes, tw;
    __host__ __device__ size_t slots_bytes() const {
        return static_cast<size_t>(nteam) * nslot * slot_bytes;
    }
    __host__ __device__ size_t bars_offset() const { return slots_bytes(); }
    __host__ __device__ size_t red_offset() const {
        return (bars_offset() + static_cast<size_t>(nteam) * nslot * sizeof(uint64_t) + 15) & ~size_t(15);
    }
    __host__ __device__ size_t abort_offset() const {
        return red_offset() + static_cast<size_t>(nteam) * 2 * tw * sizeof(float2);
    }
    __host__ __device__ size_t pipe_offset() const {   // [nteam][2][tw] row partials
        return abort_offset() + static_cast<size_t>(nteam) * 16;
    }
    __host__ __device__ size_t cursor_offset() const {
        return pipe_offset() + static_cast<size_t>(nteam) * 2 * tw * sizeof(float);
    }
    __host__ __device__ size_t total_bytes() const {
        return cursor_offset() + static_cast<size_t>(nteam) * sizeof(RingCursor) + kSlotAlign;
    }
};

__host__ __device__ inline int round_up(int v, int a) { return (v + a - 1) / a * a; }

// Row slot size: the row's BF16 bytes, rounded up to the swizzle atom.
__host__ __device__ inline int slot_bytes_for(int H) { return round_up(2 * H, kSlotAlign); }

// Shared-memory carve-up of a wide-row CTA (one 128-byte line per thread):
// row slots, the packed-weight table [8 chunks][P threads] x 16 B (only for a
// kernel that reads its weights from shared memory: wtab), slot barriers,
// per-team partial buffers [2][TW], abort words and cursors.
struct WideLayout {
    int nteam, nslot, slot_bytes, P;
    bool wtab = true;
    __host__ __device__ size_t slots_bytes() const { return static_cast<size_t>(nteam) * nslot * slot_bytes; }
    __host__ __device__ size_t wtab_offset() const { return slots_bytes(); }              // [8][P] x 16 B
    __host__ __device__ size_t bars_offset() const {
        return wtab_offset() + (wtab ? static_cast<size_t>(P) * 128 : 0);
    }
    __host__ __device__ size_t part_offset() const {                                      // [nteam][2][TW] f32
        return (bars_offset() + static_cast<size_t>(nteam) * nslot * sizeof(uint64_t) + 15) & ~size_t(15);
    }
    __host__ __device__ size_t abort_offset() const { return part_offset() + static_cast<size_t>(nteam) * 2 * (P / 32) * sizeof(float); }
    __host__ __device__ size_t cursor_offset() const { return abort_offset() + static_cast<size_t>(nteam) * 16; }
    __host__ __device__ size_t total_bytes() const {
        return cursor_offset() + static_cast<size_t>(nteam) * sizeof(RingCursor) + kSlotAlign;
    }
};

// The norm weights of a wide-row kernel in tensor memory.  Thread t of a team
// owns line t (64 elements) of every row, and warp w of the CTA reaches lane
// quadrant w % 4 only; since TW divides 4 or 4 divides TW, lane l of quadrant
// g holds the weights of line 32 (g % TW) + l, and for TW = 8 a second column
// block holds the lines of warps 4..7 of a team.  A line takes 32 columns of
// packed BF16 pairs, or with GAINS 64 columns of the FP32 gains gc + w (formed
// once, the same single rounding as forming them per row).  Lines past the
// row's end hold zeros.
template <int TW, bool GAINS>
struct WideWeightTable {
    static constexpr uint32_t kLineCols = GAINS ? 64u : 32u;
    static constexpr int kColBlocks = TW > 4 ? 2 : 1;
    static constexpr uint32_t kCols = kLineCols * kColBlocks;   // the allocation: 32..128 columns

    // Warps 0..3 of the CTA fill it (each its own quadrant).
    static __device__ __forceinline__ void fill(uint32_t base, int warp, int lane, const uint16_t* w, float gc,
                                                int lines) {
#pragma unroll
        for (int cb = 0; cb < kColBlocks; ++cb) {
            const int line = ((warp % TW) + 4 * cb) * 32 + lane;
            const bool in = line < lines;
            const uint32_t dst = base + ((32u * static_cast<uint32_t>(warp)) << 16) + kLineCols * cb;
#pragma unroll
            for (int h = 0; h < static_cast<int>(kLineCols / 32); ++h) {
                uint32_t r[32];
                if constexpr (!GAINS) {
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const uint4 v = in ? *reinterpret_cast<const uint4*>(w + 64 * line + 8 * c)
                                           : make_uint4(0u, 0u, 0u, 0u);
                        r[4 * c] = v.x;
                        r[4 * c + 1] = v.y;
                        r[4 * c + 2] = v.z;
                        r[4 * c + 3] = v.w;
                    }
                } else {   // elements 32 h .. 32 h + 31 of the line
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const uint4 v = in ? *reinterpret_cast<const uint4*>(w + 64 * line + 32 * h + 8 * c)
                                           : make_uint4(0u, 0u, 0u, 0u);
                        const uint32_t ws[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const float2 f = unpack_bf16x2(ws[q]);
                            r[8 * c + 2 * q] = __float_as_uint(in ? __fadd_rn(gc, f.x) : 0.0f);
                            r[8 * c + 2 * q + 1] = __float_as_uint(in ? __fadd_rn(gc, f.y) : 0.0f);
                        }
                    }
                }
                tmem_st32(dst + 32u * static_cast<uint32_t>(h), r);
            }
        }
    }

    // Address of this thread's line: its warp's quadrant, its column block.
    static __device__ __forceinline__ uint32_t line_addr(uint32_t base, int warp, int warp_in_team) {
        return base + ((32u * static_cast<uint32_t>(warp & 3)) << 16) +
               kLineCols * static_cast<uint32_t>(warp_in_team >> 2);
    }
};

// Team-wide sum of one float per thread, in the canonical tree order.  One
// named barrier per call when the team spans several warps.
template <int TW>
struct TeamSum {
    float* red;        // [2][TW] float2 (two partials per warp)
    int* abort_word;   // one per team
    int bar_id;
    int warp_in_team;
    int lane;
    int buf;

    // Returns the sum; `abort` becomes true on every thread of the team when
    // any thread passed fail = true.
    __device__ __forceinline__ float operator()(float v, bool fail, bool& abort) {
        v = warp_tree_sum(v);
        if constexpr (TW == 1) {
            abort = __any_sync(0xffffffffu, fail);
            __syncwarp();
            return v;
        } else {
            if (fail) *reinterpret_cast<volatile int*>(abort_word) = 1;
            if (lane == 0) red[buf * 2 * TW + warp_in_team] = v;
            named_bar_sync(bar_id, TW * 32);
            float p[TW];
            const float* src = red + buf * 2 * TW;
#pragma unroll
            for (int i = 0; i < TW; i += 2) {
                const float2 q = *reinterpret_cast<const float2*>(src + i);
                p[i] = q.x;
                p[i + 1] = q.y;
            }
            abort = *reinterpret_cast<volatile int*>(abort_word) != 0;
            buf ^= 1;
            return tree_sum_array<TW>(p);
        }
    }

    // Two independent sums with one barrier.
    __device__ __forceinline__ float2 sum2(float v0, float v1, bool fail, bool& abort) {
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float o0 = __shfl_xor_sync(0xffffffffu, v0, off);
            const float o1 = __shfl_xor_sync(0xffffffffu, v1, off);
            v0 = v0 + o0;
            v1 = v1 + o1;
        }
        if constexpr (TW == 1) {
            abort = __any_sync(0xffffffffu, fail);
            __syncwarp();
            return make_float2(v0, v1);
        } else {
            if (fail) *reinterpret_cast<volatile int*>(abort_word) = 1;
            float2* src2 = reinterpret_cast<float2*>(red) + buf * TW;
            if (lane == 0) src2[warp_in_team] = make_float2(v0, v1);
            named_bar_sync(bar_id, TW * 32);
            float p0[TW], p1[TW];
#pragma unroll
            for (int i = 0; i < TW; i += 2) {
                const float4 q = *reinterpret_cast<const float4*>(src2 + i);
                p0[i] = q.x;
                p1[i] = q.y;
                p0[i + 1] = q.z;
                p1[i + 1] = q.w;
            }
            abort = *reinterpret_cast<volatile int*>(abort_word) != 0;
            buf ^= 1;
            return make_float2(tree_sum_array<TW>(p0), tree_sum_array<TW>(p1));
        }
    }

    // Two independent sums; lane l receives the sum of v0 when l is even, of
    // v1 when l is odd.  A one-warp team splits the butterfly's first level
    // between the two sums (even lanes keep v0 and take the partner's v0, odd
    // lanes the same for v1), so every later level moves one value instead of
    // two; each sum still comes out of the balanced pairwise tree over lanes
    // 0..31 in order.
    __device__ __forceinline__ float sum2_lane(float v0, float v1, bool fail, bool& abort) {
        if constexpr (TW == 1) {
            const bool odd = (lane & 1) != 0;
            float v = (odd ? v1 : v0) + __shfl_xor_sync(0xffffffffu, odd ? v0 : v1, 1);
#pragma unroll
            for (int off = 2; off < 32; off <<= 1) v = v + __shfl_xor_sync(0xffffffffu, v, off);
            abort = __any_sync(0xffffffffu, fail);
            __syncwarp();
            return v;
        } else {
            const float2 s = sum2(v0, v1, fail, abort);
            return (lane & 1) ? s.y : s.x;
        }
    }
};

// Reads this thread's 32 elements (16 words of two BF16) of a row slot.
// nvalid (0..2) is the number of this thread's 16-element blocks inside the
// row; chunks of missing blocks read as zero.
template <bool SWZ>
__device__ __forceinline__ void read_row32(uint32_t slot_saddr, int tid, int nvalid, uint32_t (&w)[16]) {
    if constexpr (SWZ) {
        const int line = tid >> 1;
        const uint32_t base = slot_saddr + 128u * line;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (i / 2 < nvalid) {
                const int cl = 4 * (tid & 1) + i;
                v = lds128(base + 16u * static_cast<uint32_t>(cl ^ (line & 7)));
            }
            w[4 * i] = v.x;
            w[4 * i + 1] = v.y;
            w[4 * i + 2] = v.z;
            w[4 * i + 3] = v.w;
        }
    } else {
        const int shift = (tid >> 1) & 3;
        const uint32_t base = slot_saddr + 64u * tid;
        uint4 r[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int c = (i + shift) & 3;
            r[i] = (c / 2 < nvalid) ? lds128(base + 16u * c) : make_uint4(0u, 0u, 0u, 0u);
        }
        // chunk c was read at step (c - shift) mod 4
#pragma unroll
        for (int bit = 1; bit < 4; bit <<= 1) {
            if (shift & bit) {
                uint4 t[4];
#pragma unroll
                for (int c = 0; c < 4; ++c) t[c] = r[(c + 4 - bit) & 3];
#pragma unroll
                for (int c = 0; c < 4; ++c) r[c] = t[c];
            }
        }
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            w[4 * c] = r[c].x;
            w[4 * c + 1] = r[c].y;
            w[4 * c + 2] = r[c].z;
            w[4 * c + 3] = r[c].w;
        }
    }
}

// Sum-of-squares partial of this thread's two blocks: sequential fused
// multiply-adds within each block (BF16 inputs, FP32 accumulator), then
// b0 + b1.
__device__ __forceinline__ float row32_sumsq(const uint32_t (&w)[16]) {
    float b0 = 0.0f, b1 = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        b0 = fma_bf16_lo(w[i], w[i], b0);           // block 0: element 2i
        b1 = fma_bf16_lo(w[8 + i], w[8 + i], b1);   // block 1: element 2i
        b0 = fma_bf16_hi(w[i], w[i], b0);           // element 2i + 1
        b1 = fma_bf16_hi(w[8 + i], w[8 + i], b1);
    }
    return b0 + b1;
}

// 1 / sqrt(ss / H + eps); when H is a power of two ss / H is the exact
// product ss * (1 / H), which rounds like the division.
__device__ __forceinline__ float inv_rms_h(float ss, float H, float rH, bool pow2, float eps) {
    const float mean = pow2 ? __fmul_rn(ss, rH) : __fdiv_rn(ss, H);
    return __frcp_rn(__fsqrt_rn(__fadd_rn(mean, eps)));
}

// Per-thread gain pairs g = center + w for this thread's 32 elements.
__device__ __forceinline__ void load_gain32(const uint16_t* w, float center, int tid, int nvalid,
                                            float2 (&g)[16]) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        if (w != nullptr && i / 8 < nvalid) {
            const uint32_t word = *reinterpret_cast<const uint32_t*>(w + 32 * tid + 2 * i);
            const float2 f = unpack_bf16x2(word);
            g[i] = make_float2(__fadd_rn(center, f.x), __fadd_rn(center, f.y));
        } else {
            g[i] = make_float2(0.0f, 0.0f);
        }
    }
}

}  // namespace mb
