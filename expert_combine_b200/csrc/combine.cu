// combine.cu -- stage 3, post-expert RMSNorm + weighted top-k combine, and the
// gated residual join (alone, or fused after the combine).
//
// Combine, per token t (TensorRT-LLM PR 21356 "Muse Spark Open decoder fast
// paths", description, post-expert norm and combine; TensorRT-LLM PR 21042
// reference composition, MoE paragraph):
//   for j = 0 .. k-1 in slot order, when 0 <= idx[t, j] < R:
//       x    = expert_out[idx[t, j], :]
//       inv  = 1 / sqrt(ss(x) / H + eps)
//       y    = bf16((x * (gc + w)) * inv)
//       acc  = fmaf(wt[t, j], y, acc)                      acc starts at +0
//   out[t, :] = bf16(acc)
// A slot outside [0, R) is never read: its row is neither copied nor touched.
//
// Gated residual join, per token (same page, gated residual join):
//   g  = bf16(gain * branch)
//   n  = bf16(g * inv_rms(g))                               weightless norm
//   r' = alpha * r + beta * n                               FP32 residual stream
//   p  = bf16((r' * (next_gc + next_w)) * inv_rms(r'))      next prenorm, optional
// Fused after the combine, `branch` is the BF16 combine output.
#include "internal.h"
#include "ring.cuh"
#include "tmap.h"

namespace mb {

struct CombineArgs {
    const uint16_t* expert_out;
    int64_t R;
    int H;
    const int32_t* row_idx;
    const float* wt;
    int T, k;
    const uint16_t* w;
    float gc, eps;
    uint16_t* out;
    JoinArgs join;
    int nslot;
};

__device__ __forceinline__ bool slot_valid(int32_t r, int64_t R) {
    return r >= 0 && static_cast<int64_t>(r) < R;
}

__device__ __forceinline__ void load_words32(const uint16_t* p, bool valid0, bool valid1, uint32_t (&w)[16]) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if ((c < 2) ? valid0 : valid1) v = *reinterpret_cast<const uint4*>(p + 8 * c);
        w[4 * c] = v.x;
        w[4 * c + 1] = v.y;
        w[4 * c + 2] = v.z;
        w[4 * c + 3] = v.w;
    }
}

// Canonical sum of squares of this thread's 32 FP32 values (pairs r[i] =
// elements 2i, 2i+1; i < 8 is block 0).
__device__ __forceinline__ float row32_sumsq_f(const float2 (&r)[16]) {
    float2 a = make_float2(0.0f, 0.0f);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float2 lo = make_float2(r[i].x, r[8 + i].x);
        const float2 hi = make_float2(r[i].y, r[8 + i].y);
        a = fma2(lo, lo, a);
        a = fma2(hi, hi, a);
    }
    return a.x + a.y;
}

// Join epilogue for one token; this thread holds 32 branch values as BF16
// pair words.  Two or three team sums.
template <int TW>
__device__ __forceinline__ void join_token32(const uint32_t (&brw)[16], int t, int H, int tid, int nvalid,
                                             const JoinArgs& j, TeamSum<TW>& team_sum, bool pow2,
                                             float rH) {
    const float fH = static_cast<float>(H);
    const bool v0 = nvalid > 0, v1 = nvalid > 1;
    uint32_t gw[16];
    load_words32(j.gain + 32 * tid, v0, v1, gw);
    uint32_t gg[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) gg[i] = pack_bf16x2_rn(mul2(unpack_bf16x2(gw[i]), unpack_bf16x2(brw[i])));
    bool abort;
    const float ss_g = team_sum(row32_sumsq(gg), false, abort);
    const float inv_g = inv_rms_h(ss_g, fH, rH, pow2, j.eps);
    const float2 inv_g2 = make_float2(inv_g, inv_g);
    const float2 alpha2 = make_float2(j.alpha, j.alpha);
    const float2 beta2 = make_float2(j.beta, j.beta);

    float* rrow = j.residual + static_cast<size_t>(t) * H + 32 * tid;
    float2 r[16];
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if ((c < 4) ? v0 : v1) v = *reinterpret_cast<const float4*>(rrow + 4 * c);
        r[2 * c] = make_float2(v.x, v.y);
        r[2 * c + 1] = make_float2(v.z, v.w);
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const float2 n = unpack_bf16x2(pack_bf16x2_rn(mul2(unpack_bf16x2(gg[i]), inv_g2)));
        r[i] = add2(mul2(alpha2, r[i]), mul2(beta2, n));
    }
#pragma unroll
    for (int c = 0; c < 8; ++c)
        if ((c < 4) ? v0 : v1)
            *reinterpret_cast<float4*>(rrow + 4 * c) =
                make_float4(r[2 * c].x, r[2 * c].y, r[2 * c + 1].x, r[2 * c + 1].y);

    if (j.next_w != nullptr) {
        const float ss_r = team_sum(row32_sumsq_f(r), false, abort);
        const float inv_r = inv_rms_h(ss_r, fH, rH, pow2, j.next_eps);
        const float2 inv_r2 = make_float2(inv_r, inv_r);
        const float2 gc2 = make_float2(j.next_gc, j.next_gc);
        uint32_t nw[16];
        load_words32(j.next_w + 32 * tid, v0, v1, nw);
        uint32_t pw[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
            pw[i] = pack_bf16x2_rn(mul2(mul2(r[i], add2(gc2, unpack_bf16x2(nw[i]))), inv_r2));
        uint16_t* prow = j.next_prenorm + static_cast<size_t>(t) * H + 32 * tid;
#pragma unroll
        for (int c = 0; c < 4; ++c)
            if ((c < 2) ? v0 : v1)
                *reinterpret_cast<uint4*>(prow + 8 * c) =
                    make_uint4(pw[4 * c], pw[4 * c + 1], pw[4 * c + 2], pw[4 * c + 3]);
    }
}

// One normalised pair as BF16-exact floats: bf16((x * g) * inv).  With GC0
// the gain is the BF16 weight itself and x * w is formed exactly by a
// mixed-precision FMA.
template <bool GC0>
__device__ __forceinline__ float2 norm_pair(uint32_t xw, uint32_t wpw, float2 gp, float2 inv2) {
    const float2 t = GC0 ? mul_bf16x2_exact(xw, wpw) : mul2(unpack_bf16x2(xw), gp);
    return round_bf16_f2(mul2(t, inv2));
}

template <int TW, bool SWZ, bool JOIN, bool GC0>
__global__ void __launch_bounds__(kConsumerThreads, 1)
    combine_kernel(const __grid_constant__ CUtensorMap tmap, const CombineArgs a) {
    constexpr int NTEAM = kConsumerThreads / (TW * 32);
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_saddr = smem_addr(smem_raw);
    uint8_t* smem = smem_raw + (((raw_saddr + kSlotAlign - 1) & ~uint32_t(kSlotAlign - 1)) - raw_saddr);
    const int H = a.H;
    const int nslot = a.nslot;
    const int slot_bytes = slot_bytes_for(H);
    const RingLayout lay{NTEAM, nslot, slot_bytes, TW};
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + lay.bars_offset());
    float* red_all = reinterpret_cast<float*>(smem + lay.red_offset());
    int* abort_all = reinterpret_cast<int*>(smem + lay.abort_offset());

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int i = 0; i < NTEAM * nslot; ++i) mbar_init(&bars[i], 1);
        for (int i = 0; i < NTEAM; ++i) abort_all[4 * i] = 0;
        fence_mbar_init();
    }
    __syncthreads();
    griddep_wait();     // row indices and weights may come from the previous kernel
    griddep_launch();

    const int T = a.T, k = a.k;
    const int64_t R = a.R;
    const int team_stride = gridDim.x * NTEAM;
    const int team = warp / TW;
    const int warp_in_team = warp % TW;
    const int tid = warp_in_team * 32 + lane;
    const int nblocks = H / 16;
    int nvalid = nblocks - 2 * tid;
    nvalid = nvalid < 0 ? 0 : (nvalid > 2 ? 2 : nvalid);
    uint8_t* ring = smem + static_cast<size_t>(team) * nslot * slot_bytes;
    const uint32_t ring_saddr = smem_addr(ring);
    uint64_t* tb = bars + static_cast<size_t>(team) * nslot;
    TeamSum<TW> team_sum{red_all + team * 4 * TW, abort_all + 4 * team, 1 + team, warp_in_team, lane, 0};

    // ---- the leader's copy cursor over (token, slot): valid rows in order
    RingCursor* cur = reinterpret_cast<RingCursor*>(smem + lay.cursor_offset()) + team;
    auto issue = [&]() {
        int ct = cur->ct, cj = cur->cj;
        while (ct < T) {
            const int32_t r = __ldg(a.row_idx + static_cast<size_t>(ct) * k + cj);
            if (++cj == k) {
                cj = 0;
                ct += team_stride;
                if (ct + team_stride < T)
                    asm volatile("prefetch.global.L1 [%0];" ::"l"(a.row_idx + static_cast<size_t>(ct + team_stride) * k));
            }
            if (!slot_valid(r, R)) continue;
            const int ws = cur->wslot;
            mbar_arrive_expect_tx(&tb[ws], 2u * static_cast<uint32_t>(H));
            uint8_t* dst = ring + static_cast<size_t>(ws) * slot_bytes;
            if constexpr (SWZ)
                tma_load_2d(smem_addr(dst), &tmap, 0, r * (H / 64), &tb[ws]);
            else
                bulk_g2s(dst, a.expert_out + static_cast<size_t>(r) * H, 2u * static_cast<uint32_t>(H), &tb[ws]);
            cur->issued += 1;
            cur->wslot = (ws + 1 == nslot) ? 0 : ws + 1;
            break;
        }
        cur->ct = ct;
        cur->cj = cj;
    };
    // one-warp teams run the cursor together: the cursor token's row indices
    // sit one per lane, its valid slots not yet requested in a ballot mask,
    // so a refill is a shuffle and one copy instead of the leader's walk
    int wc_t = static_cast<int>(blockIdx.x) * NTEAM + team;      // cursor token
    int32_t wc_r = -1;                                          // its row index in this lane's slot
    uint32_t wc_mask = 0u;                                      // its valid slots still to request
    int wc_slot = 0, wc_issued = 0, wc_consumed = 0;
    auto warp_issue = [&]() {
        while (wc_mask == 0u) {
            wc_t += team_stride;
            if (wc_t >= T) return;
            wc_r = lane < k ? __ldg(a.row_idx + static_cast<size_t>(wc_t) * k + lane) : -1;
            wc_mask = __ballot_sync(0xffffffffu, lane < k && slot_valid(wc_r, R));
        }
        const int j = __ffs(wc_mask) - 1;
        wc_mask &= wc_mask - 1u;
        const int32_t r = __shfl_sync(0xffffffffu, wc_r, j);
        if (lane == 0) {
            mbar_arrive_expect_tx(&tb[wc_slot], 2u * static_cast<uint32_t>(H));
            uint8_t* dst = ring + static_cast<size_t>(wc_slot) * slot_bytes;
            if constexpr (SWZ)
                tma_load_2d(smem_addr(dst), &tmap, 0, r * (H / 64), &tb[wc_slot]);
            else
                bulk_g2s(dst, a.expert_out + static_cast<size_t>(r) * H, 2u * static_cast<uint32_t>(H), &tb[wc_slot]);
        }
        wc_issued += 1;
        wc_slot = (wc_slot + 1 == nslot) ? 0 : wc_slot + 1;
    };
    if constexpr (TW == 1) {
        if (wc_t < T) {
            wc_r = lane < k ? __ldg(a.row_idx + static_cast<size_t>(wc_t) * k + lane) : -1;
            wc_mask = __ballot_sync(0xffffffffu, lane < k && slot_valid(wc_r, R));
            for (int i = 0; i < nslot; ++i) warp_issue();
        }
    } else if (tid == 0) {
        *cur = RingCursor{static_cast<int>(blockIdx.x) * NTEAM + team, 0, 0, 0, 0, 0, 0, 0};
        for (int i = 0; i < nslot; ++i) issue();
    }

    // gain: with GC0 the packed BF16 weights, else FP32 pairs gc + w
    uint32_t wp[16];
    float2 g[16];
    if constexpr (GC0) {
        load_words32(a.w + 32 * tid, nvalid > 0, nvalid > 1, wp);
    } else {
        load_gain32(a.w, a.gc, tid, nvalid, g);
    }
    const float fH = static_cast<float>(H);
    const bool pow2 = (H & (H - 1)) == 0;
    const float rH = pow2 ? __frcp_rn(fH) : 0.0f;
    constexpr bool PAIR = GC0;   // two rows per team iteration (register budget allows it)

    // slot indices and weights of the token, one slot per lane (k <= 32),
    // loaded one token ahead
    int t = blockIdx.x * NTEAM + team;
    int32_t my_r = -1;
    float my_w = 0.0f;
    if (t < T && lane < k) {
        my_r = __ldg(a.row_idx + static_cast<size_t>(t) * k + lane);
        my_w = __ldg(a.wt + static_cast<size_t>(t) * k + lane);
    }
    int slot = 0, phase = 0;
    bool aborted = false;
    for (; t < T; t += team_stride) {
        const int32_t cur_r = my_r;
        const float cur_w = my_w;
        const int tn = t + team_stride;
        if (tn < T && lane < k) {
            my_r = __ldg(a.row_idx + static_cast<size_t>(tn) * k + lane);
            my_w = __ldg(a.wt + static_cast<size_t>(tn) * k + lane);
        }
        float2 acc[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) acc[i] = make_float2(0.0f, 0.0f);

        // valid slots of this token, in slot order
        unsigned vm = __ballot_sync(0xffffffffu, lane < k && slot_valid(cur_r, R));
        while (vm != 0u) {
            const int j0 = __ffs(vm) - 1;
            vm &= vm - 1u;
            const bool two = PAIR && vm != 0u;
            int j1 = j0;
            if (two) {
                j1 = __ffs(vm) - 1;
                vm &= vm - 1u;
            }
            const float w0 = __shfl_sync(0xffffffffu, cur_w, j0);
            const float w1 = __shfl_sync(0xffffffffu, cur_w, j1);
            int s1 = slot + 1, ph1 = phase;
            if (s1 == nslot) {
                s1 = 0;
                ph1 ^= 1;
            }
            bool ok = mbar_wait_bounded(&tb[slot], phase, 4u);
            if (two && ok) ok = mbar_wait_bounded(&tb[s1], ph1, 4u);
            uint32_t wv0[16], wv1[16];
            if (ok) {
                read_row32<SWZ>(ring_saddr + static_cast<uint32_t>(slot * slot_bytes), tid, nvalid, wv0);
                if (two) read_row32<SWZ>(ring_saddr + static_cast<uint32_t>(s1 * slot_bytes), tid, nvalid, wv1);
            } else {
#pragma unroll
                for (int i = 0; i < 16; ++i) wv0[i] = wv1[i] = 0u;
            }
            bool abort;
            float ss;       // lane l: the sum of squares of the step's row l & 1
            if (two) {
                ss = team_sum.sum2_lane(row32_sumsq(wv0), row32_sumsq(wv1), !ok, abort);
            } else {
                ss = team_sum(row32_sumsq(wv0), !ok, abort);
            }
            if (abort) {
                aborted = true;
                break;
            }
            if constexpr (TW == 1) {   // the warp has read these slots: refill them
                wc_consumed += two ? 2 : 1;
                if (lane == 0) fence_proxy_async_smem();
                warp_issue();
                if (two) warp_issue();
            } else if (tid == 0) {   // the whole team has read these slots: refill them
                cur->consumed += two ? 2 : 1;
                fence_proxy_async_smem();
                issue();
                if (two) issue();
            }
            slot = s1;
            phase = ph1;
            if (two) {
                if (++slot == nslot) {
                    slot = 0;
                    phase ^= 1;
                }
            }
            // each lane forms the inverse RMS of its row l & 1 (one evaluation
            // serves both rows); lanes 0 and 1 hand them out
            const float inv_l = inv_rms_h(ss, fH, rH, pow2, a.eps);
            const float inv0 = __shfl_sync(0xffffffffu, inv_l, 0);
            const float2 inv02 = make_float2(inv0, inv0);
            const float2 w02 = make_float2(w0, w0);
            if (two) {
                const float inv1 = __shfl_sync(0xffffffffu, inv_l, 1);
                const float2 inv12 = make_float2(inv1, inv1);
                const float2 w12 = make_float2(w1, w1);
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float2 y0 = norm_pair<GC0>(wv0[i], wp[i], g[i], inv02);
                    const float2 y1 = norm_pair<GC0>(wv1[i], wp[i], g[i], inv12);
                    acc[i] = fma2(w02, y0, acc[i]);
                    acc[i] = fma2(w12, y1, acc[i]);
                }
            } else {
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    acc[i] = fma2(w02, norm_pair<GC0>(wv0[i], wp[i], g[i], inv02), acc[i]);
                }
            }
        }
        if (aborted) break;

        uint32_t brw[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) brw[i] = pack_bf16x2_rn(acc[i]);
        if (a.out != nullptr) {
            uint16_t* orow = a.out + static_cast<size_t>(t) * H + 32 * tid;
#pragma unroll
            for (int c = 0; c < 4; ++c)
                if (c / 2 < nvalid)
                    __stcs(reinterpret_cast<uint4*>(orow + 8 * c),   // streaming: written once
                           make_uint4(brw[4 * c], brw[4 * c + 1], brw[4 * c + 2], brw[4 * c + 3]));
        }
        if constexpr (JOIN) join_token32<TW>(brw, t, H, tid, nvalid, a.join, team_sum, pow2, rH);
    }
    // copies still in flight (only after an abort) land before the CTA exits
    if constexpr (TW == 1) {
        if (lane == 0)
            for (int f = wc_consumed; f < wc_issued; ++f)
                mbar_wait_bounded(&tb[f % nslot], (f / nslot) & 1, 2u);
    } else if (tid == 0) {
        for (int f = cur->consumed; f < cur->issued; ++f)
            mbar_wait_bounded(&tb[f % nslot], (f / nslot) & 1, 2u);
    }
}

// ---------------------------------------------------------------------------
// Wide-row combine (H >= 2048, H % 64 == 0): thread t of a team owns the
// 128-byte line t of every row (64 elements, four 16-element blocks), so a
// team of P = H/64 (rounded up to a power of two) threads covers a row and a
// CTA holds 512/P teams.  Each row is read twice from its shared-memory slot:
// pass 1 forms the sum-of-squares partial (the team barrier then yields inv),
// pass 2 re-reads the row, normalises it and accumulates; only the FP32
// accumulator lives in registers.  A slot is handed back one row late (at the
// barrier of the team's next row, when every warp has finished pass 2).  The
// packed BF16 norm weights sit in tensor memory, not shared memory: lane l of
// lane quadrant g holds the 32 weight words of line 32 (g % TW) + l (for
// TW = 8, column block 1 holds the lines of warps 4..7 of a team), so pass 2
// fetches them with tcgen05.ld and the shared-memory port carries only the
// row copies and the two passes' reads of them.
template <int TW, bool GC0>
__global__ void __launch_bounds__(kConsumerThreads, 1)
    combine_wide_kernel(const __grid_constant__ CUtensorMap tmap, const CombineArgs a) {
    constexpr int P = TW * 32;
    constexpr int NTEAM = kConsumerThreads / P;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_saddr = smem_addr(smem_raw);
    uint8_t* smem = smem_raw + (((raw_saddr + kSlotAlign - 1) & ~uint32_t(kSlotAlign - 1)) - raw_saddr);
    const int H = a.H;
    const int nslot = a.nslot;
    const int slot_bytes = slot_bytes_for(H);
    const WideLayout lay{NTEAM, nslot, slot_bytes, P, false};   // weights in tensor memory
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + lay.bars_offset());
    float* part_all = reinterpret_cast<float*>(smem + lay.part_offset());
    int* abort_all = reinterpret_cast<int*>(smem + lay.abort_offset());

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int team = warp / TW;
    const int warp_in_team = warp % TW;
    const int tid = warp_in_team * 32 + lane;
    const int lines = H / 64;
    const bool has_line = tid < lines;
    const bool warp_has_line = warp_in_team * 32 < lines;   // the same on every lane of the warp
    using WTab = WideWeightTable<TW, !GC0>;   // with a gain centre: the FP32 gains
    __shared__ uint32_t s_tmem;
    if (warp == 0) {
        tmem_alloc(&s_tmem, WTab::kCols);
        tmem_relinquish();
    }
    if (threadIdx.x == 0) {
        for (int i = 0; i < NTEAM * nslot; ++i) mbar_init(&bars[i], 1);
        for (int i = 0; i < NTEAM; ++i) abort_all[4 * i] = 0;
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    griddep_wait();     // row indices and weights may come from the previous kernel
    griddep_launch();
    if (warp < 4) WTab::fill(s_tmem, warp, lane, a.w, a.gc, lines);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t wt_taddr = WTab::line_addr(s_tmem, warp, warp_in_team);

    const int T = a.T, k = a.k;
    const int64_t R = a.R;
    const int team_stride = gridDim.x * NTEAM;
    uint8_t* ring = smem + static_cast<size_t>(team) * nslot * slot_bytes;
    const uint32_t ring_saddr = smem_addr(ring);
    uint64_t* tb = bars + static_cast<size_t>(team) * nslot;
    int* abort_word = abort_all + 4 * team;
    float* part = part_all + team * 2 * TW;

    // warp 0 of the team runs the copy cursor together: the cursor token's
    // row indices one per lane, its valid slots not yet requested in a ballot
    // mask, so a refill is a shuffle and one copy (lane 0 issues it)
    int wc_t = static_cast<int>(blockIdx.x) * NTEAM + team;      // cursor token
    int32_t wc_r = -1;
    uint32_t wc_mask = 0u;
    int wc_slot = 0, wc_issued = 0, wc_consumed = 0;
    auto warp_issue = [&]() {
        while (wc_mask == 0u) {
            wc_t += team_stride;
            if (wc_t >= T) return;
            wc_r = lane < k ? __ldg(a.row_idx + static_cast<size_t>(wc_t) * k + lane) : -1;
            wc_mask = __ballot_sync(0xffffffffu, lane < k && slot_valid(wc_r, R));
        }
        const int j = __ffs(wc_mask) - 1;
        wc_mask &= wc_mask - 1u;
        const int32_t r = __shfl_sync(0xffffffffu, wc_r, j);
        if (lane == 0) {
            mbar_arrive_expect_tx(&tb[wc_slot], 2u * static_cast<uint32_t>(H));
            tma_load_2d(smem_addr(ring + static_cast<size_t>(wc_slot) * slot_bytes), &tmap, 0, r * lines,
                        &tb[wc_slot]);
        }
        wc_issued += 1;
        wc_slot = (wc_slot + 1 == nslot) ? 0 : wc_slot + 1;
    };
    if (warp_in_team == 0 && wc_t < T) {
        wc_r = lane < k ? __ldg(a.row_idx + static_cast<size_t>(wc_t) * k + lane) : -1;
        wc_mask = __ballot_sync(0xffffffffu, lane < k && slot_valid(wc_r, R));
        for (int i = 0; i < nslot; ++i) warp_issue();
    }

    const float fH = static_cast<float>(H);
    const bool pow2 = (H & (H - 1)) == 0;
    const float rH = pow2 ? __frcp_rn(fH) : 0.0f;
    // this thread's line in a slot (line 0 for a thread past the row's end);
    // chunk c of it sits at chunk c ^ sw (SWIZZLE_128B)
    const uint32_t line_off = has_line ? 128u * static_cast<uint32_t>(tid) : 0u;
    const int sw = tid & 7;

    int t = blockIdx.x * NTEAM + team;
    int32_t my_r = -1;
    float my_w = 0.0f;
    if (t < T && lane < k) {
        my_r = __ldg(a.row_idx + static_cast<size_t>(t) * k + lane);
        my_w = __ldg(a.wt + static_cast<size_t>(t) * k + lane);
    }
    int slot = 0, phase = 0, pbuf = 0;
    bool held = false;      // a slot waits to be handed back at the next barrier
    bool aborted = false;
    float2 acc[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) acc[i] = make_float2(0.0f, 0.0f);

    for (; t < T; t += team_stride) {
        const int32_t cur_r = my_r;
        const float cur_w = my_w;
        const int tn = t + team_stride;
        if (tn < T && lane < k) {
            my_r = __ldg(a.row_idx + static_cast<size_t>(tn) * k + lane);
            my_w = __ldg(a.wt + static_cast<size_t>(tn) * k + lane);
        }
        unsigned vm = __ballot_sync(0xffffffffu, lane < k && slot_valid(cur_r, R));
        while (vm != 0u) {
            const int j = __ffs(vm) - 1;
            vm &= vm - 1u;
            const float wj = __shfl_sync(0xffffffffu, cur_w, j);
            const bool ok = mbar_wait_bounded(&tb[slot], phase, 4u);
            const uint32_t sbase = ring_saddr + static_cast<uint32_t>(slot * slot_bytes) + line_off;
            // pass 1: sum of squares of the four blocks, two chunks per block
            float b[4] = {0.0f, 0.0f, 0.0f, 0.0f};
            if (ok && has_line) {
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const uint4 v = lds128(sbase + 16u * static_cast<uint32_t>(c ^ sw));
                    float& acc_b = b[c >> 1];
                    acc_b = fma_bf16_lo(v.x, v.x, acc_b);
                    acc_b = fma_bf16_hi(v.x, v.x, acc_b);
                    acc_b = fma_bf16_lo(v.y, v.y, acc_b);
                    acc_b = fma_bf16_hi(v.y, v.y, acc_b);
                    acc_b = fma_bf16_lo(v.z, v.z, acc_b);
                    acc_b = fma_bf16_hi(v.z, v.z, acc_b);
                    acc_b = fma_bf16_lo(v.w, v.w, acc_b);
                    acc_b = fma_bf16_hi(v.w, v.w, acc_b);
                }
            }
            if (!ok) *reinterpret_cast<volatile int*>(abort_word) = 1;
            const float v = warp_tree_sum((b[0] + b[1]) + (b[2] + b[3]));
            if (lane == 0) part[pbuf * TW + warp_in_team] = v;
            if constexpr (TW == 1) __syncwarp();
            else named_bar_sync(1 + team, P);
            if (*reinterpret_cast<volatile int*>(abort_word) != 0) {
                aborted = true;
                break;
            }
            if (warp_in_team == 0 && held) {   // every warp has finished pass 2 of the previous row
                wc_consumed += 1;
                if (lane == 0) fence_proxy_async_smem();
                warp_issue();
            }
            held = true;
            float pp[TW];
#pragma unroll
            for (int i = 0; i < TW; ++i) pp[i] = part[pbuf * TW + i];
            pbuf ^= 1;
            const float inv = inv_rms_h(tree_sum_array<TW>(pp), fH, rH, pow2, a.eps);
            const float2 inv2 = make_float2(inv, inv);
            const float2 w2 = make_float2(wj, wj);
            // pass 2: normalise and accumulate (every lane of a warp that holds
            // a line reads the weight table; a lane past the row's end reads
            // line 0 and its accumulator is never stored)
            if (warp_has_line)
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                uint32_t ws[8];
                if constexpr (GC0) {
                    const uint4 wv = tmem_ld4_ro(wt_taddr + 4u * static_cast<uint32_t>(c));
                    ws[0] = wv.x;
                    ws[1] = wv.y;
                    ws[2] = wv.z;
                    ws[3] = wv.w;
                } else {
                    tmem_ld8_ro(wt_taddr + 8u * static_cast<uint32_t>(c), ws);
                }
                const uint4 x = lds128(sbase + 16u * static_cast<uint32_t>(c ^ sw));
                const uint32_t xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float2 xg = GC0 ? mul_bf16x2_exact(xs[q], ws[q])
                                          : mul2(unpack_bf16x2(xs[q]),
                                                 make_float2(__uint_as_float(ws[2 * q]), __uint_as_float(ws[2 * q + 1])));
                    acc[4 * c + q] = fma2(w2, round_bf16_f2(mul2(xg, inv2)), acc[4 * c + q]);
                }
            }
            if (++slot == nslot) {
                slot = 0;
                phase ^= 1;
            }
        }
        if (aborted) break;
        if (has_line && a.out != nullptr) {
            uint16_t* orow = a.out + static_cast<size_t>(t) * H + 64 * tid;
#pragma unroll
            for (int c = 0; c < 8; ++c)
                __stcs(reinterpret_cast<uint4*>(orow + 8 * c),     // streaming: written once
                       make_uint4(pack_bf16x2_rn(acc[4 * c]), pack_bf16x2_rn(acc[4 * c + 1]),
                                  pack_bf16x2_rn(acc[4 * c + 2]), pack_bf16x2_rn(acc[4 * c + 3])));
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) acc[i] = make_float2(0.0f, 0.0f);
    }
    // copies still in flight land before the CTA exits
    if (tid == 0)
        for (int f = wc_consumed; f < wc_issued; ++f)
            mbar_wait_bounded(&tb[f % nslot], (f / nslot) & 1, 2u);
    tc_fence_before();
    __syncthreads();    // every warp's last weight-table read is done
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(s_tmem, WTab::kCols);
    }
}

// Standalone gated residual join: the branch comes from global memory.
template <int TW>
__global__ void __launch_bounds__(kConsumerThreads, 1)
    residual_join_kernel(const uint16_t* __restrict__ branch, int T, int H, JoinArgs join) {
    constexpr int NTEAM = kConsumerThreads / (TW * 32);
    __shared__ __align__(16) float red_all[NTEAM * 4 * TW];
    __shared__ int abort_all[NTEAM * 4];
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int team = warp / TW;
    const int warp_in_team = warp % TW;
    const int tid = warp_in_team * 32 + lane;
    const int nblocks = H / 16;
    int nvalid = nblocks - 2 * tid;
    nvalid = nvalid < 0 ? 0 : (nvalid > 2 ? 2 : nvalid);
    if (threadIdx.x < NTEAM) abort_all[4 * threadIdx.x] = 0;
    __syncthreads();
    griddep_wait();
    griddep_launch();
    TeamSum<TW> team_sum{red_all + team * 4 * TW, abort_all + 4 * team, 1 + team, warp_in_team, lane, 0};
    const bool pow2 = (H & (H - 1)) == 0;
    const float rH = pow2 ? __frcp_rn(static_cast<float>(H)) : 0.0f;
    for (int t = blockIdx.x * NTEAM + team; t < T; t += gridDim.x * NTEAM) {
        uint32_t brw[16];
        load_words32(branch + static_cast<size_t>(t) * H + 32 * tid, nvalid > 0, nvalid > 1, brw);
        join_token32<TW>(brw, t, H, tid, nvalid, join, team_sum, pow2, rH);
    }
}

namespace {

cudaLaunchConfig_t pdl_config(int grid, int block, size_t smem, cudaStream_t s, cudaLaunchAttribute* attr) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cfg;
}

template <int TW, bool SWZ, bool JOIN, bool GC0>
cudaError_t launch_cb(const CUtensorMap& tmap, const CombineArgs& args, cudaStream_t s) {
    constexpr int NTEAM = kConsumerThreads / (TW * 32);
    const int slot_bytes = slot_bytes_for(args.H);
    int nslot = kRingBytes / (NTEAM * slot_bytes);
    if (nslot > 16) nslot = 16;
    if (nslot < 2) return cudaErrorInvalidConfiguration;
    CombineArgs a = args;
    a.nslot = nslot;
    const RingLayout lay{NTEAM, nslot, slot_bytes, TW};
    const size_t smem = lay.total_bytes();
    auto kern = combine_kernel<TW, SWZ, JOIN, GC0>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    int grid = (a.T + NTEAM - 1) / NTEAM;
    const int cap = device_info().sm_count;
    if (grid > cap) grid = cap;
    cudaLaunchAttribute attr[1];
    cudaLaunchConfig_t cfg = pdl_config(grid, kConsumerThreads, smem, s, attr);
    return cudaLaunchKernelEx(&cfg, kern, tmap, a);
}

template <bool SWZ, bool JOIN, bool GC0>
cudaError_t launch_cb_tw(int TW, const CUtensorMap& tmap, const CombineArgs& a, cudaStream_t s) {
    switch (TW) {
        case 1: return launch_cb<1, SWZ, JOIN, GC0>(tmap, a, s);
        case 2: return launch_cb<2, SWZ, JOIN, GC0>(tmap, a, s);
        case 4: return launch_cb<4, SWZ, JOIN, GC0>(tmap, a, s);
        case 8: return launch_cb<8, SWZ, JOIN, GC0>(tmap, a, s);
        case 16: return launch_cb<16, SWZ, JOIN, GC0>(tmap, a, s);
        default: return cudaErrorInvalidValue;
    }
}

template <bool SWZ, bool JOIN>
cudaError_t launch_cb_gc(int TW, const CUtensorMap& tmap, const CombineArgs& a, cudaStream_t s) {
    // gc == +0 or -0: the gain is the BF16 weight itself (0 + w == w exactly)
    return a.gc == 0.0f ? launch_cb_tw<SWZ, JOIN, true>(TW, tmap, a, s)
                        : launch_cb_tw<SWZ, JOIN, false>(TW, tmap, a, s);
}

template <int TW, bool GC0>
cudaError_t launch_wide(const CUtensorMap& tmap, const CombineArgs& args, cudaStream_t s) {
    constexpr int P = TW * 32;
    constexpr int NTEAM = kConsumerThreads / P;
    const int slot_bytes = slot_bytes_for(args.H);
    WideLayout lay{NTEAM, 1, slot_bytes, P, false};
    const size_t fixed = lay.total_bytes() - static_cast<size_t>(NTEAM) * slot_bytes;
    cudaFuncAttributes fa{};   // the kernel's static shared memory counts against the same limit
    cudaError_t fe = cudaFuncGetAttributes(&fa, combine_wide_kernel<TW, GC0>);
    if (fe != cudaSuccess) return fe;
    const int avail = device_info().max_smem_optin - static_cast<int>(fixed) - static_cast<int>(fa.sharedSizeBytes) -
                      64 * NTEAM;
    int nslot = avail / (NTEAM * slot_bytes);
    if (nslot > 16) nslot = 16;
    if (nslot < 2) return cudaErrorInvalidConfiguration;
    lay.nslot = nslot;
    CombineArgs a = args;
    a.nslot = nslot;
    const size_t smem = lay.total_bytes();
    auto kern = combine_wide_kernel<TW, GC0>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    int grid = (a.T + NTEAM - 1) / NTEAM;
    const int cap = device_info().sm_count;
    if (grid > cap) grid = cap;
    cudaLaunchAttribute attr[1];
    cudaLaunchConfig_t cfg = pdl_config(grid, kConsumerThreads, smem, s, attr);
    return cudaLaunchKernelEx(&cfg, kern, tmap, a);
}

template <bool GC0>
cudaError_t launch_wide_tw(int TW, const CUtensorMap& tmap, const CombineArgs& a, cudaStream_t s) {
    switch (TW) {
        case 1: return launch_wide<1, GC0>(tmap, a, s);
        case 2: return launch_wide<2, GC0>(tmap, a, s);
        case 4: return launch_wide<4, GC0>(tmap, a, s);
        case 8: return launch_wide<8, GC0>(tmap, a, s);
        default: return cudaErrorInvalidValue;
    }
}

template <int TW>
cudaError_t launch_rj(const uint16_t* branch, int T, int H, const JoinArgs& join, cudaStream_t s) {
    constexpr int NTEAM = kConsumerThreads / (TW * 32);
    int grid = (T + NTEAM - 1) / NTEAM;
    const int cap = device_info().sm_count * 2;
    if (grid > cap) grid = cap;
    cudaLaunchAttribute attr[1];
    cudaLaunchConfig_t cfg = pdl_config(grid, kConsumerThreads, 0, s, attr);
    return cudaLaunchKernelEx(&cfg, residual_join_kernel<TW>, branch, T, H, join);
}

}  // namespace

int team_warps(int H);   // norm_quant.cu

cudaError_t launch_combine(const uint16_t* expert_out, int64_t R, int H, const int32_t* row_idx,
                           const float* wt, int T, int k, const uint16_t* w, float gc, float eps,
                           uint16_t* out, const JoinArgs& join, cudaStream_t s) {
    if (cluster_path(T, H)) return launch_combine_cluster(expert_out, R, H, row_idx, wt, T, k, w, gc, eps, out, join, s);
    const CombineArgs a{expert_out, R, H, row_idx, wt, T, k, w, gc, eps, out, join, 0};
    const int TW = team_warps(H);
    const bool fused = join.residual != nullptr;
    CUtensorMap tmap;
    const bool swz = H % 64 == 0 && R > 0 && static_cast<uint64_t>(R) * (H / 64) < (1ull << 31) &&
                     encode_line_map(&tmap, expert_out, static_cast<uint64_t>(R) * (H / 64),
                                     static_cast<uint32_t>(H / 64));
    if (!swz) std::memset(&tmap, 0, sizeof(tmap));
    if (swz && !fused && H >= 2048) {
        // one 128-byte line per thread: P = next_pow2(H / 64) threads per team
        int P = 32;
        while (P < H / 64) P <<= 1;
        return a.gc == 0.0f ? launch_wide_tw<true>(P / 32, tmap, a, s) : launch_wide_tw<false>(P / 32, tmap, a, s);
    }
    if (swz) return fused ? launch_cb_gc<true, true>(TW, tmap, a, s) : launch_cb_gc<true, false>(TW, tmap, a, s);
    return fused ? launch_cb_gc<false, true>(TW, tmap, a, s) : launch_cb_gc<false, false>(TW, tmap, a, s);
}

cudaError_t launch_residual_join(const uint16_t* branch, int T, int H, const JoinArgs& join,
                                 cudaStream_t s) {
    if (cluster_path(T, H)) return launch_join_cluster(branch, T, H, join, s);
    switch (team_warps(H)) {
        case 1: return launch_rj<1>(branch, T, H, join, s);
        case 2: return launch_rj<2>(branch, T, H, join, s);
        case 4: return launch_rj<4>(branch, T, H, join, s);
        case 8: return launch_rj<8>(branch, T, H, join, s);
        case 16: return launch_rj<16>(branch, T, H, join, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace mb
