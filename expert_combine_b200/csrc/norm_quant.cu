// norm_quant.cu -- stage 2, pre-expert RMSNorm fused with NVFP4 quantisation.
//
// Per token t (vLLM API page "prepare_trtllm_nvfp4": norm_quant_trtllm_nvfp4
// and _quantize_nvfp4_global_scale; TensorRT-LLM PR 21356, "Numerics"):
//   ss   = sum of x^2 in the canonical tree order (see ring.cuh)
//   inv  = 1 / sqrt(ss / H + eps)
//   y_h  = bf16((x_h * (gc + w_h)) * inv)                  one BF16 rounding
//   per block of 16:  amax = max |y|
//                     sf   = e4m3_satfinite(gs * (amax * fl(1/6)))
//                     os   = sf != 0 ? 1 / (sf * (1 / gs)) : 0
//                     code = e2m1_rn_satfinite(y * os), -0 carries no sign
//   packed[t, i] = code(2i) | code(2i + 1) << 4,  sf[t, b] linear [M, H/16]
// The input row is read either contiguous ([M, H]) or from the rank-block
// layout [tp, M, H/tp] (tp copies per row into one slot).
#include "internal.h"
#include "ring.cuh"
#include "route.cuh"
#include "tmap.h"

namespace mb {

struct NormQuantArgs {
    const uint16_t* x;
    int M, H, tp;
    const uint16_t* w;
    float gc, eps;
    const float* gs;
    uint8_t* packed;
    uint8_t* sf;
    int nslot;
};

// The router's arguments when the wide norm-quant kernel also routes its tokens.
struct FusedRouteArgs {
    const float* logits;
    const float* bias;
    const uint8_t* mask;
    int E, k;
    int32_t* ids;
    float* weights;
};

// Router warps added to a wide norm-quant CTA (after its 16 row warps), three
// per SM sub-partition; at 896 threads the kernel fits in 72 registers a
// thread without spilling.
constexpr int kFusedRouterWarps = 12;
constexpr int kTmemReleaseBar = 15;       // named barrier of the row warps at the end (teams use 1..8)
// The router warps use the small selection path with 8 scores per lane.
constexpr int kFusedRouteMaxExperts = 256;

template <int TW, bool SWZ, bool GC0>
__global__ void __launch_bounds__(kConsumerThreads, 1)
    norm_quant_kernel(const __grid_constant__ CUtensorMap tmap, const NormQuantArgs a) {
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
        for (int i = 0; i < NTEAM * nslot; ++i) mbar_init(&bars[i], 1);   // one arrive + the bytes
        for (int i = 0; i < NTEAM; ++i) abort_all[4 * i] = 0;
        fence_mbar_init();
    }
    __syncthreads();
    griddep_wait();     // inputs may come from the previous kernel on the stream
    griddep_launch();   // the next kernel may start its prologue as CTAs retire

    const int M = a.M;
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

    // ---- the leader's copy cursor: one row (tp segments) per token
    const int hs = H / a.tp;
    const uint32_t seg_bytes = 2u * static_cast<uint32_t>(hs);
    const int seg_lines = hs / 64;
    RingCursor* cur = reinterpret_cast<RingCursor*>(smem + lay.cursor_offset()) + team;
    auto issue = [&]() {
        const int nt = cur->ct;
        if (nt >= M) return;
        const int ws = cur->wslot;
        mbar_arrive_expect_tx(&tb[ws], 2u * static_cast<uint32_t>(H));
        uint8_t* dst = ring + static_cast<size_t>(ws) * slot_bytes;
        for (int s = 0; s < a.tp; ++s) {
            if constexpr (SWZ)
                tma_load_2d(smem_addr(dst + static_cast<size_t>(s) * seg_bytes), &tmap, 0,
                            (s * M + nt) * seg_lines, &tb[ws]);
            else
                bulk_g2s(dst + static_cast<size_t>(s) * seg_bytes,
                         a.x + (static_cast<size_t>(s) * M + nt) * hs, seg_bytes, &tb[ws]);
        }
        cur->ct = nt + team_stride;
        cur->issued += 1;
        cur->wslot = (ws + 1 == nslot) ? 0 : ws + 1;
    };
    if (tid == 0) {
        *cur = RingCursor{static_cast<int>(blockIdx.x) * NTEAM + team, 0, 0, 0, 0, 0, 0, 0};
        for (int i = 0; i < nslot; ++i) issue();
    }

    // gain: with GC0 the packed BF16 weights (x * w formed exactly by a
    // mixed-precision FMA), else FP32 pairs gc + w
    uint32_t wp[16];
    float2 g[16];
    if constexpr (GC0) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (c / 2 < nvalid) v = *reinterpret_cast<const uint4*>(a.w + 32 * tid + 8 * c);
            wp[4 * c] = v.x;
            wp[4 * c + 1] = v.y;
            wp[4 * c + 2] = v.z;
            wp[4 * c + 3] = v.w;
        }
    } else {
        load_gain32(a.w, a.gc, tid, nvalid, g);
    }
    const float gs = __ldg(a.gs);
    const float rgs = __frcp_rn(gs);
    constexpr float kR6 = (float)(1.0 / 6.0);
    const float fH = static_cast<float>(H);
    const bool pow2 = (H & (H - 1)) == 0;
    const float rH = pow2 ? __frcp_rn(fH) : 0.0f;
    const float2 zero2 = make_float2(0.0f, 0.0f);

    int slot = 0, phase = 0;
    for (int t = blockIdx.x * NTEAM + team; t < M; t += team_stride) {
        const bool ok = mbar_wait_bounded(&tb[slot], phase, 4u);
        uint32_t wv[16];
        if (ok) {
            read_row32<SWZ>(ring_saddr + static_cast<uint32_t>(slot * slot_bytes), tid, nvalid, wv);
        } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) wv[i] = 0u;
        }
        bool abort;
        const float ss = team_sum(row32_sumsq(wv), !ok, abort);
        if (abort) break;
        if (tid == 0) {   // the whole team has read this slot: refill it
            cur->consumed += 1;
            fence_proxy_async_smem();
            issue();
        }
        if (++slot == nslot) {
            slot = 0;
            phase ^= 1;
        }

        const float inv = inv_rms_h(ss, fH, rH, pow2, a.eps);
        const float2 inv2 = make_float2(inv, inv);
#pragma unroll
        for (int b = 0; b < 2; ++b) {
            if (b < nvalid) {
                uint32_t yw[8];
                uint32_t m = 0u;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float2 xg = GC0 ? mul_bf16x2_exact(wv[8 * b + i], wp[8 * b + i])
                                          : mul2(unpack_bf16x2(wv[8 * b + i]), g[8 * b + i]);
                    const float2 t2 = mul2(xg, inv2);
                    yw[i] = pack_bf16x2_rn(t2);
                    m = maxabs_bf16x2(m, yw[i]);
                }
                const float2 mf = unpack_bf16x2(m & 0x7fff7fffu);
                const float amax = fmaxf(mf.x, mf.y);
                const uint32_t sfc = cvt_e4m3_satfinite(__fmul_rn(gs, __fmul_rn(amax, kR6)));
                const float sf_f = e4m3_to_f32(sfc);
                const float os = (sf_f != 0.0f) ? __frcp_rn(__fmul_rn(sf_f, rgs)) : 0.0f;
                const float2 os2 = make_float2(os, os);
                float q[16];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    // y * os + 0 in one rounding: a -0 product becomes +0 (no sign
                    // bit for -0), any other product is rounded once as by a multiply
                    const float2 q2 = fma2(unpack_bf16x2(yw[i]), os2, zero2);
                    q[2 * i] = q2.x;
                    q[2 * i + 1] = q2.y;
                }
                uint2 codes;
                codes.x = cvt_e2m1x8(q);
                codes.y = cvt_e2m1x8(q + 8);
                const int gb = 2 * tid + b;
                *reinterpret_cast<uint2*>(a.packed + static_cast<size_t>(t) * (H / 2) + 8 * gb) = codes;
                a.sf[static_cast<size_t>(t) * nblocks + gb] = static_cast<uint8_t>(sfc);
            }
        }
    }
    // copies still in flight (only after an abort) land before the CTA exits
    if (tid == 0)
        for (int f = cur->consumed; f < cur->issued; ++f)
            mbar_wait_bounded(&tb[f % nslot], (f / nslot) & 1, 2u);
}

// ---------------------------------------------------------------------------
// Wide-row norm-quant (H >= 2048, H % 64 == 0, tensor-map copies): thread t of
// a team owns the 128-byte line t of every row (four 16-element blocks) and
// keeps its 32 words in registers across the team barrier, so the slot is
// refilled as soon as the barrier has passed.  The packed BF16 weights sit in
// a shared-memory table read without bank conflicts, or with ROUTE in tensor
// memory (below).
//
// ROUTE: the CTA carries router warps after its row warps; they route the same
// M tokens (one per warp iteration, statically interleaved over the grid's
// router warps) in the issue slots and registers the streaming row warps
// leave free, so the latency-bound router adds little to the bandwidth-bound
// norm-quant.  The router warps touch no shared memory and no barrier after
// the CTA's set-up.
template <int TW, bool GC0, bool ROUTE>
__global__ void __launch_bounds__(kConsumerThreads + (ROUTE ? 32 * kFusedRouterWarps : 0), 1)
    norm_quant_wide_kernel(const __grid_constant__ CUtensorMap tmap, const NormQuantArgs a,
                           const FusedRouteArgs ra) {
    constexpr int P = TW * 32;
    constexpr int NTEAM = kConsumerThreads / P;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_saddr = smem_addr(smem_raw);
    uint8_t* smem = smem_raw + (((raw_saddr + kSlotAlign - 1) & ~uint32_t(kSlotAlign - 1)) - raw_saddr);
    const int H = a.H;
    const int nslot = a.nslot;
    const int slot_bytes = slot_bytes_for(H);
    const WideLayout lay{NTEAM, nslot, slot_bytes, P};
    uint4* wtab = reinterpret_cast<uint4*>(smem + lay.wtab_offset());   // used without the router warps
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
    // The packed BF16 norm weights: alone, the kernel reads them from a
    // shared-memory table (chunk c of line t at [c][t]); with the router warps
    // they sit in tensor memory instead and each block's eight words are
    // fetched with tcgen05.ld, which leaves the shared-memory port to the rows
    // (40.4 against 41.4 us for the fused call at 8192 x 8192; the table in
    // tensor memory or in registers made the kernel alone slower, 35.4 against
    // 34.4 us).
    using WTab = WideWeightTable<TW, false>;
    __shared__ uint32_t s_tmem;
    if (ROUTE && warp == 0) {
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
    griddep_wait();     // inputs may come from the previous kernel on the stream
    griddep_launch();

    const int M = a.M;
    const int team_stride = gridDim.x * NTEAM;
    uint8_t* ring = smem + static_cast<size_t>(team) * nslot * slot_bytes;
    const uint32_t ring_saddr = smem_addr(ring);
    const uint32_t wtab_saddr = smem_addr(wtab);
    uint64_t* tb = bars + static_cast<size_t>(team) * nslot;
    int* abort_word = abort_all + 4 * team;
    float* part = part_all + team * 2 * TW;

    // ---- the leader's copy cursor: one row (tp segments) per token
    const int hs = H / a.tp;
    const int seg_lines = hs / 64;
    RingCursor* cur = reinterpret_cast<RingCursor*>(smem + lay.cursor_offset()) + team;
    auto issue = [&]() {
        const int nt = cur->ct;
        if (nt >= M) return;
        const int ws = cur->wslot;
        mbar_arrive_expect_tx(&tb[ws], 2u * static_cast<uint32_t>(H));
        uint8_t* dst = ring + static_cast<size_t>(ws) * slot_bytes;
        for (int s = 0; s < a.tp; ++s)
            tma_load_2d(smem_addr(dst + static_cast<size_t>(s) * 2 * hs), &tmap, 0, (s * M + nt) * seg_lines,
                        &tb[ws]);
        cur->ct = nt + team_stride;
        cur->issued += 1;
        cur->wslot = (ws + 1 == nslot) ? 0 : ws + 1;
    };
    // the row warps' leaders start their copies before the tables below are filled
    if (warp < NTEAM * TW && tid == 0) {
        *cur = RingCursor{static_cast<int>(blockIdx.x) * NTEAM + team, 0, 0, 0, 0, 0, 0, 0};
        for (int i = 0; i < nslot; ++i) issue();
    }
    if constexpr (ROUTE) {
        if (warp < 4) WTab::fill(s_tmem, warp, lane, a.w, 0.0f, lines);
    } else if (team == 0) {
#pragma unroll
        for (int c = 0; c < 8; ++c)
            wtab[c * P + tid] = has_line ? *reinterpret_cast<const uint4*>(a.w + 64 * tid + 8 * c)
                                         : make_uint4(0u, 0u, 0u, 0u);
    }
    // The output scale of each of the 256 E4M3 block-scale codes, 1 / (sf * (1 /
    // gs)) (0 where sf is 0), formed once per CTA with the same roundings as
    // per block: one shared-memory load per block instead of the decode, the
    // product and the IEEE reciprocal.  It pays where the kernel is issue-bound
    // (with the router warps: 40.6 -> 38.9 us at 8192 x 8192; with a gain
    // centre: 37.0 -> 35.7 us) and not alone with a zero centre (34.2 -> 35.0 us).
    constexpr bool kOsTable = ROUTE || !GC0;
    __shared__ float os_tab[kOsTable ? 256 : 1];
    if (kOsTable && threadIdx.x < 256) {
        const float sfv = e4m3_to_f32(threadIdx.x);
        os_tab[threadIdx.x] = (sfv != 0.0f) ? __frcp_rn(__fmul_rn(sfv, __frcp_rn(__ldg(a.gs)))) : 0.0f;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if constexpr (ROUTE) {
        constexpr int RW = kFusedRouterWarps;
        if (warp >= NTEAM * TW) {
            route_singles<8, false>(ra.logits, ra.bias, ra.mask, a.M, ra.E, ra.k, ra.ids, ra.weights,
                           static_cast<int>(blockIdx.x) * RW + (warp - NTEAM * TW),
                           static_cast<int>(gridDim.x) * RW, lane);
            return;
        }
    }

    const uint32_t wt_taddr = ROUTE ? WTab::line_addr(s_tmem, warp, warp_in_team) : 0u;

    const float gs = __ldg(a.gs);
    const float rgs = __frcp_rn(gs);
    constexpr float kR6 = (float)(1.0 / 6.0);
    const float fH = static_cast<float>(H);
    const bool pow2 = (H & (H - 1)) == 0;
    const float rH = pow2 ? __frcp_rn(fH) : 0.0f;
    const float2 zero2 = make_float2(0.0f, 0.0f);
    const float2 gc2 = make_float2(a.gc, a.gc);
    const uint32_t line_off = 128u * static_cast<uint32_t>(tid);
    const int sw = tid & 7;
    const int nblocks = H / 16;

    int slot = 0, phase = 0, pbuf = 0;
    for (int t = blockIdx.x * NTEAM + team; t < M; t += team_stride) {
        const bool ok = mbar_wait_bounded(&tb[slot], phase, 4u);
        uint32_t wv[32];
        float b[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        const uint32_t sbase = ring_saddr + static_cast<uint32_t>(slot * slot_bytes) + line_off;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (ok && has_line) v = lds128(sbase + 16u * static_cast<uint32_t>(c ^ sw));
            wv[4 * c] = v.x;
            wv[4 * c + 1] = v.y;
            wv[4 * c + 2] = v.z;
            wv[4 * c + 3] = v.w;
        }
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            float& acc_b = b[c >> 1];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                acc_b = fma_bf16_lo(wv[4 * c + q], wv[4 * c + q], acc_b);
                acc_b = fma_bf16_hi(wv[4 * c + q], wv[4 * c + q], acc_b);
            }
        }
        if (!ok) *reinterpret_cast<volatile int*>(abort_word) = 1;
        const float v = warp_tree_sum((b[0] + b[1]) + (b[2] + b[3]));
        if (lane == 0) part[pbuf * TW + warp_in_team] = v;
        if constexpr (TW == 1) __syncwarp();
        else named_bar_sync(1 + team, P);
        if (*reinterpret_cast<volatile int*>(abort_word) != 0) break;
        if (tid == 0) {   // the row is in every thread's registers: refill the slot
            cur->consumed += 1;
            fence_proxy_async_smem();
            issue();
        }
        if (++slot == nslot) {
            slot = 0;
            phase ^= 1;
        }
        float pp[TW];
#pragma unroll
        for (int i = 0; i < TW; ++i) pp[i] = part[pbuf * TW + i];
        pbuf ^= 1;
        const float inv = inv_rms_h(tree_sum_array<TW>(pp), fH, rH, pow2, a.eps);
        const float2 inv2 = make_float2(inv, inv);
        if (ROUTE ? warp_has_line : has_line) {    // with the router warps every lane of the warp reads the table
        uint32_t codes[8];
        uint32_t sfw = 0u;
#pragma unroll
        for (int blk = 0; blk < 4; ++blk) {
            uint32_t ws[8];
            if constexpr (ROUTE) {
                tmem_ld8_ro(wt_taddr + 8u * static_cast<uint32_t>(blk), ws);
            } else {
                const uint4 w0 = lds128(wtab_saddr + 16u * static_cast<uint32_t>((2 * blk) * P + tid));
                const uint4 w1 = lds128(wtab_saddr + 16u * static_cast<uint32_t>((2 * blk + 1) * P + tid));
                ws[0] = w0.x;
                ws[1] = w0.y;
                ws[2] = w0.z;
                ws[3] = w0.w;
                ws[4] = w1.x;
                ws[5] = w1.y;
                ws[6] = w1.z;
                ws[7] = w1.w;
            }
            uint32_t yw[8];
            uint32_t m = 0u;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const uint32_t xw = wv[8 * blk + i];
                const float2 xg = GC0 ? mul_bf16x2_exact(xw, ws[i])
                                      : mul2(unpack_bf16x2(xw), add2(gc2, unpack_bf16x2(ws[i])));
                yw[i] = pack_bf16x2_rn(mul2(xg, inv2));
                m = maxabs_bf16x2(m, yw[i]);
            }
            const float2 mf = unpack_bf16x2(m & 0x7fff7fffu);
            const float amax = fmaxf(mf.x, mf.y);
            const uint32_t sfc = cvt_e4m3_satfinite(__fmul_rn(gs, __fmul_rn(amax, kR6)));
            float os;
            if constexpr (kOsTable) {
                os = os_tab[sfc];
            } else {
                const float sf_f = e4m3_to_f32(sfc);
                os = (sf_f != 0.0f) ? __frcp_rn(__fmul_rn(sf_f, rgs)) : 0.0f;
            }
            const float2 os2 = make_float2(os, os);
            float q[16];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float2 q2 = fma2(unpack_bf16x2(yw[i]), os2, zero2);   // -0 -> +0, one rounding
                q[2 * i] = q2.x;
                q[2 * i + 1] = q2.y;
            }
            codes[2 * blk] = cvt_e2m1x8(q);
            codes[2 * blk + 1] = cvt_e2m1x8(q + 8);
            sfw |= sfc << (8 * blk);
        }
        if (has_line) {
            uint8_t* prow = a.packed + static_cast<size_t>(t) * (H / 2) + 32 * tid;
            *reinterpret_cast<uint4*>(prow) = make_uint4(codes[0], codes[1], codes[2], codes[3]);
            *reinterpret_cast<uint4*>(prow + 16) = make_uint4(codes[4], codes[5], codes[6], codes[7]);
            *reinterpret_cast<uint32_t*>(a.sf + static_cast<size_t>(t) * nblocks + 4 * tid) = sfw;
        }
        }
    }
    if (tid == 0)
        for (int f = cur->consumed; f < cur->issued; ++f)
            mbar_wait_bounded(&tb[f % nslot], (f / nslot) & 1, 2u);
    if constexpr (ROUTE) {
        // the row warps (the router warps have left) release the weight table
        // once every row warp's last read of it is done
        tc_fence_before();
        named_bar_sync(kTmemReleaseBar, NTEAM * P);
        if (warp == 0) {
            tc_fence_after();
            tmem_dealloc(s_tmem, WTab::kCols);
        }
    }
}

namespace {

template <int TW, bool SWZ, bool GC0>
cudaError_t launch_nq(const CUtensorMap& tmap, const NormQuantArgs& args, cudaStream_t s) {
    constexpr int NTEAM = kConsumerThreads / (TW * 32);
    const int slot_bytes = slot_bytes_for(args.H);
    int nslot = kRingBytes / (NTEAM * slot_bytes);
    if (nslot > 16) nslot = 16;
    if (nslot < 2) return cudaErrorInvalidConfiguration;
    NormQuantArgs a = args;
    a.nslot = nslot;
    const RingLayout lay{NTEAM, nslot, slot_bytes, TW};
    const size_t smem = lay.total_bytes();
    auto kern = norm_quant_kernel<TW, SWZ, GC0>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    int grid = (a.M + NTEAM - 1) / NTEAM;
    const int cap = device_info().sm_count;
    if (grid > cap) grid = cap;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kConsumerThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, tmap, a);
}

template <bool SWZ, bool GC0>
cudaError_t launch_nq_tw(int TW, const CUtensorMap& tmap, const NormQuantArgs& a, cudaStream_t s) {
    switch (TW) {
        case 1: return launch_nq<1, SWZ, GC0>(tmap, a, s);
        case 2: return launch_nq<2, SWZ, GC0>(tmap, a, s);
        case 4: return launch_nq<4, SWZ, GC0>(tmap, a, s);
        case 8: return launch_nq<8, SWZ, GC0>(tmap, a, s);
        case 16: return launch_nq<16, SWZ, GC0>(tmap, a, s);
        default: return cudaErrorInvalidValue;
    }
}

template <int TW, bool GC0, bool ROUTE>
cudaError_t launch_nq_wide(const CUtensorMap& tmap, const NormQuantArgs& args, const FusedRouteArgs& ra,
                           cudaStream_t s) {
    constexpr int P = TW * 32;
    constexpr int NTEAM = kConsumerThreads / P;
    const int slot_bytes = slot_bytes_for(args.H);
    WideLayout lay{NTEAM, 1, slot_bytes, P};
    const size_t fixed = lay.total_bytes() - static_cast<size_t>(NTEAM) * slot_bytes;
    cudaFuncAttributes fa{};   // the kernel's static shared memory counts against the same limit
    cudaError_t fe = cudaFuncGetAttributes(&fa, norm_quant_wide_kernel<TW, GC0, ROUTE>);
    if (fe != cudaSuccess) return fe;
    const int avail = device_info().max_smem_optin - static_cast<int>(fixed) - static_cast<int>(fa.sharedSizeBytes) -
                      64 * NTEAM;
    int nslot = avail / (NTEAM * slot_bytes);
    if (nslot > 16) nslot = 16;
    if (nslot < 2) return cudaErrorInvalidConfiguration;
    lay.nslot = nslot;
    NormQuantArgs a = args;
    a.nslot = nslot;
    const size_t smem = lay.total_bytes();
    auto kern = norm_quant_wide_kernel<TW, GC0, ROUTE>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    int grid = (a.M + NTEAM - 1) / NTEAM;
    const int cap = device_info().sm_count;
    if (grid > cap) grid = cap;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kConsumerThreads + (ROUTE ? 32 * kFusedRouterWarps : 0));
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, tmap, a, ra);
}

template <bool GC0, bool ROUTE>
cudaError_t launch_nq_wide_tw(int TW, const CUtensorMap& tmap, const NormQuantArgs& a, const FusedRouteArgs& ra,
                              cudaStream_t s) {
    switch (TW) {
        case 1: return launch_nq_wide<1, GC0, ROUTE>(tmap, a, ra, s);
        case 2: return launch_nq_wide<2, GC0, ROUTE>(tmap, a, ra, s);
        case 4: return launch_nq_wide<4, GC0, ROUTE>(tmap, a, ra, s);
        case 8: return launch_nq_wide<8, GC0, ROUTE>(tmap, a, ra, s);
        default: return cudaErrorInvalidValue;
    }
}

template <bool ROUTE>
cudaError_t launch_nq_wide_gc(int TW, const CUtensorMap& tmap, const NormQuantArgs& a, const FusedRouteArgs& ra,
                              cudaStream_t s) {
    return a.gc == 0.0f ? launch_nq_wide_tw<true, ROUTE>(TW, tmap, a, ra, s)
                        : launch_nq_wide_tw<false, ROUTE>(TW, tmap, a, ra, s);
}

// gc == +0 or -0: the gain is the BF16 weight itself (0 + w == w exactly)
template <bool SWZ>
cudaError_t launch_nq_gc(int TW, const CUtensorMap& tmap, const NormQuantArgs& a, cudaStream_t s) {
    return a.gc == 0.0f ? launch_nq_tw<SWZ, true>(TW, tmap, a, s) : launch_nq_tw<SWZ, false>(TW, tmap, a, s);
}

}  // namespace

// Warps per team: 32 elements per thread, P = next_pow2(H / 32) threads (at
// least one warp).
int team_warps(int H) {
    const int nblocks = H / 16;
    const int per = (nblocks + 1) / 2;
    int P = 32;
    while (P < per) P <<= 1;
    return P / 32;
}

namespace {

// The sizes the wide tensor-map norm-quant path takes.
bool wide_nq_sizes(int M, int H, int tp) {
    const int hs = H / tp;
    return (hs % 64 == 0) && (tp == 1 || (2 * hs) % kSlotAlign == 0) &&
           static_cast<uint64_t>(M) * tp * (hs / 64) < (1ull << 31) && H >= 2048;
}

// Tensor map and team width of the norm-quant row copies; false when the
// wide tensor-map path does not apply.
bool wide_nq_plan(const uint16_t* x, int M, int H, int tp, CUtensorMap& tmap, int& TW) {
    const int hs = H / tp;
    if (!wide_nq_sizes(M, H, tp)) return false;
    if (!encode_line_map(&tmap, x, static_cast<uint64_t>(M) * tp * (hs / 64), static_cast<uint32_t>(hs / 64)))
        return false;
    int P = 32;
    while (P < H / 64) P <<= 1;
    TW = P / 32;
    return true;
}

}  // namespace

cudaError_t launch_norm_quant(const uint16_t* x, int M, int H, int tp, const uint16_t* w, float gc,
                              float eps, const float* gs, uint8_t* packed, uint8_t* sf,
                              cudaStream_t s) {
    NormQuantArgs a{x, M, H, tp, w, gc, eps, gs, packed, sf, 0};
    CUtensorMap tmap;
    int TW = 0;
    if (wide_nq_plan(x, M, H, tp, tmap, TW)) return launch_nq_wide_gc<false>(TW, tmap, a, FusedRouteArgs{}, s);
    const int hs = H / tp;
    const bool swz = (hs % 64 == 0) && (tp == 1 || (2 * hs) % kSlotAlign == 0) &&
                     static_cast<uint64_t>(M) * tp * (hs / 64) < (1ull << 31);
    if (swz && encode_line_map(&tmap, x, static_cast<uint64_t>(M) * tp * (hs / 64),
                               static_cast<uint32_t>(hs / 64)))
        return launch_nq_gc<true>(team_warps(H), tmap, a, s);
    std::memset(&tmap, 0, sizeof(tmap));
    return launch_nq_gc<false>(team_warps(H), tmap, a, s);
}

bool route_beside_norm_quant(int M) { return M <= device_info().sm_count * kRouteBesideTokensPerSM; }

int route_norm_quant_kernels(int M, int H, int tp, int E) {
    if (route_beside_norm_quant(M)) return 2;
    return (E <= kFusedRouteMaxExperts && wide_nq_sizes(M, H, tp)) ? 1 : 2;
}

cudaError_t launch_route_norm_quant(const float* logits, const float* bias, const uint8_t* mask, int E, int k,
                                    int32_t* ids, float* weights, const uint16_t* x, int M, int H, int tp,
                                    const uint16_t* w, float gc, float eps, const float* gs, uint8_t* packed,
                                    uint8_t* sf, cudaStream_t s) {
    // The norm-quant is streaming-bound and holds each SM's shared memory
    // and most of its registers; the router is latency-bound, needs little of
    // either, but wants many warps in flight.  When its tokens fit one wave of
    // the warp slots a norm-quant CTA leaves free (three 2-warp CTAs per SM,
    // one token per warp), the norm-quant goes first and the router follows
    // beside it (programmatic dependent launch lets it start as soon as the
    // norm-quant kernel is running).  Larger batches on the wide norm-quant
    // path (E <= 256) route in extra warps of the norm-quant kernel itself;
    // the rest run the router first with every warp slot, then the norm-quant.
    if (route_beside_norm_quant(M)) {
        cudaError_t e = launch_norm_quant(x, M, H, tp, w, gc, eps, gs, packed, sf, s);
        if (e != cudaSuccess) return e;
        return launch_route_beside(logits, bias, mask, M, E, k, ids, weights, s);
    }
    CUtensorMap tmap;
    int TW = 0;
    if (E <= kFusedRouteMaxExperts && wide_nq_plan(x, M, H, tp, tmap, TW)) {
        const NormQuantArgs a{x, M, H, tp, w, gc, eps, gs, packed, sf, 0};
        const FusedRouteArgs ra{logits, bias, mask, E, k, ids, weights};
        return launch_nq_wide_gc<true>(TW, tmap, a, ra, s);
    }
    cudaError_t e = launch_route(logits, bias, mask, M, E, k, ids, weights, s);
    if (e != cudaSuccess) return e;
    return launch_norm_quant(x, M, H, tp, w, gc, eps, gs, packed, sf, s);
}

}  // namespace mb
