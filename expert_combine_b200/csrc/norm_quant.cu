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
// layout [tp, M, H/tp] (tp bulk copies per row into one slot).
#include "internal.h"
#include "ring.cuh"

namespace mb {

template <int B, int TW>
__global__ void __launch_bounds__(kConsumerThreads + 32, 1)
    norm_quant_kernel(const uint16_t* __restrict__ x, int M, int H, int tp,
                      const uint16_t* __restrict__ w, float gc, float eps,
                      const float* __restrict__ gs_ptr, uint8_t* __restrict__ packed,
                      uint8_t* __restrict__ sf_out, int nslot) {
    constexpr int NTEAM = kConsumerThreads / (TW * 32);
    extern __shared__ __align__(128) uint8_t smem[];
    const int slot_bytes = 2 * H;
    const RingLayout lay{NTEAM, nslot, slot_bytes, TW};
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + lay.bars_offset());
    float* red_all = reinterpret_cast<float*>(smem + lay.red_offset());
    int* flags_all = reinterpret_cast<int*>(red_all + NTEAM * 2 * TW);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int i = 0; i < NTEAM * nslot; ++i) {
            mbar_init(&bars[2 * i], 1);       // full: producer's arrive + bytes
            mbar_init(&bars[2 * i + 1], 1);   // empty: one consumer arrive
        }
        fence_mbar_init();
    }
    __syncthreads();

    const int team_stride = gridDim.x * NTEAM;

    if (warp == NTEAM * TW) {
        // ---------------- producer: lane `team` feeds that team's ring
        if (lane < NTEAM) {
            const int team = lane;
            uint8_t* ring = smem + static_cast<size_t>(team) * nslot * slot_bytes;
            uint64_t* tb = bars + static_cast<size_t>(team) * nslot * 2;
            const int hs = H / tp;
            const uint32_t seg_bytes = 2u * static_cast<uint32_t>(hs);
            int fills = 0;
            for (int t = blockIdx.x * NTEAM + team; t < M; t += team_stride) {
                const int slot = fills % nslot;
                const int use = fills / nslot;
                if (use > 0 && !mbar_wait_bounded(&tb[2 * slot + 1], (use - 1) & 1, 1u)) break;
                mbar_arrive_expect_tx(&tb[2 * slot], static_cast<uint32_t>(slot_bytes));
                uint8_t* dst = ring + static_cast<size_t>(slot) * slot_bytes;
                for (int s = 0; s < tp; ++s)
                    bulk_g2s(dst + static_cast<size_t>(s) * seg_bytes,
                             x + (static_cast<size_t>(s) * M + t) * hs, seg_bytes, &tb[2 * slot]);
                ++fills;
            }
            // drain: every issued copy has landed before the CTA exits
            for (int f = fills > nslot ? fills - nslot : 0; f < fills; ++f)
                mbar_wait_bounded(&tb[2 * (f % nslot)], (f / nslot) & 1, 2u);
        }
        return;
    }

    // ---------------- consumers
    const int team = warp / TW;
    const int warp_in_team = warp % TW;
    const int tid = warp_in_team * 32 + lane;
    const int nblocks = H / 16;
    int nvalid = nblocks - tid * B;
    nvalid = nvalid < 0 ? 0 : (nvalid > B ? B : nvalid);
    const uint8_t* ring = smem + static_cast<size_t>(team) * nslot * slot_bytes;
    uint64_t* tb = bars + static_cast<size_t>(team) * nslot * 2;
    TeamSum<TW> team_sum{red_all + team * 2 * TW, flags_all + team * 2 * TW, 1 + team, warp_in_team,
                         lane, 0};

    float g[16 * B];
#pragma unroll
    for (int i = 0; i < 16 * B; ++i) {
        const int h = 16 * B * tid + i;
        g[i] = (i / 16 < nvalid) ? __fadd_rn(gc, __uint_as_float(static_cast<uint32_t>(w[h]) << 16)) : 0.0f;
    }
    const float gs = __ldg(gs_ptr);
    const float rgs = __frcp_rn(gs);
    constexpr float kR6 = (float)(1.0 / 6.0);
    const float fH = static_cast<float>(H);

    int fills = 0;
    for (int t = blockIdx.x * NTEAM + team; t < M; t += team_stride) {
        const int slot = fills % nslot;
        const bool ok = mbar_wait_bounded(&tb[2 * slot], (fills / nslot) & 1, 4u);
        uint32_t wv[8 * B];
        if (ok) {
            read_slot_blocks<B>(ring + static_cast<size_t>(slot) * slot_bytes, tid, nvalid, wv);
        } else {
#pragma unroll
            for (int i = 0; i < 8 * B; ++i) wv[i] = 0u;
        }
        float xv[16 * B];
#pragma unroll
        for (int i = 0; i < 8 * B; ++i) {
            xv[2 * i] = bf16_lo(wv[i]);
            xv[2 * i + 1] = bf16_hi(wv[i]);
        }
        float part[B];
#pragma unroll
        for (int b = 0; b < B; ++b) part[b] = block_sumsq16(xv + 16 * b);
        bool abort;
        const float ss = team_sum(tree_sum_array<B>(part), !ok, abort);
        if (abort) break;
        if (tid == 0) mbar_arrive(&tb[2 * slot + 1]);
        ++fills;

        const float inv = inv_rms(ss, fH, eps);
#pragma unroll
        for (int b = 0; b < B; ++b) {
            if (b < nvalid) {
                float y[16];
                float amax = 0.0f;
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    y[i] = round_bf16(__fmul_rn(__fmul_rn(xv[16 * b + i], g[16 * b + i]), inv));
                    amax = fmaxf(amax, fabsf(y[i]));
                }
                const uint32_t sfc = cvt_e4m3_satfinite(__fmul_rn(gs, __fmul_rn(amax, kR6)));
                const float sf_f = e4m3_to_f32(sfc);
                const float os = (sf_f != 0.0f) ? __frcp_rn(__fmul_rn(sf_f, rgs)) : 0.0f;
                float q[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) q[i] = __fmul_rn(y[i], os);
                uint2 codes;
                codes.x = cvt_e2m1x8(q);
                codes.y = cvt_e2m1x8(q + 8);
                const int gb = tid * B + b;
                *reinterpret_cast<uint2*>(packed + static_cast<size_t>(t) * (H / 2) + 8 * gb) = codes;
                sf_out[static_cast<size_t>(t) * nblocks + gb] = static_cast<uint8_t>(sfc);
            }
        }
    }
}

namespace {

template <int B, int TW>
cudaError_t launch_nq(const uint16_t* x, int M, int H, int tp, const uint16_t* w, float gc, float eps,
                      const float* gs, uint8_t* packed, uint8_t* sf, cudaStream_t s) {
    constexpr int NTEAM = kConsumerThreads / (TW * 32);
    const int slot_bytes = 2 * H;
    int nslot = kRingBytes / (NTEAM * slot_bytes);
    if (nslot > 16) nslot = 16;
    if (nslot < 2) return cudaErrorInvalidConfiguration;
    const RingLayout lay{NTEAM, nslot, slot_bytes, TW};
    const size_t smem = lay.total_bytes();
    auto kern = norm_quant_kernel<B, TW>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    int grid = (M + NTEAM - 1) / NTEAM;
    const int cap = device_info().sm_count;
    if (grid > cap) grid = cap;
    kern<<<grid, kConsumerThreads + 32, smem, s>>>(x, M, H, tp, w, gc, eps, gs, packed, sf, nslot);
    return cudaGetLastError();
}

}  // namespace

// Team width from the row size: B blocks per thread, P = next_pow2(blocks/B)
// threads per team (at least one warp).
cudaError_t launch_norm_quant(const uint16_t* x, int M, int H, int tp, const uint16_t* w, float gc,
                              float eps, const float* gs, uint8_t* packed, uint8_t* sf,
                              cudaStream_t s) {
    const int nblocks = H / 16;
    const int B = nblocks <= 512 ? 1 : 2;
    int per = (nblocks + B - 1) / B;
    int P = 32;
    while (P < per) P <<= 1;
    const int TW = P / 32;
#define MB_NQ(Bv, TWv) \
    if (B == Bv && TW == TWv) return launch_nq<Bv, TWv>(x, M, H, tp, w, gc, eps, gs, packed, sf, s);
    MB_NQ(1, 1) MB_NQ(1, 2) MB_NQ(1, 4) MB_NQ(1, 8) MB_NQ(1, 16)
    MB_NQ(2, 16)
#undef MB_NQ
    return cudaErrorInvalidValue;
}

}  // namespace mb
