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

namespace mb {

// Join epilogue for one token: this thread holds 16 B branch values of the
// row (BF16-exact floats in br[]).  Uses two or three team sums.
template <int B, int TW>
__device__ __forceinline__ void join_token(const float (&br)[16 * B], int t, int H, int tid, int nvalid,
                                           const JoinArgs& j, const float (&gain)[16 * B],
                                           const float (&g2)[16 * B], TeamSum<TW>& team_sum) {
    float* rrow = j.residual + static_cast<size_t>(t) * H + 16 * B * tid;
    float r[16 * B];
#pragma unroll
    for (int b = 0; b < B; ++b) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (b < nvalid) v = *reinterpret_cast<const float4*>(rrow + 16 * b + 4 * q);
            r[16 * b + 4 * q + 0] = v.x;
            r[16 * b + 4 * q + 1] = v.y;
            r[16 * b + 4 * q + 2] = v.z;
            r[16 * b + 4 * q + 3] = v.w;
        }
    }
    float gg[16 * B];
#pragma unroll
    for (int i = 0; i < 16 * B; ++i) gg[i] = round_bf16(__fmul_rn(gain[i], br[i]));
    float part[B];
#pragma unroll
    for (int b = 0; b < B; ++b) part[b] = block_sumsq16(gg + 16 * b);
    bool abort;
    const float ss_g = team_sum(tree_sum_array<B>(part), false, abort);
    const float inv_g = inv_rms(ss_g, static_cast<float>(H), j.eps);
#pragma unroll
    for (int i = 0; i < 16 * B; ++i) {
        const float n = round_bf16(__fmul_rn(gg[i], inv_g));
        r[i] = __fadd_rn(__fmul_rn(j.alpha, r[i]), __fmul_rn(j.beta, n));
    }
#pragma unroll
    for (int b = 0; b < B; ++b) {
        if (b < nvalid) {
#pragma unroll
            for (int q = 0; q < 4; ++q)
                *reinterpret_cast<float4*>(rrow + 16 * b + 4 * q) =
                    make_float4(r[16 * b + 4 * q], r[16 * b + 4 * q + 1], r[16 * b + 4 * q + 2],
                                r[16 * b + 4 * q + 3]);
        }
    }
    if (j.next_w != nullptr) {
#pragma unroll
        for (int b = 0; b < B; ++b) part[b] = (b < nvalid) ? block_sumsq16(r + 16 * b) : 0.0f;
        const float ss_r = team_sum(tree_sum_array<B>(part), false, abort);
        const float inv_r = inv_rms(ss_r, static_cast<float>(H), j.next_eps);
        uint16_t* prow = j.next_prenorm + static_cast<size_t>(t) * H + 16 * B * tid;
#pragma unroll
        for (int b = 0; b < B; ++b) {
            if (b < nvalid) {
                uint32_t pk[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int e = 16 * b + 2 * i;
                    pk[i] = pack_bf16x2(__fmul_rn(__fmul_rn(r[e], g2[e]), inv_r),
                                        __fmul_rn(__fmul_rn(r[e + 1], g2[e + 1]), inv_r));
                }
                *reinterpret_cast<uint4*>(prow + 16 * b) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                *reinterpret_cast<uint4*>(prow + 16 * b + 8) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
            }
        }
    }
}

template <int B>
__device__ __forceinline__ void load_gain(const uint16_t* w, float center, int tid, int nvalid,
                                          float (&g)[16 * B]) {
#pragma unroll
    for (int i = 0; i < 16 * B; ++i)
        g[i] = (w != nullptr && i / 16 < nvalid)
                   ? __fadd_rn(center, __uint_as_float(static_cast<uint32_t>(w[16 * B * tid + i]) << 16))
                   : 0.0f;
}

__device__ __forceinline__ bool slot_valid(int32_t r, int64_t R) {
    return r >= 0 && static_cast<int64_t>(r) < R;
}

template <int B, int TW, bool JOIN>
__global__ void __launch_bounds__(kConsumerThreads + 32, 1)
    combine_kernel(const uint16_t* __restrict__ expert_out, int64_t R, int H,
                   const int32_t* __restrict__ row_idx, const float* __restrict__ wt, int T, int k,
                   const uint16_t* __restrict__ w, float gc, float eps, uint16_t* __restrict__ out,
                   JoinArgs join, int nslot) {
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
            mbar_init(&bars[2 * i], 1);
            mbar_init(&bars[2 * i + 1], 1);
        }
        fence_mbar_init();
    }
    __syncthreads();

    const int team_stride = gridDim.x * NTEAM;

    if (warp == NTEAM * TW) {
        // ---------------- producer: lane `team` copies the valid rows of the
        // team's tokens, in slot order, into the team's ring.
        if (lane < NTEAM) {
            const int team = lane;
            uint8_t* ring = smem + static_cast<size_t>(team) * nslot * slot_bytes;
            uint64_t* tb = bars + static_cast<size_t>(team) * nslot * 2;
            int fills = 0;
            bool stop = false;
            for (int t = blockIdx.x * NTEAM + team; t < T && !stop; t += team_stride) {
                const int tn = t + team_stride;
                if (tn < T)
                    asm volatile("prefetch.global.L1 [%0];" ::"l"(row_idx + static_cast<size_t>(tn) * k));
                const int32_t* ir = row_idx + static_cast<size_t>(t) * k;
                for (int j = 0; j < k; ++j) {
                    const int32_t r = __ldg(ir + j);
                    if (!slot_valid(r, R)) continue;
                    const int slot = fills % nslot;
                    const int use = fills / nslot;
                    if (use > 0 && !mbar_wait_bounded(&tb[2 * slot + 1], (use - 1) & 1, 1u)) {
                        stop = true;
                        break;
                    }
                    mbar_arrive_expect_tx(&tb[2 * slot], static_cast<uint32_t>(slot_bytes));
                    bulk_g2s(ring + static_cast<size_t>(slot) * slot_bytes,
                             expert_out + static_cast<size_t>(r) * H, static_cast<uint32_t>(slot_bytes),
                             &tb[2 * slot]);
                    ++fills;
                }
            }
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
    load_gain<B>(w, gc, tid, nvalid, g);
    float gain[16 * B], g2[16 * B];
    if constexpr (JOIN) {
        load_gain<B>(join.gain, 0.0f, tid, nvalid, gain);
        load_gain<B>(join.next_w, join.next_gc, tid, nvalid, g2);
    }
    const float fH = static_cast<float>(H);

    // slot indices and weights of the token, one slot per lane (k <= 32),
    // loaded one token ahead
    int t = blockIdx.x * NTEAM + team;
    int32_t my_r = -1;
    float my_w = 0.0f;
    if (t < T && lane < k) {
        my_r = __ldg(row_idx + static_cast<size_t>(t) * k + lane);
        my_w = __ldg(wt + static_cast<size_t>(t) * k + lane);
    }
    int fills = 0;
    bool aborted = false;
    for (; t < T; t += team_stride) {
        const int32_t cur_r = my_r;
        const float cur_w = my_w;
        const int tn = t + team_stride;
        if (tn < T && lane < k) {
            my_r = __ldg(row_idx + static_cast<size_t>(tn) * k + lane);
            my_w = __ldg(wt + static_cast<size_t>(tn) * k + lane);
        }
        float acc[16 * B];
#pragma unroll
        for (int i = 0; i < 16 * B; ++i) acc[i] = 0.0f;

        for (int j = 0; j < k; ++j) {
            const int32_t r = __shfl_sync(0xffffffffu, cur_r, j);
            if (!slot_valid(r, R)) continue;
            const float wj = __shfl_sync(0xffffffffu, cur_w, j);
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
            if (abort) {
                aborted = true;
                break;
            }
            if (tid == 0) mbar_arrive(&tb[2 * slot + 1]);
            ++fills;
            const float inv = inv_rms(ss, fH, eps);
#pragma unroll
            for (int i = 0; i < 16 * B; ++i)
                acc[i] = fmaf(wj, round_bf16(__fmul_rn(__fmul_rn(xv[i], g[i]), inv)), acc[i]);
        }
        if (aborted) break;

        float br[16 * B];
#pragma unroll
        for (int i = 0; i < 16 * B; ++i) br[i] = round_bf16(acc[i]);
        if (out != nullptr) {
            uint16_t* orow = out + static_cast<size_t>(t) * H + 16 * B * tid;
#pragma unroll
            for (int b = 0; b < B; ++b) {
                if (b < nvalid) {
                    uint32_t pk[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) pk[i] = pack_bf16x2(br[16 * b + 2 * i], br[16 * b + 2 * i + 1]);
                    *reinterpret_cast<uint4*>(orow + 16 * b) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                    *reinterpret_cast<uint4*>(orow + 16 * b + 8) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
                }
            }
        }
        if constexpr (JOIN) join_token<B, TW>(br, t, H, tid, nvalid, join, gain, g2, team_sum);
    }
}

// Standalone gated residual join: the branch comes from global memory.
template <int B, int TW>
__global__ void __launch_bounds__(kConsumerThreads, 1)
    residual_join_kernel(const uint16_t* __restrict__ branch, int T, int H, JoinArgs join) {
    constexpr int NTEAM = kConsumerThreads / (TW * 32);
    __shared__ float red_all[NTEAM * 2 * TW];
    __shared__ int flags_all[NTEAM * 2 * TW];
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int team = warp / TW;
    const int warp_in_team = warp % TW;
    const int tid = warp_in_team * 32 + lane;
    const int nblocks = H / 16;
    int nvalid = nblocks - tid * B;
    nvalid = nvalid < 0 ? 0 : (nvalid > B ? B : nvalid);
    TeamSum<TW> team_sum{red_all + team * 2 * TW, flags_all + team * 2 * TW, 1 + team, warp_in_team,
                         lane, 0};
    float gain[16 * B], g2[16 * B];
    load_gain<B>(join.gain, 0.0f, tid, nvalid, gain);
    load_gain<B>(join.next_w, join.next_gc, tid, nvalid, g2);
    for (int t = blockIdx.x * NTEAM + team; t < T; t += gridDim.x * NTEAM) {
        const uint16_t* brow = branch + static_cast<size_t>(t) * H + 16 * B * tid;
        float br[16 * B];
#pragma unroll
        for (int b = 0; b < B; ++b) {
            uint4 lo = make_uint4(0u, 0u, 0u, 0u), hi = lo;
            if (b < nvalid) {
                lo = ld_nc_v4(brow + 16 * b);
                hi = ld_nc_v4(brow + 16 * b + 8);
            }
            const uint32_t v[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                br[16 * b + 2 * i] = bf16_lo(v[i]);
                br[16 * b + 2 * i + 1] = bf16_hi(v[i]);
            }
        }
        join_token<B, TW>(br, t, H, tid, nvalid, join, gain, g2, team_sum);
    }
}

namespace {

template <int B, int TW>
cudaError_t launch_cb(const uint16_t* expert_out, int64_t R, int H, const int32_t* row_idx, const float* wt,
                      int T, int k, const uint16_t* w, float gc, float eps, uint16_t* out,
                      const JoinArgs& join, cudaStream_t s) {
    constexpr int NTEAM = kConsumerThreads / (TW * 32);
    const int slot_bytes = 2 * H;
    int nslot = kRingBytes / (NTEAM * slot_bytes);
    if (nslot > 16) nslot = 16;
    if (nslot < 2) return cudaErrorInvalidConfiguration;
    const RingLayout lay{NTEAM, nslot, slot_bytes, TW};
    const size_t smem = lay.total_bytes();
    int grid = (T + NTEAM - 1) / NTEAM;
    const int cap = device_info().sm_count;
    if (grid > cap) grid = cap;
    if (join.residual != nullptr) {
        auto kern = combine_kernel<B, TW, true>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(smem));
        if (e != cudaSuccess) return e;
        kern<<<grid, kConsumerThreads + 32, smem, s>>>(expert_out, R, H, row_idx, wt, T, k, w, gc, eps,
                                                        out, join, nslot);
    } else {
        auto kern = combine_kernel<B, TW, false>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(smem));
        if (e != cudaSuccess) return e;
        kern<<<grid, kConsumerThreads + 32, smem, s>>>(expert_out, R, H, row_idx, wt, T, k, w, gc, eps,
                                                        out, join, nslot);
    }
    return cudaGetLastError();
}

template <int B, int TW>
cudaError_t launch_rj(const uint16_t* branch, int T, int H, const JoinArgs& join, cudaStream_t s) {
    constexpr int NTEAM = kConsumerThreads / (TW * 32);
    int grid = (T + NTEAM - 1) / NTEAM;
    const int cap = device_info().sm_count * 2;
    if (grid > cap) grid = cap;
    residual_join_kernel<B, TW><<<grid, kConsumerThreads, 0, s>>>(branch, T, H, join);
    return cudaGetLastError();
}

void team_shape(int H, int& B, int& TW) {
    const int nblocks = H / 16;
    B = nblocks <= 512 ? 1 : 2;
    const int per = (nblocks + B - 1) / B;
    int P = 32;
    while (P < per) P <<= 1;
    TW = P / 32;
}

}  // namespace

cudaError_t launch_combine(const uint16_t* expert_out, int64_t R, int H, const int32_t* row_idx,
                           const float* wt, int T, int k, const uint16_t* w, float gc, float eps,
                           uint16_t* out, const JoinArgs& join, cudaStream_t s) {
    int B, TW;
    team_shape(H, B, TW);
#define MB_CB(Bv, TWv) \
    if (B == Bv && TW == TWv) return launch_cb<Bv, TWv>(expert_out, R, H, row_idx, wt, T, k, w, gc, eps, out, join, s);
    MB_CB(1, 1) MB_CB(1, 2) MB_CB(1, 4) MB_CB(1, 8) MB_CB(1, 16)
    MB_CB(2, 16)
#undef MB_CB
    return cudaErrorInvalidValue;
}

cudaError_t launch_residual_join(const uint16_t* branch, int T, int H, const JoinArgs& join,
                                 cudaStream_t s) {
    int B, TW;
    team_shape(H, B, TW);
#define MB_RJ(Bv, TWv) \
    if (B == Bv && TW == TWv) return launch_rj<Bv, TWv>(branch, T, H, join, s);
    MB_RJ(1, 1) MB_RJ(1, 2) MB_RJ(1, 4) MB_RJ(1, 8) MB_RJ(1, 16)
    MB_RJ(2, 16)
#undef MB_RJ
    return cudaErrorInvalidValue;
}

}  // namespace mb
