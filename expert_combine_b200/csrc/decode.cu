// decode.cu -- the MoE boundary's post-expert side for a few tokens (decode
// batches): combine, gated residual join and next prenorm, one token per
// thread-block cluster.
//
// Same arithmetic as combine.cu (TensorRT-LLM PR 21356 "Muse Spark Open
// decoder fast paths", description: post-expert norm and combine, gated
// residual join, the fused decoder boundary), bit for bit: the results equal
// the row kernels' and the oracle's.  Only the work split differs.  With few
// tokens the row kernels give each token to one team, which then reads the
// token's k expert rows one after the other -- a chain of dependent DRAM
// trips.  Here a token's hidden dimension is split across the C CTAs of a
// cluster (C <= 8), each thread owning one 16-element block, so all k rows of
// the token are in flight at once, and the three row statistics (sum of
// squares of each expert row, of the joined branch g, of the updated
// residual) are reduced across the cluster through distributed shared memory
// between hardware cluster barriers.  No CTA waits on another except at
// those barriers, and every CTA of a cluster takes the same path.
//
// Canonical reduction order: thread l of warp w of cluster rank c owns block
// b = (c * NW + w) * 32 + l of the row (blocks padded with zeros to
// P2 = TPB * C = next_pow2(H / 16)); its partial is the sequential fused
// multiply-add over the block's 16 elements, then a butterfly over the warp's
// 32 blocks, a pairwise tree over the CTA's warps and one over the cluster's
// CTAs in rank order -- the balanced pairwise tree over the padded blocks.
#include "internal.h"
#include "common.cuh"
#include "ring.cuh"

namespace mb {

namespace {

struct DecodeArgs {
    const uint16_t* expert_out;   // [R, H] BF16 (combine)
    int64_t R;
    int H;
    const int32_t* row_idx;       // [T, k]
    const float* wt;              // [T, k]
    int T, k;
    const uint16_t* w;            // [H] post-expert norm weight
    float gc, eps;
    uint16_t* out;                // [T, H] combine output, may be NULL
    const uint16_t* branch;       // [T, H] BF16 branch (join without combine)
    JoinArgs join;
};

__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Final barrier: only keeps every CTA's shared memory alive until all remote
// reads of it are done (their values were consumed before this point), so no
// memory ordering is needed and pending global stores are not waited for.
__device__ __forceinline__ void cluster_exit_sync() {
    asm volatile("barrier.cluster.arrive.relaxed.aligned;\n\tbarrier.cluster.wait.aligned;" ::: "memory");
}

// The float at `local` (a shared-memory address of this CTA) in the CTA of
// cluster rank `rank`.
__device__ __forceinline__ float ld_cluster_f32(const float* local, uint32_t rank) {
    uint32_t remote;
    float v;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_addr(local)), "r"(rank));
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
    return v;
}

// Pairwise tree, in rank order, over the C CTAs' values at `local`.
template <int C>
__device__ __forceinline__ float cluster_tree(const float* local) {
    if constexpr (C == 1) {
        return *local;
    } else {
        float v[C];
#pragma unroll
        for (int r = 0; r < C; ++r) v[r] = ld_cluster_f32(local, r);
        return tree_sum_array<C>(v);
    }
}

// Sequential fused multiply-add of the squares of one 16-element block held
// as 8 BF16 pair words (element 2i in the low half of word i).
__device__ __forceinline__ float block_sumsq_bf16(const uint32_t (&w)[8]) {
    float s = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        s = fma_bf16_lo(w[i], w[i], s);
        s = fma_bf16_hi(w[i], w[i], s);
    }
    return s;
}

__device__ __forceinline__ float block_sumsq_f32(const float2 (&v)[8]) {
    float s = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        s = __fmaf_rn(v[i].x, v[i].x, s);
        s = __fmaf_rn(v[i].y, v[i].y, s);
    }
    return s;
}

__device__ __forceinline__ void load_block16(const uint16_t* p, uint32_t (&w)[8]) {
    const uint4 a = *reinterpret_cast<const uint4*>(p);
    const uint4 b = *reinterpret_cast<const uint4*>(p + 8);
    w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
    w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
}

__device__ __forceinline__ void store_block16(uint16_t* p, const uint32_t (&w)[8]) {
    *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
    *reinterpret_cast<uint4*>(p + 8) = make_uint4(w[4], w[5], w[6], w[7]);
}

// Statistic of one value per thread over the whole token row: warp butterfly,
// CTA tree (through `wpart`, NW floats), cluster tree (through `cpart`, one
// float).  Every thread returns the same sum.
template <int NW, int C>
__device__ __forceinline__ float row_sum(float v, float* wpart, float* cpart) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    v = warp_tree_sum(v);
    if (lane == 0) wpart[warp] = v;
    __syncthreads();
    if (threadIdx.x == 0) *cpart = tree_sum_array<NW>(wpart);
    if constexpr (C > 1) cluster_sync_all();
    else __syncthreads();
    return cluster_tree<C>(cpart);
}

constexpr int kGroup = 8;   // expert rows fetched together

template <int TPB, int C, bool COMBINE, bool JOIN, bool GC0>
__global__ void __launch_bounds__(TPB) boundary_cluster_kernel(const DecodeArgs a) {
    constexpr int NW = TPB / 32;
    __shared__ float wpart[kMaxTopK][NW];
    __shared__ __align__(16) float cpart[kMaxTopK];
    __shared__ float sinv[kMaxTopK];
    __shared__ float wg[NW], cg[1], wr[NW], cr[1];

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int t = blockIdx.x / C;
    const int rank = blockIdx.x % C;
    const int H = a.H;
    const int blk = rank * TPB + threadIdx.x;
    const bool has = blk < H / 16;
    const int col = 16 * blk;
    const float fH = static_cast<float>(H);
    const bool pow2 = (H & (H - 1)) == 0;
    const float rH = pow2 ? __frcp_rn(fH) : 0.0f;
    griddep_wait();
    griddep_launch();

    uint32_t bw[8];   // this block of the branch (the combine output), BF16 pairs
    if constexpr (COMBINE) {
        const int k = a.k;
        int32_t r_l = -1;
        float w_l = 0.0f;
        if (lane < k) {
            r_l = __ldg(a.row_idx + static_cast<size_t>(t) * k + lane);
            w_l = __ldg(a.wt + static_cast<size_t>(t) * k + lane);
        }
        const bool v_l = lane < k && r_l >= 0 && static_cast<int64_t>(r_l) < a.R;
        const unsigned vm = __ballot_sync(0xffffffffu, v_l);

        // pass 1: the partial sum of squares of each valid row
        for (int j0 = 0; j0 < k; j0 += kGroup) {
            uint32_t x[kGroup][8];
#pragma unroll
            for (int jj = 0; jj < kGroup; ++jj) {
                const int j = j0 + jj;
                const int r = __shfl_sync(0xffffffffu, r_l, j & 31);
                if (j < k && ((vm >> j) & 1u) && has)
                    load_block16(a.expert_out + static_cast<size_t>(r) * H + col, x[jj]);
                else
#pragma unroll
                    for (int i = 0; i < 8; ++i) x[jj][i] = 0u;
            }
#pragma unroll
            for (int jj = 0; jj < kGroup; ++jj) {
                const int j = j0 + jj;
                const float s = warp_tree_sum(block_sumsq_bf16(x[jj]));
                if (j < k && lane == 0) wpart[j][warp] = s;
            }
        }
        __syncthreads();
        if (threadIdx.x < k) cpart[threadIdx.x] = tree_sum_array<NW>(wpart[threadIdx.x]);
        if constexpr (C > 1) cluster_sync_all();
        else __syncthreads();
        if (threadIdx.x < k && ((vm >> threadIdx.x) & 1u))
            sinv[threadIdx.x] = inv_rms_h(cluster_tree<C>(&cpart[threadIdx.x]), fH, rH, pow2, a.eps);
        __syncthreads();

        // pass 2: normalise and accumulate in slot order
        uint32_t nw[8];
        float2 gp[8];
        if (has) load_block16(a.w + col, nw);
        else
#pragma unroll
            for (int i = 0; i < 8; ++i) nw[i] = 0u;
        const float2 gc2 = make_float2(a.gc, a.gc);
#pragma unroll
        for (int i = 0; i < 8; ++i) gp[i] = GC0 ? make_float2(0.0f, 0.0f) : add2(gc2, unpack_bf16x2(nw[i]));
        float2 acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = make_float2(0.0f, 0.0f);
        for (int j0 = 0; j0 < k; j0 += kGroup) {
            uint32_t x[kGroup][8];
#pragma unroll
            for (int jj = 0; jj < kGroup; ++jj) {
                const int j = j0 + jj;
                const int r = __shfl_sync(0xffffffffu, r_l, j & 31);
                if (j < k && ((vm >> j) & 1u) && has)
                    load_block16(a.expert_out + static_cast<size_t>(r) * H + col, x[jj]);
                else
#pragma unroll
                    for (int i = 0; i < 8; ++i) x[jj][i] = 0u;
            }
#pragma unroll
            for (int jj = 0; jj < kGroup; ++jj) {
                const int j = j0 + jj;
                const float wj = __shfl_sync(0xffffffffu, w_l, j & 31);
                if (j < k && ((vm >> j) & 1u)) {
                    const float inv = sinv[j];
                    const float2 inv2 = make_float2(inv, inv);
                    const float2 w2 = make_float2(wj, wj);
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const float2 tt = GC0 ? mul_bf16x2_exact(x[jj][i], nw[i]) : mul2(unpack_bf16x2(x[jj][i]), gp[i]);
                        acc[i] = fma2(w2, round_bf16_f2(mul2(tt, inv2)), acc[i]);
                    }
                }
            }
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) bw[i] = pack_bf16x2_rn(acc[i]);
        if constexpr (!JOIN)
            if (a.out != nullptr && has) store_block16(a.out + static_cast<size_t>(t) * H + col, bw);
    } else {
        if (has) load_block16(a.branch + static_cast<size_t>(t) * H + col, bw);
        else
#pragma unroll
            for (int i = 0; i < 8; ++i) bw[i] = 0u;
    }

    if constexpr (JOIN) {
        const JoinArgs& jn = a.join;
        // g = bf16(gain * branch), n = bf16(g * inv(g)), r' = alpha r + beta n; every
        // global store waits until the last cluster reduction is done
        uint32_t gw[8], nw2[8];
        float2 r[8];
        const bool hn = has && jn.next_w != nullptr;
        const float* rrow = jn.residual + static_cast<size_t>(t) * H + col;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            uint4 g4 = make_uint4(0u, 0u, 0u, 0u), n4 = make_uint4(0u, 0u, 0u, 0u);
            if (has) g4 = *reinterpret_cast<const uint4*>(jn.gain + col + 8 * c);
            if (hn) n4 = *reinterpret_cast<const uint4*>(jn.next_w + col + 8 * c);
            gw[4 * c] = g4.x; gw[4 * c + 1] = g4.y; gw[4 * c + 2] = g4.z; gw[4 * c + 3] = g4.w;
            nw2[4 * c] = n4.x; nw2[4 * c + 1] = n4.y; nw2[4 * c + 2] = n4.z; nw2[4 * c + 3] = n4.w;
        }
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (has) v = *reinterpret_cast<const float4*>(rrow + 4 * c);
            r[2 * c] = make_float2(v.x, v.y);
            r[2 * c + 1] = make_float2(v.z, v.w);
        }
        uint32_t gg[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) gg[i] = pack_bf16x2_rn(mul2(unpack_bf16x2(gw[i]), unpack_bf16x2(bw[i])));
        const float inv_g = inv_rms_h(row_sum<NW, C>(block_sumsq_bf16(gg), wg, cg), fH, rH, pow2, jn.eps);
        const float2 inv_g2 = make_float2(inv_g, inv_g);
        const float2 alpha2 = make_float2(jn.alpha, jn.alpha);
        const float2 beta2 = make_float2(jn.beta, jn.beta);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float2 n = unpack_bf16x2(pack_bf16x2_rn(mul2(unpack_bf16x2(gg[i]), inv_g2)));
            r[i] = add2(mul2(alpha2, r[i]), mul2(beta2, n));
        }
        uint32_t pw[8];
        if (jn.next_w != nullptr) {
            // p = bf16((r' * (next_gc + next_w)) * inv(r'))
            const float inv_r = inv_rms_h(row_sum<NW, C>(block_sumsq_f32(r), wr, cr), fH, rH, pow2, jn.next_eps);
            const float2 inv_r2 = make_float2(inv_r, inv_r);
            const float2 ngc2 = make_float2(jn.next_gc, jn.next_gc);
#pragma unroll
            for (int i = 0; i < 8; ++i) pw[i] = pack_bf16x2_rn(mul2(mul2(r[i], add2(ngc2, unpack_bf16x2(nw2[i]))), inv_r2));
        }
        if (has) {
            if (COMBINE && a.out != nullptr) store_block16(a.out + static_cast<size_t>(t) * H + col, bw);
            float* rw = jn.residual + static_cast<size_t>(t) * H + col;
#pragma unroll
            for (int c = 0; c < 4; ++c)
                *reinterpret_cast<float4*>(rw + 4 * c) =
                    make_float4(r[2 * c].x, r[2 * c].y, r[2 * c + 1].x, r[2 * c + 1].y);
            if (jn.next_w != nullptr) store_block16(jn.next_prenorm + static_cast<size_t>(t) * H + col, pw);
        }
    }
    // no CTA leaves while another may still read its shared memory
    if constexpr (C > 1) cluster_exit_sync();
}

// Threads per CTA and CTAs per cluster for row length H: TPB * C equals the
// padded block count next_pow2(H / 16), with C <= 8.
struct ClusterShape {
    int tpb, c;
};
ClusterShape cluster_shape(int H) {
    int p2 = 1;
    while (p2 < H / 16) p2 <<= 1;
    if (p2 <= 32) return {32, 1};
    if (p2 <= 512) return {64, p2 / 64};
    return {p2 / 8, 8};
}

template <int TPB, int C, bool COMBINE, bool JOIN, bool GC0>
cudaError_t launch_bc(const DecodeArgs& a, cudaStream_t s) {
    cudaLaunchAttribute attr[2];
    cudaLaunchConfig_t cfg = pdl_config(a.T * C, TPB, 0, s, attr);
    if constexpr (C > 1) {
        attr[1].id = cudaLaunchAttributeClusterDimension;
        attr[1].val.clusterDim.x = C;
        attr[1].val.clusterDim.y = 1;
        attr[1].val.clusterDim.z = 1;
        cfg.numAttrs = 2;
    }
    return cudaLaunchKernelEx(&cfg, boundary_cluster_kernel<TPB, C, COMBINE, JOIN, GC0>, a);
}

template <bool COMBINE, bool JOIN, bool GC0>
cudaError_t launch_bc_shape(const DecodeArgs& a, cudaStream_t s) {
    const ClusterShape sh = cluster_shape(a.H);
    switch (sh.tpb * 16 + sh.c) {
        case 32 * 16 + 1: return launch_bc<32, 1, COMBINE, JOIN, GC0>(a, s);
        case 64 * 16 + 1: return launch_bc<64, 1, COMBINE, JOIN, GC0>(a, s);
        case 64 * 16 + 2: return launch_bc<64, 2, COMBINE, JOIN, GC0>(a, s);
        case 64 * 16 + 4: return launch_bc<64, 4, COMBINE, JOIN, GC0>(a, s);
        case 64 * 16 + 8: return launch_bc<64, 8, COMBINE, JOIN, GC0>(a, s);
        case 128 * 16 + 8: return launch_bc<128, 8, COMBINE, JOIN, GC0>(a, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

// The cluster path while one wave of it fits the GPU at 16 warps per SM
// (T * next_pow2(H / 16) threads); past that the row kernels' streaming wins.
bool cluster_path(int T, int H) {
    if (T < 1 || H < 16 || H > kMaxHidden) return false;
    const ClusterShape sh = cluster_shape(H);
    return static_cast<int64_t>(T) * sh.tpb * sh.c <= static_cast<int64_t>(device_info().sm_count) * kClusterThreadsPerSM;
}

cudaError_t launch_combine_cluster(const uint16_t* expert_out, int64_t R, int H, const int32_t* row_idx,
                                   const float* wt, int T, int k, const uint16_t* w, float gc, float eps,
                                   uint16_t* out, const JoinArgs& join, cudaStream_t s) {
    DecodeArgs a{expert_out, R, H, row_idx, wt, T, k, w, gc, eps, out, nullptr, join};
    const bool fused = join.residual != nullptr;
    if (fused) return gc == 0.0f ? launch_bc_shape<true, true, true>(a, s) : launch_bc_shape<true, true, false>(a, s);
    return gc == 0.0f ? launch_bc_shape<true, false, true>(a, s) : launch_bc_shape<true, false, false>(a, s);
}

cudaError_t launch_join_cluster(const uint16_t* branch, int T, int H, const JoinArgs& join, cudaStream_t s) {
    DecodeArgs a{nullptr, 0, H, nullptr, nullptr, T, 0, nullptr, 0.0f, 0.0f, nullptr, branch, join};
    return launch_bc_shape<false, true, true>(a, s);
}

}  // namespace mb
