// finalize_ar.cu -- the expert finalize fused with the tensor-parallel
// all-reduce of its partials, one shot over peer memory.
//
// Per token t on rank r (TensorRT-LLM PR 21356 "Muse Spark Open decoder fast
// paths", description, "Fused finalize + all-reduce": the expert finalize and
// the TP all-reduce as one kernel, a one-shot exchange, FP32 accumulation;
// PR 21042 reference composition, MoE paragraph: the finalize all-reduces
// partials in FP32):
//   p_r[t, :] = the combine's FP32 accumulator over the slots j of t whose
//               row lives on rank r (0 <= row_idx_r[t, j] < R_r), in slot
//               order from +0, not rounded
//   out[t, :] = bf16(((p_0 + p_1) + p_2) + ...)          on every rank
//
// Exchange: each rank writes p_r into its own workspace, then raises, in
// every rank's workspace, the flag (r, t) with this call's epoch; a rank
// reduces token t once it has seen the flags (q, t) of all ranks q, reading
// the peers' partials with plain loads from their memory (no multicast, no
// staging copy).  Partials and flags are double-buffered by the epoch's
// parity, so a rank never overwrites a buffer a peer may still read: a rank
// reaches call n + 2 only after every peer has raised its flags of call
// n + 1, which it does only after its call n has ended.
//
// Every CTA of a launch must be resident at once (each waits on other CTAs'
// flags): the launch is cooperative and the grid is capped at one wave.
// The one-device form runs all ranks of the exchange in one launch (grid.y
// = ranks), each with its own workspace; it computes exactly what the
// multi-process form does.
#include "common.cuh"
#include "internal.h"
#include "ring.cuh"

namespace mb {

namespace {

// One rank's workspace (device memory that the peers map):
//   [0, 256)       header: epoch of the last finished call, CTA exit count
//   flags          [2][world][Tmax] uint32
//   partials       [2][Tmax][H] float
struct FarHeader {
    unsigned int epoch;
    unsigned int done;
};

__host__ __device__ inline size_t far_flags_offset() { return 256; }
__host__ __device__ inline size_t far_partial_offset(int world, int Tmax) {
    const size_t end = far_flags_offset() + 2ull * world * Tmax * sizeof(uint32_t);
    return (end + 255) & ~size_t(255);
}
__host__ __device__ inline size_t far_workspace_bytes(int world, int Tmax, int H) {
    return far_partial_offset(world, Tmax) + 2ull * Tmax * H * sizeof(float);
}

struct FarRankIO {
    const uint16_t* expert_out;
    int64_t R;
    const int32_t* row_idx;
    const float* wt;
    uint16_t* out;
};

struct FarArgs {
    FarRankIO io[kFarMaxWorld];   // the ranks this launch computes: io[i] is rank rank0 + i
    uint8_t* ws[kFarMaxWorld];    // every rank's workspace as mapped on this device
    const uint16_t* w;
    float gc, eps;
    int H, T, k, Tmax, world, rank0;
};

constexpr unsigned int kFarWaitCode = 16u;   // mb_device_status bit 4

// Release / acquire as fence + relaxed access: a thread's fence orders every
// write it has observed (the CTA's, through the barrier before it) before its
// later flag stores, and its flag loads before every later read of the CTA
// (through the barrier after it).  SYS: some ranks are other processes'
// GPUs (system scope); otherwise every rank is on this device (GPU scope).
template <bool SYS>
__device__ __forceinline__ void fence_scope() {
    if constexpr (SYS) asm volatile("fence.acq_rel.sys;" ::: "memory");
    else asm volatile("fence.acq_rel.gpu;" ::: "memory");
}
template <bool SYS>
__device__ __forceinline__ void st_relaxed(uint32_t* p, uint32_t v) {
    if constexpr (SYS) asm volatile("st.relaxed.sys.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
    else asm volatile("st.relaxed.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
template <bool SYS>
__device__ __forceinline__ uint32_t ld_relaxed(const uint32_t* p) {
    uint32_t v;
    if constexpr (SYS) asm volatile("ld.relaxed.sys.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    else asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
// A peer's partial: cached in L2 only (the line may have changed since an
// earlier call cached it closer).
__device__ __forceinline__ float4 ld_cg_f4(const float* p) {
    float4 v;
    asm volatile("ld.global.cg.v4.f32 {%0,%1,%2,%3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "l"(p));
    return v;
}

// This thread's 32 elements of a BF16 row (two 16-element blocks, nvalid of
// them inside the row; missing blocks read as zero).
__device__ __forceinline__ void load_row32(const uint16_t* row, int tid, int nvalid, uint32_t (&w)[16]) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (c / 2 < nvalid) v = ld_nc_v4(row + 32 * tid + 8 * c);
        w[4 * c] = v.x;
        w[4 * c + 1] = v.y;
        w[4 * c + 2] = v.z;
        w[4 * c + 3] = v.w;
    }
}

// CTA-wide canonical sums of two per-thread partials (lane butterfly, then a
// balanced tree over the NW warps in order).  red holds 2 * NW floats.
template <int NW>
__device__ __forceinline__ float2 cta_sum2(float a, float b, float* red) {
    a = warp_tree_sum(a);
    b = warp_tree_sum(b);
    const int warp = threadIdx.x >> 5;
    if ((threadIdx.x & 31) == 0) {
        red[warp] = a;
        red[NW + warp] = b;
    }
    __syncthreads();
    float pa[NW], pb[NW];
#pragma unroll
    for (int i = 0; i < NW; ++i) {
        pa[i] = red[i];
        pb[i] = red[NW + i];
    }
    __syncthreads();   // red is reused by the next call
    return make_float2(tree_sum_array<NW>(pa), tree_sum_array<NW>(pb));
}

template <bool GC0>
__device__ __forceinline__ float2 far_norm_pair(uint32_t xw, uint32_t wpw, float2 gp, float2 inv2) {
    const float2 t = GC0 ? mul_bf16x2_exact(xw, wpw) : mul2(unpack_bf16x2(xw), gp);
    return round_bf16_f2(mul2(t, inv2));
}

// One CTA of NW warps per (token group, rank); thread tid owns elements
// [32 tid, 32 tid + 32).
template <int NW, bool GC0, bool SYS>
__global__ void __launch_bounds__(NW * 32) finalize_ar_kernel(const FarArgs a) {
    __shared__ float red[2 * NW];
    __shared__ int s_abort;
    const int li = blockIdx.y;
    const int rank = a.rank0 + li;
    const FarRankIO io = a.io[li];
    const int H = a.H, T = a.T, k = a.k, world = a.world;
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    int nvalid = H / 16 - 2 * tid;
    nvalid = nvalid < 0 ? 0 : (nvalid > 2 ? 2 : nvalid);

    uint8_t* my_ws = a.ws[rank];
    FarHeader* hdr = reinterpret_cast<FarHeader*>(my_ws);
    const uint32_t epoch = *reinterpret_cast<volatile unsigned int*>(&hdr->epoch) + 1u;
    const int par = static_cast<int>(epoch & 1u);
    const size_t poff = far_partial_offset(world, a.Tmax) + static_cast<size_t>(par) * a.Tmax * H * sizeof(float);
    const size_t foff = far_flags_offset() + static_cast<size_t>(par) * world * a.Tmax * sizeof(uint32_t);
    float* my_part = reinterpret_cast<float*>(my_ws + poff);
    if (tid == 0) s_abort = 0;

    // gain: with GC0 the BF16 weight words, else FP32 pairs gc + w
    uint32_t wp[16];
    float2 g[16];
    if constexpr (GC0) {
        load_row32(a.w, tid, nvalid, wp);
    } else {
        load_gain32(a.w, a.gc, tid, nvalid, g);
    }
    const float fH = static_cast<float>(H);
    const bool pow2 = (H & (H - 1)) == 0;
    const float rH = pow2 ? __frcp_rn(fH) : 0.0f;

    // ---- phase 1: this rank's partial of each of the CTA's tokens
    for (int t = blockIdx.x; t < T; t += gridDim.x) {
        int32_t my_r = -1;
        float my_w = 0.0f;
        if (lane < k) {
            my_r = __ldg(io.row_idx + static_cast<size_t>(t) * k + lane);
            my_w = __ldg(io.wt + static_cast<size_t>(t) * k + lane);
        }
        const bool valid = lane < k && my_r >= 0 && static_cast<int64_t>(my_r) < io.R;
        unsigned vm = __ballot_sync(0xffffffffu, valid);
        float2 acc[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) acc[i] = make_float2(0.0f, 0.0f);
        while (vm != 0u) {
            const int j0 = __ffs(vm) - 1;
            vm &= vm - 1u;
            const bool two = vm != 0u;
            int j1 = j0;
            if (two) {
                j1 = __ffs(vm) - 1;
                vm &= vm - 1u;
            }
            const int32_t r0 = __shfl_sync(0xffffffffu, my_r, j0);
            const int32_t r1 = __shfl_sync(0xffffffffu, my_r, j1);
            const float w0 = __shfl_sync(0xffffffffu, my_w, j0);
            const float w1 = __shfl_sync(0xffffffffu, my_w, j1);
            uint32_t x0[16], x1[16];
            load_row32(io.expert_out + static_cast<size_t>(r0) * H, tid, nvalid, x0);
            if (two) load_row32(io.expert_out + static_cast<size_t>(r1) * H, tid, nvalid, x1);
            else {
#pragma unroll
                for (int i = 0; i < 16; ++i) x1[i] = 0u;
            }
            const float2 ss = cta_sum2<NW>(row32_sumsq(x0), row32_sumsq(x1), red);
            // each lane forms the inverse RMS of row l & 1 of the step (one
            // evaluation serves both rows); lanes 0 and 1 hand them out
            const float inv_l = inv_rms_h((lane & 1) ? ss.y : ss.x, fH, rH, pow2, a.eps);
            const float inv0 = __shfl_sync(0xffffffffu, inv_l, 0);
            const float2 inv02 = make_float2(inv0, inv0);
            const float2 w02 = make_float2(w0, w0);
#pragma unroll
            for (int i = 0; i < 16; ++i) acc[i] = fma2(w02, far_norm_pair<GC0>(x0[i], wp[i], g[i], inv02), acc[i]);
            if (two) {
                const float inv1 = __shfl_sync(0xffffffffu, inv_l, 1);
                const float2 inv12 = make_float2(inv1, inv1);
                const float2 w12 = make_float2(w1, w1);
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    acc[i] = fma2(w12, far_norm_pair<GC0>(x1[i], wp[i], g[i], inv12), acc[i]);
            }
        }
        float* prow = my_part + static_cast<size_t>(t) * H + 32 * tid;
#pragma unroll
        for (int c = 0; c < 8; ++c)
            if (c / 4 < nvalid)
                *reinterpret_cast<float4*>(prow + 4 * c) =
                    make_float4(acc[2 * c].x, acc[2 * c].y, acc[2 * c + 1].x, acc[2 * c + 1].y);
    }

    // ---- the CTA's partials are in memory: thread q tells rank q (one
    // system-scope fence per thread, then plain flag stores), then waits for
    // rank q's flags of the CTA's tokens (plain loads, one fence after them)
    __syncthreads();
    if (tid < world) {
        fence_scope<SYS>();
        uint32_t* f = reinterpret_cast<uint32_t*>(a.ws[tid] + foff) + static_cast<size_t>(rank) * a.Tmax;
        for (int t = blockIdx.x; t < T; t += gridDim.x) st_relaxed<SYS>(f + t, epoch);
        const uint32_t* mine = reinterpret_cast<const uint32_t*>(my_ws + foff) + static_cast<size_t>(tid) * a.Tmax;
        const unsigned long long t0 = globaltimer_ns();
        bool ok = true;
        for (int t = blockIdx.x; t < T && ok; t += gridDim.x) {
            while (ld_relaxed<SYS>(mine + t) != epoch) {
                if (globaltimer_ns() - t0 > kWaitLimitNs) {
                    atomicOr(&g_wait_timeout, kFarWaitCode);
                    ok = false;
                    break;
                }
            }
        }
        fence_scope<SYS>();
        if (!ok) s_abort = 1;
    }
    __syncthreads();

    // ---- phase 2: every rank's partial of the CTA's tokens, summed in rank
    // order; here thread tid takes the float4 columns tid, tid + 32 NW, ...
    // (every warp access one contiguous run)
    const int ncol = H / 4;
    for (int t = blockIdx.x; t < T && s_abort == 0; t += gridDim.x) {
        uint16_t* orow = io.out + static_cast<size_t>(t) * H;
        for (int c0 = tid; c0 < ncol; c0 += 4 * NW * 32) {
            float4 sum[4];
#pragma unroll
            for (int q = 0; q < kFarMaxWorld; ++q) {
                if (q >= world) break;
                const float4* src = reinterpret_cast<const float4*>(a.ws[q] + poff) + static_cast<size_t>(t) * ncol;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int c = c0 + u * NW * 32;
                    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
                    if (c < ncol) v = ld_cg_f4(reinterpret_cast<const float*>(src + c));
                    if (q == 0) {
                        sum[u] = v;
                    } else {
                        sum[u].x = __fadd_rn(sum[u].x, v.x);
                        sum[u].y = __fadd_rn(sum[u].y, v.y);
                        sum[u].z = __fadd_rn(sum[u].z, v.z);
                        sum[u].w = __fadd_rn(sum[u].w, v.w);
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int c = c0 + u * NW * 32;
                if (c < ncol)
                    *reinterpret_cast<uint2*>(orow + 4 * c) =
                        make_uint2(pack_bf16x2_rn(make_float2(sum[u].x, sum[u].y)),
                                   pack_bf16x2_rn(make_float2(sum[u].z, sum[u].w)));
            }
        }
    }

    // ---- the last CTA of this rank to finish publishes the epoch for the next call
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        const unsigned int n = atomicAdd(&hdr->done, 1u);
        if (n + 1u == gridDim.x) {
            hdr->done = 0u;
            __threadfence();
            *reinterpret_cast<volatile unsigned int*>(&hdr->epoch) = epoch;
        }
    }
}

template <int NW, bool GC0, bool SYS>
cudaError_t launch_far_nw(const FarArgs& a, int nloc, cudaStream_t s) {
    auto kern = finalize_ar_kernel<NW, GC0, SYS>;
    int per_sm = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, NW * 32, 0);
    if (e != cudaSuccess) return e;
    const int wave = per_sm * device_info().sm_count / nloc;   // every CTA resident at once
    if (wave < 1) return cudaErrorCooperativeLaunchTooLarge;
    const int nblk = a.T < wave ? a.T : wave;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(nblk, nloc);
    cfg.blockDim = dim3(NW * 32);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, a);
}

template <bool GC0, bool SYS>
cudaError_t launch_far_gc(const FarArgs& a, int nloc, cudaStream_t s) {
    switch (far_warps(a.H)) {
        case 1: return launch_far_nw<1, GC0, SYS>(a, nloc, s);
        case 2: return launch_far_nw<2, GC0, SYS>(a, nloc, s);
        case 4: return launch_far_nw<4, GC0, SYS>(a, nloc, s);
        case 8: return launch_far_nw<8, GC0, SYS>(a, nloc, s);
        case 16: return launch_far_nw<16, GC0, SYS>(a, nloc, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

// Warps per CTA: 32 elements per thread, next_pow2(H / 32) threads (at least
// one warp).
int far_warps(int H) {
    int P = 32;
    while (P * 32 < H) P <<= 1;
    return P / 32;
}

size_t finalize_ar_workspace_bytes(int world, int Tmax, int H) { return far_workspace_bytes(world, Tmax, H); }

size_t finalize_ar_flags_bytes(int world, int Tmax) {
    return far_flags_offset() + 2ull * world * Tmax * sizeof(uint32_t);
}

cudaError_t launch_finalize_ar(const FarLaunch& L, cudaStream_t s) {
    FarArgs a = {};
    for (int i = 0; i < L.nloc; ++i)
        a.io[i] = FarRankIO{L.expert_out[i], L.R[i], L.row_idx[i], L.wt[i], L.out[i]};
    for (int q = 0; q < L.world; ++q) a.ws[q] = static_cast<uint8_t*>(L.ws[q]);
    a.w = L.w;
    a.gc = L.gc;
    a.eps = L.eps;
    a.H = L.H;
    a.T = L.T;
    a.k = L.k;
    a.Tmax = L.Tmax;
    a.world = L.world;
    a.rank0 = L.rank0;
    // every rank on this device: GPU-scope ordering suffices; else system scope
    if (L.nloc == L.world)
        return L.gc == 0.0f ? launch_far_gc<true, false>(a, L.nloc, s) : launch_far_gc<false, false>(a, L.nloc, s);
    return L.gc == 0.0f ? launch_far_gc<true, true>(a, L.nloc, s) : launch_far_gc<false, true>(a, L.nloc, s);
}

}  // namespace mb
