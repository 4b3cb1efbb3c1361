// router_proj.cu -- the router projection: logits = scale * x W^T with an
// FP32 router weight, on the 5th-generation tensor cores (tcgen05, BF16
// operands, FP32 accumulator in tensor memory).
//
// TensorRT-LLM PR 21356 "Muse Spark Open decoder fast paths", description,
// "Router projection": FP32 weights and FP32 accumulation for up to 128
// tokens, the input cast and a scale folded in, tensor cores with a split of
// the FP32 operand from 16 tokens (the same page lists a BF16x3 router among
// its experiments).
//
// Precision.  The hidden states are BF16, so x needs no split.  The FP32
// weight is prepared once into three BF16 parts, w = w1 + w2 + w3 + d with
// w1 = bf16(w), w2 = bf16(w - w1), w3 = bf16(w - w1 - w2) (each remainder is
// exact in FP32) and |d| <= 2^-27 |w|.  A product of two BF16 values is exact
// in FP32, so x W^T = x w1^T + x w2^T + x w3^T.  The three parts of a CTA's
// experts sit side by side as one B operand, so each K step is a single MMA
// (M = 128, N = 3 x experts) that reads the x slice from shared memory once;
// the tensor core accumulates each part in its own FP32 columns, and the
// epilogue adds them, the two small parts first: w1 + (w2 + w3).
//
// Work split (one M tile of 128 token rows per grid row; rows >= T read as
// zero): each CTA owns NE experts (16, or 32 when the 16-expert grid would
// take more than one wave) and one of C contiguous K chunks, C <= 8 CTAs of a
// thread-block cluster.  One thread streams the chunk's slabs of 64 K elements
// with TMA into a ring of 4 (NE = 16) or 3 (NE = 32) stages (x: 128 rows x 128
// bytes, the three weight parts: NE rows x 128 bytes each, all 128-byte
// swizzled, which is the K-major layout the MMA reads, the parts back to
// back); another thread issues each slab's 4 MMAs (K steps of 16, M = 128,
// N = 3 NE) into a 128 x 3 NE FP32 accumulator in tensor memory and hands the
// stage back with tcgen05.commit.
// No CTA-wide barrier runs inside the K loop.  The C partial accumulators are
// then summed across the cluster in rank order through distributed shared
// memory (no atomics: the same result run to run), scaled, and written for the
// tokens below T.
#include "internal.h"
#include "common.cuh"
#include "tmem.cuh"
#include "tmap.h"

namespace mb {

namespace {

constexpr int kRpThreads = 128;           // 4 warps: one per tensor-memory lane quadrant
constexpr int kRpM = 128;                 // token rows per MMA tile
constexpr int kRpSlabK = 64;              // K elements per slab (one 128-byte swizzle row of BF16)
constexpr int kRpXTile = kRpM * 128;      // 16 KB

// Shape of a CTA's tile for NE experts per CTA (16, or 32 when the 16-expert
// grid would need more than one wave): the MMA N is 3 NE (the three weight
// parts side by side), part p of expert n accumulates in column NE p + n.
template <int NE>
struct RpShape {
    static constexpr int kN = NE;
    static constexpr int kNParts = 3 * NE;
    static constexpr int kStages = NE == 16 ? 4 : 3;          // 2 CTAs per SM either way
    static constexpr int kWTile = NE * 128;                   // one weight part's slab
    static constexpr int kStageBytes = kRpXTile + 3 * kWTile; // parts back to back: one 3 NE-row B operand
    static constexpr size_t kSmemBytes = 1024 + static_cast<size_t>(kStages) * kStageBytes + kRpM * NE * 4;
    static constexpr int kTmemCols = kNParts <= 64 ? 64 : 128;   // allocation unit >= kNParts
    // Instruction descriptor: FP32 accumulator, BF16 A and B, both K-major, N = kNParts, M = kRpM.
    static constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) |
                                       (static_cast<uint32_t>(kNParts >> 3) << 17) |
                                       (static_cast<uint32_t>(kRpM >> 4) << 24);
    static_assert(NE % 16 == 0, "the epilogue reads 16 columns at a time");
    static_assert(kNParts % 16 == 0 && kNParts <= 256, "an M = 128 MMA takes N in steps of 16 up to 256");
    static_assert(kNParts <= kTmemCols, "the accumulator fits its tensor-memory allocation");
    static_assert(2 * (kSmemBytes + 1024) <= 228 * 1024, "two CTAs fit one SM's shared memory");
};

struct RouterProjArgs {
    float* logits;        // [T, E] FP32
    int T, H, E;
    int kc;               // K elements per CTA (a multiple of 64)
    float scale;
};

// ---- tcgen05 MMA primitives (cta_group::1; tensor-memory helpers in tmem.cuh)
// D[128 x N] (+)= A[128 x 16] B[N x 16]^T, BF16 operands from shared memory.
__device__ __forceinline__ void mma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(0u), "r"(0u), "r"(0u), "r"(0u)
        : "memory");
}
// Arrive on `bar` once every MMA this thread issued so far has completed.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_addr(bar))
                 : "memory");
}
// Shared-memory matrix descriptor, K-major, 128-byte swizzle: 8-row groups
// 1024 bytes apart (stride byte offset), leading byte offset unused (1),
// descriptor version 1, swizzle mode 2.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr) {
    return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (static_cast<uint64_t>(1u) << 16) |
           (static_cast<uint64_t>(1024u >> 4) << 32) | (static_cast<uint64_t>(1u) << 46) |
           (static_cast<uint64_t>(2u) << 61);
}

template <int C, int NE>
__global__ void __launch_bounds__(kRpThreads) router_proj_kernel(const __grid_constant__ CUtensorMap xmap,
                                                                 const __grid_constant__ CUtensorMap wmap,
                                                                 const RouterProjArgs a) {
    extern __shared__ uint8_t rp_smem_raw[];
    const uint32_t raw = smem_addr(rp_smem_raw);
    uint8_t* stages = rp_smem_raw + (((raw + 1023u) & ~1023u) - raw);   // 1024-byte aligned (128-byte swizzle)
    using S = RpShape<NE>;
    float* part = reinterpret_cast<float*>(stages + S::kStages * S::kStageBytes);   // [128][NE] partial sums
    __shared__ __align__(8) uint64_t full[S::kStages];    // slab landed (TMA)
    __shared__ __align__(8) uint64_t empty[S::kStages];   // slab's MMAs done (tcgen05.commit)
    __shared__ __align__(8) uint64_t done;               // every MMA done
    __shared__ uint32_t s_tmem;
    __shared__ int s_issued, s_consumed;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int krank = blockIdx.x % C;
    const int e0 = (blockIdx.x / C) * NE;
    const int m0 = blockIdx.y * kRpM;
    const int kbase = krank * a.kc;
    const int J = a.kc / kRpSlabK;

    if (threadIdx.x == 0) {
        for (int i = 0; i < S::kStages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        mbar_init(&done, 1);
        s_issued = 0;
        s_consumed = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(&s_tmem, S::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_d = s_tmem;
    griddep_wait();
    griddep_launch();

    // One lane of warp 0 produces, one lane of warp 1 issues the MMAs; their
    // warp-mates wait at __syncwarp (not on the barriers, which would make the
    // whole warp sleep with them).
    if (warp == 0) {
        if (lane == 0) {                // TMA producer
        int j = 0;
        for (; j < J; ++j) {
            const int s = j % S::kStages;
            if (j >= S::kStages &&
                !mbar_wait_bounded(&empty[s], static_cast<uint32_t>((j / S::kStages - 1) & 1), 8u))
                break;
            uint8_t* st = stages + s * S::kStageBytes;
            const int k0 = kbase + j * kRpSlabK;
            mbar_arrive_expect_tx(&full[s], S::kStageBytes);
            tma_load_2d(smem_addr(st), &xmap, k0, m0, &full[s]);
#pragma unroll
            for (int p = 0; p < 3; ++p)
                tma_load_2d(smem_addr(st + kRpXTile + p * S::kWTile), &wmap, k0, p * a.E + e0, &full[s]);
        }
        s_issued = j;
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {                // MMA issuer
        int j = 0;
        for (; j < J; ++j) {
            const int s = j % S::kStages;
            if (!mbar_wait_bounded(&full[s], static_cast<uint32_t>((j / S::kStages) & 1), 8u)) break;
            tc_fence_after();
            const uint32_t sa = smem_addr(stages + s * S::kStageBytes);
#pragma unroll
            for (int ks = 0; ks < kRpSlabK / 16; ++ks)   // K steps of 16 BF16 = 32 bytes; B = parts 0..2
                mma_bf16(tmem_d, smem_desc_sw128(sa + 32u * ks), smem_desc_sw128(sa + kRpXTile + 32u * ks), S::kIdesc,
                         (j | ks) != 0 ? 1u : 0u);
            mma_commit(&empty[s]);
        }
        s_consumed = j;
        mma_commit(&done);   // arrives once every MMA issued above has completed
        }
        __syncwarp();
    }
    const bool finished = mbar_wait_bounded(&done, 0u, 8u);
    __syncthreads();
    const bool complete = finished && s_consumed == J;
    if (threadIdx.x == 0)   // copies issued but never consumed (an early stop) land before the CTA exits
        for (int j = s_consumed; j < s_issued; ++j)
            mbar_wait_bounded(&full[j % S::kStages], static_cast<uint32_t>((j / S::kStages) & 1), 8u);
    tc_fence_after();

    // partial accumulator: warp w holds token rows 32w .. 32w + 31; part p of
    // expert n in column NE p + n, read 16 experts at a time
    const uint32_t trow = tmem_d + (static_cast<uint32_t>(32 * warp) << 16);
#pragma unroll
    for (int h = 0; h < NE / 16; ++h) {
        float v[16], u[16];
        tmem_ld16(trow + static_cast<uint32_t>(NE + 16 * h), v);
        tmem_ld16(trow + static_cast<uint32_t>(2 * NE + 16 * h), u);
#pragma unroll
        for (int n = 0; n < 16; ++n) u[n] = v[n] + u[n];
        tmem_ld16(trow + static_cast<uint32_t>(16 * h), v);
#pragma unroll
        for (int n = 0; n < 16; ++n) part[(32 * warp + lane) * NE + 16 * h + n] = complete ? v[n] + u[n] : 0.0f;
    }
    tc_fence_before();
    if constexpr (C > 1) {
        asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
    } else {
        __syncthreads();
    }
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem_d, S::kTmemCols);
    }

    // this CTA's rows of the tile: the C partials summed in rank order
    constexpr int kRows = kRpM / C;
    for (int o = threadIdx.x; o < kRows * NE; o += kRpThreads) {
        const int m = krank * kRows + o / NE, n = o % NE;
        const float* src = part + m * NE + n;
        float pv[C];
#pragma unroll
        for (int q = 0; q < C; ++q) {
            if constexpr (C == 1) {
                pv[q] = *src;
            } else {
                uint32_t remote;
                asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_addr(src)), "r"(q));
                asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(pv[q]) : "r"(remote) : "memory");
            }
        }
        const float sum = tree_sum_array<C>(pv);
        if (m0 + m < a.T) a.logits[static_cast<size_t>(m0 + m) * a.E + e0 + n] = __fmul_rn(a.scale, sum);
    }
    if constexpr (C > 1)
        asm volatile("barrier.cluster.arrive.relaxed.aligned;\n\tbarrier.cluster.wait.aligned;" ::: "memory");
}

__device__ __forceinline__ uint16_t bf16_bits_rn(float x) {
    uint16_t r;
    asm("cvt.rn.bf16.f32 %0, %1;" : "=h"(r) : "f"(x));
    return r;
}

// w3[p][e][h], p = 0, 1, 2: the BF16 parts of w (see the file comment).
__global__ void router_weight_split_kernel(const float* __restrict__ w, int64_t n, uint16_t* __restrict__ w3) {
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const float x = w[i];
        const uint16_t b1 = bf16_bits_rn(x);
        const float r1 = __fsub_rn(x, __uint_as_float(static_cast<uint32_t>(b1) << 16));
        const uint16_t b2 = bf16_bits_rn(r1);
        const float r2 = __fsub_rn(r1, __uint_as_float(static_cast<uint32_t>(b2) << 16));
        w3[i] = b1;
        w3[n + i] = b2;
        w3[2 * n + i] = bf16_bits_rn(r2);
    }
}

template <int C, int NE>
cudaError_t launch_rp(const CUtensorMap& xmap, const CUtensorMap& wmap, const RouterProjArgs& a, cudaStream_t s) {
    using S = RpShape<NE>;
    cudaError_t e = cudaFuncSetAttribute(reinterpret_cast<const void*>(router_proj_kernel<C, NE>),
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(S::kSmemBytes));
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((a.E / NE) * C, (a.T + kRpM - 1) / kRpM);
    cfg.blockDim = dim3(kRpThreads);
    cfg.dynamicSmemBytes = S::kSmemBytes;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if constexpr (C > 1) {
        attr[1].id = cudaLaunchAttributeClusterDimension;
        attr[1].val.clusterDim.x = C;
        attr[1].val.clusterDim.y = 1;
        attr[1].val.clusterDim.z = 1;
        cfg.numAttrs = 2;
    }
    return cudaLaunchKernelEx(&cfg, router_proj_kernel<C, NE>, xmap, wmap, a);
}

template <int C>
cudaError_t launch_rp_ne(int NE, const CUtensorMap& xmap, const CUtensorMap& wmap, const RouterProjArgs& a,
                         cudaStream_t s) {
    return NE == 32 ? launch_rp<C, 32>(xmap, wmap, a, s) : launch_rp<C, 16>(xmap, wmap, a, s);
}

}  // namespace

// K chunks per expert tile: the largest C in {8, 4, 2, 1} with H % (64 C) == 0.
int router_proj_chunks(int H) {
    for (int c = 8; c > 1; c >>= 1)
        if (H % (kRpSlabK * c) == 0) return c;
    return 1;
}

// Experts per CTA: 32 when E allows it and the 16-expert grid would take more
// than one wave at two CTAs per SM, else 16.  Every output element is summed
// the same way either way, so the choice changes no result.
int router_proj_experts_per_cta(int T, int E, int C) {
    if (E % 32 != 0) return 16;
    const int64_t ctas16 = static_cast<int64_t>(E / 16) * C * ((T + kRpM - 1) / kRpM);
    return ctas16 > 2LL * device_info().sm_count ? 32 : 16;
}

cudaError_t launch_router_weight_split(const float* w, int E, int H, uint16_t* w3, cudaStream_t s) {
    const int64_t n = static_cast<int64_t>(E) * H;
    int grid = static_cast<int>((n + 255) / 256);
    if (grid > device_info().sm_count * 8) grid = device_info().sm_count * 8;
    router_weight_split_kernel<<<grid, 256, 0, s>>>(w, n, w3);
    return cudaGetLastError();
}

cudaError_t launch_router_proj(const uint16_t* x, int T, int H, const uint16_t* w3, int E, float scale, float* logits,
                               cudaStream_t s) {
    const int C = router_proj_chunks(H);
    const int NE = router_proj_experts_per_cta(T, E, C);
    const RouterProjArgs a{logits, T, H, E, H / C, scale};
    CUtensorMap xmap, wmap;
    if (!encode_2d_map(&xmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, x, static_cast<uint64_t>(T), static_cast<uint64_t>(H),
                       static_cast<uint64_t>(H) * 2, kRpM, kRpSlabK, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_2d_map(&wmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, w3, static_cast<uint64_t>(3) * E,
                       static_cast<uint64_t>(H), static_cast<uint64_t>(H) * 2, static_cast<uint32_t>(NE), kRpSlabK,
                       CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    switch (C) {
        case 8: return launch_rp_ne<8>(NE, xmap, wmap, a, s);
        case 4: return launch_rp_ne<4>(NE, xmap, wmap, a, s);
        case 2: return launch_rp_ne<2>(NE, xmap, wmap, a, s);
        default: return launch_rp_ne<1>(NE, xmap, wmap, a, s);
    }
}

}  // namespace mb
