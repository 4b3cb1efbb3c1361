// route.cu -- stage 1, the sigmoid router gate (one warp per token).
//
// Computes, per valid token t (TensorRT-LLM PR 21356 "Muse Spark Open decoder
// fast paths", description, Routing; lmdeploy PR 4835 "MoE gate v2", token
// mask):
//   s_e = sigmoid(l_e)            FP32, the project's exp (below)
//   c_e = s_e + bias_e            selection score only
//   picks = first k experts in the order (c descending, id ascending)
//   w_j   = s_{pick j} / (s_{pick 0} + ... + s_{pick k-1})   summed in pick order
// and for an invalid token ids = -1, weights = 0 without reading its logits.
//
// Selection: every lane streams E/32 scores with 128-bit loads and keeps a
// sorted register list of its best L candidates as 64-bit keys
// (orderable(c) << 32 | ~id, so a larger key is the better pick and keys are
// unique); k rounds of a warp-wide max over the lanes' list heads then emit
// the picks in order.  Nothing is staged in shared or global scratch memory.
#include "common.cuh"
#include "internal.h"

namespace mb {

// ---------------------------------------------------------------- exp / sigmoid
// Range reduction x = n ln2 + r with a Cody-Waite split of ln2 (a 15-fraction-bit
// head, so n * head is exact), a degree-7 Taylor polynomial of e^r (Horner,
// fused multiply-adds) and 2^n from the exponent field.  Inputs are clamped to
// [-87, 88] so 2^n stays a normal number.
__device__ __forceinline__ float exp_fixed(float x) {
    constexpr float kLn2Hi = 22713.0f / 32768.0f;
    constexpr float kLn2Lo = (float)(0.6931471805599453094 - 22713.0 / 32768.0);
    constexpr float kLog2e = (float)1.4426950408889634074;
    x = (x < -87.0f) ? -87.0f : x;
    x = (x > 88.0f) ? 88.0f : x;
    const float t = __fmul_rn(x, kLog2e);
    const float n = rintf(t);
    float r = fmaf(-n, kLn2Hi, x);
    r = fmaf(-n, kLn2Lo, r);
    float p = (float)(1.0 / 5040.0);
    p = fmaf(p, r, (float)(1.0 / 720.0));
    p = fmaf(p, r, (float)(1.0 / 120.0));
    p = fmaf(p, r, (float)(1.0 / 24.0));
    p = fmaf(p, r, (float)(1.0 / 6.0));
    p = fmaf(p, r, 0.5f);
    p = fmaf(p, r, 1.0f);
    p = fmaf(p, r, 1.0f);
    const float two_n = __uint_as_float(static_cast<uint32_t>(static_cast<int>(n) + 127) << 23);
    return __fmul_rn(p, two_n);
}

__device__ __forceinline__ float sigmoid_fixed(float x) {
    const float e = exp_fixed(-x);
    return __frcp_rn(__fadd_rn(1.0f, e));
}

// Key of expert e with selection score c: larger key = earlier pick.
__device__ __forceinline__ uint64_t select_key(float c, int e) {
    c = __fadd_rn(c, 0.0f);                                  // -0 -> +0
    const uint32_t u = __float_as_uint(c);
    uint32_t hi = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    if (c != c) hi = 0u;                                     // NaN sorts last
    return (static_cast<uint64_t>(hi) << 32) | static_cast<uint32_t>(~static_cast<uint32_t>(e));
}

template <int L>
__device__ __forceinline__ void list_insert(uint64_t (&list)[L], uint64_t key) {
    if (key > list[L - 1]) {
#pragma unroll
        for (int i = 0; i < L; ++i) {
            const uint64_t hi = list[i] > key ? list[i] : key;
            key = list[i] > key ? key : list[i];
            list[i] = hi;
        }
    }
}

__device__ __forceinline__ uint64_t warp_max_u64(uint64_t v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        const uint64_t o = __shfl_xor_sync(0xffffffffu, v, off);
        v = o > v ? o : v;
    }
    return v;
}

template <int L>
__global__ void __launch_bounds__(256) route_kernel(const float* __restrict__ logits,
                                                    const float* __restrict__ bias,
                                                    const uint8_t* __restrict__ mask, int T, int E,
                                                    int k, int32_t* __restrict__ ids,
                                                    float* __restrict__ weights) {
    griddep_wait();     // inputs may come from the previous kernel on the stream
    griddep_launch();
    const int lane = threadIdx.x & 31;
    const int warp = static_cast<int>((blockIdx.x * blockDim.x + threadIdx.x) >> 5);
    const int nwarps = static_cast<int>((gridDim.x * blockDim.x) >> 5);
    const bool vec = (E & 3) == 0;

    for (int t = warp; t < T; t += nwarps) {
        int32_t* id_row = ids + static_cast<size_t>(t) * k;
        float* w_row = weights + static_cast<size_t>(t) * k;
        if (mask[t] == 0) {
            if (lane < k) {
                id_row[lane] = -1;
                w_row[lane] = 0.0f;
            }
            continue;
        }
        const float* l = logits + static_cast<size_t>(t) * E;
        uint64_t list[L];
#pragma unroll
        for (int i = 0; i < L; ++i) list[i] = 0ull;

        if (vec) {
            const int nq = E >> 2;
            for (int q0 = lane; q0 < nq; q0 += 128) {
                float4 v[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int q = q0 + 32 * u;
                    if (q < nq) v[u] = ld_nc_f4(l + 4 * q);
                }
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int q = q0 + 32 * u;
                    if (q < nq) {
                        const float4 b = __ldg(reinterpret_cast<const float4*>(bias) + q);
                        const int e = 4 * q;
                        list_insert<L>(list, select_key(__fadd_rn(sigmoid_fixed(v[u].x), b.x), e));
                        list_insert<L>(list, select_key(__fadd_rn(sigmoid_fixed(v[u].y), b.y), e + 1));
                        list_insert<L>(list, select_key(__fadd_rn(sigmoid_fixed(v[u].z), b.z), e + 2));
                        list_insert<L>(list, select_key(__fadd_rn(sigmoid_fixed(v[u].w), b.w), e + 3));
                    }
                }
            }
        } else {
            for (int e = lane; e < E; e += 32)
                list_insert<L>(list, select_key(__fadd_rn(sigmoid_fixed(__ldg(l + e)), __ldg(bias + e)), e));
        }

        // k rounds: the lane holding the best remaining head pops it.
        uint64_t mine = 0ull;
        for (int j = 0; j < k; ++j) {
            const uint64_t best = warp_max_u64(list[0]);
            if (list[0] == best) {
#pragma unroll
                for (int i = 0; i < L - 1; ++i) list[i] = list[i + 1];
                list[L - 1] = 0ull;
            }
            if (lane == j) mine = best;
        }
        const int e = static_cast<int>(~static_cast<uint32_t>(mine));
        float s = 0.0f;
        if (lane < k) s = sigmoid_fixed(__ldg(l + e));
        float S = 0.0f;
        for (int j = 0; j < k; ++j) S = __fadd_rn(S, __shfl_sync(0xffffffffu, s, j));
        if (lane < k) {
            id_row[lane] = e;
            w_row[lane] = __fdiv_rn(s, S);
        }
    }
}

cudaError_t launch_route(const float* logits, const float* bias, const uint8_t* mask, int T, int E,
                         int k, int32_t* ids, float* weights, cudaStream_t s) {
    const int per_lane = (E + 31) / 32;
    const int need = per_lane < k ? per_lane : k;
    const int warps_per_cta = 8;
    int grid = (T + warps_per_cta - 1) / warps_per_cta;
    const int cap = device_info().sm_count * 8;
    if (grid > cap) grid = cap;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(256);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (need <= 8) return cudaLaunchKernelEx(&cfg, route_kernel<8>, logits, bias, mask, T, E, k, ids, weights);
    if (need <= 16) return cudaLaunchKernelEx(&cfg, route_kernel<16>, logits, bias, mask, T, E, k, ids, weights);
    return cudaLaunchKernelEx(&cfg, route_kernel<32>, logits, bias, mask, T, E, k, ids, weights);
}

}  // namespace mb
