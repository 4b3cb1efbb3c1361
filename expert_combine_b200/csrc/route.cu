// route.cu -- stage 1, the sigmoid router gate (one token per warp iteration).
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
// Selection (route.cuh): a shortlist from a fast sigmoid with a bounded
// error, then the exact sigmoid and an exact ranking of the shortlisted
// experts only.  For E <= 512 a lane holds its E/32 logits in registers; for
// larger E the approximate keys of the token go through one shared-memory row
// per warp.  When the shortlist overflows (massive exact ties), the token
// takes the exact merge rounds: k warp maxima (redux.sync) over the lanes'
// best keys, the lowest expert id winning among equal keys.  Nothing is
// staged in global scratch memory.
#include "internal.h"
#include "route.cuh"

namespace mb {

// MODE > 0: E <= 32 MODE, EPL = MODE logits per lane in registers (exact
// rounds up to 8 per lane, the shortlist at 16); MODE < 0:
// larger E, each lane keeping a sorted list of its L = -MODE best exact
// scores (the router beside the norm-quant, which has no shared memory to
// spare).
//
// BESIDE: launched right after the norm-quant kernel of the same tokens, to
// run in the registers and warp slots that kernel leaves free on every SM.
// It then starts without waiting for that kernel (it does not read its
// outputs; the norm-quant kernel lets it launch only after its own wait for
// the kernels before it, so the router's inputs are ready and the previous
// readers of ids / weights are done), and waits for it at the end, so that
// the router finishes after the norm-quant and the kernels after it may rely
// on both.
// (the shortlist instantiation is held to four CTAs' registers per SM: more
// warps hide its dependent chains; measured 115 -> 109 us at 65536 x 512, k = 22)
template <int MODE, bool BESIDE>
__global__ void __launch_bounds__(256, (MODE > 8 && !BESIDE) ? 4 : 1) route_kernel(const float* __restrict__ logits,
                                                    const float* __restrict__ bias,
                                                    const uint8_t* __restrict__ mask, int T, int E,
                                                    int k, int32_t* __restrict__ ids,
                                                    float* __restrict__ weights) {
    if constexpr (!BESIDE) griddep_wait();     // inputs may come from the previous kernel on the stream
    griddep_launch();
    const int lane = threadIdx.x & 31;
    const int warp = static_cast<int>((blockIdx.x * blockDim.x + threadIdx.x) >> 5);
    const int nwarps = static_cast<int>((gridDim.x * blockDim.x) >> 5);
    const bool vec = (E & 3) == 0;

    // one token per warp iteration: each token's selection is one dependent
    // chain, and more warps with one chain each measured faster than fewer
    // warps interleaving two
    if constexpr (MODE > 8) {
        route_shortlist_tokens<MODE>(logits, bias, mask, T, E, k, ids, weights, warp, nwarps, lane);
    } else if constexpr (MODE > 0) {
        route_singles<MODE, !BESIDE>(logits, bias, mask, T, E, k, ids, weights, warp, nwarps, lane);
    } else {
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
            uint32_t pick_key = 0u, pick_id = 0u;
            route_token_list<-MODE>(l, bias, E, k, lane, vec, pick_key, pick_id);
            route_write(l, k, lane, pick_id, id_row, w_row);
        }
    }
    if constexpr (BESIDE) griddep_wait();
}

// E > 512 on its own: the shortlist over approximate keys staged in one
// shared-memory row per warp (kRouteWideWarps warps per CTA).
constexpr int kRouteWideWarps = 4;

__global__ void __launch_bounds__(32 * kRouteWideWarps) route_wide_kernel(const float* __restrict__ logits,
                                                                          const float* __restrict__ bias,
                                                                          const uint8_t* __restrict__ mask, int T,
                                                                          int E, int k, int32_t* __restrict__ ids,
                                                                          float* __restrict__ weights) {
    extern __shared__ __align__(16) uint16_t route_keys[];
    griddep_wait();
    griddep_launch();
    const int lane = threadIdx.x & 31;
    const int warp = static_cast<int>((blockIdx.x * blockDim.x + threadIdx.x) >> 5);
    const int nwarps = static_cast<int>((gridDim.x * blockDim.x) >> 5);
    uint16_t* keys = route_keys + static_cast<size_t>(threadIdx.x >> 5) * 128 * ((E + 127) >> 7);
    route_shortlist_tokens<0>(logits, bias, mask, T, E, k, ids, weights, warp, nwarps, lane, keys);
}

namespace {

template <bool BESIDE>
cudaError_t launch_route_cfg(const float* logits, const float* bias, const uint8_t* mask, int T, int E, int k,
                             int32_t* ids, float* weights, int threads, int grid_cap, cudaStream_t s) {
    const int per_lane = (E + 31) / 32;
    const int warps_per_cta = threads / 32;
    // scores per lane, rounded up to whole 128-bit loads
    const int epl = (per_lane + 3) / 4 * 4;
    int grid = (T + warps_per_cta - 1) / warps_per_cta;   // one token per warp, up to the cap
    if (grid > grid_cap) grid = grid_cap;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(threads);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (epl <= 4) return cudaLaunchKernelEx(&cfg, route_kernel<4, BESIDE>, logits, bias, mask, T, E, k, ids, weights);
    if (epl <= 8) return cudaLaunchKernelEx(&cfg, route_kernel<8, BESIDE>, logits, bias, mask, T, E, k, ids, weights);
    if (epl <= 16) return cudaLaunchKernelEx(&cfg, route_kernel<16, BESIDE>, logits, bias, mask, T, E, k, ids, weights);
    if constexpr (!BESIDE) {
        // the shortlist with its keys in shared memory
        const size_t smem = static_cast<size_t>(kRouteWideWarps) * 128 * ((E + 127) / 128) * sizeof(uint16_t);
        cudaError_t e = cudaFuncSetAttribute(reinterpret_cast<const void*>(route_wide_kernel),
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
        if (e != cudaSuccess) return e;
        int per_sm = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, route_wide_kernel, 32 * kRouteWideWarps, smem);
        if (e != cudaSuccess) return e;
        if (per_sm < 1) per_sm = 1;
        int g = (T + kRouteWideWarps - 1) / kRouteWideWarps;
        if (g > device_info().sm_count * per_sm) g = device_info().sm_count * per_sm;
        cfg.gridDim = dim3(g);
        cfg.blockDim = dim3(32 * kRouteWideWarps);
        cfg.dynamicSmemBytes = smem;
        return cudaLaunchKernelEx(&cfg, route_wide_kernel, logits, bias, mask, T, E, k, ids, weights);
    }
    if (k <= 8) return cudaLaunchKernelEx(&cfg, route_kernel<-8, BESIDE>, logits, bias, mask, T, E, k, ids, weights);
    if (k <= 16) return cudaLaunchKernelEx(&cfg, route_kernel<-16, BESIDE>, logits, bias, mask, T, E, k, ids, weights);
    return cudaLaunchKernelEx(&cfg, route_kernel<-32, BESIDE>, logits, bias, mask, T, E, k, ids, weights);
}

}  // namespace

// Every binary32 input once: the largest |sigmoid_fast(x) - sigmoid_fixed(x)|
// (NaN inputs skipped), as the bits of a non-negative float, max-combined into
// *err_bits (which starts at 0).
__global__ void __launch_bounds__(256) fast_sigmoid_check_kernel(unsigned int* __restrict__ err_bits) {
    const uint64_t n = 1ull << 32;
    const uint64_t stride = static_cast<uint64_t>(gridDim.x) * blockDim.x;
    uint32_t worst = 0u;
    for (uint64_t i = static_cast<uint64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += stride) {
        const float x = __uint_as_float(static_cast<uint32_t>(i));
        if (x != x) continue;
        const float d = fabsf(__fsub_rn(sigmoid_fast(x), sigmoid_fixed(x)));
        worst = max(worst, (d == d) ? __float_as_uint(d) : 0x7F800000u);
    }
    worst = __reduce_max_sync(0xffffffffu, worst);
    if ((threadIdx.x & 31) == 0) atomicMax(err_bits, worst);
}

cudaError_t launch_fast_sigmoid_check(float* max_err, cudaStream_t s) {
    cudaError_t e = cudaMemsetAsync(max_err, 0, sizeof(float), s);
    if (e != cudaSuccess) return e;
    fast_sigmoid_check_kernel<<<device_info().sm_count * 8, 256, 0, s>>>(reinterpret_cast<unsigned int*>(max_err));
    return cudaGetLastError();
}

cudaError_t launch_route(const float* logits, const float* bias, const uint8_t* mask, int T, int E,
                         int k, int32_t* ids, float* weights, cudaStream_t s) {
    return launch_route_cfg<false>(logits, bias, mask, T, E, k, ids, weights, 256, device_info().sm_count * 8, s);
}

cudaError_t launch_route_beside(const float* logits, const float* bias, const uint8_t* mask, int T, int E,
                                int k, int32_t* ids, float* weights, cudaStream_t s) {
    // 64-thread CTAs, at most three per SM: six warps of 64 registers fit
    // beside a norm-quant CTA (512 threads x 104 registers); one token per warp
    return launch_route_cfg<true>(logits, bias, mask, T, E, k, ids, weights, 64, device_info().sm_count * 3, s);
}

}  // namespace mb
