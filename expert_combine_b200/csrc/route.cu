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
// Selection: every lane reads E/32 scores with 128-bit loads and turns each
// into a 32-bit order-preserving key; k merge rounds then emit the picks in
// order, each a warp max (redux.sync) over the lanes' current bests with the
// lowest expert id winning among equal keys (a warp min over the tied
// lanes).  For E <= 512 a lane keeps its best and second-best remaining
// scores, promotes the second when its best is picked and rescans its <= 16
// scores only when picked again before a rescan; beyond that it keeps a
// sorted list of its best k.  Nothing is staged in
// shared or global scratch memory.
#include "internal.h"
#include "route.cuh"

namespace mb {

// MODE > 0: the small path with EPL = MODE scores per lane; MODE < 0: the
// list path with L = -MODE entries.
//
// BESIDE: launched right after the norm-quant kernel of the same tokens, to
// run in the registers and warp slots that kernel leaves free on every SM.
// It then starts without waiting for that kernel (it does not read its
// outputs; the norm-quant kernel lets it launch only after its own wait for
// the kernels before it, so the router's inputs are ready and the previous
// readers of ids / weights are done), and waits for it at the end, so that
// the router finishes after the norm-quant and the kernels after it may rely
// on both.
template <int MODE, bool BESIDE>
__global__ void __launch_bounds__(256) route_kernel(const float* __restrict__ logits,
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
    // chain of warp reductions, and more warps with one chain each measured
    // faster than fewer warps interleaving two
    if constexpr (MODE > 0) {
        route_singles<MODE>(logits, bias, mask, T, E, k, ids, weights, warp, nwarps, lane);
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
    if (k <= 8) return cudaLaunchKernelEx(&cfg, route_kernel<-8, BESIDE>, logits, bias, mask, T, E, k, ids, weights);
    if (k <= 16) return cudaLaunchKernelEx(&cfg, route_kernel<-16, BESIDE>, logits, bias, mask, T, E, k, ids, weights);
    return cudaLaunchKernelEx(&cfg, route_kernel<-32, BESIDE>, logits, bias, mask, T, E, k, ids, weights);
}

}  // namespace

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
