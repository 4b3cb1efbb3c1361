// api.cu -- the C ABI (include/moe_boundary.h): argument checks, status codes
// and launches.  No allocation, no synchronisation, no host fallback.
#include <climits>
#include <cstring>
#include <cstdarg>
#include <cstdio>
#include <mutex>

#include "moe_boundary.h"
#include "common.cuh"
#include "internal.h"

namespace mb {

namespace {

thread_local char t_last_error[512] = "";

int fail(int code, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(t_last_error, sizeof(t_last_error), fmt, ap);
    va_end(ap);
    return code;
}

int cuda_status(cudaError_t e, const char* where) {
    if (e == cudaSuccess) return MB_OK;
    return fail(MB_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned256(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 255u) == 0; }

constexpr int kMaxDevices = 64;
DeviceInfo g_info[kMaxDevices];
std::once_flag g_once[kMaxDevices];

bool hidden_ok(int H) { return H > 0 && H % 16 == 0 && H <= kMaxHidden; }

}  // namespace

const DeviceInfo& device_info() {
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= kMaxDevices) dev = 0;
    std::call_once(g_once[dev], [dev] {
        int sms = 148, smem = 227 * 1024;
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        cudaDeviceGetAttribute(&smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        g_info[dev].sm_count = sms;
        g_info[dev].max_smem_optin = smem;
    });
    return g_info[dev];
}

}  // namespace mb

using namespace mb;

extern "C" {

const char* mb_last_error(void) { return t_last_error; }

int moe_boundary_supported(int stage, int T, int H, int E, int k, int tp) {
    if (T < 0) return 0;
    switch (stage) {
        case MB_STAGE_ROUTE:
            return (k >= 1 && k <= kMaxTopK && E >= k && E <= kMaxExperts) ? 1 : 0;
        case MB_STAGE_NORM_QUANT:
            return (hidden_ok(H) && tp >= 1 && H % tp == 0 && (H / tp) % 16 == 0) ? 1 : 0;
        case MB_STAGE_COMBINE:
        case MB_STAGE_COMBINE_JOIN:
            return (hidden_ok(H) && k >= 1 && k <= kMaxTopK) ? 1 : 0;
        case MB_STAGE_JOIN:
            return hidden_ok(H) ? 1 : 0;
        case MB_STAGE_ROUTER_LOGITS:
            return (H >= 64 && H % 64 == 0 && H <= kMaxHidden && E >= 16 && E % 16 == 0 && E <= kMaxExperts &&
                    (static_cast<int64_t>(T) + 127) / 128 <= 65535)
                       ? 1
                       : 0;
        case MB_STAGE_DISPATCH:
            return (k >= 1 && k <= kMaxTopK && E >= 1 && E <= kMaxExperts &&
                    static_cast<int64_t>(T) * k <= INT32_MAX)
                       ? 1
                       : 0;
        case MB_STAGE_FINALIZE_AR:
            return (H >= 16 && H % 16 == 0 && H <= kMaxHidden && k >= 1 && k <= kMaxTopK && tp >= 1 &&
                    tp <= kFarMaxWorld)
                       ? 1
                       : 0;
        case MB_STAGE_ROUTE_NORM_QUANT:
            return (moe_boundary_supported(MB_STAGE_ROUTE, T, H, E, k, tp) &&
                    moe_boundary_supported(MB_STAGE_NORM_QUANT, T, H, E, k, tp))
                       ? 1
                       : 0;
        default:
            return 0;
    }
}

static int check_route(const char* fn, const float* logits, const float* bias, const uint8_t* token_mask,
                       int T, int E, int k, int32_t* topk_ids, float* topk_weights) {
    if (T < 0 || E < 0 || k < 0) return fail(MB_ERR_INVALID_ARG, "%s: negative size", fn);
    if (!moe_boundary_supported(MB_STAGE_ROUTE, T, 0, E, k, 1))
        return fail(MB_ERR_UNSUPPORTED, "%s: needs 1 <= k <= %d and k <= E <= %d (k=%d, E=%d)", fn,
                    kMaxTopK, kMaxExperts, k, E);
    if (T == 0) return MB_OK;
    if (!logits || !bias || !token_mask || !topk_ids || !topk_weights)
        return fail(MB_ERR_INVALID_ARG, "%s: null pointer", fn);
    if (!aligned16(logits) || !aligned16(bias) || !aligned16(token_mask) || !aligned16(topk_ids) ||
        !aligned16(topk_weights))
        return fail(MB_ERR_INVALID_ARG, "%s: pointers must be 16-byte aligned", fn);
    return MB_OK;
}

int moe_route_check_fast_sigmoid(float* max_err, void* stream) {
    const char* fn = "moe_route_check_fast_sigmoid";
    if (!max_err) return fail(MB_ERR_INVALID_ARG, "%s: null pointer", fn);
    if ((reinterpret_cast<uintptr_t>(max_err) & 3u) != 0)
        return fail(MB_ERR_INVALID_ARG, "%s: max_err must be 4-byte aligned", fn);
    return cuda_status(launch_fast_sigmoid_check(max_err, static_cast<cudaStream_t>(stream)), fn);
}

static int check_norm_quant(const char* fn, const uint16_t* x, int M, int H, int tp, const uint16_t* norm_w,
                            const float* global_scale, uint8_t* packed, uint8_t* sf) {
    if (M < 0 || H < 0 || tp < 0) return fail(MB_ERR_INVALID_ARG, "%s: negative size", fn);
    if (tp == 0 || H % 16 != 0 || H % tp != 0 || (H / tp) % 16 != 0)
        return fail(MB_ERR_INVALID_ARG,
                    "%s: needs H %% 16 == 0, tp >= 1, H %% tp == 0, (H/tp) %% 16 == 0 (H=%d, tp=%d)", fn, H,
                    tp);
    if (!moe_boundary_supported(MB_STAGE_NORM_QUANT, M, H, 0, 0, tp))
        return fail(MB_ERR_UNSUPPORTED, "%s: H=%d outside 16..%d", fn, H, kMaxHidden);
    if (M == 0) return MB_OK;
    if (!x || !norm_w || !global_scale || !packed || !sf) return fail(MB_ERR_INVALID_ARG, "%s: null pointer", fn);
    if (!aligned16(x) || !aligned16(norm_w) || !aligned16(packed) || !aligned16(sf) ||
        (reinterpret_cast<uintptr_t>(global_scale) & 3u))
        return fail(MB_ERR_INVALID_ARG, "%s: pointers must be 16-byte aligned", fn);
    return MB_OK;
}

int moe_route(const float* logits, const float* bias, const uint8_t* token_mask, int T, int E, int k,
              int32_t* topk_ids, float* topk_weights, void* stream) {
    const int st = check_route("moe_route", logits, bias, token_mask, T, E, k, topk_ids, topk_weights);
    if (st != MB_OK || T == 0) return st;
    return cuda_status(launch_route(logits, bias, token_mask, T, E, k, topk_ids, topk_weights,
                                    static_cast<cudaStream_t>(stream)),
                       "moe_route");
}

int norm_quant_nvfp4(const uint16_t* x, int M, int H, int tp, const uint16_t* norm_w, float gain_center,
                     float eps, const float* global_scale, uint8_t* packed, uint8_t* sf, void* stream) {
    const int st = check_norm_quant("norm_quant_nvfp4", x, M, H, tp, norm_w, global_scale, packed, sf);
    if (st != MB_OK || M == 0) return st;
    return cuda_status(launch_norm_quant(x, M, H, tp, norm_w, gain_center, eps, global_scale, packed, sf,
                                         static_cast<cudaStream_t>(stream)),
                       "norm_quant_nvfp4");
}

int moe_route_norm_quant(const float* logits, const float* bias, const uint8_t* token_mask, int E, int k,
                         int32_t* topk_ids, float* topk_weights, const uint16_t* x, int M, int H, int tp,
                         const uint16_t* norm_w, float gain_center, float eps, const float* global_scale,
                         uint8_t* packed, uint8_t* sf, void* stream) {
    int st = check_route("moe_route_norm_quant", logits, bias, token_mask, M, E, k, topk_ids, topk_weights);
    if (st != MB_OK) return st;
    st = check_norm_quant("moe_route_norm_quant", x, M, H, tp, norm_w, global_scale, packed, sf);
    if (st != MB_OK || M == 0) return st;
    return cuda_status(launch_route_norm_quant(logits, bias, token_mask, E, k, topk_ids, topk_weights, x, M, H,
                                               tp, norm_w, gain_center, eps, global_scale, packed, sf,
                                               static_cast<cudaStream_t>(stream)),
                       "moe_route_norm_quant");
}

int moe_route_norm_quant_kernels(int M, int H, int tp, int E, int k) {
    if (!moe_boundary_supported(MB_STAGE_ROUTE_NORM_QUANT, M, H, E, k, tp)) return -1;
    if (M == 0) return 0;
    int n = 0;
    if (cudaGetDeviceCount(&n) != cudaSuccess || n == 0) {
        cudaGetLastError();
        return -1;
    }
    return route_norm_quant_kernels(M, H, tp, E);
}

static int check_combine(const char* fn, const uint16_t* expert_out, int64_t num_rows, int H,
                         const int32_t* row_idx, const float* weights, int T, int k,
                         const uint16_t* norm_w) {
    if (T < 0 || H < 0 || k < 0 || num_rows < 0) return fail(MB_ERR_INVALID_ARG, "%s: negative size", fn);
    if (H % 16 != 0) return fail(MB_ERR_INVALID_ARG, "%s: H %% 16 != 0 (H=%d)", fn, H);
    if (!moe_boundary_supported(MB_STAGE_COMBINE, T, H, 0, k, 1))
        return fail(MB_ERR_UNSUPPORTED, "%s: needs 16 <= H <= %d and 1 <= k <= %d (H=%d, k=%d)", fn,
                    kMaxHidden, kMaxTopK, H, k);
    if (T == 0) return MB_OK;
    if ((num_rows > 0 && !expert_out) || !row_idx || !weights || !norm_w)
        return fail(MB_ERR_INVALID_ARG, "%s: null pointer", fn);
    if (!aligned16(expert_out) || !aligned16(row_idx) || !aligned16(weights) || !aligned16(norm_w))
        return fail(MB_ERR_INVALID_ARG, "%s: pointers must be 16-byte aligned", fn);
    return MB_OK;
}

static int check_join(const char* fn, float* residual, const uint16_t* gain, const uint16_t* next_w,
                      uint16_t* next_prenorm) {
    if (!residual || !gain) return fail(MB_ERR_INVALID_ARG, "%s: null pointer", fn);
    if ((next_w == nullptr) != (next_prenorm == nullptr))
        return fail(MB_ERR_INVALID_ARG, "%s: next_w and next_prenorm must both be set or both be NULL", fn);
    if (!aligned16(residual) || !aligned16(gain) || !aligned16(next_w) || !aligned16(next_prenorm))
        return fail(MB_ERR_INVALID_ARG, "%s: pointers must be 16-byte aligned", fn);
    return MB_OK;
}

int expert_combine(const uint16_t* expert_out, int64_t num_rows, int H, const int32_t* row_idx,
                   const float* weights, int T, int k, const uint16_t* norm_w, float gain_center, float eps,
                   uint16_t* out, void* stream) {
    int st = check_combine("expert_combine", expert_out, num_rows, H, row_idx, weights, T, k, norm_w);
    if (st != MB_OK || T == 0) return st;
    if (!out) return fail(MB_ERR_INVALID_ARG, "expert_combine: null pointer");
    if (!aligned16(out)) return fail(MB_ERR_INVALID_ARG, "expert_combine: pointers must be 16-byte aligned");
    JoinArgs none{};
    return cuda_status(launch_combine(expert_out, num_rows, H, row_idx, weights, T, k, norm_w, gain_center,
                                      eps, out, none, static_cast<cudaStream_t>(stream)),
                       "expert_combine");
}

int residual_join(float* residual, const uint16_t* branch, const uint16_t* gain, float alpha, float beta,
                  float eps, const uint16_t* next_w, float next_gc, float next_eps, uint16_t* next_prenorm,
                  int T, int H, void* stream) {
    if (T < 0 || H < 0) return fail(MB_ERR_INVALID_ARG, "residual_join: negative size");
    if (H % 16 != 0) return fail(MB_ERR_INVALID_ARG, "residual_join: H %% 16 != 0 (H=%d)", H);
    if (!moe_boundary_supported(MB_STAGE_JOIN, T, H, 0, 0, 1))
        return fail(MB_ERR_UNSUPPORTED, "residual_join: H=%d outside 16..%d", H, kMaxHidden);
    if (T == 0) return MB_OK;
    int st = check_join("residual_join", residual, gain, next_w, next_prenorm);
    if (st != MB_OK) return st;
    if (!branch) return fail(MB_ERR_INVALID_ARG, "residual_join: null pointer");
    if (!aligned16(branch)) return fail(MB_ERR_INVALID_ARG, "residual_join: pointers must be 16-byte aligned");
    JoinArgs j{residual, gain, alpha, beta, eps, next_w, next_gc, next_eps, next_prenorm};
    return cuda_status(launch_residual_join(branch, T, H, j, static_cast<cudaStream_t>(stream)),
                       "residual_join");
}

int expert_combine_join(const uint16_t* expert_out, int64_t num_rows, int H, const int32_t* row_idx,
                        const float* weights, int T, int k, const uint16_t* norm_w, float gain_center,
                        float eps, uint16_t* out, float* residual, const uint16_t* gain, float alpha,
                        float beta, float join_eps, const uint16_t* next_w, float next_gc, float next_eps,
                        uint16_t* next_prenorm, void* stream) {
    int st = check_combine("expert_combine_join", expert_out, num_rows, H, row_idx, weights, T, k, norm_w);
    if (st != MB_OK || T == 0) return st;
    st = check_join("expert_combine_join", residual, gain, next_w, next_prenorm);
    if (st != MB_OK) return st;
    if (!aligned16(out))
        return fail(MB_ERR_INVALID_ARG, "expert_combine_join: pointers must be 16-byte aligned");
    JoinArgs j{residual, gain, alpha, beta, join_eps, next_w, next_gc, next_eps, next_prenorm};
    return cuda_status(launch_combine(expert_out, num_rows, H, row_idx, weights, T, k, norm_w, gain_center,
                                      eps, out, j, static_cast<cudaStream_t>(stream)),
                       "expert_combine_join");
}

int router_weight_prepare(const float* w, int E, int H, uint16_t* w3, void* stream) {
    const char* fn = "router_weight_prepare";
    if (E < 0 || H < 0) return fail(MB_ERR_INVALID_ARG, "%s: negative size", fn);
    if (!moe_boundary_supported(MB_STAGE_ROUTER_LOGITS, 1, H, E, 0, 1))
        return fail(MB_ERR_UNSUPPORTED, "%s: needs H %% 64 == 0, 64 <= H <= %d, E %% 16 == 0, 16 <= E <= %d (H=%d, E=%d)",
                    fn, kMaxHidden, kMaxExperts, H, E);
    if (!w || !w3) return fail(MB_ERR_INVALID_ARG, "%s: null pointer", fn);
    if (!aligned16(w) || !aligned16(w3)) return fail(MB_ERR_INVALID_ARG, "%s: pointers must be 16-byte aligned", fn);
    return cuda_status(launch_router_weight_split(w, E, H, w3, static_cast<cudaStream_t>(stream)), fn);
}

int router_logits(const uint16_t* x, int T, int H, const uint16_t* w3, int E, float scale, float* logits,
                  void* stream) {
    const char* fn = "router_logits";
    if (T < 0 || H < 0 || E < 0) return fail(MB_ERR_INVALID_ARG, "%s: negative size", fn);
    if (!moe_boundary_supported(MB_STAGE_ROUTER_LOGITS, T, H, E, 0, 1))
        return fail(MB_ERR_UNSUPPORTED, "%s: needs H %% 64 == 0, 64 <= H <= %d, E %% 16 == 0, 16 <= E <= %d (H=%d, E=%d)",
                    fn, kMaxHidden, kMaxExperts, H, E);
    if (T == 0) return MB_OK;
    if (!x || !w3 || !logits) return fail(MB_ERR_INVALID_ARG, "%s: null pointer", fn);
    if (!aligned16(x) || !aligned16(w3) || !aligned16(logits))
        return fail(MB_ERR_INVALID_ARG, "%s: pointers must be 16-byte aligned", fn);
    return cuda_status(launch_router_proj(x, T, H, w3, E, scale, logits, static_cast<cudaStream_t>(stream)), fn);
}

size_t moe_dispatch_workspace_size(int T, int k, int E) {
    if (T < 0 || k < 1 || E < 1) return 0;
    return dispatch_workspace_bytes(static_cast<int64_t>(T) * k, E);
}

}  // extern "C"

namespace mb {

// The checks of moe_dispatch's arguments other than the workspace (shared with
// moe_dispatch_noalloc, which must refuse the same inputs the same way).
int check_dispatch(const char* fn, const int32_t* topk_ids, int T, int k, int expert_begin, int E,
                   const int32_t* expert_offsets, const int32_t* row_idx, const int32_t* row_token) {
    if (T < 0 || k < 0 || E < 0 || expert_begin < 0) return fail(MB_ERR_INVALID_ARG, "%s: negative argument", fn);
    if (static_cast<int64_t>(expert_begin) + E > INT32_MAX)
        return fail(MB_ERR_INVALID_ARG, "%s: expert_begin + E overflows int32", fn);
    if (!moe_boundary_supported(MB_STAGE_DISPATCH, T, 0, E, k, 1))
        return fail(MB_ERR_UNSUPPORTED, "%s: needs 1 <= k <= %d, 1 <= E <= %d and T * k < 2^31 (T=%d, k=%d, E=%d)",
                    fn, kMaxTopK, kMaxExperts, T, k, E);
    if (!expert_offsets || (T > 0 && (!topk_ids || !row_idx || !row_token)))
        return fail(MB_ERR_INVALID_ARG, "%s: null pointer", fn);
    if (!aligned16(expert_offsets) || !aligned16(topk_ids) || !aligned16(row_idx) || !aligned16(row_token))
        return fail(MB_ERR_INVALID_ARG, "%s: pointers must be 16-byte aligned", fn);
    return MB_OK;
}

}  // namespace mb

extern "C" {

int moe_dispatch(const int32_t* topk_ids, int T, int k, int expert_begin, int E, int32_t* expert_offsets,
                 int32_t* row_idx, int32_t* row_token, void* workspace, size_t workspace_bytes, void* stream) {
    const char* fn = "moe_dispatch";
    const int st = check_dispatch(fn, topk_ids, T, k, expert_begin, E, expert_offsets, row_idx, row_token);
    if (st != MB_OK) return st;
    const size_t need = dispatch_workspace_bytes(static_cast<int64_t>(T) * k, E);
    if (need > 0) {
        if (!workspace || workspace_bytes < need)
            return fail(MB_ERR_INVALID_ARG, "%s: needs a workspace of %zu bytes (got %zu)", fn, need,
                        workspace ? workspace_bytes : static_cast<size_t>(0));
        if (!aligned16(workspace)) return fail(MB_ERR_INVALID_ARG, "%s: workspace must be 16-byte aligned", fn);
    }
    return cuda_status(launch_dispatch(topk_ids, T, k, expert_begin, E, expert_offsets, row_idx, row_token,
                                       workspace, static_cast<cudaStream_t>(stream)),
                       fn);
}

// ------------------------------------------------------------------ finalize + all-reduce
static_assert(kFarMaxWorld == MB_FAR_MAX_WORLD, "one limit on the ranks");

static bool far_sizes_ok(int world, int T_max, int H, int k) {
    return world >= 1 && world <= kFarMaxWorld && T_max >= 1 && H >= 16 && H % 16 == 0 && H <= kMaxHidden &&
           k >= 1 && k <= kMaxTopK;
}

size_t finalize_ar_workspace_size(int world, int T_max, int H) {
    if (!far_sizes_ok(world, T_max, H, 1)) return 0;
    return finalize_ar_workspace_bytes(world, T_max, H);
}

int finalize_ar_workspace_init(void* workspace, int world, int T_max, int H, void* stream) {
    const char* fn = "finalize_ar_workspace_init";
    if (!far_sizes_ok(world, T_max, H, 1))
        return fail(MB_ERR_UNSUPPORTED, "%s: needs 1 <= world <= %d, T_max >= 1, H %% 16 == 0, 16 <= H <= %d", fn,
                    kFarMaxWorld, kMaxHidden);
    if (!workspace || !aligned256(workspace)) return fail(MB_ERR_INVALID_ARG, "%s: workspace must be 256-byte aligned", fn);
    return cuda_status(cudaMemsetAsync(workspace, 0, finalize_ar_flags_bytes(world, T_max),
                                       static_cast<cudaStream_t>(stream)),
                       fn);
}

static int check_far_common(const char* fn, int H, int T, int k, int world, int T_max, const uint16_t* norm_w,
                            void* const* workspaces) {
    if (T < 0 || H < 0 || k < 0 || world < 0 || T_max < 0) return fail(MB_ERR_INVALID_ARG, "%s: negative size", fn);
    if (!far_sizes_ok(world, T_max, H, k))
        return fail(MB_ERR_UNSUPPORTED,
                    "%s: needs 1 <= world <= %d, H %% 16 == 0, 16 <= H <= %d, 1 <= k <= %d (world=%d, H=%d, k=%d)", fn,
                    kFarMaxWorld, kMaxHidden, kMaxTopK, world, H, k);
    if (T > T_max) return fail(MB_ERR_INVALID_ARG, "%s: T = %d exceeds the workspace's T_max = %d", fn, T, T_max);
    if (!workspaces || !norm_w) return fail(MB_ERR_INVALID_ARG, "%s: null pointer", fn);
    if (!aligned16(norm_w)) return fail(MB_ERR_INVALID_ARG, "%s: norm_w must be 16-byte aligned", fn);
    for (int q = 0; q < world; ++q)
        if (!workspaces[q] || !aligned256(workspaces[q]))
            return fail(MB_ERR_INVALID_ARG, "%s: workspace of rank %d missing or not 256-byte aligned", fn, q);
    return MB_OK;
}

static int check_far_rank(const char* fn, int r, const uint16_t* expert_out, int64_t num_rows, const int32_t* row_idx,
                          const float* weights, const uint16_t* out) {
    if (num_rows < 0) return fail(MB_ERR_INVALID_ARG, "%s: rank %d: negative num_rows", fn, r);
    if (!row_idx || !weights || !out || (num_rows > 0 && !expert_out))
        return fail(MB_ERR_INVALID_ARG, "%s: rank %d: null pointer", fn, r);
    if (!aligned16(expert_out) || !aligned16(out))
        return fail(MB_ERR_INVALID_ARG, "%s: rank %d: expert_out and out must be 16-byte aligned", fn, r);
    return MB_OK;
}

int expert_finalize_allreduce(const uint16_t* expert_out, int64_t num_rows, int H, const int32_t* row_idx,
                              const float* weights, int T, int k, const uint16_t* norm_w, float gain_center, float eps,
                              void* const* workspaces, int world, int rank, int T_max, uint16_t* out, void* stream) {
    const char* fn = "expert_finalize_allreduce";
    int st = check_far_common(fn, H, T, k, world, T_max, norm_w, workspaces);
    if (st != MB_OK) return st;
    if (rank < 0 || rank >= world) return fail(MB_ERR_INVALID_ARG, "%s: rank %d outside [0, %d)", fn, rank, world);
    if (T == 0) return MB_OK;
    st = check_far_rank(fn, rank, expert_out, num_rows, row_idx, weights, out);
    if (st != MB_OK) return st;
    FarLaunch L = {};
    L.nloc = 1;
    L.expert_out[0] = expert_out;
    L.R[0] = num_rows;
    L.row_idx[0] = row_idx;
    L.wt[0] = weights;
    L.out[0] = out;
    for (int q = 0; q < world; ++q) L.ws[q] = workspaces[q];
    L.w = norm_w;
    L.gc = gain_center;
    L.eps = eps;
    L.H = H;
    L.T = T;
    L.k = k;
    L.Tmax = T_max;
    L.world = world;
    L.rank0 = rank;
    return cuda_status(launch_finalize_ar(L, static_cast<cudaStream_t>(stream)), fn);
}

int expert_finalize_allreduce_local(const uint16_t* const* expert_out, const int64_t* num_rows, int H,
                                    const int32_t* const* row_idx, const float* const* weights, int T, int k,
                                    const uint16_t* norm_w, float gain_center, float eps, void* const* workspaces,
                                    int world, int T_max, uint16_t* const* out, void* stream) {
    const char* fn = "expert_finalize_allreduce_local";
    int st = check_far_common(fn, H, T, k, world, T_max, norm_w, workspaces);
    if (st != MB_OK) return st;
    if (T == 0) return MB_OK;
    if (!expert_out || !num_rows || !row_idx || !weights || !out)
        return fail(MB_ERR_INVALID_ARG, "%s: null pointer", fn);
    FarLaunch L = {};
    L.nloc = world;
    for (int r = 0; r < world; ++r) {
        st = check_far_rank(fn, r, expert_out[r], num_rows[r], row_idx[r], weights[r], out[r]);
        if (st != MB_OK) return st;
        L.expert_out[r] = expert_out[r];
        L.R[r] = num_rows[r];
        L.row_idx[r] = row_idx[r];
        L.wt[r] = weights[r];
        L.out[r] = out[r];
        L.ws[r] = workspaces[r];
    }
    L.w = norm_w;
    L.gc = gain_center;
    L.eps = eps;
    L.H = H;
    L.T = T;
    L.k = k;
    L.Tmax = T_max;
    L.world = world;
    L.rank0 = 0;
    return cuda_status(launch_finalize_ar(L, static_cast<cudaStream_t>(stream)), fn);
}

// ------------------------------------------------------------------ peer memory
int mb_ipc_alloc(size_t bytes, void** ptr) {
    if (!ptr || bytes == 0) return fail(MB_ERR_INVALID_ARG, "mb_ipc_alloc: null pointer or zero size");
    *ptr = nullptr;
    return cuda_status(cudaMalloc(ptr, bytes), "mb_ipc_alloc");
}

int mb_ipc_free(void* ptr) {
    if (!ptr) return MB_OK;
    return cuda_status(cudaFree(ptr), "mb_ipc_free");
}

int mb_ipc_get_handle(const void* ptr, void* handle) {
    static_assert(sizeof(cudaIpcMemHandle_t) == MB_IPC_HANDLE_BYTES, "IPC handle size");
    if (!ptr || !handle) return fail(MB_ERR_INVALID_ARG, "mb_ipc_get_handle: null pointer");
    cudaIpcMemHandle_t h;
    const int st = cuda_status(cudaIpcGetMemHandle(&h, const_cast<void*>(ptr)), "mb_ipc_get_handle");
    if (st == MB_OK) std::memcpy(handle, &h, sizeof(h));
    return st;
}

int mb_ipc_open(const void* handle, void** ptr) {
    if (!handle || !ptr) return fail(MB_ERR_INVALID_ARG, "mb_ipc_open: null pointer");
    *ptr = nullptr;
    cudaIpcMemHandle_t h;
    std::memcpy(&h, handle, sizeof(h));
    return cuda_status(cudaIpcOpenMemHandle(ptr, h, cudaIpcMemLazyEnablePeerAccess), "mb_ipc_open");
}

int mb_ipc_close(void* ptr) {
    if (!ptr) return MB_OK;
    return cuda_status(cudaIpcCloseMemHandle(ptr), "mb_ipc_close");
}

int mb_device_status(void) {
    unsigned int v = 0u, zero = 0u;
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_wait_timeout, sizeof(v));
    if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_wait_timeout, &zero, sizeof(zero));
    if (e != cudaSuccess) {
        fail(MB_ERR_CUDA, "mb_device_status: %s", cudaGetErrorString(e));
        return -1;
    }
    return static_cast<int>(v);
}

}  // extern "C"
