// internal.h -- launchers shared between the kernel files and the C-ABI
// entry points (host side).  Each returns a cudaError_t from the launch.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace mb {

struct DeviceInfo {
    int sm_count;
    int max_smem_optin;
};
const DeviceInfo& device_info();   // current device, cached per device

// The exhaustive check of the router's fast sigmoid against the exact one.
cudaError_t launch_fast_sigmoid_check(float* max_err, cudaStream_t s);
cudaError_t launch_route(const float* logits, const float* bias, const uint8_t* mask, int T, int E,
                         int k, int32_t* ids, float* weights, cudaStream_t s);

// The router launched right after the norm-quant of the same tokens, running
// beside it (see route.cu); used for batches up to kRouteBesideTokensPerSM
// tokens per SM.
constexpr int kRouteBesideTokensPerSM = 6;
cudaError_t launch_route_beside(const float* logits, const float* bias, const uint8_t* mask, int T, int E,
                                int k, int32_t* ids, float* weights, cudaStream_t s);

cudaError_t launch_norm_quant(const uint16_t* x, int M, int H, int tp, const uint16_t* w, float gc,
                              float eps, const float* gs, uint8_t* packed, uint8_t* sf,
                              cudaStream_t s);

// Kernels launch_route_norm_quant enqueues for these sizes (x 16-byte aligned).
int route_norm_quant_kernels(int M, int H, int tp, int E);
cudaError_t launch_route_norm_quant(const float* logits, const float* bias, const uint8_t* mask, int E, int k,
                                    int32_t* ids, float* weights, const uint16_t* x, int M, int H, int tp,
                                    const uint16_t* w, float gc, float eps, const float* gs, uint8_t* packed,
                                    uint8_t* sf, cudaStream_t s);

struct JoinArgs {
    float* residual;            // [T, H] FP32 in/out; NULL = no join
    const uint16_t* gain;       // [H] BF16
    float alpha, beta, eps;
    const uint16_t* next_w;     // [H] BF16, NULL = no next prenorm
    float next_gc, next_eps;
    uint16_t* next_prenorm;     // [T, H] BF16
};

cudaError_t launch_combine(const uint16_t* expert_out, int64_t R, int H, const int32_t* row_idx,
                           const float* wt, int T, int k, const uint16_t* w, float gc, float eps,
                           uint16_t* out, const JoinArgs& join, cudaStream_t s);

cudaError_t launch_residual_join(const uint16_t* branch, int T, int H, const JoinArgs& join,
                                 cudaStream_t s);

// Few tokens (decode): combine / join with one token per thread-block cluster
// (decode.cu) while T * next_pow2(H / 16) <= SMs * kClusterThreadsPerSM (148
// tokens at H = 8192 on B200); the row kernels take larger T.  Bit-identical
// results.
constexpr int kClusterThreadsPerSM = 512;
bool cluster_path(int T, int H);
cudaError_t launch_combine_cluster(const uint16_t* expert_out, int64_t R, int H, const int32_t* row_idx,
                                   const float* wt, int T, int k, const uint16_t* w, float gc, float eps,
                                   uint16_t* out, const JoinArgs& join, cudaStream_t s);
cudaError_t launch_join_cluster(const uint16_t* branch, int T, int H, const JoinArgs& join, cudaStream_t s);

// Router projection (router_proj.cu): logits = scale * x W^T on the tensor
// cores from the FP32 weight prepared into three BF16 parts; C K-chunks per
// expert tile (a cluster of C CTAs).
int router_proj_chunks(int H);
cudaError_t launch_router_weight_split(const float* w, int E, int H, uint16_t* w3, cudaStream_t s);
cudaError_t launch_router_proj(const uint16_t* x, int T, int H, const uint16_t* w3, int E, float scale, float* logits,
                               cudaStream_t s);

// Dispatch: workspace bytes for n = T * k entries (0 when one tile holds
// them all), and the launch (one kernel, or three with the workspace).
size_t dispatch_workspace_bytes(int64_t n, int E);
cudaError_t launch_dispatch(const int32_t* ids, int T, int k, int e0, int E, int32_t* offsets, int32_t* row_idx,
                            int32_t* row_token, void* workspace, cudaStream_t s);

// Largest H the row kernels take (16-element blocks, at most 1024 per row).
constexpr int kMaxHidden = 16384;
constexpr int kMaxTopK = 32;
constexpr int kMaxExperts = 4096;

// Expert finalize fused with the tensor-parallel all-reduce (finalize_ar.cu).
constexpr int kFarMaxWorld = 8;
struct FarLaunch {
    int nloc;                                   // ranks computed by this launch: rank0 .. rank0 + nloc - 1
    const uint16_t* expert_out[kFarMaxWorld];   // per local rank
    int64_t R[kFarMaxWorld];
    const int32_t* row_idx[kFarMaxWorld];
    const float* wt[kFarMaxWorld];
    uint16_t* out[kFarMaxWorld];
    void* ws[kFarMaxWorld];                     // every rank's workspace, as mapped on this device
    const uint16_t* w;
    float gc, eps;
    int H, T, k, Tmax, world, rank0;
};
int far_warps(int H);
size_t finalize_ar_workspace_bytes(int world, int Tmax, int H);
size_t finalize_ar_flags_bytes(int world, int Tmax);
cudaError_t launch_finalize_ar(const FarLaunch& L, cudaStream_t s);

}  // namespace mb
