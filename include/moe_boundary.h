/*
 * moe_boundary.h -- C ABI of the per-token MoE boundary of a sparse decoder
 * layer on NVIDIA B200 (sm_100a): router gate, pre-expert RMSNorm fused with
 * NVFP4 quantisation, post-expert norm + weighted combine, gated residual join.
 *
 * Entry points: moe_route, norm_quant_nvfp4, moe_route_norm_quant (both
 * pre-expert stages in one call), expert_combine, residual_join,
 * expert_combine_join (the combine with the join fused), moe_dispatch and
 * moe_dispatch_noalloc (expert-grouped rows of the routing entries),
 * router_weight_prepare and router_logits (the router projection),
 * expert_finalize_allreduce and expert_finalize_allreduce_local (the combine
 * of an expert-parallel layer fused with its tensor-parallel all-reduce) with
 * their workspace calls and the mb_ipc_* peer-memory helpers; queries
 * moe_boundary_supported, moe_route_norm_quant_kernels, the workspace sizes,
 * mb_last_error and mb_device_status.
 *
 * Library: libmoe_boundary.so (CUDA runtime only; no PyTorch types).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Tensors are DEVICE pointers owned by the caller, row-major and
 *    contiguous; every base pointer must be 16-byte aligned.  BF16 values are
 *    passed as uint16_t bit patterns, E4M3 and packed E2M1 as uint8_t.
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream).  Work is
 *    only enqueued; nothing is synchronised, allocated or freed (except by the
 *    calls whose job that is: mb_ipc_alloc / mb_ipc_free / mb_ipc_open /
 *    mb_ipc_close, and mb_device_status, which synchronises to read its word).
 *  - Return value: MB_OK, or an error code.  Arguments are checked before
 *    anything is enqueued, so on an error nothing runs; mb_last_error()
 *    returns a message for the calling thread's most recent failure.
 *  - A call with zero tokens returns MB_OK without launching (the empty-input
 *    rule of norm_quant_trtllm_nvfp4 on the vLLM API page
 *    "prepare_trtllm_nvfp4").
 *  - Floating point: FP32 arithmetic in a fixed order with one IEEE rounding
 *    per operation; fused multiply-adds only where stated.  Results are
 *    bitwise reproducible run to run.
 */
#ifndef MOE_BOUNDARY_H
#define MOE_BOUNDARY_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum {
    MB_OK = 0,
    MB_ERR_INVALID_ARG = 1,  /* null pointer, negative size, misaligned pointer, shape mismatch */
    MB_ERR_UNSUPPORTED = 2,  /* valid, but outside the sizes the kernels take (see each call)  */
    MB_ERR_CUDA = 3,         /* the CUDA runtime reported an error while enqueuing             */
};

/*
 * moe_route -- sigmoid router gate with selection bias and token mask.
 *
 * Source: TensorRT-LLM PR 21356 "Add the Muse Spark Open decoder fast paths",
 * description, "Routing" (sigmoid, bias, top-k, renormalised weights, picks
 * sorted with exact ties to the lowest expert id); TensorRT-LLM PR 21042
 * (router in FP32); lmdeploy PR 4835 "MoE gate v2", commit notes (a required
 * token mask; invalid tokens produce no routing entries).
 *
 * For a valid token t (token_mask[t] != 0):
 *   s_e = 1 / (1 + exp(-logits[t, e]))          exp: the library's own FP32 exp
 *   c_e = s_e + bias[e]                          used for selection only
 *   topk_ids[t, j]     = j-th expert in the order (c descending, id ascending)
 *   topk_weights[t, j] = s_{id j} / (s_{id 0} + ... + s_{id k-1})
 * For an invalid token: topk_ids[t, :] = -1, topk_weights[t, :] = 0, and its
 * logits are not read (they may hold NaN).
 *
 *   logits        [T, E] FP32          bias          [E] FP32
 *   token_mask    [T] uint8 (required) topk_ids      [T, k] int32 (out)
 *   topk_weights  [T, k] FP32 (out)
 * Supported: 1 <= k <= 32, k <= E <= 4096.
 *
 * The kernels shortlist experts with a fast sigmoid whose error against the
 * exact one is bounded by MB_ROUTE_FAST_SIGMOID_BOUND and decide among the
 * shortlist with the exact sigmoid, so the results are those of the exact
 * definition above (moe_route_check_fast_sigmoid re-measures the bound).
 */
#define MB_ROUTE_FAST_SIGMOID_BOUND 4.76837158203125e-07f   /* 2^-21 */
int moe_route(const float* logits, const float* bias, const uint8_t* token_mask, int T, int E,
              int k, int32_t* topk_ids, float* topk_weights, void* stream);

/*
 * moe_route_check_fast_sigmoid -- measure the router's fast-sigmoid bound.
 *
 * No counterpart on the reference pages: moe_route picks its candidates with
 * an approximate sigmoid built from the GPU's approximate 2^x and reciprocal
 * and is exact only while that approximation stays within
 * MB_ROUTE_FAST_SIGMOID_BOUND of the exact sigmoid.  This call evaluates both
 * on the device for every binary32 input (NaNs skipped) and writes the largest
 * absolute difference to *max_err (a device float the caller owns; set to 0
 * first, then max-combined by the kernel).  Enqueued on `stream`; read
 * *max_err after synchronising.  Takes about a millisecond on a B200.
 */
int moe_route_check_fast_sigmoid(float* max_err, void* stream);

/*
 * norm_quant_nvfp4 -- pre-expert RMSNorm fused with NVFP4 quantisation.
 *
 * Source: vLLM API page "prepare_trtllm_nvfp4", norm_quant_trtllm_nvfp4 and
 * _quantize_nvfp4_global_scale; TensorRT-LLM PR 21356, "Numerics" (the gain
 * centre is added in FP32 and the norm's result is rounded to BF16 once).
 *
 * Per token t, over logical x[t, 0..H-1]:
 *   inv  = 1 / sqrt(sum(x^2) / H + eps)
 *   y    = bf16((x * (gain_center + norm_w)) * inv)
 *   per block of 16 consecutive y:
 *     sf   = e4m3_rn_satfinite(gs * (max|y| * fl(1/6)))        -> sf[t, block]
 *     os   = sf != 0 ? 1 / (sf * (1 / gs)) : 0
 *     code = e2m1 round-to-nearest-even, saturating, of y * os (sign bit iff < 0)
 *   packed[t, i] = code(2i) | code(2i + 1) << 4
 *
 *   x        tp == 1: [M, H] BF16; tp > 1: rank-block [tp, M, H/tp] BF16, the
 *            layout a dim-0 all-gather of column shards leaves (logical
 *            x[t, h] is at ((h / (H/tp)) * M + t) * (H/tp) + h % (H/tp))
 *   norm_w   [H] BF16
 *   global_scale  device pointer to one FP32 value gs > 0
 *   packed   [M, H/2] uint8 (out)       sf  [M, H/16] uint8 E4M3 (out, linear)
 * Supported: H % 16 == 0, H <= 16384, tp >= 1, H % tp == 0, (H/tp) % 16 == 0.
 */
int norm_quant_nvfp4(const uint16_t* x, int M, int H, int tp, const uint16_t* norm_w,
                     float gain_center, float eps, const float* global_scale, uint8_t* packed,
                     uint8_t* sf, void* stream);

/*
 * moe_route_norm_quant -- moe_route and norm_quant_nvfp4 of the same M tokens
 * in one call.
 *
 * Source: as moe_route and norm_quant_nvfp4.  The two pre-expert stages read
 * disjoint inputs and are independent (TensorRT-LLM PR 21356, "Where they
 * plug in", runs the pre-expert norm beside the router).  The work is
 * enqueued on `stream` in one of three arrangements: for small batches (up to
 * 6 tokens per SM) the router kernel runs concurrently with the norm-quant
 * kernel, in the registers and warp slots that kernel leaves free; for larger
 * batches on the wide norm-quant path (H >= 2048, H / tp % 64 == 0, E <= 256)
 * one kernel does both, its router warps beside its row warps; otherwise the
 * router kernel runs first.  The call completes, in stream order, when both
 * stages have.  Results are those of the two calls with T = M, bit for bit.
 * Supported: both calls' rules.
 */
int moe_route_norm_quant(const float* logits, const float* bias, const uint8_t* token_mask, int E, int k,
                         int32_t* topk_ids, float* topk_weights, const uint16_t* x, int M, int H, int tp,
                         const uint16_t* norm_w, float gain_center, float eps, const float* global_scale,
                         uint8_t* packed, uint8_t* sf, void* stream);

/*
 * moe_route_norm_quant_kernels -- how many kernels moe_route_norm_quant
 * enqueues for these sizes on the current device (1 or 2), for an input x
 * whose address is 16-byte aligned (an unaligned x takes a two-kernel
 * arrangement); 0 for M == 0.  Returns -1 when the sizes are not supported or
 * no CUDA device is present.  No device work.
 */
int moe_route_norm_quant_kernels(int M, int H, int tp, int E, int k);

/*
 * expert_combine -- post-expert RMSNorm of each selected row + weighted sum.
 *
 * Source: TensorRT-LLM PR 21356, description, "Post-expert norm and combine"
 * (weight-first RMSNorm of each selected expert row, the routing weights and
 * the top-k sum in one pass; a row behind an invalid slot -- -1, or past the
 * end of the expert output -- is never read); TensorRT-LLM PR 21042 (the
 * finalize applies the post-expert norm before the weighted top-k sum);
 * lmdeploy PR 4835 (absent rows marked -1).
 *
 * Per token t, acc = +0, then for j = 0 .. k-1 in order, when
 * 0 <= row_idx[t, j] < num_rows:
 *   x   = expert_out[row_idx[t, j], :]
 *   y   = bf16((x * (gain_center + norm_w)) * (1 / sqrt(sum(x^2) / H + eps)))
 *   acc = fmaf(weights[t, j], y, acc)
 * out[t, :] = bf16(acc).  Slots outside [0, num_rows) contribute nothing and
 * their rows are never read; a token without a valid slot outputs zeros.
 *
 *   expert_out  [num_rows, H] BF16     row_idx  [T, k] int32
 *   weights     [T, k] FP32            norm_w   [H] BF16
 *   out         [T, H] BF16 (out)
 * Supported: H % 16 == 0, H <= 16384, 1 <= k <= 32, num_rows >= 0.
 */
int expert_combine(const uint16_t* expert_out, int64_t num_rows, int H, const int32_t* row_idx,
                   const float* weights, int T, int k, const uint16_t* norm_w, float gain_center,
                   float eps, uint16_t* out, void* stream);

/*
 * residual_join -- gated residual join over the FP32 residual stream, with
 * the next branch's prenorm optionally fused.
 *
 * Source: TensorRT-LLM PR 21356, description, "Gated residual join"
 * (alpha * residual + beta * rmsnorm(gain * branch) over the FP32 residual
 * stream, alone or with the next branch's Gemma prenorm; BF16 rounding where
 * the reference composition rounds).
 *
 * Per token t:
 *   g  = bf16(gain * branch[t, :])
 *   n  = bf16(g * (1 / sqrt(sum(g^2) / H + eps)))
 *   residual[t, :] = alpha * residual[t, :] + beta * n        (in place, FP32)
 *   if next_w != NULL:
 *     next_prenorm[t, :] = bf16((r * (next_gc + next_w)) * (1 / sqrt(sum(r^2) / H + next_eps)))
 *     with r the updated residual row.
 *
 *   residual [T, H] FP32 (in/out)   branch [T, H] BF16   gain [H] BF16
 *   next_w   [H] BF16 or NULL        next_prenorm [T, H] BF16 (out) or NULL
 *   (next_w and next_prenorm are both NULL or both non-NULL)
 * Supported: H % 16 == 0, H <= 16384.
 */
int residual_join(float* residual, const uint16_t* branch, const uint16_t* gain, float alpha,
                  float beta, float eps, const uint16_t* next_w, float next_gc, float next_eps,
                  uint16_t* next_prenorm, int T, int H, void* stream);

/*
 * expert_combine_join -- expert_combine followed by residual_join in one
 * kernel, the combine's BF16 output serving as the branch.
 *
 * Source: as expert_combine and residual_join (the fused decoder boundary of
 * TensorRT-LLM PR 21356).  Arguments are those of the two calls; `out`
 * (the combine output) may be NULL when only the residual and the prenorm are
 * wanted.  Results equal expert_combine then residual_join bit for bit.
 */
int expert_combine_join(const uint16_t* expert_out, int64_t num_rows, int H, const int32_t* row_idx,
                        const float* weights, int T, int k, const uint16_t* norm_w,
                        float gain_center, float eps, uint16_t* out, float* residual,
                        const uint16_t* gain, float alpha, float beta, float join_eps,
                        const uint16_t* next_w, float next_gc, float next_eps,
                        uint16_t* next_prenorm, void* stream);

/*
 * router_weight_prepare -- the FP32 router weight in the form router_logits
 * reads: three BF16 parts of each weight (done once, when the weight loads).
 *
 * Source: TensorRT-LLM PR 21356, description, "Router projection" (FP32
 * weights on tensor cores with a split of the FP32 operand; the page lists a
 * BF16x3 router among its experiments).
 *
 *   w1 = bf16(w), w2 = bf16(w - w1), w3 = bf16(w - w1 - w2)   (round to
 *   nearest even; each remainder is exact in FP32), |w - w1 - w2 - w3| <=
 *   2^-27 |w|.
 *
 *   w    [E, H] FP32 (row e: expert e)
 *   w3   [3, E, H] BF16 (out): w1, then w2, then w3; 6 * E * H bytes
 * Supported: as router_logits.
 */
int router_weight_prepare(const float* w, int E, int H, uint16_t* w3, void* stream);

/*
 * router_logits -- the router projection: logits = scale * x W^T.
 *
 * Source: TensorRT-LLM PR 21356, description, "Router projection" (FP32
 * weights and FP32 accumulation for up to 128 tokens, the input cast and a
 * scale folded in, tensor cores from 16 tokens).
 *
 *   logits[t, e] = scale * sum_h float(x[t, h]) * w[e, h]
 *
 * computed on the tensor cores from the prepared weight: x w1^T + x w2^T +
 * x w3^T with BF16 operands (every product exact in FP32) accumulated in FP32
 * in a fixed order, so results are reproducible run to run.  The error against
 * the exact sum is below (2^-27 + (3 H / C / 16 + 12) * 2^-23) *
 * sum_h |scale * x * w|, with C = 8, 4, 2 or 1 the largest such that
 * H % (64 C) == 0.
 *
 *   x       [T, H] BF16          w3      [3, E, H] BF16 from router_weight_prepare
 *   logits  [T, E] FP32 (out)
 * Supported: H % 64 == 0, 64 <= H <= 16384, E % 16 == 0, 16 <= E <= 4096.
 */
int router_logits(const uint16_t* x, int T, int H, const uint16_t* w3, int E, float scale, float* logits,
                  void* stream);

/*
 * moe_dispatch -- expert-grouped rows of the routing entries: the dispatch
 * step between the router (moe_route) and the experts, producing the
 * row_idx that expert_combine reads.
 *
 * Source: lmdeploy PR 4835 "MoE gate v2", commit notes (the routing entries
 * are grouped per expert by a histogram and an exclusive scan, hierarchical
 * over CTAs for large expert counts; tokens without routing entries get no
 * rows; en2f, the row of each routing entry, is cleared to -1 where no row
 * exists; the routed count is passed on).
 *
 * Entry i = t * k + j of topk_ids is valid iff expert_begin <= topk_ids[i] <
 * expert_begin + E (the experts of this rank; -1, the router's mark for a
 * masked token, is never valid); its local expert is e = topk_ids[i] -
 * expert_begin.  Rows are grouped by e ascending; inside one expert the
 * entries keep the order of i (a stable counting sort), so tokens ascend.
 *
 *   topk_ids        [T, k] int32 (global expert ids)
 *   expert_offsets  [E + 1] int32 (out): first row of each expert;
 *                   expert_offsets[E] = R, the number of valid entries
 *   row_idx         [T, k] int32 (out): the row of entry i (en2f), -1 when
 *                   the entry is invalid
 *   row_token       [T * k] int32 (out): the token of row r for r < R, -1 for
 *                   R <= r < T * k
 *   workspace       device scratch of moe_dispatch_workspace_size(T, k, E)
 *                   bytes, 16-byte aligned, owned by the caller; may be NULL
 *                   when that size is 0 (T * k <= 4096).  Its contents need
 *                   no initialisation and are not kept between calls, but
 *                   two calls that overlap on the GPU need two workspaces.
 * Returns MB_ERR_INVALID_ARG when the workspace is missing or too small.
 * T == 0 still writes expert_offsets (all zero); the other pointers may then
 * be NULL.  Integer only: the result does not depend on the launch shape.
 * Supported: 1 <= k <= 32, 1 <= E <= 4096, T * k < 2^31, expert_begin >= 0.
 */
size_t moe_dispatch_workspace_size(int T, int k, int E);
int moe_dispatch(const int32_t* topk_ids, int T, int k, int expert_begin, int E, int32_t* expert_offsets,
                 int32_t* row_idx, int32_t* row_token, void* workspace, size_t workspace_bytes, void* stream);

/*
 * moe_dispatch_noalloc -- moe_dispatch without a caller workspace, for
 * callers that cannot allocate device memory.
 *
 * No counterpart on the reference pages: this entry point exists for callers
 * that have no device memory to hand over -- their memory belongs to an
 * allocator they cannot reach from this call site, or they must not call
 * cudaMalloc/cudaFree on the hot path (those calls can synchronise the whole
 * device), or the GPU's memory is already spoken for.  The call allocates
 * nothing: its scratch is a fixed 1 MiB array compiled into the library,
 * which every GPU that loads the library holds until the process exits.
 *
 * Arguments, outputs and results are those of moe_dispatch (bit for bit), and
 * so are the argument checks and their status codes; only then is the size
 * limit below checked.
 * Limit: the inputs must fit the array, (ceil(T * k / 4096) + 1) * E * 4 <=
 * 1 MiB (for example T * k up to about 4.19 M entries at E = 256, 413 K at
 * E = 2560); larger calls return MB_ERR_UNSUPPORTED without launching.
 * Every call on a device shares the one array: two calls whose kernels
 * overlap on the GPU (different streams, no ordering between them) race on
 * it and can return wrong rows.  Nothing in the array needs to start at zero
 * (each call writes every count it reads), and it keeps the last call's
 * counts.  The first call on a device looks up the array's device address
 * (synchronous, with that device current) and keeps it once the lookup has
 * succeeded (a failed lookup is retried by the next call); make that first
 * call before any stream capture begins.  The kept address assumes the
 * device's context lives as long as the process: after cudaDeviceReset, do
 * not call this entry point again in the same process.
 */
int moe_dispatch_noalloc(const int32_t* topk_ids, int T, int k, int expert_begin, int E, int32_t* expert_offsets,
                         int32_t* row_idx, int32_t* row_token, void* stream);

/*
 * Expert finalize fused with the tensor-parallel all-reduce of its partials.
 *
 * Source: TensorRT-LLM PR 21356, description, "Fused finalize + all-reduce"
 * (with the experts split over the ranks, the expert finalize and the TP
 * all-reduce run as one kernel, a one-shot exchange through peer memory, FP32
 * accumulation; construction is collective) and PR 21042, MoE paragraph (the
 * finalize all-reduces partials in FP32).
 *
 * Per token t, rank r's partial is the combine's FP32 accumulator over the
 * slots whose row it holds (0 <= row_idx_r[t, j] < num_rows_r), in slot order
 * from +0:  acc = fmaf(weights[t, j], bf16((x * (gain_center + norm_w)) *
 * inv_rms(x)), acc).  Every rank outputs out[t, :] = bf16(((p_0 + p_1) + p_2)
 * + ...), the partials added in FP32 in rank order.  Slots whose row lives on
 * another rank are marked -1 (or any value outside [0, num_rows_r)) and never
 * read.
 *
 * Exchange: every rank owns a workspace of finalize_ar_workspace_size()
 * bytes of device memory that every other rank maps (mb_ipc_* below, or any
 * other peer mapping); `workspaces` lists all ranks' workspaces as mapped in
 * the calling process, in rank order.  A call writes this rank's partials
 * into its own workspace, raises a per-token flag in every rank's workspace,
 * waits (up to 2 s; then bit 4 of mb_device_status is set and the remaining
 * tokens are left unwritten) for every rank's flag of each token it reduces,
 * and reads the peers' partials with plain loads from their memory.  Every
 * rank must make the same sequence of calls, with the same T, world and T_max;
 * calls are counted in the workspace (graph replays included), so nothing on
 * the host changes between calls.  Each launch is cooperative (all CTAs
 * resident at once).  After a wait ran out the workspaces are out of step:
 * initialise them again on every rank.
 *
 *   expert_out [num_rows, H] BF16    row_idx [T, k] int32   weights [T, k] FP32
 *   norm_w [H] BF16                  out [T, H] BF16 (out)
 * Supported: 1 <= world <= 8, H % 16 == 0, 16 <= H <= 16384, 1 <= k <= 32,
 * T <= T_max.  Pointers 16-byte aligned, workspaces 256-byte aligned.
 */
#define MB_FAR_MAX_WORLD 8

/* Bytes of one rank's workspace (0 when the sizes are not supported). */
size_t finalize_ar_workspace_size(int world, int T_max, int H);

/* Zero a workspace's call counter and flags (enqueued on `stream`); every
 * rank initialises its own before the first call and after a wait ran out. */
int finalize_ar_workspace_init(void* workspace, int world, int T_max, int H, void* stream);

/* One rank's call (one process per GPU). */
int expert_finalize_allreduce(const uint16_t* expert_out, int64_t num_rows, int H, const int32_t* row_idx,
                              const float* weights, int T, int k, const uint16_t* norm_w, float gain_center, float eps,
                              void* const* workspaces, int world, int rank, int T_max, uint16_t* out, void* stream);

/* All `world` ranks' calls in one launch on the current device, each rank
 * with its own inputs, output and workspace (host arrays of `world` entries):
 * the same exchange and the same results as `world` processes, for tests and
 * for measuring the kernel on one GPU. */
int expert_finalize_allreduce_local(const uint16_t* const* expert_out, const int64_t* num_rows, int H,
                                    const int32_t* const* row_idx, const float* const* weights, int T, int k,
                                    const uint16_t* norm_w, float gain_center, float eps, void* const* workspaces,
                                    int world, int T_max, uint16_t* const* out, void* stream);

/*
 * Peer memory through CUDA IPC (one process per GPU, one node).
 * mb_ipc_alloc: a whole cudaMalloc allocation (its handle maps from its
 * first byte).  mb_ipc_get_handle: the MB_IPC_HANDLE_BYTES-byte handle of such
 * an allocation, to send to the peers.  mb_ipc_open: map a peer's handle in
 * this process.  mb_ipc_close: unmap it.  A rank frees its own allocation only
 * after every peer has closed its mapping of it.
 */
#define MB_IPC_HANDLE_BYTES 64
int mb_ipc_alloc(size_t bytes, void** ptr);
int mb_ipc_free(void* ptr);
int mb_ipc_get_handle(const void* ptr, void* handle);
int mb_ipc_open(const void* handle, void** ptr);
int mb_ipc_close(void* ptr);

/* Stage ids for moe_boundary_supported(). */
enum {
    MB_STAGE_ROUTE = 0,
    MB_STAGE_NORM_QUANT = 1,
    MB_STAGE_COMBINE = 2,
    MB_STAGE_JOIN = 3,
    MB_STAGE_COMBINE_JOIN = 4,
    MB_STAGE_ROUTE_NORM_QUANT = 5,
    MB_STAGE_DISPATCH = 6,
    MB_STAGE_ROUTER_LOGITS = 7,
    MB_STAGE_FINALIZE_AR = 8,   /* tp = world */
};

/*
 * moe_boundary_supported -- 1 when the stage takes these sizes, else 0 (the
 * `*_supported` predicates of TensorRT-LLM PR 21356, description).  No side
 * effects; arguments a stage does not use are ignored.
 */
int moe_boundary_supported(int stage, int T, int H, int E, int k, int tp);

/* Message of the calling thread's last failed call ("" if none). */
const char* mb_last_error(void);

/*
 * mb_device_status -- reads and clears the device-side status word of the
 * current device (synchronous).  Bit 0: a producer's bounded wait for a free
 * shared-memory slot ran out; bit 1: a drain wait ran out; bit 2: a
 * consumer's wait for a copied row ran out; bit 3: the router projection's
 * wait for its tensor-core MMAs ran out; bit 4: the finalize all-reduce's
 * wait for a peer's partial ran out.  0 means no kernel reported a
 * timeout since the last call.  Returns -1 (and sets mb_last_error) when the
 * CUDA runtime fails.
 */
int mb_device_status(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_BOUNDARY_H */
