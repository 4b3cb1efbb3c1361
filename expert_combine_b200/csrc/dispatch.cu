// dispatch.cu -- expert-grouped rows of the routing entries (the dispatch step
// between the router and the experts).
//
// lmdeploy PR 4835 "MoE gate v2", commit notes: the gate's routing entries are
// grouped per expert by a histogram and an exclusive scan (hierarchical over
// CTAs for large expert counts), tokens without routing entries get no rows,
// and en2f -- the row of each routing entry -- is -1 where no row exists.
//
// Entry i = t * k + j of ids [T, k] is valid iff expert_begin <= ids[i] <
// expert_begin + E; its local expert is e = ids[i] - expert_begin.  Rows are
// grouped by e ascending, and inside one expert the entries keep their order
// i (a stable counting sort).  Outputs: offsets [E + 1] (first row of each
// expert, offsets[E] = R valid entries), row_idx [T, k] (en2f, -1 for an
// invalid entry) and row_token [T * k] (token of row r for r < R, -1 after).
//
// Work split.  A tile is 4096 consecutive entries handled by one CTA of eight
// warps; warp w takes the tile's w-th run of 512 entries, 32 at a time.  In
// each step the lanes holding the same expert form a group (one warp ballot
// per bit of the expert id), so a lane's rank among the warp's entries of its
// expert is the warp's running count of that expert plus the number of lower
// lanes in its group: the order of i is kept without sorting.  Per-warp counts are then scanned across the
// eight warps of the tile (shared memory), across tiles per expert, and over
// experts.  One tile (T * k <= 4096, decode batches) runs as one kernel;
// larger inputs run the tile counts and the placement, with the per-tile
// counts in the caller's workspace; above 32 tiles a column scan over the
// tiles (one CTA per 32 experts) runs between them, below it each placement
// CTA sums the counts of the tiles before its own.  Everything is integer, so the result is exact and
// independent of the launch shape.
#include <mutex>

#include "internal.h"
#include "common.cuh"

namespace mb {

namespace {

constexpr int kDispWarps = 8;
constexpr int kDispThreads = kDispWarps * 32;
constexpr int kDispIter = 16;                                  // 32-entry steps per warp
constexpr int kDispWarpSpan = 32 * kDispIter;                  // 512 entries per warp
constexpr int kDispTile = kDispWarps * kDispWarpSpan;          // 4096 entries per CTA
constexpr int kDispFoldTiles = 32;   // up to this many tiles the placement scans the tile counts itself

struct DispatchArgs {
    const int32_t* ids;
    int64_t n;              // T * k
    int k;
    int e0, E;
    int32_t* offsets;       // [E + 1]
    int32_t* row_idx;       // [n]
    int32_t* row_token;     // [n]
    int32_t* tile_counts;   // [ntiles][E]  (several tiles only)
    int32_t* totals;        // [E]          (several tiles only)
    int ntiles;
};

// Local expert of an id, or -1.
__device__ __forceinline__ int local_expert(const DispatchArgs& a, int32_t id) {
    const int64_t d = static_cast<int64_t>(id) - a.e0;
    return (d >= 0 && d < a.E) ? static_cast<int>(d) : -1;
}

// This CTA's tile of a [n] int32 array into registers, four consecutive
// entries per 16-byte load: v[m] holds entries 4 * (threadIdx.x + 256 m) ..
// + 3 of the tile.  Entries at or past n read as `fill`.  The array's base
// is 16-byte aligned and a tile starts at a multiple of 4096 entries.  NC:
// the array is read-only while the kernel runs (the read-only data path).
template <bool NC>
__device__ __forceinline__ void load_tile4(const int32_t* p, int64_t n, int32_t fill,
                                           int4 (&v)[kDispTile / 4 / kDispThreads]) {
    const int64_t tile0 = static_cast<int64_t>(blockIdx.x) * kDispTile;
#pragma unroll
    for (int m = 0; m < kDispTile / 4 / kDispThreads; ++m) {
        const int64_t i = tile0 + 4 * (threadIdx.x + m * kDispThreads);
        if (i + 3 < n) {
            if constexpr (NC) {
                const uint4 u = ld_nc_v4(p + i);
                v[m] = make_int4(static_cast<int>(u.x), static_cast<int>(u.y), static_cast<int>(u.z),
                                 static_cast<int>(u.w));
            } else {
                v[m] = *reinterpret_cast<const int4*>(p + i);
            }
        } else {
            v[m].x = i < n ? p[i] : fill;
            v[m].y = i + 1 < n ? p[i + 1] : fill;
            v[m].z = i + 2 < n ? p[i + 2] : fill;
            v[m].w = i + 3 < n ? p[i + 3] : fill;
        }
    }
}

// In-place exclusive scan of a[0..n) in shared memory by the whole CTA
// (kDispThreads threads, n <= 16 * kDispThreads); returns the total.  ws holds
// kDispWarps ints.
__device__ int block_exclusive_scan(int32_t* a, int n, int32_t* ws) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int per = (n + kDispThreads - 1) / kDispThreads;
    const int b = threadIdx.x * per;
    int s = 0;
    for (int j = 0; j < per; ++j)
        if (b + j < n) s += a[b + j];
    int v = s;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, v, off);
        if (lane >= off) v += u;
    }
    if (lane == 31) ws[warp] = v;
    __syncthreads();
    int run = v - s, total = 0;
#pragma unroll
    for (int w = 0; w < kDispWarps; ++w) {
        if (w < warp) run += ws[w];
        total += ws[w];
    }
    for (int j = 0; j < per; ++j)
        if (b + j < n) {
            const int c = a[b + j];
            a[b + j] = run;
            run += c;
        }
    __syncthreads();
    return total;
}

// Ranks of one tile's entries.  sid holds the tile's local experts (-1 when
// invalid or past n), staged by the whole CTA.  Leaves in cnt[w * E + e] the
// first rank of warp w's entries of expert e inside the tile, and in tot[e]
// (when not null) or tile_counts[tile][e] the tile's count of expert e.  ex /
// rk receive each step's expert and the entry's rank inside its warp.
__device__ void tile_ranks(const DispatchArgs& a, const int32_t* sid, int32_t* cnt, int32_t* tot,
                           int (&ex)[kDispIter], int (&rk)[kDispIter]) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int E = a.E;
#pragma unroll
    for (int it = 0; it < kDispIter; ++it) ex[it] = sid[warp * kDispWarpSpan + it * 32 + lane];
    int32_t* wc = cnt + warp * E;
    const unsigned below = (1u << lane) - 1u;
    // the groups of all steps first (independent of the counts), then the
    // running counts, one step after the other
    // Group of lane l: the valid lanes whose expert agrees with l's in every
    // bit, one ballot per bit of the expert id (an invalid lane is alone).
    const int nbits = E > 1 ? 32 - __clz(E - 1) : 0;
    unsigned peers[kDispIter];
#pragma unroll
    for (int it = 0; it < kDispIter; ++it) peers[it] = __ballot_sync(0xffffffffu, ex[it] >= 0);
    for (int b = 0; b < nbits; ++b) {
#pragma unroll
        for (int it = 0; it < kDispIter; ++it) {
            const bool bit = (ex[it] >> b) & 1;
            const unsigned set = __ballot_sync(0xffffffffu, bit);
            peers[it] &= bit ? set : ~set;
        }
    }
#pragma unroll
    for (int it = 0; it < kDispIter; ++it)
        if (ex[it] < 0) peers[it] = 1u << lane;
#pragma unroll
    for (int it = 0; it < kDispIter; ++it) {
        const int e = ex[it];
        const int base = e >= 0 ? wc[e] : 0;
        __syncwarp();
        if (e >= 0 && (peers[it] >> lane) == 1u) wc[e] = base + __popc(peers[it]);   // highest lane of the group
        __syncwarp();
        rk[it] = base + __popc(peers[it] & below);
    }
    __syncthreads();
    // exclusive scan of the per-warp counts over the warps, per expert
    for (int e = threadIdx.x; e < E; e += kDispThreads) {
        int run = 0;
#pragma unroll
        for (int w = 0; w < kDispWarps; ++w) {
            const int c = cnt[w * E + e];
            cnt[w * E + e] = run;
            run += c;
        }
        if (tot != nullptr) tot[e] = run;
        else a.tile_counts[static_cast<int64_t>(blockIdx.x) * E + e] = run;
    }
    __syncthreads();
}

// Zeroes the per-warp counts, waits for the previous kernel, and stages the
// tile's local experts in sid.
__device__ __forceinline__ void tile_prologue(const DispatchArgs& a, int32_t* cnt, int32_t* sid) {
    for (int i = threadIdx.x; i < kDispWarps * a.E; i += kDispThreads) cnt[i] = 0;
    griddep_wait();
    griddep_launch();
    int4 v[kDispTile / 4 / kDispThreads];
    load_tile4<true>(a.ids, a.n, INT32_MIN, v);
    const int64_t tile0 = static_cast<int64_t>(blockIdx.x) * kDispTile;
#pragma unroll
    for (int m = 0; m < kDispTile / 4 / kDispThreads; ++m) {
        const int q = 4 * (threadIdx.x + m * kDispThreads);
        const int64_t i = tile0 + q;
        *reinterpret_cast<int4*>(sid + q) =
            make_int4(i < a.n ? local_expert(a, v[m].x) : -1, i + 1 < a.n ? local_expert(a, v[m].y) : -1,
                      i + 2 < a.n ? local_expert(a, v[m].z) : -1, i + 3 < a.n ? local_expert(a, v[m].w) : -1);
    }
    __syncthreads();
}

__device__ __forceinline__ int32_t token_of(const DispatchArgs& a, int64_t i) {
    return static_cast<int32_t>(static_cast<uint32_t>(i) / static_cast<uint32_t>(a.k));
}

// One tile holds every entry: ranks, offsets and rows in one kernel.
__global__ void __launch_bounds__(kDispThreads) dispatch_single_kernel(const DispatchArgs a) {
    extern __shared__ __align__(16) int32_t dsm[];
    int32_t* sid = dsm;                        // [4096]
    int32_t* cnt = sid + kDispTile;            // [8][E]
    int32_t* tot = cnt + kDispWarps * a.E;     // [E]
    int32_t* ws = tot + a.E;                   // [8]
    tile_prologue(a, cnt, sid);
    int ex[kDispIter], rk[kDispIter];
    tile_ranks(a, sid, cnt, tot, ex, rk);
    const int R = block_exclusive_scan(tot, a.E, ws);
    for (int e = threadIdx.x; e <= a.E; e += kDispThreads) a.offsets[e] = e < a.E ? tot[e] : R;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t wbase = static_cast<int64_t>(warp) * kDispWarpSpan;
#pragma unroll
    for (int it = 0; it < kDispIter; ++it) {
        const int64_t i = wbase + it * 32 + lane;
        if (i >= a.n) continue;
        const int e = ex[it];
        if (e >= 0) {
            const int row = tot[e] + cnt[warp * a.E + e] + rk[it];
            a.row_idx[i] = row;
            a.row_token[row] = token_of(a, i);
        } else {
            a.row_idx[i] = -1;
        }
        if (i >= R) a.row_token[i] = -1;
    }
}

// Several tiles, kernel 1: per-tile counts into the workspace, and each
// valid entry's rank inside its tile packed with its expert into row_idx
// (expert << 16 | rank; the rank is below 4096) for the placement kernel.
__global__ void __launch_bounds__(kDispThreads) dispatch_count_kernel(const DispatchArgs a) {
    extern __shared__ __align__(16) int32_t dsm[];
    int32_t* sid = dsm;               // [4096]
    int32_t* cnt = sid + kDispTile;   // [8][E]
    tile_prologue(a, cnt, sid);
    int ex[kDispIter], rk[kDispIter];
    tile_ranks(a, sid, cnt, nullptr, ex, rk);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t wbase = static_cast<int64_t>(blockIdx.x) * kDispTile + warp * kDispWarpSpan;
#pragma unroll
    for (int it = 0; it < kDispIter; ++it) {
        const int64_t i = wbase + it * 32 + lane;
        if (i >= a.n) continue;
        const int e = ex[it];
        a.row_idx[i] = e >= 0 ? ((e << 16) | (cnt[warp * a.E + e] + rk[it])) : -1;
    }
}

// Kernel 2: per expert, the exclusive scan of its tile counts over the tiles
// (in place) and its total.  One CTA of 32 warps per 32 experts; warp w scans
// the w-th 32nd of the tiles, lane l expert 32 * blockIdx.x + l.
constexpr int kScanWarps = 32;

__global__ void __launch_bounds__(kScanWarps * 32) dispatch_scan_kernel(const DispatchArgs a) {
    __shared__ int32_t part[kScanWarps][32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int e = blockIdx.x * 32 + lane;
    const bool ok = e < a.E;
    const int per = (a.ntiles + kScanWarps - 1) / kScanWarps;
    const int t0 = warp * per;
    const int t1 = min(a.ntiles, t0 + per);
    griddep_wait();
    griddep_launch();
    int32_t* col = a.tile_counts + e;
    int s = 0;
    if (ok) {
#pragma unroll 8
        for (int t = t0; t < t1; ++t) s += col[static_cast<int64_t>(t) * a.E];
    }
    part[warp][lane] = s;
    __syncthreads();
    int base = 0, total = 0;
#pragma unroll
    for (int w = 0; w < kScanWarps; ++w) {
        if (w < warp) base += part[w][lane];
        total += part[w][lane];
    }
    if (ok) {
#pragma unroll 8
        for (int t = t0; t < t1; ++t) {
            const int c = col[static_cast<int64_t>(t) * a.E];
            col[static_cast<int64_t>(t) * a.E] = base;
            base += c;
        }
        if (warp == 0) a.totals[e] = total;
    }
}

// Kernel 3: offsets from the totals (every CTA scans them; CTA 0 writes them
// out), then each entry's row = offsets[e] + tile base of e + rank in tile.
// FOLD (few tiles): kernel 2 is skipped and every CTA forms its own tile
// bases and the totals from the raw per-tile counts (ntiles * E loads per
// CTA, all of them L2 hits).
template <bool FOLD>
__global__ void __launch_bounds__(kDispThreads) dispatch_place_kernel(const DispatchArgs a) {
    extern __shared__ __align__(16) int32_t dsm[];
    int32_t* add = dsm;          // [E]
    int32_t* ws = dsm + a.E;     // [8]
    griddep_wait();
    griddep_launch();
    int4 v[kDispTile / 4 / kDispThreads];
    load_tile4<false>(a.row_idx, a.n, -1, v);   // packed (expert, rank) from kernel 1; rewritten below
    // this tile's bases per expert, fetched beside the totals (E <= 16 * 256)
    constexpr int kPer = kMaxExperts / kDispThreads;
    int base[kPer];
    if constexpr (FOLD) {
#pragma unroll
        for (int j = 0; j < kPer; ++j) {
            const int e = threadIdx.x + j * kDispThreads;
            int sum = 0, mine = 0;
            if (e < a.E) {
#pragma unroll 8
                for (int t = 0; t < a.ntiles; ++t) {
                    const int c = __ldg(a.tile_counts + static_cast<int64_t>(t) * a.E + e);
                    mine = (t == static_cast<int>(blockIdx.x)) ? sum : mine;
                    sum += c;
                }
                add[e] = sum;
            }
            base[j] = mine;
        }
    } else {
        const int32_t* tb = a.tile_counts + static_cast<int64_t>(blockIdx.x) * a.E;
#pragma unroll
        for (int j = 0; j < kPer; ++j) {
            const int e = threadIdx.x + j * kDispThreads;
            base[j] = e < a.E ? __ldg(tb + e) : 0;
            if (e < a.E) add[e] = __ldg(a.totals + e);
        }
    }
    __syncthreads();
    const int R = block_exclusive_scan(add, a.E, ws);
    if (blockIdx.x == 0)
        for (int e = threadIdx.x; e <= a.E; e += kDispThreads) a.offsets[e] = e < a.E ? add[e] : R;
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
        const int e = threadIdx.x + j * kDispThreads;
        if (e < a.E) add[e] += base[j];
    }
    __syncthreads();
    const int64_t tile0 = static_cast<int64_t>(blockIdx.x) * kDispTile;
#pragma unroll
    for (int m = 0; m < kDispTile / 4 / kDispThreads; ++m) {
        const int64_t i = tile0 + 4 * (threadIdx.x + m * kDispThreads);
        if (i >= a.n) break;
        int r[4] = {v[m].x, v[m].y, v[m].z, v[m].w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            if (r[q] >= 0) {
                r[q] = add[r[q] >> 16] + (r[q] & 0xffff);
                if (i + q < a.n) a.row_token[r[q]] = token_of(a, i + q);
            }
            if (i + q >= R && i + q < a.n) a.row_token[i + q] = -1;
        }
        if (i + 3 < a.n) {
            *reinterpret_cast<int4*>(a.row_idx + i) = make_int4(r[0], r[1], r[2], r[3]);
        } else {
            for (int q = 0; q < 4; ++q)
                if (i + q < a.n) a.row_idx[i + q] = r[q];
        }
    }
}

int64_t dispatch_tiles(int64_t n) { return (n + kDispTile - 1) / kDispTile; }

// The shared-memory opt-in of the two kernels that take per-warp counts,
// set once per device for the largest expert count.
cudaError_t set_smem_once() {
    constexpr int kMaxDev = 64;
    static std::once_flag once[kMaxDev];
    static cudaError_t err[kMaxDev];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDev) return cudaErrorInvalidDevice;
    std::call_once(once[dev], [dev] {
        const int single = (kDispTile + (kDispWarps + 1) * kMaxExperts + kDispWarps) * 4;
        const int count = (kDispTile + kDispWarps * kMaxExperts) * 4;
        cudaError_t r = cudaFuncSetAttribute(reinterpret_cast<const void*>(dispatch_single_kernel),
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, single);
        if (r == cudaSuccess)
            r = cudaFuncSetAttribute(reinterpret_cast<const void*>(dispatch_count_kernel),
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, count);
        err[dev] = r;
    });
    return err[dev];
}

}  // namespace

size_t dispatch_workspace_bytes(int64_t n, int E) {
    const int64_t nt = dispatch_tiles(n);
    if (nt <= 1) return 0;
    return static_cast<size_t>((nt + 1) * E) * sizeof(int32_t);
}

cudaError_t launch_dispatch(const int32_t* ids, int T, int k, int e0, int E, int32_t* offsets, int32_t* row_idx,
                            int32_t* row_token, void* workspace, cudaStream_t s) {
    DispatchArgs a{};
    a.ids = ids;
    a.n = static_cast<int64_t>(T) * k;
    a.k = k;
    a.e0 = e0;
    a.E = E;
    a.offsets = offsets;
    a.row_idx = row_idx;
    a.row_token = row_token;
    const int64_t nt = dispatch_tiles(a.n);
    a.ntiles = static_cast<int>(nt);
    cudaLaunchAttribute attr[1];
    cudaError_t err = set_smem_once();
    if (err != cudaSuccess) return err;
    if (nt <= 1) {
        const size_t smem = (kDispTile + static_cast<size_t>(kDispWarps + 1) * E + kDispWarps) * sizeof(int32_t);
        cudaLaunchConfig_t cfg = pdl_config(1, kDispThreads, smem, s, attr);
        return cudaLaunchKernelEx(&cfg, dispatch_single_kernel, a);
    }
    a.tile_counts = static_cast<int32_t*>(workspace);
    a.totals = a.tile_counts + nt * E;
    const size_t smem1 = (kDispTile + static_cast<size_t>(kDispWarps) * E) * sizeof(int32_t);
    cudaLaunchConfig_t c1 = pdl_config(static_cast<int>(nt), kDispThreads, smem1, s, attr);
    err = cudaLaunchKernelEx(&c1, dispatch_count_kernel, a);
    if (err != cudaSuccess) return err;
    const size_t smem3 = (static_cast<size_t>(E) + kDispWarps) * sizeof(int32_t);
    cudaLaunchConfig_t c3 = pdl_config(static_cast<int>(nt), kDispThreads, smem3, s, attr);
    if (nt <= kDispFoldTiles) return cudaLaunchKernelEx(&c3, dispatch_place_kernel<true>, a);
    cudaLaunchConfig_t c2 = pdl_config((E + 31) / 32, kScanWarps * 32, 0, s, attr);
    err = cudaLaunchKernelEx(&c2, dispatch_scan_kernel, a);
    if (err != cudaSuccess) return err;
    return cudaLaunchKernelEx(&c3, dispatch_place_kernel<false>, a);
}

}  // namespace mb
