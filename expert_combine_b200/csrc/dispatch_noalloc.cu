// dispatch_noalloc.cu -- moe_dispatch for callers that cannot allocate device
// memory.
//
// moe_dispatch needs a caller-provided workspace once T * k exceeds one tile
// (4096 entries).  Some callers have no way to provide one: their device
// memory is owned by an allocator they cannot reach from this call site (a
// framework's caching pool behind a plain C interface), or they must not call
// cudaMalloc / cudaFree on the hot path because those calls can synchronise
// the whole device and stall the other streams of a serving loop, or the
// weights and caches already hold nearly all of the GPU's memory.  For them,
// moe_dispatch_noalloc takes its scratch from a fixed array compiled into the
// library instead.
//
// The array lives in device memory for as long as the library is loaded, on
// every GPU that loads it.  Its address is looked up once per device
// (cudaGetSymbolAddress, with that device current) on the first call made on
// that device that succeeds; in host code the array's name only stands for it.
// A failed lookup (for example an error left over from an earlier launch) is
// not remembered: the next call looks again.  The remembered address belongs
// to the device's context as it was at the lookup, so it assumes that context
// lives as long as the process: after cudaDeviceReset the array is a new
// allocation and this entry point must not be called again in that process.
#include <mutex>

#include "moe_boundary.h"
#include "internal.h"

namespace mb {

namespace {

// 1 MiB of int32 counts: (ceil(T * k / 4096) + 1) * E of them per call.
constexpr size_t kNoAllocScratchBytes = size_t(1) << 20;

static __device__ __align__(256) int32_t g_dispatch_scratch[kNoAllocScratchBytes / sizeof(int32_t)];

constexpr int kScratchDevices = 64;
std::mutex g_scratch_mutex;
void* g_scratch_address[kScratchDevices] = {};   // null until a lookup on that device succeeded

// Device address of g_dispatch_scratch on the current device.
cudaError_t scratch_address(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kScratchDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (g_scratch_address[dev] == nullptr) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_dispatch_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_address[dev] = p;
    }
    *out = g_scratch_address[dev];
    return cudaSuccess;
}

}  // namespace

}  // namespace mb

extern "C" int moe_dispatch_noalloc(const int32_t* topk_ids, int T, int k, int expert_begin, int E,
                                    int32_t* expert_offsets, int32_t* row_idx, int32_t* row_token, void* stream) {
    using namespace mb;
    const char* fn = "moe_dispatch_noalloc";
    const int st = check_dispatch(fn, topk_ids, T, k, expert_begin, E, expert_offsets, row_idx, row_token);
    if (st != MB_OK) return st;
    const size_t need = moe_dispatch_workspace_size(T, k, E);
    if (need > kNoAllocScratchBytes)
        return fail(MB_ERR_UNSUPPORTED,
                    "%s: T=%d, k=%d, E=%d needs %zu bytes of scratch; the library's "
                    "fixed array holds %zu (call moe_dispatch with a workspace instead)",
                    fn, T, k, E, need, kNoAllocScratchBytes);
    void* scratch = nullptr;
    if (need > 0) {
        const cudaError_t e = scratch_address(&scratch);
        if (e != cudaSuccess) return cuda_status(e, "moe_dispatch_noalloc: scratch address");
    }
    return moe_dispatch(topk_ids, T, k, expert_begin, E, expert_offsets, row_idx, row_token, scratch,
                        need > 0 ? kNoAllocScratchBytes : 0, stream);
}
