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
// that device; in host code the array's name only stands for it.
#include <mutex>

#include "moe_boundary.h"
#include "internal.h"

namespace mb {

namespace {

// 1 MiB of int32 counts: (ceil(T * k / 4096) + 1) * E of them per call.
constexpr size_t kNoAllocScratchBytes = size_t(1) << 20;

static __device__ __align__(256) int32_t g_dispatch_scratch[kNoAllocScratchBytes / sizeof(int32_t)];

struct ScratchAddress {
    std::once_flag once;
    void* ptr = nullptr;
    cudaError_t err = cudaSuccess;
};
constexpr int kScratchDevices = 64;
ScratchAddress g_scratch_address[kScratchDevices];

// Device address of g_dispatch_scratch on the current device.
cudaError_t scratch_address(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kScratchDevices) return cudaErrorInvalidDevice;
    ScratchAddress& s = g_scratch_address[dev];
    std::call_once(s.once, [&s] { s.err = cudaGetSymbolAddress(&s.ptr, g_dispatch_scratch); });
    *out = s.ptr;
    return s.err;
}

}  // namespace

}  // namespace mb

extern "C" int moe_dispatch_noalloc(const int32_t* topk_ids, int T, int k, int expert_begin, int E,
                                    int32_t* expert_offsets, int32_t* row_idx, int32_t* row_token, void* stream) {
    using namespace mb;
    const size_t need = moe_dispatch_workspace_size(T, k, E);
    if (need > kNoAllocScratchBytes)
        return fail(MB_ERR_UNSUPPORTED,
                    "moe_dispatch_noalloc: T=%d, k=%d, E=%d needs %zu bytes of scratch; the library's "
                    "fixed array holds %zu (call moe_dispatch with a workspace instead)",
                    T, k, E, need, kNoAllocScratchBytes);
    void* scratch = nullptr;
    if (need > 0) {
        const cudaError_t e = scratch_address(&scratch);
        if (e != cudaSuccess) return cuda_status(e, "moe_dispatch_noalloc (scratch address)");
    }
    return moe_dispatch(topk_ids, T, k, expert_begin, E, expert_offsets, row_idx, row_token, scratch,
                        need > 0 ? kNoAllocScratchBytes : 0, stream);
}
