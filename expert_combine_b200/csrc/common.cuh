// common.cuh -- device helpers shared by the MoE-boundary kernels (sm_100a).
//
// Arithmetic contract (all kernels are compiled with --fmad=false): every
// float operation below is a single IEEE binary32 operation, fused
// multiply-adds appear only as explicit fmaf(), divisions and square roots are
// the correctly rounded __fdiv_rn / __frcp_rn / __fsqrt_rn.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace mb {

// ------------------------------------------------------------------ errors
// Set (bitwise OR) by a kernel whose bounded wait on an mbarrier ran out.
// The host reads and clears it through mb_device_status().  (The library is
// one translation unit, so this is its single definition.)
__device__ unsigned int g_wait_timeout = 0u;

constexpr unsigned long long kWaitLimitNs = 2000000000ull;   // 2 s

__device__ __forceinline__ unsigned long long globaltimer_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ------------------------------------------------------------------ BF16
__device__ __forceinline__ float bf16_lo(uint32_t packed) { return __uint_as_float(packed << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t packed) { return __uint_as_float(packed & 0xffff0000u); }

// Round two floats to BF16 (nearest even) and pack them, a in the low half.
__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&v);
}

// Round to BF16 and return the rounded value as a float.
__device__ __forceinline__ float round_bf16(float a) {
    return __bfloat162float(__float2bfloat16_rn(a));
}

// ------------------------------------------------------------------ mbarrier / bulk copy
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_addr(bar))
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
                     smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for the phase with the given parity to complete, for at most
// kWaitLimitNs.  Returns false (and flags g_wait_timeout) when the limit ran out.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, unsigned int code) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer_ns();
    while (true) {
        for (int i = 0; i < 64; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
            atomicOr(&g_wait_timeout, code);
            return false;
        }
    }
}

// One-dimensional bulk copy global -> shared, completing on an mbarrier.
// dst, src and bytes must be multiples of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_addr(dst)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

// Named barrier over `count` threads (a multiple of 32).
__device__ __forceinline__ void named_bar_sync(int id, int count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// ------------------------------------------------------------------ loads
__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ float4 ld_nc_f4(const void* p) {
    float4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.f32 {%0,%1,%2,%3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ void st_v4(void* p, uint4 v) {
    asm volatile("st.global.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

// ------------------------------------------------------------------ canonical sums of squares
// Sequential fused multiply-add over the 16 values of one block.
__device__ __forceinline__ float block_sumsq16(const float* v) {
    float a = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) a = fmaf(v[i], v[i], a);
    return a;
}

// Butterfly over the 32 lanes: level by level, lane pairs (l, l^1), then
// pairs of pairs, ...  Every lane ends with the same bits, equal to the
// balanced pairwise tree over lanes 0..31 in order (IEEE addition commutes).
__device__ __forceinline__ float warp_tree_sum(float v) {
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) v = v + __shfl_xor_sync(0xffffffffu, v, off);
    return v;
}

// Balanced pairwise tree over n (a power of two) values in order.
template <int N>
__device__ __forceinline__ float tree_sum_array(const float* v) {
    if constexpr (N == 1) {
        return v[0];
    } else {
        float tmp[N / 2];
#pragma unroll
        for (int i = 0; i < N / 2; ++i) tmp[i] = v[2 * i] + v[2 * i + 1];
        return tree_sum_array<N / 2>(tmp);
    }
}

// 1 / sqrt(ss / H + eps), three correctly rounded steps.
__device__ __forceinline__ float inv_rms(float ss, float H, float eps) {
    float mean = __fdiv_rn(ss, H);
    float d = __fadd_rn(mean, eps);
    float r = __fsqrt_rn(d);
    return __frcp_rn(r);
}

// ------------------------------------------------------------------ FP8 / FP4 conversions
// E4M3 round-to-nearest-even with saturation to +-448 (no NaN for finite input).
__device__ __forceinline__ uint32_t cvt_e4m3_satfinite(float a) {
    uint16_t r;
    asm("{\n\t.reg .b16 t;\n\tcvt.rn.satfinite.e4m3x2.f32 t, %2, %1;\n\tmov.b16 %0, t;\n\t}"
        : "=h"(r)
        : "f"(a), "f"(0.0f));
    return r & 0xffu;
}

// Decode an E4M3 byte to float (exact).
__device__ __forceinline__ float e4m3_to_f32(uint32_t c) {
    uint32_t packed;
    uint16_t in = static_cast<uint16_t>(c);
    asm("{\n\t.reg .b32 t;\n\tcvt.rn.f16x2.e4m3x2 t, %1;\n\tmov.b32 %0, t;\n\t}" : "=r"(packed) : "h"(in));
    __half h = __ushort_as_half(static_cast<unsigned short>(packed & 0xffffu));
    return __half2float(h);
}

// Eight E2M1 codes packed in a 32-bit word, v[0] in the lowest nibble
// (round-to-nearest-even on the E2M1 grid, saturating).  The caller passes no
// -0 (a -0 would come back with the sign bit set).
__device__ __forceinline__ uint32_t cvt_e2m1x8(const float* v) {
    uint32_t r;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(r)
        : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
    return r;
}

}  // namespace mb

// ------------------------------------------------------------------ paired FP32 (sm_100 f32x2)
// Two independent IEEE binary32 operations per instruction; each lane of the
// pair is rounded exactly like the scalar operation.
namespace mb {

__device__ __forceinline__ uint64_t f2_bits(float2 a) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a.x), "f"(a.y));
    return r;
}
__device__ __forceinline__ float2 bits_f2(uint64_t r) {
    float2 a;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a.x), "=f"(a.y) : "l"(r));
    return a;
}
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(f2_bits(a)), "l"(f2_bits(b)));
    return bits_f2(d);
}
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(f2_bits(a)), "l"(f2_bits(b)));
    return bits_f2(d);
}
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(f2_bits(a)), "l"(f2_bits(b)), "l"(f2_bits(c)));
    return bits_f2(d);
}
// Mixed-precision fused multiply-add on the BF16 halves of two pair words:
// fl32(a_h * b_h + c), the product exact (BF16 inputs widen exactly), one
// rounding -- the same bits as fmaf(float(a_h), float(b_h), c).
__device__ __forceinline__ float fma_bf16_lo(uint32_t a, uint32_t b, float c) {
    float d;
    asm("{\n\t.reg .b16 al, ah, bl, bh;\n\tmov.b32 {al, ah}, %1;\n\tmov.b32 {bl, bh}, %2;\n\t"
        "fma.rn.f32.bf16 %0, al, bl, %3;\n\t}"
        : "=f"(d)
        : "r"(a), "r"(b), "f"(c));
    return d;
}
__device__ __forceinline__ float fma_bf16_hi(uint32_t a, uint32_t b, float c) {
    float d;
    asm("{\n\t.reg .b16 al, ah, bl, bh;\n\tmov.b32 {al, ah}, %1;\n\tmov.b32 {bl, bh}, %2;\n\t"
        "fma.rn.f32.bf16 %0, ah, bh, %3;\n\t}"
        : "=f"(d)
        : "r"(a), "r"(b), "f"(c));
    return d;
}
// Exact product of the BF16 halves as a float pair: (a_lo * b_lo, a_hi * b_hi)
// (adding -0 keeps the sign of a zero product).
__device__ __forceinline__ float2 mul_bf16x2_exact(uint32_t a, uint32_t b) {
    return make_float2(fma_bf16_lo(a, b, -0.0f), fma_bf16_hi(a, b, -0.0f));
}

// BF16 pair word -> two floats (exact).
__device__ __forceinline__ float2 unpack_bf16x2(uint32_t w) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}
// Two floats -> BF16 pair word, round to nearest even, x in the low half.
__device__ __forceinline__ uint32_t pack_bf16x2_rn(float2 v) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %2, %1;" : "=r"(r) : "f"(v.x), "f"(v.y));
    return r;
}
// Round one float to BF16 (nearest even) and return it as a float: the
// conversion packs (a, 0) so the result word is exactly the float's bits.
__device__ __forceinline__ float round_bf16_f(float a) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(a), "f"(0.0f));
    return __uint_as_float(r);
}
__device__ __forceinline__ float2 round_bf16_f2(float2 v) {
    return make_float2(round_bf16_f(v.x), round_bf16_f(v.y));
}

// Largest magnitude of the two BF16 halves of a and b, per half (signs are
// not meaningful in the result; only the magnitudes are used).
__device__ __forceinline__ uint32_t maxabs_bf16x2(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr));
    return v;
}

// 2-D tiled TMA load global -> shared (no multicast), completing on an mbarrier.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void* tmap, int x, int y, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(tmap), "r"(x), "r"(y), "r"(smem_addr(bar))
        : "memory");
}

// Orders this thread's earlier generic-proxy shared-memory accesses before
// its later async-proxy (TMA) ones.
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

}  // namespace mb
