// route.cuh -- device-side pieces of the sigmoid router gate, shared by the
// router kernels (route.cu) and the router warps of the fused norm-quant
// kernel (norm_quant.cu).
//
// Per valid token t (TensorRT-LLM PR 21356 "Muse Spark Open decoder fast
// paths", description, Routing; lmdeploy PR 4835 "MoE gate v2", token mask):
//   s_e = sigmoid(l_e)            FP32, the project's exp (below)
//   c_e = s_e + bias_e            selection score only
//   picks = first k experts in the order (c descending, id ascending)
//   w_j   = s_{pick j} / (s_{pick 0} + ... + s_{pick k-1})   summed in pick order
// and for an invalid token ids = -1, weights = 0 without reading its logits.
//
// Selection takes two steps per token.  A shortlist from a fast sigmoid (the
// hardware's approximate 2^x and reciprocal, within kSigFastErr of the exact
// one): k rounds of one warp max over each lane's two best approximate scores
// give a value tau that at least k experts reach, and only experts whose
// approximate score lies within twice the error bound below tau can belong to
// the exact top k (every other one is exactly below k others).  Those
// candidates -- typically k or a few more -- get the exact sigmoid, move to
// one lane each and are put in pick order by broadcast ranks or a bitonic
// network across the lanes, with no dependent chain of warp reductions.  When more than 32 remain
// (massive exact ties) the token takes the exact merge rounds over all its
// experts instead.
#pragma once

#include "common.cuh"

namespace mb {

// ---------------------------------------------------------------- exp / sigmoid
// Range reduction x = n ln2 + r with a Cody-Waite split of ln2 (a 15-fraction-bit
// head, so n * head is exact), a degree-7 Taylor polynomial of e^r (Horner,
// fused multiply-adds) and 2^n from the exponent field.  Inputs are clamped to
// [-87, 88] so 2^n stays a normal number.  (The clamp and the rounding of n
// use max/min and an add-and-subtract of 1.5 * 2^23: the same values as
// compare-and-select and rintf, in fewer instructions.)
__device__ __forceinline__ float exp_fixed(float x) {
    constexpr float kLn2Hi = 22713.0f / 32768.0f;
    constexpr float kLn2Lo = (float)(0.6931471805599453094 - 22713.0 / 32768.0);
    constexpr float kLog2e = (float)1.4426950408889634074;
    {   // clamp, a NaN passing through
        float y;
        asm("max.NaN.f32 %0, %1, %2;" : "=f"(y) : "f"(x), "f"(-87.0f));
        asm("min.NaN.f32 %0, %1, %2;" : "=f"(x) : "f"(y), "f"(88.0f));
    }
    const float t = __fmul_rn(x, kLog2e);
    // n = t rounded to the nearest integer, ties to even (|t| < 128): adding
    // 1.5 * 2^23 leaves the integer in the low bits of `big`
    const float big = __fadd_rn(t, 12582912.0f);
    const float n = __fsub_rn(big, 12582912.0f);
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
    // 2^n: big's bits are 0x4B400000 + n, and 0x4B400000 << 23 vanishes mod 2^32
    const float two_n = __uint_as_float((__float_as_uint(big) + 127u) << 23);
    return __fmul_rn(p, two_n);
}

__device__ __forceinline__ float sigmoid_fixed(float x) {
    const float e = exp_fixed(-x);
    return __frcp_rn(__fadd_rn(1.0f, e));
}

// 32-bit selection key of a score: order-preserving image of the float
// (larger key = larger score), -0 and +0 equal, NaN = 1 (below every number),
// 0 = "no candidate".  Equal keys are broken by the lower expert id.
__device__ __forceinline__ uint32_t score_key(float c) {
    c = __fadd_rn(c, 0.0f);                                  // -0 -> +0
    const uint32_t u = __float_as_uint(c);
    const uint32_t k = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    return (c != c) ? 1u : k;
}

__device__ __forceinline__ uint32_t warp_max_u32(uint32_t v) { return __reduce_max_sync(0xffffffffu, v); }
__device__ __forceinline__ uint32_t warp_min_u32(uint32_t v) { return __reduce_min_sync(0xffffffffu, v); }

// One merge round: the warp's best (key, id) over every lane's best
// candidate; returns true on the lane that owns it.
__device__ __forceinline__ bool pick_round(uint32_t my_key, uint32_t my_id, uint32_t& key, uint32_t& id) {
    key = warp_max_u32(my_key);
    id = warp_min_u32(my_key == key ? my_id : 0xffffffffu);
    return my_key == key && my_id == id;
}

// This lane's EPL logits of a token row (4 per 128-bit load, ids
// 4 * (lane + 32 u) + i ascending with the register index; 0 past E).
template <int EPL>
__device__ __forceinline__ void load_logits(const float* l, int E, int lane, bool vec, float (&lv)[EPL]) {
#pragma unroll
    for (int u = 0; u < EPL / 4; ++u) {
        const int q = lane + 32 * u;
        if (vec && 4 * q + 3 < E) {
            const float4 v = ld_nc_f4(l + 4 * q);
            lv[4 * u + 0] = v.x;
            lv[4 * u + 1] = v.y;
            lv[4 * u + 2] = v.z;
            lv[4 * u + 3] = v.w;
        } else {
#pragma unroll
            for (int i = 0; i < 4; ++i) lv[4 * u + i] = (4 * q + i < E) ? __ldg(l + 4 * q + i) : 0.0f;
        }
    }
}

// Expert id of position p of this lane's scores (4 per 128-bit load,
// ids 4 * (lane + 32 u) + i for position 4 u + i).
__device__ __forceinline__ uint32_t lane_pos_id(int p, int lane) {
    return 4u * static_cast<uint32_t>(lane + 32 * (p >> 2)) + static_cast<uint32_t>(p & 3);
}

// A lane's remaining candidates for the merge rounds: its best and
// second-best keys not yet picked (largest key, lowest position -- hence
// lowest id -- among equals) and the positions already picked.  When its
// best is picked the second is promoted; only a lane picked twice in a row
// without a rescan in between scans its scores again, so most rounds cost a
// few instructions instead of a rescan.
template <int EPL>
struct LaneTop2 {
    uint32_t k1, k2, id1, id2;
    int p1, p2;
    uint32_t used;
    bool have2;

    __device__ __forceinline__ void scan(const uint32_t (&key)[EPL], int lane) {
        k1 = k2 = 0u;
        p1 = p2 = 0;
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
            const uint32_t v = ((used >> i) & 1u) ? 0u : key[i];
            if (v > k1) {
                k2 = k1;
                p2 = p1;
                k1 = v;
                p1 = i;
            } else if (v > k2) {
                k2 = v;
                p2 = i;
            }
        }
        id1 = lane_pos_id(p1, lane);
        id2 = lane_pos_id(p2, lane);
        have2 = true;
    }
    __device__ __forceinline__ void init(const uint32_t (&key)[EPL], int lane) {
        used = 0u;
        scan(key, lane);
    }
    // this lane's best was picked
    __device__ __forceinline__ void pop(const uint32_t (&key)[EPL], int lane) {
        used |= 1u << p1;
        if (have2) {
            k1 = k2;
            p1 = p2;
            id1 = id2;
            have2 = false;
        } else {
            scan(key, lane);
        }
    }
};

// E <= 32 * EPL: every lane keeps its EPL scores; k merge rounds, each a warp
// max over the lanes' best remaining keys, the lowest id among the lanes
// holding it winning.
template <int EPL>
__device__ __forceinline__ void select_small(const float (&lv)[EPL], const float* bias, int E, int k, int lane,
                                             bool vec, uint32_t& pick_key, uint32_t& pick_id) {
    uint32_t key[EPL];
#pragma unroll
    for (int u = 0; u < EPL / 4; ++u) {
        const int q = lane + 32 * u;
        if (vec && 4 * q + 3 < E) {
            const float4 b = __ldg(reinterpret_cast<const float4*>(bias) + q);
            key[4 * u + 0] = score_key(__fadd_rn(sigmoid_fixed(lv[4 * u + 0]), b.x));
            key[4 * u + 1] = score_key(__fadd_rn(sigmoid_fixed(lv[4 * u + 1]), b.y));
            key[4 * u + 2] = score_key(__fadd_rn(sigmoid_fixed(lv[4 * u + 2]), b.z));
            key[4 * u + 3] = score_key(__fadd_rn(sigmoid_fixed(lv[4 * u + 3]), b.w));
        } else {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int e = 4 * q + i;
                key[4 * u + i] = e < E ? score_key(__fadd_rn(sigmoid_fixed(lv[4 * u + i]), __ldg(bias + e))) : 0u;
            }
        }
    }
    LaneTop2<EPL> c;
    c.init(key, lane);
    for (int j = 0; j < k; ++j) {
        uint32_t key_j, id_j;
        if (pick_round(c.k1, c.id1, key_j, id_j)) c.pop(key, lane);
        if (lane == j) {
            pick_key = key_j;
            pick_id = id_j;
        }
    }
}

// The picks' unbiased sigmoids, renormalised in pick order (lane j < k holds
// pick j), written with the ids.
__device__ __forceinline__ void route_write(const float* l, int k, int lane, uint32_t pick_id, int32_t* id_row,
                                            float* w_row) {
    const int e = static_cast<int>(pick_id);
    float s = 0.0f;
    if (lane < k) s = sigmoid_fixed(__ldg(l + e));
    float S = 0.0f;
    for (int j = 0; j < k; ++j) S = __fadd_rn(S, __shfl_sync(0xffffffffu, s, j));
    if (lane < k) {
        id_row[lane] = e;
        w_row[lane] = __fdiv_rn(s, S);
    }
}

// ---------------------------------------------------------------- shortlist and verify
// Fast sigmoid for the shortlist: 1 / (1 + 2^(-x log2 e)) with the hardware's
// approximate 2^x and reciprocal (flush-to-zero).  Over all 2^32 binary32
// inputs it differs from sigmoid_fixed by at most 1.79e-7 (2^-22.4) on sm_100a;
// moe_route_check_fast_sigmoid measures that on the device, and kSigFastErr
// bounds it with a margin.
constexpr float kSigFastErr = 0x1p-21f;
constexpr float kInf = __builtin_huge_valf();

__device__ __forceinline__ float sigmoid_fast(float x) {
    const float t = __fmul_rn(x, -1.4426950408889634f);
    float e, r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e) : "f"(t));
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(__fadd_rn(1.0f, e)));
    return r;
}

// The number a key > 1 stands for (inverse of score_key).
__device__ __forceinline__ float key_value(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// Twice an upper bound on |c_fast - c| over a token's experts, where
// c = fl(s + b) and c_fast = fl(s_fast + b): the sigmoid's error plus one ulp
// of the largest |s + b| <= max|b| + 2 (a half-ulp rounding on each side);
// infinite when a bias is not finite.  bmax_bits: the bits of max |b|.
__device__ __forceinline__ float shortlist_width(uint32_t bmax_bits) {
    const float B = __fadd_ru(__uint_as_float(bmax_bits), 2.0f);
    const uint32_t ex = (__float_as_uint(B) >> 23) & 0xFFu;
    if (ex == 0xFFu) return kInf;
    const float ulp_b = __uint_as_float((ex - 23u) << 23);
    return __fmul_ru(2.0f, __fadd_ru(kSigFastErr, ulp_b));
}

// The window's floor: an expert whose fast score is below it scores exactly
// below every expert whose fast score reached tau (the k-th round's maximum,
// as a key), and at least k did.  Rounded down; -inf keeps every number.
__device__ __forceinline__ float shortlist_floor(uint32_t tau, float width) {
    if (!(width < kInf)) return -kInf;
    return __fsub_rd(key_value(tau), width);
}

// k rounds of the warp's best offer over each lane's two best fast scores
// (as keys): every lane holding the round's maximum gives it up, so each round
// removes at least one expert scoring at least the final maximum, returned.
__device__ __forceinline__ uint32_t shortlist_tau(float a1f, float a2f, int k) {
    uint32_t a1 = score_key(a1f), a2 = score_key(a2f), tau = 0u;
    for (int j = 0; j < k; ++j) {
        tau = warp_max_u32(a1);
        if (a1 == tau) {
            a1 = a2;
            a2 = 0u;
        }
    }
    return tau;
}

// Running best two of a lane's fast scores (NaN counts as -inf here).
__device__ __forceinline__ void top2_update(float v, float& a1, float& a2) {
    v = fmaxf(v, -kInf);
    a2 = fmaxf(a2, fminf(v, a1));
    a1 = fmaxf(a1, v);
}

// Position of the n-th (from 0) set bit of m; m has more than n set bits.
__device__ __forceinline__ int nth_set_bit(uint32_t m, int n) {
    int pos = 0;
#pragma unroll
    for (int w = 16; w > 0; w >>= 1) {
        const int c = __popc(m & ((1u << w) - 1u));
        if (n >= c) {
            n -= c;
            m >>= w;
            pos += w;
        }
    }
    return pos;
}

// Largest expert id the shortlist's 64-bit order can carry (27 bits).
constexpr uint32_t kShortlistIdMax = (1u << 27) - 1u;
static_assert(kMaxExperts <= static_cast<int>(kShortlistIdMax) + 1, "expert ids fit the shortlist's order");

// The warp's 64-bit values sorted descending over lanes 0..N-1 (N = 16 or 32;
// lane l ends with the l-th largest): a bitonic network of compare-exchanges
// between lanes l and l ^ stride, block l / size descending when even.
template <int N>
__device__ __forceinline__ uint64_t warp_sort_desc(uint64_t v, int lane) {
#pragma unroll
    for (int size = 2; size <= N; size <<= 1) {
#pragma unroll
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            const uint64_t o = __shfl_xor_sync(0xffffffffu, v, stride);
            const bool keep_max = ((lane & stride) == 0) == ((lane & size) == 0);
            v = keep_max ? (o > v ? o : v) : (o < v ? o : v);
        }
    }
    return v;
}

// Rank a token's shortlisted experts exactly and write its picks.  Each lane
// holds `cnt` of them; next_id() yields the lane's next expert id (cnt calls).
// The ids move to one lane each, every lane computes its expert's exact
// sigmoid and selection key at once, and broadcast ranks (up to 16) or a
// bitonic network across the lanes (above) put them in pick order.
// Returns false, writing nothing, when the warp holds more than 32 or fewer
// than k shortlisted experts.
template <bool SORT32, class NextId>
__device__ __forceinline__ bool shortlist_finish(int cnt, int lane, int k, NextId&& next_id,
                                                 const float* __restrict__ row, const float* __restrict__ bias,
                                                 int32_t* id_row, float* w_row) {
    constexpr uint32_t kAll = 0xffffffffu;
    int incl = cnt;                                  // inclusive prefix of the counts
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(kAll, incl, o);
        if (lane >= o) incl += v;
    }
    const int nc = __shfl_sync(kAll, incl, 31);
    if (nc > 32 || nc < k) return false;
    // slot d (lane d < nc) takes id d - start of the lane whose slots begin at
    // `start`, the highest slot start at or below d
    const int off = incl - cnt;
    const uint32_t starts = __reduce_or_sync(kAll, cnt > 0 ? (1u << off) : 0u);
    const uint32_t holders = __ballot_sync(kAll, cnt > 0);
    int src = lane, rd = -1;
    if (lane < nc) {
        const int start = 31 - __clz(starts & (0xffffffffu >> (31 - lane)));
        src = nth_set_bit(holders, __popc(starts & ((1u << start) - 1u)));
        rd = lane - start;
    }
    const int rounds = __reduce_max_sync(kAll, cnt);
    uint32_t mid = 0u;
    for (int r = 0; r < rounds; ++r) {
        const uint32_t cid = (r < cnt) ? next_id() : 0u;
        const uint32_t g = __shfl_sync(kAll, cid, src);
        if (rd == r) mid = g;
    }
    // the order (key descending, id ascending) as one 64-bit number, larger
    // first: key, then ~id -- or, for the network, 2^27 - 1 - id and the lane
    // (ids are distinct, so the lane never decides; it tells where the
    // candidate's sigmoid sits)
    uint64_t mine = 0u;                              // lanes without a candidate sort last
    float ms = 0.0f;
    if (lane < nc) {
        ms = sigmoid_fixed(__ldg(row + mid));
        const uint32_t key = score_key(__fadd_rn(ms, __ldg(bias + mid)));
        mine = (static_cast<uint64_t>(key) << 32) |
               (SORT32 ? (static_cast<uint64_t>(kShortlistIdMax - mid) << 5) | static_cast<uint64_t>(lane)
                       : static_cast<uint64_t>(~mid));
    }
    // `from` on lane p: the lane holding the p-th largest.  With SORT32 and
    // above 16 candidates a bitonic network over the 32 lanes sorts them (the
    // lane travels in the low bits); otherwise each candidate's rank comes
    // from broadcasts, eight per step so that they overlap, and lane p learns
    // which lane holds rank p from one warp OR per bit of the lane index.  The
    // network is cheaper at k = 22 (85.8 against 89.0 us at 65536 x 512); the
    // broadcast ranks are cheaper up to 16 candidates (8.5 against 8.7 us at
    // 8192 x 256, k = 8), and the large-E kernel, whose k is 8 in practice,
    // runs faster without the network's code (115.5 against 118.2 us).
    int from = 0;
    if (SORT32 && nc > 16) {
        from = static_cast<int>(warp_sort_desc<32>(mine, lane) & 31u);
    } else {
        int rank = 0;
        for (int i0 = 0; i0 < nc; i0 += 8) {
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const uint64_t other = __shfl_sync(kAll, mine, (i0 + q) & 31);
                rank += (other > mine) ? 1 : 0;
            }
        }
#pragma unroll
        for (int bit = 0; bit < 5; ++bit) {
            const uint32_t m = __reduce_or_sync(kAll, (lane < nc && ((lane >> bit) & 1)) ? (1u << rank) : 0u);
            from |= static_cast<int>((m >> lane) & 1u) << bit;
        }
    }
    const float sp = __shfl_sync(kAll, ms, from);    // lane p < k: the sigmoid of pick p
    const uint32_t idp = __shfl_sync(kAll, mid, from);
    float S = 0.0f;                                  // summed in pick order
    for (int p = 0; p < k; ++p) S = __fadd_rn(S, __shfl_sync(kAll, sp, p));
    if (lane < k) {
        id_row[lane] = static_cast<int32_t>(idp);
        w_row[lane] = __fdiv_rn(sp, S);
    }
    return true;
}

// One token with E <= 32 EPL: the lane's EPL fast scores in registers.
// Returns false (nothing written) when the shortlist does not fit.
template <int EPL>
__device__ __forceinline__ bool route_token_shortlist(const float* __restrict__ row, const float* __restrict__ bias,
                                                      int E, int k, int lane, bool vec, float width, int32_t* id_row,
                                                      float* w_row) {
    float av[EPL];
    float a1 = -kInf, a2 = -kInf;
    {
        float lv[EPL], bv[EPL];
        load_logits<EPL>(row, E, lane, vec, lv);
        load_logits<EPL>(bias, E, lane, vec, bv);
        if (E == 32 * EPL) {                         // every position holds an expert
#pragma unroll
            for (int p = 0; p < EPL; ++p) {
                av[p] = __fadd_rn(sigmoid_fast(lv[p]), bv[p]);
                top2_update(av[p], a1, a2);
            }
        } else {
#pragma unroll
            for (int p = 0; p < EPL; ++p) {
                av[p] = lane_pos_id(p, lane) < static_cast<uint32_t>(E) ? __fadd_rn(sigmoid_fast(lv[p]), bv[p])
                                                                        : __int_as_float(0x7fc00000);
                top2_update(av[p], a1, a2);
            }
        }
    }
    const float lo = shortlist_floor(shortlist_tau(a1, a2, k), width);
    uint32_t rem = 0u;
#pragma unroll
    for (int p = 0; p < EPL; ++p) rem |= (av[p] >= lo) ? (1u << p) : 0u;
    const int cnt = __popc(rem);
    auto next_id = [&]() {
        const int p = __ffs(rem) - 1;
        rem &= rem - 1u;
        return lane_pos_id(p, lane);
    };
    return shortlist_finish<true>(cnt, lane, k, next_id, row, bias, id_row, w_row);
}

// Large E (more than 16 experts per lane): the fast scores go through the
// warp's shared-memory row `keys` as FP16 (128 ceil(E / 128) halves, 2 bytes
// each: half the space of FP32, so more warps fit per SM); the score of
// expert e is half e, lane l handling experts 128 c + 4 l .. + 3 of each chunk
// c (one 8-byte store or load per chunk, conflict-free).  The FP16 rounding
// widens the window by `store_err` (half an FP16 ulp of the largest score), so
// every expert whose fast score reaches the floor still does after storing.
// A lane keeps up to kWideLaneCands shortlisted experts; when one has more,
// or the warp more than 32, it returns false and writes nothing.
constexpr int kWideLaneCands = 8;

__device__ __forceinline__ uint2 pack_f16x4(float a, float b, float c, float d) {
    uint2 r;
    asm("cvt.rn.f16x2.f32 %0, %2, %1;" : "=r"(r.x) : "f"(a), "f"(b));
    asm("cvt.rn.f16x2.f32 %0, %2, %1;" : "=r"(r.y) : "f"(c), "f"(d));
    return r;
}
__device__ __forceinline__ float f16_lo(uint32_t w) {
    float f;
    asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %1;\n\tcvt.f32.f16 %0, lo;\n\t}" : "=f"(f) : "r"(w));
    return f;
}
__device__ __forceinline__ float f16_hi(uint32_t w) {
    float f;
    asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %1;\n\tcvt.f32.f16 %0, hi;\n\t}" : "=f"(f) : "r"(w));
    return f;
}

// Half an FP16 ulp of the largest |fast score| (at most max|b| + 2), or
// infinity when FP16 cannot hold it (every expert is then shortlisted).
__device__ __forceinline__ float f16_store_err(uint32_t bmax_bits) {
    const float B = __fadd_ru(__uint_as_float(bmax_bits), 2.0f);
    if (!(B < 32768.0f)) return kInf;
    const uint32_t ex = (__float_as_uint(B) >> 23) & 0xFFu;    // B >= 2: ex >= 128
    return __uint_as_float((ex - 11u) << 23);                  // 2^(e - 11) = ulp_f16(B) / 2
}

__device__ __forceinline__ bool route_token_wide(const float* __restrict__ row, const float* __restrict__ bias, int E,
                                                 int k, int lane, bool vec, float width, float store_err,
                                                 uint16_t* keys, int32_t* id_row, float* w_row) {
    const int nch = (E + 127) >> 7;
    const float nan = __int_as_float(0x7fc00000);
    float a1 = -kInf, a2 = -kInf;
    for (int c0 = 0; c0 < nch; c0 += 4) {          // four chunks' loads in flight at a time
        float4 v[4], b[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int e0 = 128 * (c0 + u) + 4 * lane;
            if (vec && e0 + 3 < E) {
                v[u] = ld_nc_f4(row + e0);
                b[u] = __ldg(reinterpret_cast<const float4*>(bias + e0));
            } else {
                v[u].x = (e0 + 0 < E) ? __ldg(row + e0 + 0) : 0.0f;
                v[u].y = (e0 + 1 < E) ? __ldg(row + e0 + 1) : 0.0f;
                v[u].z = (e0 + 2 < E) ? __ldg(row + e0 + 2) : 0.0f;
                v[u].w = (e0 + 3 < E) ? __ldg(row + e0 + 3) : 0.0f;
                b[u].x = (e0 + 0 < E) ? __ldg(bias + e0 + 0) : 0.0f;
                b[u].y = (e0 + 1 < E) ? __ldg(bias + e0 + 1) : 0.0f;
                b[u].z = (e0 + 2 < E) ? __ldg(bias + e0 + 2) : 0.0f;
                b[u].w = (e0 + 3 < E) ? __ldg(bias + e0 + 3) : 0.0f;
            }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int c = c0 + u;
            if (c < nch) {
                const int e0 = 128 * c + 4 * lane;
                float f0, f1, f2, f3;
                if (128 * (c + 1) <= E) {                // a full chunk (the same for the whole warp)
                    f0 = __fadd_rn(sigmoid_fast(v[u].x), b[u].x);
                    f1 = __fadd_rn(sigmoid_fast(v[u].y), b[u].y);
                    f2 = __fadd_rn(sigmoid_fast(v[u].z), b[u].z);
                    f3 = __fadd_rn(sigmoid_fast(v[u].w), b[u].w);
                } else {
                    f0 = (e0 + 0 < E) ? __fadd_rn(sigmoid_fast(v[u].x), b[u].x) : nan;
                    f1 = (e0 + 1 < E) ? __fadd_rn(sigmoid_fast(v[u].y), b[u].y) : nan;
                    f2 = (e0 + 2 < E) ? __fadd_rn(sigmoid_fast(v[u].z), b[u].z) : nan;
                    f3 = (e0 + 3 < E) ? __fadd_rn(sigmoid_fast(v[u].w), b[u].w) : nan;
                }
                *reinterpret_cast<uint2*>(keys + e0) = pack_f16x4(f0, f1, f2, f3);
                top2_update(f0, a1, a2);
                top2_update(f1, a1, a2);
                top2_update(f2, a1, a2);
                top2_update(f3, a1, a2);
            }
        }
    }
    const float lo = __fsub_rd(shortlist_floor(shortlist_tau(a1, a2, k), width), store_err);
    int cnt = 0;
    uint32_t cand[kWideLaneCands];                    // shortlisted experts, newest first
#pragma unroll
    for (int i = 0; i < kWideLaneCands; ++i) cand[i] = 0u;
    for (int c = 0; c < nch; ++c) {
        const int e0 = 128 * c + 4 * lane;
        const uint2 h = *reinterpret_cast<const uint2*>(keys + e0);
        const float fv[4] = {f16_lo(h.x), f16_hi(h.x), f16_lo(h.y), f16_hi(h.y)};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            if (fv[i] >= lo) {                        // NaN (past E) never
#pragma unroll
                for (int q = kWideLaneCands - 1; q > 0; --q) cand[q] = cand[q - 1];
                cand[0] = static_cast<uint32_t>(e0 + i);
                ++cnt;
            }
        }
    }
    int taken = 0;
    auto next_id = [&]() {
        const int q = cnt - 1 - taken;                // oldest first
        ++taken;
        uint32_t e = cand[0];
#pragma unroll
        for (int i = 1; i < kWideLaneCands; ++i) e = (q == i) ? cand[i] : e;
        return e;
    };
    return shortlist_finish<false>(cnt > kWideLaneCands ? 33 : cnt, lane, k, next_id, row, bias, id_row, w_row);
}

// Exact merge rounds for the large-E path when its shortlist does not fit,
// with no scratch: each lane tracks its best two remaining (key, position) of
// its experts 128 c + 4 lane + i, recomputing their exact keys from memory
// when it rescans (only after both were taken); taken positions are bits of
// a 128-bit mask (E <= 4096: at most 128 positions a lane).  k rounds as in
// select_small.  Sets the lane's pick (lane j < k: pick j).
__device__ __forceinline__ void select_wide_exact(const float* __restrict__ l, const float* __restrict__ bias, int E,
                                                  int k, int lane, uint32_t& pick_id) {
    const int npos = 4 * ((E + 127) >> 7);
    auto expert = [&](int p) { return static_cast<uint32_t>(128 * (p >> 2) + 4 * lane + (p & 3)); };
    uint32_t taken[4] = {0u, 0u, 0u, 0u};
    auto is_taken = [&](int p) {
        const uint32_t w = (p < 32) ? taken[0] : (p < 64) ? taken[1] : (p < 96) ? taken[2] : taken[3];
        return ((w >> (p & 31)) & 1u) != 0u;
    };
    auto take = [&](int p) {
        const uint32_t m = 1u << (p & 31);
        if (p < 32) taken[0] |= m;
        else if (p < 64) taken[1] |= m;
        else if (p < 96) taken[2] |= m;
        else taken[3] |= m;
    };
    uint32_t k1 = 0u, k2 = 0u;
    int p1 = 0, p2 = 0;
    bool have2 = true;
    auto scan = [&]() {
        k1 = k2 = 0u;
        p1 = p2 = 0;
        for (int p = 0; p < npos; ++p) {
            const uint32_t e = expert(p);
            const uint32_t v = (e < static_cast<uint32_t>(E) && !is_taken(p))
                                   ? score_key(__fadd_rn(sigmoid_fixed(__ldg(l + e)), __ldg(bias + e)))
                                   : 0u;
            if (v > k1) {
                k2 = k1;
                p2 = p1;
                k1 = v;
                p1 = p;
            } else if (v > k2) {
                k2 = v;
                p2 = p;
            }
        }
        have2 = true;
    };
    scan();
    for (int j = 0; j < k; ++j) {
        uint32_t key_j, id_j;
        if (pick_round(k1, expert(p1), key_j, id_j)) {
            take(p1);
            if (have2) {
                k1 = k2;
                p1 = p2;
                have2 = false;
            } else {
                scan();
            }
        }
        if (lane == j) pick_id = id_j;
    }
}

// The bits of max |bias| over the call's experts (from memory).
__device__ __forceinline__ uint32_t bias_max_bits(const float* bias, int E, int lane) {
    uint32_t m = 0u;
    for (int e = lane; e < E; e += 32) m = max(m, __float_as_uint(fabsf(__ldg(bias + e))));
    return warp_max_u32(m);
}

// The shortlist window of a call, from the biases in memory.
__device__ __forceinline__ float bias_width(const float* bias, int E, int lane) {
    return shortlist_width(bias_max_bits(bias, E, lane));
}

// Larger E: every lane keeps a sorted list of its L best (key, id); ids arrive
// in ascending order, so inserting strictly below equal keys keeps ties in id
// order.
template <int L>
__device__ __forceinline__ void route_token_list(const float* l, const float* bias, int E, int k, int lane,
                                                 bool vec, uint32_t& pick_key, uint32_t& pick_id) {
    uint32_t lk[L], li[L];
#pragma unroll
    for (int i = 0; i < L; ++i) {
        lk[i] = 0u;
        li[i] = 0xffffffffu;
    }
    auto insert = [&](uint32_t key, uint32_t id) {
        if (key > lk[L - 1]) {
#pragma unroll
            for (int i = 0; i < L; ++i) {
                const bool gt = key > lk[i];
                const uint32_t tk = lk[i], ti = li[i];
                lk[i] = gt ? key : tk;
                li[i] = gt ? id : ti;
                key = gt ? tk : key;
                id = gt ? ti : id;
            }
        }
    };
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
                    const uint32_t e = 4u * static_cast<uint32_t>(q);
                    insert(score_key(__fadd_rn(sigmoid_fixed(v[u].x), b.x)), e);
                    insert(score_key(__fadd_rn(sigmoid_fixed(v[u].y), b.y)), e + 1);
                    insert(score_key(__fadd_rn(sigmoid_fixed(v[u].z), b.z)), e + 2);
                    insert(score_key(__fadd_rn(sigmoid_fixed(v[u].w), b.w)), e + 3);
                }
            }
        }
    } else {
        for (int e = lane; e < E; e += 32)
            insert(score_key(__fadd_rn(sigmoid_fixed(__ldg(l + e)), __ldg(bias + e))), static_cast<uint32_t>(e));
    }
    for (int j = 0; j < k; ++j) {
        uint32_t key_j, id_j;
        if (pick_round(lk[0], li[0], key_j, id_j)) {
#pragma unroll
            for (int i = 0; i < L - 1; ++i) {
                lk[i] = lk[i + 1];
                li[i] = li[i + 1];
            }
            lk[L - 1] = 0u;
            li[L - 1] = 0xffffffffu;
        }
        if (lane == j) {
            pick_key = key_j;
            pick_id = id_j;
        }
    }
}


// One token per warp iteration (t, t + nwarps, ...) for E <= 32 MODE (MODE
// <= 8), the next token's mask byte read at the end of each iteration: one
// selection chain at a time measured faster than two interleaved (or than the
// next token's logits held in registers).  SHORTLIST: the shortlist selection
// (the standalone router kernels, where it measured faster: 10.2 -> 8.6 us at
// 8192 x 256); otherwise the exact merge rounds over the lane's registers (the
// router warps inside the norm-quant kernel, whose row warps the shortlist's
// shuffles slowed: 41.3 -> 44.3 us for the fused call).
template <int MODE, bool SHORTLIST>
__device__ __forceinline__ void route_singles(const float* __restrict__ logits, const float* __restrict__ bias,
                                              const uint8_t* __restrict__ mask, int T, int E, int k,
                                              int32_t* __restrict__ ids, float* __restrict__ weights, int warp,
                                              int nwarps, int lane) {
    const bool vec = (E & 3) == 0;
    int t = warp;
    if (t >= T) return;
    bool valid = mask[t] != 0;
    if constexpr (SHORTLIST) {
        const float width = bias_width(bias, E, lane);
        for (;;) {
            const int tn = t + nwarps;
            int32_t* id_row = ids + static_cast<size_t>(t) * k;
            float* w_row = weights + static_cast<size_t>(t) * k;
            const float* row = logits + static_cast<size_t>(t) * E;
            if (!valid) {
                if (lane < k) {
                    id_row[lane] = -1;
                    w_row[lane] = 0.0f;
                }
            } else if (!route_token_shortlist<MODE>(row, bias, E, k, lane, vec, width, id_row, w_row)) {
                float lv[MODE];
                load_logits<MODE>(row, E, lane, vec, lv);
                uint32_t pick_key = 0u, pick_id = 0u;
                select_small<MODE>(lv, bias, E, k, lane, vec, pick_key, pick_id);
                route_write(row, k, lane, pick_id, id_row, w_row);
            }
            if (tn >= T) break;
            t = tn;
            valid = mask[t] != 0;
        }
    } else {
        float lv[MODE];
#pragma unroll
        for (int i = 0; i < MODE; ++i) lv[i] = 0.0f;
        for (;;) {
            const int tn = t + nwarps;
            if (valid) load_logits<MODE>(logits + static_cast<size_t>(t) * E, E, lane, vec, lv);
            int32_t* id_row = ids + static_cast<size_t>(t) * k;
            float* w_row = weights + static_cast<size_t>(t) * k;
            if (!valid) {
                if (lane < k) {
                    id_row[lane] = -1;
                    w_row[lane] = 0.0f;
                }
            } else {
                uint32_t pick_key = 0u, pick_id = 0u;
                select_small<MODE>(lv, bias, E, k, lane, vec, pick_key, pick_id);
                route_write(logits + static_cast<size_t>(t) * E, k, lane, pick_id, id_row, w_row);
            }
            if (tn >= T) break;
            t = tn;
            valid = mask[t] != 0;
        }
    }
}

// Validity of this warp's tokens t0, t0 + nwarps, ..., 32 of them, one mask
// byte per lane in one load (bit j: token t0 + j nwarps is valid).
__device__ __forceinline__ uint32_t warp_token_mask(const uint8_t* __restrict__ mask, int T, int64_t t0, int nwarps,
                                                    int lane) {
    const int64_t t = t0 + static_cast<int64_t>(lane) * nwarps;
    return __ballot_sync(0xffffffffu, t < T && mask[t] != 0);
}

// Bring a logits row (E floats) into L2 ahead of its use, 128 bytes a lane.
__device__ __forceinline__ void prefetch_row_l2(const float* row, int E, int lane) {
    for (int e = 32 * lane; e < E; e += 32 * 32) asm volatile("prefetch.global.L2 [%0];" ::"l"(row + e));
}

// One token per warp iteration with the shortlist: MODE > 0, E <= 32 MODE
// with the fast scores in registers; MODE == 0, larger E through the warp's
// shared-memory row `keys`.  The mask bytes of 32 tokens come in one load and
// the next valid token's logits are prefetched into L2 while this one is
// selected.  A token whose shortlist does not fit takes the exact rounds.
template <int MODE>
__device__ __forceinline__ void route_shortlist_tokens(const float* __restrict__ logits,
                                                       const float* __restrict__ bias,
                                                       const uint8_t* __restrict__ mask, int T, int E, int k,
                                                       int32_t* __restrict__ ids, float* __restrict__ weights,
                                                       int warp, int nwarps, int lane, uint16_t* keys = nullptr) {
    const bool vec = (E & 3) == 0;
    if (warp >= T) return;
    const uint32_t bmax = bias_max_bits(bias, E, lane);
    const float width = shortlist_width(bmax);
    const float store_err = MODE > 0 ? 0.0f : f16_store_err(bmax);
    uint32_t vbits = 0u;
    for (int64_t j = 0, t = warp; t < T; ++j, t += nwarps) {
        if ((j & 31) == 0) vbits = warp_token_mask(mask, T, t, nwarps, lane);
        const bool valid = (vbits >> (j & 31)) & 1u;
        const float* row = logits + static_cast<size_t>(t) * E;
        const int64_t tn = t + nwarps;
        const bool next_valid = ((j & 31) != 31) ? ((vbits >> ((j + 1) & 31)) & 1u) : (tn < T);
        if (next_valid && tn < T) prefetch_row_l2(logits + static_cast<size_t>(tn) * E, E, lane);
        int32_t* id_row = ids + static_cast<size_t>(t) * k;
        float* w_row = weights + static_cast<size_t>(t) * k;
        if (!valid) {
            if (lane < k) {
                id_row[lane] = -1;
                w_row[lane] = 0.0f;
            }
            continue;
        }
        uint32_t pick_id = 0u;
        if constexpr (MODE > 0) {
            if (route_token_shortlist<MODE>(row, bias, E, k, lane, vec, width, id_row, w_row)) continue;
            float lv[MODE];
            load_logits<MODE>(row, E, lane, vec, lv);
            uint32_t pick_key = 0u;
            select_small<MODE>(lv, bias, E, k, lane, vec, pick_key, pick_id);
        } else {
            if (route_token_wide(row, bias, E, k, lane, vec, width, store_err, keys, id_row, w_row)) continue;
            select_wide_exact(row, bias, E, k, lane, pick_id);
        }
        route_write(row, k, lane, pick_id, id_row, w_row);
    }
}

}  // namespace mb
