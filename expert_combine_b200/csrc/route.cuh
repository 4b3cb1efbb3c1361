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
#pragma once

#include "common.cuh"

namespace mb {

// ---------------------------------------------------------------- exp / sigmoid
// Range reduction x = n ln2 + r with a Cody-Waite split of ln2 (a 15-fraction-bit
// head, so n * head is exact), a degree-7 Taylor polynomial of e^r (Horner,
// fused multiply-adds) and 2^n from the exponent field.  Inputs are clamped to
// [-87, 88] so 2^n stays a normal number.
__device__ __forceinline__ float exp_fixed(float x) {
    constexpr float kLn2Hi = 22713.0f / 32768.0f;
    constexpr float kLn2Lo = (float)(0.6931471805599453094 - 22713.0 / 32768.0);
    constexpr float kLog2e = (float)1.4426950408889634074;
    x = (x < -87.0f) ? -87.0f : x;
    x = (x > 88.0f) ? 88.0f : x;
    const float t = __fmul_rn(x, kLog2e);
    const float n = rintf(t);
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
    const float two_n = __uint_as_float(static_cast<uint32_t>(static_cast<int>(n) + 127) << 23);
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


// One token per warp iteration (t, t + nwarps, ...) on the small path
// (E <= 32 * MODE), for the router kernels and the router warps of the fused
// norm-quant kernel: one selection chain at a time measured faster than two
// interleaved (or than the next token's logits held in registers).  The next
// token's mask byte is read at the end of each iteration.
template <int MODE>
__device__ __forceinline__ void route_singles(const float* __restrict__ logits, const float* __restrict__ bias,
                                              const uint8_t* __restrict__ mask, int T, int E, int k,
                                              int32_t* __restrict__ ids, float* __restrict__ weights, int warp,
                                              int nwarps, int lane) {
    const bool vec = (E & 3) == 0;
    int t = warp;
    if (t >= T) return;
    bool valid = mask[t] != 0;
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

}  // namespace mb
