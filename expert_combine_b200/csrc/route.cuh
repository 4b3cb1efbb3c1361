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

// Two tokens at once (independent selection chains interleaved round by
// round); tokens that are absent or masked are given all-zero keys and their
// picks are ignored by the caller.
template <int EPL>
__device__ __forceinline__ void select_small2(const float (&la)[EPL], const float (&lb)[EPL], bool va, bool vb,
                                              const float* bias, int E, int k, int lane, bool vec,
                                              uint32_t& pick_a, uint32_t& pick_b) {
    uint32_t ka[EPL], kb[EPL];
#pragma unroll
    for (int u = 0; u < EPL / 4; ++u) {
        const int q = lane + 32 * u;
        float4 b;
        if (vec && 4 * q + 3 < E) {
            b = __ldg(reinterpret_cast<const float4*>(bias) + q);
        } else {
            b.x = 4 * q + 0 < E ? __ldg(bias + 4 * q + 0) : 0.0f;
            b.y = 4 * q + 1 < E ? __ldg(bias + 4 * q + 1) : 0.0f;
            b.z = 4 * q + 2 < E ? __ldg(bias + 4 * q + 2) : 0.0f;
            b.w = 4 * q + 3 < E ? __ldg(bias + 4 * q + 3) : 0.0f;
        }
        const float bb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const bool in = 4 * q + i < E;
            ka[4 * u + i] = (va && in) ? score_key(__fadd_rn(sigmoid_fixed(la[4 * u + i]), bb[i])) : 0u;
            kb[4 * u + i] = (vb && in) ? score_key(__fadd_rn(sigmoid_fixed(lb[4 * u + i]), bb[i])) : 0u;
        }
    }
    LaneTop2<EPL> ca, cb;
    ca.init(ka, lane);
    cb.init(kb, lane);
    for (int j = 0; j < k; ++j) {
        const uint32_t ma = warp_max_u32(ca.k1);
        const uint32_t mb = warp_max_u32(cb.k1);
        const uint32_t wa = warp_min_u32(ca.k1 == ma ? ca.id1 : 0xffffffffu);
        const uint32_t wb = warp_min_u32(cb.k1 == mb ? cb.id1 : 0xffffffffu);
        if (ca.k1 == ma && ca.id1 == wa) ca.pop(ka, lane);
        if (cb.k1 == mb && cb.id1 == wb) cb.pop(kb, lane);
        if (lane == j) {
            pick_a = wa;
            pick_b = wb;
        }
    }
}

// Picks of two tokens written together (lane j < k holds pick j of each);
// a token that is absent (t >= T) is skipped, a masked one gets -1 / 0.
__device__ __forceinline__ void route_write2(const float* logits, int E, int k, int lane, int ta, int tb,
                                             bool pa, bool pb, bool va, bool vb, uint32_t id_a, uint32_t id_b,
                                             int32_t* ids, float* weights) {
    const float* la = logits + static_cast<size_t>(ta) * E;
    const float* lb = logits + static_cast<size_t>(tb) * E;
    float sa = 0.0f, sb = 0.0f;
    if (lane < k) {
        if (va) sa = sigmoid_fixed(__ldg(la + id_a));
        if (vb) sb = sigmoid_fixed(__ldg(lb + id_b));
    }
    float Sa = 0.0f, Sb = 0.0f;
    for (int j = 0; j < k; ++j) {
        Sa = __fadd_rn(Sa, __shfl_sync(0xffffffffu, sa, j));
        Sb = __fadd_rn(Sb, __shfl_sync(0xffffffffu, sb, j));
    }
    if (lane < k) {
        if (pa) {
            ids[static_cast<size_t>(ta) * k + lane] = va ? static_cast<int32_t>(id_a) : -1;
            weights[static_cast<size_t>(ta) * k + lane] = va ? __fdiv_rn(sa, Sa) : 0.0f;
        }
        if (pb) {
            ids[static_cast<size_t>(tb) * k + lane] = vb ? static_cast<int32_t>(id_b) : -1;
            weights[static_cast<size_t>(tb) * k + lane] = vb ? __fdiv_rn(sb, Sb) : 0.0f;
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


// Two tokens per warp iteration (t and t + nwarps), for the small path
// (E <= 32 * MODE).  The next pair's mask bytes and logits are loaded one
// iteration ahead, so a warp that routes many tokens keeps a load in flight
// while it selects.
template <int MODE>
__device__ __forceinline__ void route_pairs(const float* __restrict__ logits, const float* __restrict__ bias,
                                            const uint8_t* __restrict__ mask, int T, int E, int k,
                                            int32_t* __restrict__ ids, float* __restrict__ weights, int warp,
                                            int nwarps, int lane) {
    const bool vec = (E & 3) == 0;
    int t = warp;
    if (t >= T) return;
    bool va = mask[t] != 0;
    bool pb = t + nwarps < T;
    bool vb = pb && mask[t + nwarps] != 0;
    float la[MODE], lb[MODE];
#pragma unroll
    for (int i = 0; i < MODE; ++i) la[i] = lb[i] = 0.0f;
    if (va) load_logits<MODE>(logits + static_cast<size_t>(t) * E, E, lane, vec, la);
    if (vb) load_logits<MODE>(logits + static_cast<size_t>(t + nwarps) * E, E, lane, vec, lb);
    for (;;) {
        const int tn = t + 2 * nwarps;
        const bool pn = tn < T;
        const bool pnb = tn + nwarps < T;
        const bool vna = pn && mask[tn] != 0;
        const bool vnb = pnb && mask[tn + nwarps] != 0;
        float na[MODE], nb[MODE];
#pragma unroll
        for (int i = 0; i < MODE; ++i) na[i] = nb[i] = 0.0f;
        if (vna) load_logits<MODE>(logits + static_cast<size_t>(tn) * E, E, lane, vec, na);
        if (vnb) load_logits<MODE>(logits + static_cast<size_t>(tn + nwarps) * E, E, lane, vec, nb);
        uint32_t ida = 0u, idb = 0u;
        select_small2<MODE>(la, lb, va, vb, bias, E, k, lane, vec, ida, idb);
        const int tb = pb ? t + nwarps : t;
        route_write2(logits, E, k, lane, t, tb, true, pb, va, vb, ida, idb, ids, weights);
        if (!pn) break;
        t = tn;
        va = vna;
        vb = vnb;
        pb = pnb;
#pragma unroll
        for (int i = 0; i < MODE; ++i) {
            la[i] = na[i];
            lb[i] = nb[i];
        }
    }
}

// One token per warp iteration (t, t + nwarps, ...), for the router warps of
// the fused norm-quant kernel: with a fixed number of warps each warp routes
// several tokens, and one selection chain at a time measured faster there
// than two interleaved (or than the next token's logits held in registers).
// The next token's mask byte is read at the end of each iteration.
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
