/*
 * oracle.c -- plain, slow CPU oracle for the per-token MoE boundary.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark load this code.  The CUDA library never
 * links, includes or calls it, and it includes nothing from the CUDA side.
 *
 * Every floating-point step is written out as a scalar IEEE-754 binary32
 * operation in program order (compile with -ffp-contract=off and without
 * -ffast-math); fmaf() appears only where the arithmetic spec names a fused
 * multiply-add.  Sources, by page title and section:
 *
 *  - "[TRTLLM-17146][feat] Add the Muse Spark Open decoder fast paths"
 *    (TensorRT-LLM PR 21356), description: the routing kernel (sigmoid, bias,
 *    top-8, renormalised weights, sorted picks, ties to the lowest id), the
 *    post-expert norm + combine (invalid slots never read), the gated
 *    residual join, and the "Numerics" paragraph (the norm adds the 1 of the
 *    gain in FP32 and rounds its result to BF16 once).
 *  - "Muse Spark Open reference composition" (TensorRT-LLM PR 21042), MoE
 *    paragraph: FP32 router, post-expert RMSNorm of each expert output before
 *    the weighted top-k sum, weight-first norms.
 *  - "prepare_trtllm_nvfp4" (vLLM API page), functions
 *    _quantize_nvfp4_global_scale and norm_quant_trtllm_nvfp4: per-16 amax,
 *    E4M3 block scale from the global scale, E2M1 thresholds, sign bit,
 *    nibble packing, linear scale layout, the rank-block input layout.
 *  - TensorRT-LLM PR 21356, description, "Router projection": the router
 *    logits come from a projection with FP32 weights and FP32 accumulation,
 *    the BF16 input cast to FP32 and a scale folded in.
 *  - TensorRT-LLM PR 21356, description, "Fused finalize + all-reduce", and
 *    PR 21042, MoE paragraph: the expert finalize and the tensor-parallel
 *    all-reduce of its partials with FP32 accumulation.
 *  - "MoE gate v2" (lmdeploy PR 4835), commit notes: a required token mask;
 *    invalid tokens produce no routing entries; absent rows marked -1; the
 *    gate's routing entries are grouped per expert by a histogram and a scan
 *    (the dispatch step), and en2f, the map from a routing entry to its row,
 *    is cleared to -1 where no row exists.
 *
 * Where the pages leave a step open the oracle takes one fixed reading
 * (listed in the repository's design notes): the sigmoid's exp is the
 * project's own range-reduced Taylor polynomial, sums of squares use a fixed
 * balanced tree over 16-element block partials, and the scale reciprocals are
 * IEEE divisions.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------ */
/* threads (the oracle is parallel over tokens only; results do not    */
/* depend on the thread count)                                         */
/* ------------------------------------------------------------------ */
void oc_set_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int oc_get_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------ */
/* bit views                                                           */
/* ------------------------------------------------------------------ */
static uint32_t f2u(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }
static float u2f(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }

/* ------------------------------------------------------------------ */
/* BF16: 1 sign, 8 exponent, 7 fraction bits (the top half of binary32) */
/* ------------------------------------------------------------------ */
float oc_bf16_to_f32(uint16_t b) { return u2f((uint32_t)b << 16); }

/* Round-to-nearest-even of binary32 to bfloat16.  NaN stays NaN (quiet). */
uint16_t oc_bf16_rn(float x) {
    uint32_t u = f2u(x);
    if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t keep_lsb = (u >> 16) & 1u;          /* ties go to the even result */
    u += 0x7fffu + keep_lsb;
    return (uint16_t)(u >> 16);
}

/* ------------------------------------------------------------------ */
/* E4M3 (OCP FP8, "fn" variant): bias 7, 3 fraction bits, no infinity,  */
/* S.1111.111 is NaN, largest finite 448, subnormal step 2^-9.          */
/* ------------------------------------------------------------------ */
float oc_e4m3_decode(uint8_t c) {
    int s = c >> 7, e = (c >> 3) & 15, m = c & 7;
    float v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = (float)m * ldexpf(1.0f, -9);
    else v = (1.0f + (float)m / 8.0f) * ldexpf(1.0f, e - 7);
    return s ? -v : v;
}

/* Round to the nearest E4M3 value, ties to the even code, saturating to
 * +-448 (never NaN for a non-NaN input).  Written as a brute-force search
 * over the 127 finite magnitudes so that it can be read against the format
 * definition. */
uint8_t oc_e4m3_rn_sat(float x) {
    if (x != x) return 0x7f;
    uint8_t sign = signbit(x) ? 0x80 : 0x00;
    double a = fabs((double)x);
    if (a >= 448.0) return (uint8_t)(sign | 0x7e);
    if (a <= ldexp(1.0, -10)) return sign;      /* at or below half the smallest subnormal */
    int best = 0;
    double best_d = a;                           /* distance to code 0 (value 0) */
    for (int c = 1; c <= 0x7e; ++c) {
        double d = fabs(a - (double)oc_e4m3_decode((uint8_t)c));
        if (d < best_d || (d == best_d && (c & 1) == 0)) { best = c; best_d = d; }
    }
    return (uint8_t)(sign | best);
}

/* ------------------------------------------------------------------ */
/* E2M1 code of a scaled value, the threshold rule of                  */
/* _quantize_nvfp4_global_scale: the magnitude code counts the          */
/* thresholds that |q| passes, the sign bit is set when q < 0.          */
/* ------------------------------------------------------------------ */
uint8_t oc_e2m1_code(float q) {
    float m = fabsf(q);
    uint8_t c = 0;
    c += (m > 0.25f);
    c += (m >= 0.75f);
    c += (m > 1.25f);
    c += (m >= 1.75f);
    c += (m > 2.5f);
    c += (m >= 3.5f);
    c += (m > 5.0f);
    if (q < 0.0f) c |= 8;
    return c;
}

/* ------------------------------------------------------------------ */
/* the project's exp and sigmoid (the pages do not say how the sigmoid */
/* is evaluated; one definition is fixed so that selection is exact)    */
/* ------------------------------------------------------------------ */
float oc_exp(float x) {
    /* ln 2 split into a head with 15 fraction bits (so n * head is exact
     * for |n| <= 256) and the binary32 rounding of the remainder. */
    const float ln2_hi = (float)(floor(M_LN2 * 32768.0) / 32768.0);
    const float ln2_lo = (float)(M_LN2 - (double)ln2_hi);
    const float log2e = (float)M_LOG2E;
    if (x < -87.0f) x = -87.0f;
    if (x > 88.0f) x = 88.0f;
    float t = x * log2e;
    float n = rintf(t);                          /* round half to even */
    float r = fmaf(-n, ln2_hi, x);
    r = fmaf(-n, ln2_lo, r);
    /* Taylor polynomial of e^r to degree 7, coefficients 1/i!, Horner. */
    float p = (float)(1.0 / 5040.0);
    p = fmaf(p, r, (float)(1.0 / 720.0));
    p = fmaf(p, r, (float)(1.0 / 120.0));
    p = fmaf(p, r, (float)(1.0 / 24.0));
    p = fmaf(p, r, (float)(1.0 / 6.0));
    p = fmaf(p, r, 0.5f);
    p = fmaf(p, r, 1.0f);
    p = fmaf(p, r, 1.0f);
    /* 2^n from the exponent field; n is in [-126, 127] after the clamp. */
    float two_n = u2f((uint32_t)((int)n + 127) << 23);
    return p * two_n;
}

float oc_sigmoid(float x) {
    float e = oc_exp(-x);
    float d = 1.0f + e;
    return 1.0f / d;
}

/* ------------------------------------------------------------------ */
/* Stage 1: router gate                                                */
/* ------------------------------------------------------------------ */
typedef struct { float c; int e; } oc_cand;

/* Selection order: larger score first; equal scores go to the lower id;
 * a NaN score sorts after every number. */
static int oc_cand_cmp(const void* pa, const void* pb) {
    const oc_cand* a = (const oc_cand*)pa;
    const oc_cand* b = (const oc_cand*)pb;
    int an = (a->c != a->c), bn = (b->c != b->c);
    if (an != bn) return an - bn;
    if (!an) {
        if (a->c > b->c) return -1;
        if (a->c < b->c) return 1;
    }
    return (a->e > b->e) - (a->e < b->e);
}

/* logits [T,E] FP32, bias [E] FP32, mask [T] (nonzero = valid token)
 * -> ids [T,k] int32, weights [T,k] FP32. */
void oc_route(const float* logits, const float* bias, const uint8_t* mask,
              int T, int E, int k, int32_t* ids, float* weights) {
#pragma omp parallel for schedule(dynamic, 16)
    for (int t = 0; t < T; ++t) {
        int32_t* id_row = ids + (size_t)t * k;
        float* w_row = weights + (size_t)t * k;
        if (!mask[t]) {                          /* invalid token: no entries, logits unread */
            for (int j = 0; j < k; ++j) { id_row[j] = -1; w_row[j] = 0.0f; }
            continue;
        }
        const float* l = logits + (size_t)t * E;
        float* s = (float*)malloc(sizeof(float) * (size_t)E);
        oc_cand* cand = (oc_cand*)malloc(sizeof(oc_cand) * (size_t)E);
        for (int e = 0; e < E; ++e) {
            s[e] = oc_sigmoid(l[e]);
            float c = s[e] + bias[e];            /* bias steers selection only */
            if (c == 0.0f) c = 0.0f;             /* -0 and +0 are one score */
            cand[e].c = c;
            cand[e].e = e;
        }
        qsort(cand, (size_t)E, sizeof(oc_cand), oc_cand_cmp);
        float S = 0.0f;
        for (int j = 0; j < k; ++j) S = S + s[cand[j].e];
        for (int j = 0; j < k; ++j) {
            id_row[j] = cand[j].e;
            w_row[j] = s[cand[j].e] / S;         /* unbiased sigmoid, renormalised */
        }
        free(cand);
        free(s);
    }
}

/* ------------------------------------------------------------------ */
/* RMSNorm pieces                                                      */
/* ------------------------------------------------------------------ */

/* Sum of squares of n values (n a multiple of 16): a sequential fused
 * multiply-add over each block of 16, then a balanced pairwise tree over the
 * block partials, level by level, an odd last element carried up unchanged. */
float oc_sumsq(const float* v, int n) {
    int nb = n / 16;
    if (nb <= 0) return 0.0f;
    float* lev = (float*)malloc(sizeof(float) * (size_t)nb);
    for (int i = 0; i < nb; ++i) {
        float a = 0.0f;
        for (int j = 0; j < 16; ++j) a = fmaf(v[16 * i + j], v[16 * i + j], a);
        lev[i] = a;
    }
    while (nb > 1) {
        int m = 0;
        for (int i = 0; i + 1 < nb; i += 2) lev[m++] = lev[i] + lev[i + 1];
        if (nb & 1) lev[m++] = lev[nb - 1];
        nb = m;
    }
    float r = lev[0];
    free(lev);
    return r;
}

/* 1 / sqrt(ss / H + eps), three correctly rounded steps. */
float oc_inv_rms(float ss, int H, float eps) {
    float mean = ss / (float)H;
    float d = mean + eps;
    float r = sqrtf(d);
    return 1.0f / r;
}

/* Weight-first RMSNorm of one row, rounded once to BF16:
 * y = bf16((x * (gc + w)) * inv). */
static void oc_norm_row(const float* x, const uint16_t* w, float gc, float inv,
                        int H, uint16_t* y) {
    for (int h = 0; h < H; ++h) {
        float g = gc + oc_bf16_to_f32(w[h]);
        float t = x[h] * g;
        y[h] = oc_bf16_rn(t * inv);
    }
}

/* Logical element x[t, h] of an [M, H] activation stored either contiguous
 * (tp == 1) or in the rank-block layout [tp, M, H/tp] that a dim-0
 * all-gather of column shards leaves. */
static size_t oc_rank_block_offset(int t, int h, int M, int H, int tp) {
    int hs = H / tp;
    return ((size_t)(h / hs) * (size_t)M + (size_t)t) * (size_t)hs + (size_t)(h % hs);
}

/* ------------------------------------------------------------------ */
/* Stage 2: RMSNorm fused with NVFP4 quantisation                      */
/* ------------------------------------------------------------------ */

/* Quantise one 16-element block of BF16 values.  Writes 8 packed bytes
 * (even element in the low nibble) and returns the E4M3 scale byte.
 * near_code / near_sf (may be NULL) count values whose FP32 input lies
 * within one ulp of a rounding threshold. */
static uint8_t oc_quant_block(const uint16_t* y16, float gs, uint8_t* packed8,
                              long* near_code, long* near_sf) {
    float amax = 0.0f;
    for (int i = 0; i < 16; ++i) {
        float a = fabsf(oc_bf16_to_f32(y16[i]));
        if (a > amax) amax = a;
    }
    const float r6 = (float)(1.0 / 6.0);
    float t = amax * r6;
    float u = gs * t;
    uint8_t sf = oc_e4m3_rn_sat(u);
    if (near_sf) {
        float lo = nextafterf(u, 0.0f), hi = nextafterf(u, INFINITY);
        if (oc_e4m3_rn_sat(lo) != sf || oc_e4m3_rn_sat(hi) != sf) ++*near_sf;
    }
    float sf_f = oc_e4m3_decode(sf);
    float os = 0.0f;
    if (sf_f != 0.0f) {
        float rgs = 1.0f / gs;
        float m = sf_f * rgs;
        os = 1.0f / m;
    }
    uint8_t codes[16];
    for (int i = 0; i < 16; ++i) {
        float q = oc_bf16_to_f32(y16[i]) * os;
        codes[i] = oc_e2m1_code(q);
        if (near_code) {
            float lo = nextafterf(q, -INFINITY), hi = nextafterf(q, INFINITY);
            if (oc_e2m1_code(lo) != codes[i] || oc_e2m1_code(hi) != codes[i]) ++*near_code;
        }
    }
    for (int i = 0; i < 8; ++i)
        packed8[i] = (uint8_t)((codes[2 * i] & 0x0f) | (codes[2 * i + 1] << 4));
    return sf;
}

/* Pre-expert RMSNorm rounded to BF16 (no quantisation): y [M,H] BF16. */
void oc_norm_bf16(const uint16_t* x, int M, int H, int tp, const uint16_t* w,
                  float gc, float eps, uint16_t* y) {
#pragma omp parallel for schedule(dynamic, 4)
    for (int t = 0; t < M; ++t) {
        float* xf = (float*)malloc(sizeof(float) * (size_t)H);
        for (int h = 0; h < H; ++h) xf[h] = oc_bf16_to_f32(x[oc_rank_block_offset(t, h, M, H, tp)]);
        float inv = oc_inv_rms(oc_sumsq(xf, H), H, eps);
        oc_norm_row(xf, w, gc, inv, H, y + (size_t)t * H);
        free(xf);
    }
}

/* RMSNorm + NVFP4 of M rows: packed [M, H/2] u8, sf [M, H/16] u8 (linear).
 * gs is the FP32 global scale.  near[0] / near[1] (may be NULL) receive the
 * counts of near-threshold codes and scales. */
void oc_norm_quant(const uint16_t* x, int M, int H, int tp, const uint16_t* w,
                   float gc, float eps, float gs, uint8_t* packed, uint8_t* sf,
                   long* near) {
    long nc = 0, ns = 0;
#pragma omp parallel for schedule(dynamic, 4) reduction(+ : nc, ns)
    for (int t = 0; t < M; ++t) {
        float* xf = (float*)malloc(sizeof(float) * (size_t)H);
        uint16_t* y = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)H);
        for (int h = 0; h < H; ++h) xf[h] = oc_bf16_to_f32(x[oc_rank_block_offset(t, h, M, H, tp)]);
        float inv = oc_inv_rms(oc_sumsq(xf, H), H, eps);
        oc_norm_row(xf, w, gc, inv, H, y);
        for (int b = 0; b < H / 16; ++b)
            sf[(size_t)t * (H / 16) + b] =
                oc_quant_block(y + 16 * b, gs, packed + (size_t)t * (H / 2) + 8 * b, &nc, &ns);
        free(y);
        free(xf);
    }
    if (near) { near[0] = nc; near[1] = ns; }
}

/* ------------------------------------------------------------------ */
/* Stage 3: post-expert norm + weighted combine                        */
/* ------------------------------------------------------------------ */

/* expert_out [R, H] BF16; row_idx [T, k] int32 (a slot is valid iff
 * 0 <= idx < R; an invalid slot's row is never touched); wt [T, k] FP32
 * -> out [T, H] BF16.  Sum in slot order with one fused multiply-add per
 * slot, starting from +0; a token with no valid slot outputs +0. */
void oc_combine(const uint16_t* expert_out, int64_t R, int H, const int32_t* row_idx,
                const float* wt, int T, int k, const uint16_t* w, float gc, float eps,
                uint16_t* out) {
#pragma omp parallel for schedule(dynamic, 4)
    for (int t = 0; t < T; ++t) {
        float* acc = (float*)malloc(sizeof(float) * (size_t)H);
        float* xf = (float*)malloc(sizeof(float) * (size_t)H);
        uint16_t* y = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)H);
        for (int h = 0; h < H; ++h) acc[h] = 0.0f;
        for (int j = 0; j < k; ++j) {
            int64_t r = row_idx[(size_t)t * k + j];
            if (r < 0 || r >= R) continue;
            const uint16_t* row = expert_out + (size_t)r * H;
            for (int h = 0; h < H; ++h) xf[h] = oc_bf16_to_f32(row[h]);
            float inv = oc_inv_rms(oc_sumsq(xf, H), H, eps);
            oc_norm_row(xf, w, gc, inv, H, y);
            float wj = wt[(size_t)t * k + j];
            for (int h = 0; h < H; ++h) acc[h] = fmaf(wj, oc_bf16_to_f32(y[h]), acc[h]);
        }
        for (int h = 0; h < H; ++h) out[(size_t)t * H + h] = oc_bf16_rn(acc[h]);
        free(y);
        free(xf);
        free(acc);
    }
}

/* ------------------------------------------------------------------ */
/* Expert finalize fused with the tensor-parallel all-reduce           */
/* ------------------------------------------------------------------ */

/* TensorRT-LLM PR 21356, description, "Fused finalize + all-reduce" (BF16
 * TP4 with EP4, the expert finalize and the TP all-reduce in one kernel, FP32
 * accumulation) and PR 21042, MoE paragraph (the finalize all-reduces
 * partials in FP32).  Reading: rank r holds the rows of its own experts,
 * expert_out[r] [R[r], H] BF16, and row_idx[r] [T, k] maps slot j of token t
 * to a local row, or to -1 / >= R[r] where the slot's expert lives on another
 * rank (never read).  The routing weights wt [T, k] and the norm weight are
 * the same on every rank.  Rank r's partial is the combine's FP32
 * accumulator over its own valid slots in slot order from +0, not rounded;
 * the all-reduce adds the partials in rank order in FP32 (s = p_0, then
 * s = s + p_r for r = 1 .. world-1) and every rank outputs bf16(s).
 * row_idx is [world][T][k]; partial (may be NULL) receives [world][T][H]. */
void oc_finalize_allreduce(const uint16_t* const* expert_out, const int64_t* R, int world, int H,
                           const int32_t* row_idx, const float* wt, int T, int k,
                           const uint16_t* w, float gc, float eps, float* partial,
                           uint16_t* out) {
#pragma omp parallel for schedule(dynamic, 4)
    for (int t = 0; t < T; ++t) {
        float* acc = (float*)malloc(sizeof(float) * (size_t)H);
        float* s = (float*)malloc(sizeof(float) * (size_t)H);
        float* xf = (float*)malloc(sizeof(float) * (size_t)H);
        uint16_t* y = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)H);
        for (int r = 0; r < world; ++r) {
            for (int h = 0; h < H; ++h) acc[h] = 0.0f;
            const int32_t* idx = row_idx + ((size_t)r * T + t) * k;
            for (int j = 0; j < k; ++j) {
                int64_t row = idx[j];
                if (row < 0 || row >= R[r]) continue;
                const uint16_t* src = expert_out[r] + (size_t)row * H;
                for (int h = 0; h < H; ++h) xf[h] = oc_bf16_to_f32(src[h]);
                float inv = oc_inv_rms(oc_sumsq(xf, H), H, eps);
                oc_norm_row(xf, w, gc, inv, H, y);
                float wj = wt[(size_t)t * k + j];
                for (int h = 0; h < H; ++h) acc[h] = fmaf(wj, oc_bf16_to_f32(y[h]), acc[h]);
            }
            if (partial)
                memcpy(partial + ((size_t)r * T + t) * H, acc, sizeof(float) * (size_t)H);
            for (int h = 0; h < H; ++h) s[h] = (r == 0) ? acc[h] : s[h] + acc[h];
        }
        for (int h = 0; h < H; ++h) out[(size_t)t * H + h] = oc_bf16_rn(s[h]);
        free(y);
        free(xf);
        free(s);
        free(acc);
    }
}

/* ------------------------------------------------------------------ */
/* Gated residual join (+ the next branch's prenorm)                   */
/* ------------------------------------------------------------------ */

/* residual [T, H] FP32 in/out; branch [T, H] BF16; gain [H] BF16.
 *   g  = bf16(gain * branch)
 *   n  = bf16(g * inv_rms(g))                 (weightless RMSNorm)
 *   r' = alpha * r + beta * n                 (two products, one sum)
 * and, when next_w is not NULL,
 *   p  = bf16((r' * (next_gc + next_w)) * inv_rms(r'))  -> next_prenorm [T, H].
 * normed (may be NULL) receives the BF16 bits of n [T, H]: the term whose
 * BF16 step bounds the residual's tolerance. */
void oc_join(float* residual, const uint16_t* branch, const uint16_t* gain, float alpha,
             float beta, float eps, const uint16_t* next_w, float next_gc, float next_eps,
             uint16_t* next_prenorm, int T, int H, uint16_t* normed) {
#pragma omp parallel for schedule(dynamic, 4)
    for (int t = 0; t < T; ++t) {
        float* g = (float*)malloc(sizeof(float) * (size_t)H);
        float* r = residual + (size_t)t * H;
        for (int h = 0; h < H; ++h)
            g[h] = oc_bf16_to_f32(oc_bf16_rn(oc_bf16_to_f32(gain[h]) *
                                             oc_bf16_to_f32(branch[(size_t)t * H + h])));
        float inv = oc_inv_rms(oc_sumsq(g, H), H, eps);
        for (int h = 0; h < H; ++h) {
            uint16_t nb = oc_bf16_rn(g[h] * inv);
            float n = oc_bf16_to_f32(nb);
            if (normed) normed[(size_t)t * H + h] = nb;
            float a = alpha * r[h];
            float b = beta * n;
            r[h] = a + b;
        }
        if (next_w) {
            float inv2 = oc_inv_rms(oc_sumsq(r, H), H, next_eps);
            oc_norm_row(r, next_w, next_gc, inv2, H, next_prenorm + (size_t)t * H);
        }
        free(g);
    }
}

/* ------------------------------------------------------------------ */
/* Router projection                                                    */
/* ------------------------------------------------------------------ */

/* x [T, H] BF16 (the hidden states), W [E, H] FP32 (the router weight).
 *   logits[t, e] = scale * sum_h float(x[t, h]) * W[e, h]
 * evaluated in binary64: every product of a BF16 and a binary32 value is
 * exact in binary64, the sum is accumulated in binary64 in h order.  out64
 * receives the binary64 value, abs64 (if not NULL) the binary64 sum of
 * |scale * x * W| -- the scale of the rounding error an FP32 evaluation may
 * make. */
void oc_router_logits(const uint16_t* x, int T, int H, const float* W, int E, float scale,
                      double* out64, double* abs64) {
#pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t) {
        for (int e = 0; e < E; ++e) {
            double s = 0.0, a = 0.0;
            const uint16_t* xr = x + (size_t)t * H;
            const float* wr = W + (size_t)e * H;
            for (int h = 0; h < H; ++h) {
                double p = (double)oc_bf16_to_f32(xr[h]) * (double)wr[h];
                s += p;
                a += fabs(p);
            }
            out64[(size_t)t * E + e] = (double)scale * s;
            if (abs64) abs64[(size_t)t * E + e] = fabs((double)scale) * a;
        }
    }
}

/* ------------------------------------------------------------------ */
/* Dispatch: expert-grouped row layout of the routing entries           */
/* ------------------------------------------------------------------ */

/* ids [T, k] int32 holds global expert ids (-1: no entry).  This rank owns
 * experts [e0, e0 + E); entry (t, j) is valid iff e0 <= ids[t, j] < e0 + E,
 * and its local expert is ids[t, j] - e0.  Rows are grouped by local expert
 * in ascending order; within one expert the entries keep their flattened
 * order t * k + j (a stable counting sort: histogram, exclusive scan, then
 * one ordered pass).  Outputs:
 *   offsets   [E + 1]  first row of each expert; offsets[E] = R, the number
 *                      of valid entries
 *   row_idx   [T, k]   the row of entry (t, j) (the pages' en2f), -1 when the
 *                      entry is invalid
 *   row_token [T * k]  the token of row r for r < R, -1 for R <= r < T * k. */
void oc_dispatch(const int32_t* ids, int T, int k, int e0, int E, int32_t* offsets,
                 int32_t* row_idx, int32_t* row_token) {
    const int64_t n = (int64_t)T * k;
    int64_t* count = (int64_t*)calloc((size_t)E + 1, sizeof(int64_t));
    for (int64_t i = 0; i < n; ++i) {
        int64_t e = (int64_t)ids[i] - e0;
        if (e >= 0 && e < E) count[e] += 1;
    }
    int64_t run = 0;
    for (int e = 0; e < E; ++e) {
        offsets[e] = (int32_t)run;
        run += count[e];
    }
    offsets[E] = (int32_t)run;
    int64_t* next = (int64_t*)malloc(sizeof(int64_t) * ((size_t)E + 1));
    for (int e = 0; e < E; ++e) next[e] = offsets[e];
    for (int64_t r = 0; r < n; ++r) row_token[r] = -1;
    for (int64_t i = 0; i < n; ++i) {
        int64_t e = (int64_t)ids[i] - e0;
        if (e >= 0 && e < E) {
            int64_t r = next[e]++;
            row_idx[i] = (int32_t)r;
            row_token[r] = (int32_t)(i / k);
        } else {
            row_idx[i] = -1;
        }
    }
    free(next);
    free(count);
}

/* ------------------------------------------------------------------ */
/* element-wise array forms of the scalar helpers (for the pin tests)  */
/* ------------------------------------------------------------------ */
void oc_bf16_rn_n(const float* x, int64_t n, uint16_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = oc_bf16_rn(x[i]);
}
void oc_e4m3_rn_sat_n(const float* x, int64_t n, uint8_t* out) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = oc_e4m3_rn_sat(x[i]);
}
void oc_e2m1_code_n(const float* q, int64_t n, uint8_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = oc_e2m1_code(q[i]);
}
void oc_exp_n(const float* x, int64_t n, float* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = oc_exp(x[i]);
}
void oc_sigmoid_n(const float* x, int64_t n, float* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = oc_sigmoid(x[i]);
}
