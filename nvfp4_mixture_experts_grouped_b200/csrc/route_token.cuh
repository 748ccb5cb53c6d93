// route_token.cuh -- grouped sigmoid top-k routing of one token by one warp,
// shared by the routing kernel and the fused router-projection kernel.
//
// "MiMo-V2.6-Flash -- REAP-50", "Model Summary" and "Pruning Method" 1: experts
// reshaped to [n_group, E / n_group], keep topk_group groups, top-k experts
// inside them, weights scaled by routed_scaling_factor; an
// e_score_correction_bias steers the selection only.  Group score = sum of the
// group's two largest biased scores; ties go to the lower index; output order is
// selection order; weights w_j = (s_j / sum s) * rsf (renormalised) or s_j * rsf.
//
// Every floating point operation that decides an id or produces a weight is an
// explicit IEEE FP32 intrinsic (no contraction), and sigmoid uses the specified
// exp below, so ids and weights are bit-reproducible.  Files including this one
// are built with -fmad=false.
#pragma once

#include <climits>
#include <cstring>

#include "common.cuh"

namespace nvfp4moe {

struct ExpSpecConsts {
    float log2e, ln2_hi, ln2_lo;
};

// Specified FP32 exp: clamp to [-87, 88]; n = rint(y * log2e); Cody-Waite
// r = fma(-n, ln2_hi, y), r = fma(-n, ln2_lo, r); p = degree-7 Taylor series of
// e^r in Horner form with fma, coefficients FP32(1/i!); result p * 2^n with 2^n
// assembled from its exponent bits (n in [-126, 127], always a normal float).
__device__ __forceinline__ float exp_spec(float y, const ExpSpecConsts& k) {
    y = fminf(fmaxf(y, -87.0f), 88.0f);
    const float n = rintf(__fmul_rn(y, k.log2e));
    float r = __fmaf_rn(-n, k.ln2_hi, y);
    r = __fmaf_rn(-n, k.ln2_lo, r);
    float p = (float)(1.0 / 5040.0);
    p = __fmaf_rn(p, r, (float)(1.0 / 720.0));
    p = __fmaf_rn(p, r, (float)(1.0 / 120.0));
    p = __fmaf_rn(p, r, (float)(1.0 / 24.0));
    p = __fmaf_rn(p, r, (float)(1.0 / 6.0));
    p = __fmaf_rn(p, r, 0.5f);
    p = __fmaf_rn(p, r, 1.0f);
    p = __fmaf_rn(p, r, 1.0f);
    const float two_n = __uint_as_float((uint32_t)((int)n + 127) << 23);
    return __fmul_rn(p, two_n);
}

__device__ __forceinline__ float sigmoid_spec(float x, const ExpSpecConsts& k) {
    if (x >= 0.0f) return __fdiv_rn(1.0f, __fadd_rn(1.0f, exp_spec(-x, k)));
    const float e = exp_spec(x, k);
    return __fdiv_rn(e, __fadd_rn(1.0f, e));
}

// A NaN biased score (a NaN in the selection bias) or a NaN group score (an
// infinite bias of each sign in one group) counts as -infinity, so every
// comparison below is a total order and every chosen id is a real expert.
__device__ __forceinline__ float nan_to_neg_inf(float v) { return v != v ? -INFINITY : v; }

// (value desc, index asc) lexicographic "better than"
__device__ __forceinline__ bool better(float va, int ia, float vb, int ib) {
    return va > vb || (va == vb && ia < ib);
}

__device__ __forceinline__ void warp_argmax(float& v, int& i) {
#pragma unroll
    for (int o = 16; o; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, v, o);
        const int oi = __shfl_xor_sync(0xffffffffu, i, o);
        if (better(ov, oi, v, i)) {
            v = ov;
            i = oi;
        }
    }
}

constexpr int RT_WARPS = 8;
constexpr int RT_MAX_E = 1024;
constexpr int RT_MAX_NPL = RT_MAX_E / 32;

// Logits written by other CTAs of the same launch are read through L2 (COHERENT);
// logits that are inputs of the launch through the read-only path.
template <bool COHERENT>
__device__ __forceinline__ float load_logit(const float* p) {
    return COHERENT ? __ldcg(p) : __ldg(p);
}

// Any group shape.  s_c: this warp's shared scratch of RT_MAX_E + 32 floats.
template <int NPL, bool COHERENT>
__device__ __forceinline__ void route_token_general(const float* __restrict__ lg, const float* __restrict__ bias,
                                                    int64_t t, int E, int n_group, int topk_group, int top_k,
                                                    float rsf, int renorm, const ExpSpecConsts& kc,
                                                    int32_t* __restrict__ ids, float* __restrict__ wts, float* s_c) {
    // biased scores laid out group by group with one pad word per group
    const int lane = lane_id();
    const int gsz = E / n_group;
    float s[NPL], c[NPL];
    // all of the lane's logits are loaded before any sigmoid, so the loads overlap
#pragma unroll
    for (int i = 0; i < NPL; ++i) s[i] = lane + 32 * i < E ? load_logit<COHERENT>(lg + lane + 32 * i) : 0.0f;
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
        const int e = lane + 32 * i;
        if (e < E) {
            s[i] = sigmoid_spec(s[i], kc);
            c[i] = nan_to_neg_inf(__fadd_rn(s[i], bias ? __ldg(bias + e) : 0.0f));
            const int g = e / gsz;
            s_c[g * (gsz + 1) + (e - g * gsz)] = c[i];
        } else {
            s[i] = 0.0f;
            c[i] = -INFINITY;
        }
    }
    __syncwarp();
    // group scores: lane g scans group g
    float score = -INFINITY;
    if (lane < n_group) {
        const float* gp = &s_c[lane * (gsz + 1)];
        int i1 = 0;
        for (int j = 1; j < gsz; ++j)
            if (gp[j] > gp[i1]) i1 = j;
        int i2 = -1;
        for (int j = 0; j < gsz; ++j)
            if (j != i1 && (i2 < 0 || gp[j] > gp[i2])) i2 = j;
        score = nan_to_neg_inf(i2 < 0 ? gp[i1] : __fadd_rn(gp[i1], gp[i2]));
    }
    // keep topk_group groups
    uint32_t chosen = 0;
    for (int r = 0; r < topk_group; ++r) {
        float v = (lane < n_group && !((chosen >> lane) & 1u)) ? score : -INFINITY;
        int idx = (lane < n_group && !((chosen >> lane) & 1u)) ? lane : 0x7fffffff;
        warp_argmax(v, idx);
        if ((unsigned)idx < 32u) chosen |= 1u << idx;  // always: a group lane beats the -inf non-groups
    }
    // top_k experts inside the chosen groups
    uint32_t taken = 0;
    int my_id = 0;
    float my_s = 0.0f;
    for (int j = 0; j < top_k; ++j) {
        float v = -INFINITY;
        int idx = 0x7fffffff;
#pragma unroll
        for (int i = 0; i < NPL; ++i) {
            const int e = lane + 32 * i;
            if (e < E && ((chosen >> (e / gsz)) & 1u) && !((taken >> i) & 1u) && better(c[i], e, v, idx)) {
                v = c[i];
                idx = e;
            }
        }
        warp_argmax(v, idx);
        idx = min(idx, E - 1);  // never taken: the kept groups hold >= top_k candidates, none NaN
        float sv = 0.0f;
        if ((idx & 31) == lane) {
            const int i = idx >> 5;
            taken |= 1u << i;
#pragma unroll
            for (int ii = 0; ii < NPL; ++ii)
                if (ii == i) sv = s[ii];
        }
        sv = __shfl_sync(0xffffffffu, sv, idx & 31);
        if (lane == j) {
            my_id = idx;
            my_s = sv;
        }
    }
    float S = 0.0f;
    for (int j = 0; j < top_k; ++j) S = __fadd_rn(S, __shfl_sync(0xffffffffu, my_s, j));
    if (lane < top_k) {
        ids[(int64_t)t * top_k + lane] = my_id;
        wts[(int64_t)t * top_k + lane] = renorm ? __fmul_rn(__fdiv_rn(my_s, S), rsf) : __fmul_rn(my_s, rsf);
    }
}

// Fast path for the common group shapes: group size G a power of two <= 32
// (a group is an aligned run of G lanes of one register row) or a multiple of
// 32 (a group is G/32 whole register rows).  Group scores come from a
// segmented warp reduction of (largest, second largest) instead of a
// sequential scan, and every element's group bit is computed once.  Same
// arithmetic and tie rules as k_route: the group score is the FP32 sum of the
// two largest values, which does not depend on which of equal values is taken.
// s_score: this warp's shared scratch of 32 floats.
template <int NPL, bool COHERENT>
__device__ __forceinline__ void route_token_fast(const float* __restrict__ lg, const float* __restrict__ bias,
                                                 int64_t t, int E, int n_group, int topk_group, int top_k, float rsf,
                                                 int renorm, const ExpSpecConsts& kc, int32_t* __restrict__ ids,
                                                 float* __restrict__ wts, float* s_score) {
    const int lane = lane_id();
    const int gsz = E / n_group;
    float s[NPL], c[NPL];
    uint32_t gbit[NPL];
    // all of the lane's logits are loaded before any sigmoid, so the loads overlap
#pragma unroll
    for (int i = 0; i < NPL; ++i) s[i] = lane + 32 * i < E ? load_logit<COHERENT>(lg + lane + 32 * i) : 0.0f;
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
        const int e = lane + 32 * i;
        if (e < E) {
            s[i] = sigmoid_spec(s[i], kc);
            c[i] = nan_to_neg_inf(__fadd_rn(s[i], bias ? __ldg(bias + e) : 0.0f));
            gbit[i] = 1u << (e / gsz);
        } else {
            s[i] = 0.0f;
            c[i] = -INFINITY;
            gbit[i] = 0u;
        }
    }
    if (gsz <= 32) {
        // per row: segments of gsz lanes
#pragma unroll
        for (int i = 0; i < NPL; ++i) {
            float a = c[i], b = -INFINITY;
            for (int o = gsz >> 1; o; o >>= 1) {
                const float pa = __shfl_xor_sync(0xffffffffu, a, o);
                const float pb = __shfl_xor_sync(0xffffffffu, b, o);
                b = fmaxf(fminf(a, pa), fmaxf(b, pb));
                a = fmaxf(a, pa);
            }
            const int e = lane + 32 * i;
            if ((lane & (gsz - 1)) == 0 && e < E) s_score[e / gsz] = nan_to_neg_inf(__fadd_rn(a, b));
        }
    } else {
        // per group: its rows, then the whole warp
        const int rows = gsz >> 5;
        for (int g = 0; g < n_group; ++g) {
            float a = -INFINITY, b = -INFINITY;
#pragma unroll
            for (int i = 0; i < NPL; ++i)
                if (i >= g * rows && i < (g + 1) * rows) {
                    b = fmaxf(b, fminf(a, c[i]));
                    a = fmaxf(a, c[i]);
                }
#pragma unroll
            for (int o = 16; o; o >>= 1) {
                const float pa = __shfl_xor_sync(0xffffffffu, a, o);
                const float pb = __shfl_xor_sync(0xffffffffu, b, o);
                b = fmaxf(fminf(a, pa), fmaxf(b, pb));
                a = fmaxf(a, pa);
            }
            if (lane == 0) s_score[g] = nan_to_neg_inf(__fadd_rn(a, b));
        }
    }
    __syncwarp();
    const float score = lane < n_group ? s_score[lane] : -INFINITY;
    // keep topk_group groups
    uint32_t chosen = 0;
    for (int r = 0; r < topk_group; ++r) {
        float v = (lane < n_group && !((chosen >> lane) & 1u)) ? score : -INFINITY;
        int idx = (lane < n_group && !((chosen >> lane) & 1u)) ? lane : 0x7fffffff;
        warp_argmax(v, idx);
        if ((unsigned)idx < 32u) chosen |= 1u << idx;  // always: a group lane beats the -inf non-groups
    }
    // top_k experts inside the chosen groups; bit i of `cand`: register row i is
    // still a candidate (a score of -inf is one too)
    uint32_t cand = 0;
#pragma unroll
    for (int i = 0; i < NPL; ++i)
        if (chosen & gbit[i]) cand |= 1u << i;
    int my_id = 0;
    float my_s = 0.0f;
    for (int j = 0; j < top_k; ++j) {
        float v = -INFINITY;
        int idx = 0x7fffffff;
#pragma unroll
        for (int i = 0; i < NPL; ++i) {
            const int e = lane + 32 * i;
            if (((cand >> i) & 1u) && better(c[i], e, v, idx)) {
                v = c[i];
                idx = e;
            }
        }
        warp_argmax(v, idx);
        idx = min(idx, E - 1);  // never taken: the kept groups hold >= top_k candidates, none NaN
        float sv = 0.0f;
        if ((idx & 31) == lane) {
            const int hit = idx >> 5;
#pragma unroll
            for (int i = 0; i < NPL; ++i)
                if (i == hit) {
                    sv = s[i];
                    cand &= ~(1u << i);
                }
        }
        sv = __shfl_sync(0xffffffffu, sv, idx & 31);
        if (lane == j) {
            my_id = idx;
            my_s = sv;
        }
    }
    float S = 0.0f;
    for (int j = 0; j < top_k; ++j) S = __fadd_rn(S, __shfl_sync(0xffffffffu, my_s, j));
    if (lane < top_k) {
        ids[(int64_t)t * top_k + lane] = my_id;
        wts[(int64_t)t * top_k + lane] = renorm ? __fmul_rn(__fdiv_rn(my_s, S), rsf) : __fmul_rn(my_s, rsf);
    }
}

// Order-preserving int key of a float (larger float -> larger key; -0 and NaN
// do not occur here: c = sigmoid + bias with NaN taken as -inf).  KEY_NONE is
// below every key, -inf's included.
__device__ __forceinline__ int32_t okey(float v) {
    const int32_t b = __float_as_int(v);
    return b >= 0 ? b : b ^ 0x7FFFFFFF;
}
__device__ __forceinline__ float okey_value(int32_t k) { return __int_as_float(k >= 0 ? k : k ^ 0x7FFFFFFF); }
constexpr int32_t KEY_NONE = INT32_MIN;

// Group size a multiple of 32 (a group is whole register rows): the same
// selections as route_token_fast, with every warp-wide arg-max done by two
// warp reductions -- the largest key, then the lowest index holding it (the
// lower-index tie rule) -- instead of shuffle butterflies.
template <int NPL, bool COHERENT>
__device__ __forceinline__ void route_token_rows(const float* __restrict__ lg, const float* __restrict__ bias,
                                                 int64_t t, int E, int n_group, int topk_group, int top_k, float rsf,
                                                 int renorm, const ExpSpecConsts& kc, int32_t* __restrict__ ids,
                                                 float* __restrict__ wts) {
    const int lane = lane_id();
    const int rows = (E / n_group) >> 5;  // register rows per group
    float s[NPL];
    int32_t key[NPL];
    // all of the lane's logits are loaded before any sigmoid, so the loads overlap
#pragma unroll
    for (int i = 0; i < NPL; ++i) s[i] = lane + 32 * i < E ? load_logit<COHERENT>(lg + lane + 32 * i) : 0.0f;
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
        const int e = lane + 32 * i;
        if (e < E) {
            s[i] = sigmoid_spec(s[i], kc);
            key[i] = okey(nan_to_neg_inf(__fadd_rn(s[i], bias ? __ldg(bias + e) : 0.0f)));
        } else {
            s[i] = 0.0f;
            key[i] = KEY_NONE;
        }
    }
    // group scores: the group's largest and second largest c (equal values count twice)
    int32_t gkey = KEY_NONE;  // lane g: key of group g's score
    if (rows == 1) {
        // one register row per group: the rows' reductions are independent and overlap
#pragma unroll
        for (int g = 0; g < NPL; ++g)
            if (g < n_group) {
                const int32_t m1 = __reduce_max_sync(0xffffffffu, key[g]);
                const uint32_t holders = __ballot_sync(0xffffffffu, key[g] == m1);
                const int32_t m2 = __popc(holders) >= 2
                                       ? m1
                                       : __reduce_max_sync(0xffffffffu, (holders >> lane) & 1u ? KEY_NONE : key[g]);
                if (lane == g) gkey = okey(nan_to_neg_inf(__fadd_rn(okey_value(m1), okey_value(m2))));
            }
    } else {
        for (int g = 0; g < n_group; ++g) {
            int32_t a = KEY_NONE, b = KEY_NONE;  // this lane's largest, second largest in the group
#pragma unroll
            for (int i = 0; i < NPL; ++i)
                if (i >= g * rows && i < (g + 1) * rows) {
                    const int32_t k = key[i];
                    b = max(b, min(a, k));
                    a = max(a, k);
                }
            const int32_t m1 = __reduce_max_sync(0xffffffffu, a);
            const uint32_t holders = __ballot_sync(0xffffffffu, a == m1);
            int32_t m2;
            if (__popc(holders) >= 2)
                m2 = m1;
            else
                m2 = __reduce_max_sync(0xffffffffu, (holders >> lane) & 1u ? b : a);
            if (lane == g) gkey = okey(nan_to_neg_inf(__fadd_rn(okey_value(m1), okey_value(m2))));
        }
    }
    // keep topk_group groups: largest score, ties to the lower group
    uint32_t chosen = 0;
    for (int r = 0; r < topk_group; ++r) {
        const bool elig = lane < n_group && !((chosen >> lane) & 1u);
        const int32_t m = __reduce_max_sync(0xffffffffu, elig ? gkey : KEY_NONE);
        const uint32_t g = __reduce_min_sync(0xffffffffu, elig && gkey == m ? (uint32_t)lane : 32u);
        if (g < 32u) chosen |= 1u << g;  // always: every group's key is above KEY_NONE
    }
    // top_k experts inside the chosen groups: largest c, ties to the lower expert
#pragma unroll
    for (int i = 0; i < NPL; ++i)
        if (!((chosen >> (i / rows)) & 1u)) key[i] = KEY_NONE;
    int my_id = 0;
    float my_s = 0.0f;
    for (int j = 0; j < top_k; ++j) {
        int32_t lk = KEY_NONE;
        int li = 0;
#pragma unroll
        for (int i = 0; i < NPL; ++i)
            if (key[i] > lk) {  // strict: the lower row (lower expert) keeps a tie
                lk = key[i];
                li = i;
            }
        const int32_t m = __reduce_max_sync(0xffffffffu, lk);
        uint32_t idx =
            __reduce_min_sync(0xffffffffu, lk == m && lk != KEY_NONE ? (uint32_t)(lane + 32 * li) : 0x7fffffffu);
        idx = min(idx, (uint32_t)(E - 1));  // never taken: the kept groups hold >= top_k candidates
        float sv = 0.0f;
        if ((int)(idx & 31) == lane) {
            const int hit = (int)(idx >> 5);
#pragma unroll
            for (int i = 0; i < NPL; ++i)
                if (i == hit) {
                    sv = s[i];
                    key[i] = KEY_NONE;
                }
        }
        sv = __shfl_sync(0xffffffffu, sv, idx & 31);
        if (lane == j) {
            my_id = (int)idx;
            my_s = sv;
        }
    }
    float S = 0.0f;
    for (int j = 0; j < top_k; ++j) S = __fadd_rn(S, __shfl_sync(0xffffffffu, my_s, j));
    if (lane < top_k) {
        ids[t * top_k + lane] = my_id;
        wts[t * top_k + lane] = renorm ? __fmul_rn(__fdiv_rn(my_s, S), rsf) : __fmul_rn(my_s, rsf);
    }
}

// Which per-token routine a group shape takes: whole register rows per group
// (group size a multiple of 32), segments of one row (a power of two <= 32), or
// the general one.
enum RouteShape { ROUTE_GENERAL = 0, ROUTE_SEGMENTS = 1, ROUTE_ROWS = 2 };
inline RouteShape route_shape(int E, int n_group) {
    const int gsz = E / n_group;
    if (n_group > 32) return ROUTE_GENERAL;
    if (gsz % 32 == 0) return ROUTE_ROWS;
    if (gsz >= 2 && gsz <= 32 && (gsz & (gsz - 1)) == 0) return ROUTE_SEGMENTS;
    return ROUTE_GENERAL;
}

inline ExpSpecConsts exp_spec_consts() {
    // ln2_hi = ln 2 rounded to FP32 with its 12 low mantissa bits cleared;
    // ln2_lo = FP32(ln 2 - ln2_hi); log2e = FP32(log2 e).
    const double ln2 = 0.69314718055994530942;
    float hi = (float)ln2;
    uint32_t u;
    memcpy(&u, &hi, 4);
    u &= 0xFFFFF000u;
    memcpy(&hi, &u, 4);
    ExpSpecConsts k;
    k.log2e = (float)1.44269504088896340736;
    k.ln2_hi = hi;
    k.ln2_lo = (float)(ln2 - (double)hi);
    return k;
}

}  // namespace nvfp4moe
