/*
 * nvfp4_oracle.c -- plain, slow CPU oracle for the routed-expert MoE layer with
 * 4-bit block-scaled expert weights.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or calls
 * this file: only the tests, the smoke check and the CPU-baseline leg of the
 * benchmark do.  It shares no code, header, table or constant generator with the
 * CUDA library; every table here is built from the format definitions below.
 *
 * Sources (web pages; cited by page title and section):
 *  [P1] "AxionML / MiMo-V2.6-Flash-MOPD-NVFP4" model card: introduction,
 *       "About NVFP4 quantization", "Quantization Details / Why a unit activation
 *       scale", "Reproduce the checkpoint".
 *  [P2] "ProCreations/MiMo-V2.6-Flash-RL-NVFP4": "What changed", "Verification".
 *  [P4] "MiMo-V2.6-Flash -- REAP-50": "Model Summary", "Pruning Method" section 1
 *       (grouped sigmoid top-k router and the SwiGLU expert formula).
 *  [P3] "baekpica MiMo-V2.6-Flash-RL mixed-quant GGUF": tensor precision table
 *       (routers kept in F32).
 *  [P5] "MiMo-V2.6-Flash-MOPD on one RTX PRO 6000": "Speed v6" and "What makes it
 *       fast" (the router's matmul followed by a fused top-k; the compact
 *       4.125-bit expert encoding).
 *
 * Arithmetic: floating point decisions that produce integers (quantised codes,
 * routing choices) are taken in IEEE FP32, exactly as written below; everything
 * else (GEMMs, SwiGLU, the combine) is float64.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------- */
/* Codebooks                                                                  */
/* ------------------------------------------------------------------------- */

/* E2M1 (FP4): 1 sign, 2 exponent, 1 mantissa bit; magnitudes up to 6, no NaN
 * or Inf ([P1] "About NVFP4 quantization").  Decoded by an explicit table. */
static const double E2M1_MAGNITUDE[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

double orc_e2m1_value(uint8_t code) {
    double m = E2M1_MAGNITUDE[code & 7];
    return (code & 8) ? -m : m;
}

/* E4M3 (FP8) from its definition: sign, 4 exponent bits with bias 7, 3 mantissa
 * bits; exponent field 0 is subnormal (m/8 * 2^-6); S.1111.111 is NaN; there is
 * no infinity, so the largest finite magnitude is 1.75 * 2^8 = 448.  NVFP4 uses
 * it as the per-16 block scale ([P1] "About NVFP4 quantization"). */
double orc_e4m3_value(uint8_t byte) {
    int s = byte >> 7, e = (byte >> 3) & 15, m = byte & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0)
        v = ldexp((double)m / 8.0, -6);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return s ? -v : v;
}

/* E8M0: an unsigned power-of-two exponent with bias 127; 0xFF is NaN.  The MXFP4
 * block scale over 32 codes ([P4] "Model Summary": E2M1 + E8M0 scale, block 32). */
double orc_e8m0_value(uint8_t byte) {
    if (byte == 0xFF) return NAN;
    return ldexp(1.0, (int)byte - 127);
}

/* BF16 is the upper half of an IEEE binary32. */
float orc_bf16_to_float(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* Round an FP32 value to BF16, round-to-nearest-even (finite inputs). */
uint16_t orc_float_to_bf16(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7F800000u) == 0x7F800000u) return (uint16_t)(u >> 16); /* inf / nan kept */
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7FFFu + lsb;
    return (uint16_t)(u >> 16);
}

/* Nearest E4M3 byte to x, ties to the even mantissa, saturating to +-448 instead
 * of producing NaN ("satfinite").  Plain search over the finite codes. */
uint8_t orc_e4m3_rne_satfinite(float x) {
    if (isnan(x)) return 0x7F;
    double a = fabs((double)x);
    int best = 0;
    double best_d = INFINITY;
    for (int c = 0; c <= 0x7E; ++c) { /* values increase with c over 0x00..0x7E */
        double d = fabs(orc_e4m3_value((uint8_t)c) - a);
        if (d < best_d || (d == best_d && (c & 1) == 0)) {
            best_d = d;
            best = c;
        }
    }
    return (uint8_t)(signbit(x) ? (best | 0x80) : best);
}

/* Nearest E2M1 code to x, ties to the even mantissa bit, saturating to +-6; the
 * sign is kept, so a negative value that rounds to zero gives code 0x8.  Every
 * magnitude above 6 is the saturated code 7 outright: a nearest search alone
 * loses it once |x| is so large (or infinite) that the distances to 4 and 6 are
 * equal in double, where the even-code tie rule would pick 4. */
uint8_t orc_e2m1_rne_sat(float x) {
    double a = fabs((double)x);
    int best = 0;
    double best_d = INFINITY;
    if (a > 6.0) return (uint8_t)(signbit(x) ? 0xF : 0x7);
    for (int c = 0; c < 8; ++c) {
        double d = fabs(E2M1_MAGNITUDE[c] - a);
        if (d < best_d || (d == best_d && (c & 1) == 0)) {
            best_d = d;
            best = c;
        }
    }
    return (uint8_t)(signbit(x) ? (best | 8) : best);
}

/* ------------------------------------------------------------------------- */
/* Tensor decoders (used by the transcode invariant and by the layer)         */
/* ------------------------------------------------------------------------- */

static inline uint8_t nibble(const uint8_t* packed, int64_t i) {
    /* two codes per byte; the even element is the low nibble */
    uint8_t b = packed[i >> 1];
    return (i & 1) ? (uint8_t)(b >> 4) : (uint8_t)(b & 15);
}

/* MXFP4 [N,K]: value = e2m1 * 2^(e8m0-127), one scale per 32 along K. */
void orc_decode_mxfp4(const uint8_t* codes, const uint8_t* e8m0, int64_t N, int64_t K, double* out) {
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k)
            out[n * K + k] = orc_e2m1_value(nibble(codes + n * (K / 2), k)) * orc_e8m0_value(e8m0[n * (K / 32) + k / 32]);
}

/* NVFP4 [N,K]: value = e2m1 * e4m3 * global, one E4M3 scale per 16 along K. */
void orc_decode_nvfp4(const uint8_t* codes, const uint8_t* e4m3, float global, int64_t N, int64_t K, double* out) {
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k)
            out[n * K + k] = orc_e2m1_value(nibble(codes + n * (K / 2), k)) *
                             orc_e4m3_value(e4m3[n * (K / 16) + k / 16]) * (double)global;
}

/* ------------------------------------------------------------------------- */
/* MXFP4 -> NVFP4 transcode                                                   */
/* ------------------------------------------------------------------------- */
/* [P1] introduction and [P2] "What changed": every E2M1 code is kept byte for
 * byte; each E8M0 scale over 32 codes becomes two exact E4M3 scales over the two
 * 16-code halves, times one exact power-of-two FP32 global scale per tensor;
 * nothing is re-rounded.  [P1] "Reproduce the checkpoint" reports the count of
 * scale blocks, of all-zero blocks and of out-of-E4M3-range blocks.
 *
 * Reading of the open points: the global is 2^g with g = k_max - 8 over the
 * non-zero blocks of the tensor (the largest block maps to the scale 256); a
 * tensor whose exponent spread k_max - k_min exceeds 17 has no exact transcode
 * (E4M3 holds exactly the powers 2^-9 .. 2^8) and is reported, its scales
 * zero-filled and its global 0; all-zero blocks take scale 0; a tensor with no
 * non-zero block takes g = 0.  A NaN E8M0 scale (0xFF) on a non-zero block is
 * reported the same way as a non-representable tensor, with its own status.
 *
 * Per-tensor status: 0 exact, 1 not representable, 2 NaN scale.
 * report[0] blocks, [1] all-zero blocks, [2] non-representable tensors,
 * [3] NaN-scale tensors.  Returns the worst status seen (2 > 1 > 0).        */

static int e4m3_byte_of_power_of_two(int e) {
    /* search the definition table for the byte whose value is exactly 2^e */
    double target = ldexp(1.0, e);
    for (int c = 0; c <= 0x7E; ++c)
        if (orc_e4m3_value((uint8_t)c) == target) return c;
    return -1;
}

int orc_transcode(const uint8_t* codes_in, const uint8_t* e8m0, int64_t num_tensors, int64_t N, int64_t K,
                  uint8_t* codes_out, uint8_t* e4m3_out, float* global_out, int32_t* tensor_status,
                  int64_t* report) {
    const int64_t blocks = N * K / 32;
    int worst = 0;
    int64_t r0 = 0, r1 = 0, r2 = 0, r3 = 0;
    /* tensors are independent: one per thread, counts summed at the end */
#pragma omp parallel for schedule(dynamic, 1) reduction(+ : r0, r1, r2, r3) reduction(max : worst)
    for (int64_t t = 0; t < num_tensors; ++t) {
        int64_t zero_blocks = 0;
        const uint8_t* c = codes_in + t * blocks * 16;
        const uint8_t* s = e8m0 + t * blocks;
        uint8_t* so = e4m3_out + t * blocks * 2;
        /* codes are copied byte for byte */
        memcpy(codes_out + t * blocks * 16, c, (size_t)(blocks * 16));

        int have = 0, kmin = 0, kmax = 0, nan_seen = 0;
        for (int64_t b = 0; b < blocks; ++b) {
            int zero = 1;
            for (int i = 0; i < 32; ++i)
                if (nibble(c + b * 16, i) & 7) zero = 0;
            if (zero) {
                zero_blocks++;
                continue;
            }
            if (s[b] == 0xFF) {
                nan_seen = 1;
                continue;
            }
            int k = (int)s[b] - 127;
            if (!have || k < kmin) kmin = k;
            if (!have || k > kmax) kmax = k;
            have = 1;
        }
        r0 += blocks;
        r1 += zero_blocks;

        int status = 0;
        if (nan_seen) status = 2;
        else if (have && kmax - kmin > 17) status = 1;
        if (status) {
            memset(so, 0, (size_t)(blocks * 2));
            global_out[t] = 0.0f;
            tensor_status[t] = status;
            if (status == 1) r2++;
            else r3++;
            if (status > worst) worst = status;
            continue;
        }
        int g = have ? kmax - 8 : 0;
        for (int64_t b = 0; b < blocks; ++b) {
            int zero = 1;
            for (int i = 0; i < 32; ++i)
                if (nibble(c + b * 16, i) & 7) zero = 0;
            uint8_t byte = 0;
            if (!zero) {
                int e = (int)s[b] - 127 - g; /* in [-9, 8] */
                int found = e4m3_byte_of_power_of_two(e);
                byte = (uint8_t)(found < 0 ? 0 : found);
            }
            so[2 * b] = byte;     /* first 16-code half  */
            so[2 * b + 1] = byte; /* second 16-code half */
        }
        global_out[t] = ldexpf(1.0f, g);
        tensor_status[t] = 0;
    }
    report[0] = r0, report[1] = r1, report[2] = r2, report[3] = r3;
    return worst;
}

/* ------------------------------------------------------------------------- */
/* Compact scales: 4.125 bits per weight                                      */
/* ------------------------------------------------------------------------- */
/* [P5] "Speed v6" lists a lossless compact expert encoding ("nvfp4c": 4.125
 * instead of 4.5 bits per weight, the same values).  It is possible because of
 * [P1] introduction: after the transcode, the two E4M3 scales of every 32 codes
 * are the same power of two.  The pages give no layout; the reading here:
 *
 *   per row of K codes one exponent r (int8) and per 32 codes one 4-bit field
 *   n; the block's scale is 2^(r - n) for n = 0..14 and 0 for n = 15.
 *
 * 4 bits per 32 codes = 0.125 bits per weight (plus 8 bits per row).  A row is
 * representable when, in every 32-code block, the two E4M3 scales have equal
 * value and that value is either 0 (then all 32 codes must be +-0, so the
 * block decodes to zeros whatever its scale) or an exact positive power of two
 * 2^e; then r is the largest e of the row's non-zero-scale blocks (0 if none)
 * and every such block needs r - e <= 14.
 *
 * Outputs: nib [rows, K/64] (byte j: low nibble = block 2j, high nibble =
 * block 2j+1), row_exp [rows], status [rows] (0 representable, 1 not).  A row
 * that is not representable gets nibbles 0xFF and r = 0.  Returns the number
 * of rows that are not representable.                                       */
static int power_of_two_exponent(double v, int* e) {
    /* v = 2^e exactly, v > 0 */
    if (!(v > 0.0)) return 0;
    int ex;
    double m = frexp(v, &ex); /* v = m * 2^ex, m in [0.5, 1) */
    if (m != 0.5) return 0;
    *e = ex - 1;
    return 1;
}

int64_t orc_compact_scales(const uint8_t* codes, const uint8_t* e4m3, int64_t rows, int64_t K, uint8_t* nib,
                           int8_t* row_exp, int32_t* status) {
    const int64_t nb = K / 32;
    int64_t bad = 0;
    int* e_of = (int*)malloc(sizeof(int) * (size_t)(nb > 0 ? nb : 1));
    int* zero_of = (int*)malloc(sizeof(int) * (size_t)(nb > 0 ? nb : 1));
    for (int64_t r = 0; r < rows; ++r) {
        const uint8_t* c = codes + r * (K / 2);
        const uint8_t* s = e4m3 + r * (K / 16);
        int ok = 1, have = 0, emax = 0;
        for (int64_t b = 0; b < nb; ++b) {
            double v0 = orc_e4m3_value(s[2 * b]), v1 = orc_e4m3_value(s[2 * b + 1]);
            zero_of[b] = 0;
            if (!(v0 == v1)) { /* unequal, or NaN */
                ok = 0;
                continue;
            }
            if (v0 == 0.0) {
                for (int i = 0; i < 32; ++i)
                    if (nibble(c + b * 16, i) & 7) ok = 0;
                zero_of[b] = 1;
                continue;
            }
            int e;
            if (!power_of_two_exponent(v0, &e)) {
                ok = 0;
                continue;
            }
            e_of[b] = e;
            if (!have || e > emax) emax = e;
            have = 1;
        }
        if (ok)
            for (int64_t b = 0; b < nb; ++b)
                if (!zero_of[b] && emax - e_of[b] > 14) ok = 0;
        status[r] = ok ? 0 : 1;
        if (!ok) {
            ++bad;
            row_exp[r] = 0;
            memset(nib + r * (K / 64), 0xFF, (size_t)(K / 64));
            continue;
        }
        row_exp[r] = (int8_t)(have ? emax : 0);
        for (int64_t j = 0; j < K / 64; ++j) {
            int lo = zero_of[2 * j] ? 15 : emax - e_of[2 * j];
            int hi = zero_of[2 * j + 1] ? 15 : emax - e_of[2 * j + 1];
            nib[r * (K / 64) + j] = (uint8_t)(lo | (hi << 4));
        }
    }
    free(e_of);
    free(zero_of);
    return bad;
}

/* The scale of every 32-code block of a compact row: 2^(r - n), or 0 for n = 15. */
void orc_compact_decode(const uint8_t* nib, const int8_t* row_exp, int64_t rows, int64_t K, double* scale_out) {
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t b = 0; b < K / 32; ++b) {
            const uint8_t byte = nib[r * (K / 64) + b / 2];
            const int n = (b & 1) ? (byte >> 4) : (byte & 15);
            scale_out[r * (K / 32) + b] = n == 15 ? 0.0 : ldexp(1.0, (int)row_exp[r] - n);
        }
}

/* ------------------------------------------------------------------------- */
/* Specified FP32 exp and sigmoid                                             */
/* ------------------------------------------------------------------------- */
/* The router needs sigmoid ([P4] "Pruning Method" 1: grouped sigmoid top-k).
 * The pages do not fix its rounding; to make routing choices reproducible on
 * both sides, the exp below is specified operation by operation in IEEE FP32:
 *   clamp y to [-87, 88]; n = rint(y * log2(e)); Cody-Waite reduction
 *   r = fma(-n, ln2_hi, y); r = fma(-n, ln2_lo, r) with ln2_hi = ln 2 rounded to
 *   FP32 with its 12 low mantissa bits cleared and ln2_lo = FP32(ln 2 - ln2_hi);
 *   p = degree-7 Taylor polynomial sum r^i / i! in Horner form with fmaf, the
 *   coefficients being FP32(1 / i!); result = p * 2^n (2^n built exactly).
 * sigmoid(x) = 1 / (1 + exp(-x)) for x >= 0, else e / (1 + e) with e = exp(x). */

static float orc_ln2_hi(void) {
    float f = (float)0.69314718055994530942;
    uint32_t u;
    memcpy(&u, &f, 4);
    u &= 0xFFFFF000u;
    memcpy(&f, &u, 4);
    return f;
}

float orc_exp_spec(float y) {
    const float log2e = (float)1.44269504088896340736;
    const float ln2_hi = orc_ln2_hi();
    const float ln2_lo = (float)(0.69314718055994530942 - (double)ln2_hi);
    if (y > 88.0f) y = 88.0f;
    if (y < -87.0f) y = -87.0f;
    float n = rintf(y * log2e);
    float r = fmaf(-n, ln2_hi, y);
    r = fmaf(-n, ln2_lo, r);
    float p = (float)(1.0 / 5040.0);
    p = fmaf(p, r, (float)(1.0 / 720.0));
    p = fmaf(p, r, (float)(1.0 / 120.0));
    p = fmaf(p, r, (float)(1.0 / 24.0));
    p = fmaf(p, r, (float)(1.0 / 6.0));
    p = fmaf(p, r, 0.5f);
    p = fmaf(p, r, 1.0f);
    p = fmaf(p, r, 1.0f);
    int ni = (int)n; /* in [-126, 127] */
    uint32_t bits = (uint32_t)(ni + 127) << 23;
    float two_n;
    memcpy(&two_n, &bits, 4);
    return p * two_n;
}

float orc_sigmoid_spec(float x) {
    if (x >= 0.0f) return 1.0f / (1.0f + orc_exp_spec(-x));
    float e = orc_exp_spec(x);
    return e / (1.0f + e);
}

/* ------------------------------------------------------------------------- */
/* Grouped sigmoid top-k routing                                              */
/* ------------------------------------------------------------------------- */
/* [P4] "Model Summary" and "Pruning Method" 1: n_routed_experts experts are
 * reshaped into [n_group, n_routed_experts / n_group]; topk_group groups are
 * kept, top-k experts are chosen inside them, and the weights are scaled by
 * routed_scaling_factor.  A selection-only correction bias exists
 * (e_score_correction_bias).  Readings: s = sigmoid(logit); c = s + bias (bias 0
 * when absent) decides the selection; a group's score is the sum of its two
 * largest c (its largest when a group has one expert); groups and experts are
 * taken by descending value, ties to the lower index; the output order is the
 * selection order.  A NaN biased score, and a NaN group score (biases of +inf
 * and -inf in one group), count as -inf, so the order is total and a selection
 * always exists.  With renormalize: S = sum of the chosen s in output order
 * (sequential FP32 adds), w_j = (s_j / S) * rsf; without: w_j = s_j * rsf.   */
void orc_route(const float* logits, const float* bias, int T, int E, int n_group, int topk_group, int top_k,
               float rsf, int renormalize, int32_t* topk_ids, float* topk_weights) {
    const int gsize = E / n_group;
    float* s = (float*)malloc(sizeof(float) * (size_t)E);
    float* c = (float*)malloc(sizeof(float) * (size_t)E);
    float* gscore = (float*)malloc(sizeof(float) * (size_t)n_group);
    char* gsel = (char*)malloc((size_t)n_group);
    char* taken = (char*)malloc((size_t)E);
    for (int t = 0; t < T; ++t) {
        const float* lg = logits + (int64_t)t * E;
        for (int e = 0; e < E; ++e) {
            s[e] = orc_sigmoid_spec(lg[e]);
            c[e] = s[e] + (bias ? bias[e] : 0.0f);
            if (isnan(c[e])) c[e] = -INFINITY; /* a NaN bias: the expert ranks last */
        }
        for (int g = 0; g < n_group; ++g) {
            int i1 = -1, i2 = -1;
            for (int e = g * gsize; e < (g + 1) * gsize; ++e)
                if (i1 < 0 || c[e] > c[i1]) i1 = e;
            for (int e = g * gsize; e < (g + 1) * gsize; ++e)
                if (e != i1 && (i2 < 0 || c[e] > c[i2])) i2 = e;
            gscore[g] = (i2 < 0) ? c[i1] : c[i1] + c[i2];
            if (isnan(gscore[g])) gscore[g] = -INFINITY; /* +inf and -inf biases in one group */
            gsel[g] = 0;
        }
        for (int r = 0; r < topk_group; ++r) {
            int best = -1;
            for (int g = 0; g < n_group; ++g)
                if (!gsel[g] && (best < 0 || gscore[g] > gscore[best])) best = g;
            gsel[best] = 1;
        }
        for (int e = 0; e < E; ++e) taken[e] = 0;
        for (int j = 0; j < top_k; ++j) {
            int best = -1;
            for (int e = 0; e < E; ++e)
                if (gsel[e / gsize] && !taken[e] && (best < 0 || c[e] > c[best])) best = e;
            taken[best] = 1;
            topk_ids[(int64_t)t * top_k + j] = best;
        }
        float S = 0.0f;
        for (int j = 0; j < top_k; ++j) S = S + s[topk_ids[(int64_t)t * top_k + j]];
        for (int j = 0; j < top_k; ++j) {
            float sj = s[topk_ids[(int64_t)t * top_k + j]];
            topk_weights[(int64_t)t * top_k + j] = renormalize ? (sj / S) * rsf : sj * rsf;
        }
    }
    free(s);
    free(c);
    free(gscore);
    free(gsel);
    free(taken);
}

/* ------------------------------------------------------------------------- */
/* Token permutation                                                          */
/* ------------------------------------------------------------------------- */
/* Groups the (token, slot) pairs by expert so each expert's rows are contiguous
 * ("grouped" experts: [P1] "Deploy" runs a fused grouped MoE; [P5] "Speed v4"
 * names an exact grouped kernel).  Order inside an expert: by token, then slot.
 * counts[E], offsets[E+1] (exclusive prefix sums), row_of_pair[T*k],
 * pair_of_row[T*k]; pair index = t * k + j.                                  */
/* ------------------------------------------------------------------------- */
/* Router projection [P3 precision table; P5 "What makes it fast"]: the gate   */
/* logits of each token are the dot products of its BF16 hidden row with the   */
/* FP32 router rows: logits[t][e] = sum_h x[t][h] * w[e][h], computed here in   */
/* float64 in h order and rounded once to FP32.  The routing of those logits   */
/* is orc_route.                                                               */
/* ------------------------------------------------------------------------- */
void orc_router_logits(const uint16_t* x, const float* w, int T, int H, int E, float* logits_out,
                       double* abs_sum_out) {
    for (int t = 0; t < T; ++t)
        for (int e = 0; e < E; ++e) {
            double acc = 0.0, mag = 0.0;
            for (int h = 0; h < H; ++h) {
                const double a = (double)orc_bf16_to_float(x[(int64_t)t * H + h]);
                const double b = (double)w[(int64_t)e * H + h];
                acc += a * b;
                mag += fabs(a * b);
            }
            logits_out[(int64_t)t * E + e] = (float)acc;
            if (abs_sum_out) abs_sum_out[(int64_t)t * E + e] = mag;
        }
}

void orc_permute(const int32_t* topk_ids, int T, int top_k, int E, int32_t* counts, int32_t* offsets,
                 int32_t* row_of_pair, int32_t* pair_of_row) {
    const int64_t P = (int64_t)T * top_k;
    for (int e = 0; e < E; ++e) counts[e] = 0;
    for (int64_t p = 0; p < P; ++p) counts[topk_ids[p]]++;
    offsets[0] = 0;
    for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
    int64_t row = 0;
    for (int e = 0; e < E; ++e)
        for (int64_t p = 0; p < P; ++p)
            if (topk_ids[p] == e) {
                row_of_pair[p] = (int32_t)row;
                pair_of_row[row] = (int32_t)p;
                row++;
            }
}

/* ------------------------------------------------------------------------- */
/* NVFP4 quantisation                                                         */
/* ------------------------------------------------------------------------- */
/* [P1] "About NVFP4 quantization" (E2M1 codes with an E4M3 scale per 16) and
 * "Why a unit activation scale" (one activation global scale, set to 1).
 * Per 16-element block of a row, with gs the dequantisation global scale:
 *   amax = max |x|;  sf = E4M3_rne_satfinite((amax / 6) / gs)  (IEEE FP32);
 *   if value(sf) == 0 every code is 0x0;
 *   else q_i = E2M1_rne_sat(x_i / (value(sf) * gs))            (IEEE FP32).
 * Codes are packed two per byte (even element in the low nibble); scales are
 * row-major [M, K/16].                                                       */
void orc_quantize_f32(const float* x, int64_t M, int64_t K, float gs, uint8_t* codes, uint8_t* scales) {
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t b = 0; b < K / 16; ++b) {
            const float* xb = x + m * K + b * 16;
            float amax = 0.0f;
            for (int i = 0; i < 16; ++i) {
                float a = fabsf(xb[i]);
                if (a > amax) amax = a;
            }
            float v = amax / 6.0f;
            v = v / gs;
            uint8_t sf = orc_e4m3_rne_satfinite(v);
            scales[m * (K / 16) + b] = sf;
            double sfv = orc_e4m3_value(sf);
            uint8_t q[16];
            if (sfv == 0.0) {
                for (int i = 0; i < 16; ++i) q[i] = 0;
            } else {
                float denom = (float)sfv * gs;
                for (int i = 0; i < 16; ++i) q[i] = orc_e2m1_rne_sat(xb[i] / denom);
            }
            for (int i = 0; i < 8; ++i) codes[m * (K / 2) + b * 8 + i] = (uint8_t)(q[2 * i] | (q[2 * i + 1] << 4));
        }
    }
}

void orc_quantize_bf16(const uint16_t* x, int64_t M, int64_t K, float gs, uint8_t* codes, uint8_t* scales) {
    float* xf = (float*)malloc(sizeof(float) * (size_t)K);
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t k = 0; k < K; ++k) xf[k] = orc_bf16_to_float(x[m * K + k]);
        orc_quantize_f32(xf, 1, K, gs, codes + m * (K / 2), scales + m * (K / 16));
    }
    free(xf);
}

/* ------------------------------------------------------------------------- */
/* MXFP8 quantisation                                                         */
/* ------------------------------------------------------------------------- */
/* [P5] "Speed v5.2" and "Quantization, context and quality": prefill expert
 * GEMMs take MXFP8 activations, E4M3 elements with one power-of-two scale per 32
 * values, on the block-scaled FP8 x FP4 tensor cores.  The pages do not spell
 * out the scale choice; the reading here is the OCP microscaling one: per 32
 * elements of a row, with amax = max |x|,
 *   X = floor(log2 amax) - 8   (8 = exponent of the largest E4M3 normal),
 *   clamped to [-127, 127]; amax == 0 gives X = -127;
 *   scale byte = X + 127 (E8M0);  q_i = E4M3_rne_satfinite(x_i / 2^X).
 * x_i / 2^X is exact in FP32 (a power-of-two step that stays in range), so the
 * only rounding is the E4M3 one.  codes [M, K] (one byte each), scales
 * [M, K/32].                                                                 */
void orc_quantize_mxfp8_f32(const float* x, int64_t M, int64_t K, uint8_t* codes, uint8_t* scales) {
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t b = 0; b < K / 32; ++b) {
            const float* xb = x + m * K + b * 32;
            double amax = 0.0;
            for (int i = 0; i < 32; ++i) {
                double a = fabs((double)xb[i]);
                if (a > amax) amax = a;
            }
            int X = -127;
            if (amax > 0.0) {
                int ex;
                frexp(amax, &ex); /* amax = f * 2^ex, f in [0.5, 1): floor(log2 amax) = ex - 1 */
                X = ex - 1 - 8;
                if (X < -127) X = -127;
                if (X > 127) X = 127;
            }
            scales[m * (K / 32) + b] = (uint8_t)(X + 127);
            for (int i = 0; i < 32; ++i) codes[m * K + b * 32 + i] = orc_e4m3_rne_satfinite(ldexpf(xb[i], -X));
        }
    }
}

void orc_quantize_mxfp8_bf16(const uint16_t* x, int64_t M, int64_t K, uint8_t* codes, uint8_t* scales) {
    float* xf = (float*)malloc(sizeof(float) * (size_t)K);
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t k = 0; k < K; ++k) xf[k] = orc_bf16_to_float(x[m * K + k]);
        orc_quantize_mxfp8_f32(xf, 1, K, codes + m * K, scales + m * (K / 32));
    }
    free(xf);
}

/* value of element k of an MXFP8 row */
static double mxfp8_value(const uint8_t* codes, const uint8_t* scales, int64_t k) {
    return orc_e4m3_value(codes[k]) * orc_e8m0_value(scales[k / 32]);
}

/* ------------------------------------------------------------------------- */
/* The MoE layer                                                              */
/* ------------------------------------------------------------------------- */
/* Expert MLP ([P4] "Pruning Method" 1, the expert output inside the saliency
 * formula): y_j = W_down,j( SiLU(W_gate,j h) (.) (W_up,j h) ), combined as
 * sum_j g_{t,j} y_j over the token's selected experts.
 * Modes ([P1] "Usage"/"Accuracy"): W4A16 keeps the activations in BF16 (the
 * SwiGLU output is rounded FP32 -> BF16 before the down projection); W4A4
 * quantises the activations to NVFP4 with the unit global scale ([P1] "Why a
 * unit activation scale") and requantises the SwiGLU output per 16 the same way;
 * W4A8 (mode 3, [P5] "Speed v5.2") quantises the layer input and the SwiGLU
 * output to MXFP8 (above) and keeps the NVFP4 weights.
 * Weights: NVFP4, gate/up [E, I, H] and down [E, H, I] (out x in), scales per 16
 * along the input dimension, w_global[E][3] = gate, up, down global scales.
 * Everything after decoding is float64; out is [n_tokens, H] for the listed
 * tokens (tokens are independent, so a sample of tokens is exact for them).  */

static double silu(double g) { return g / (1.0 + exp(-g)); }

static void decode_row(const uint8_t* codes, const uint8_t* sf, double global, int64_t K, double* out) {
    for (int64_t k = 0; k < K; ++k)
        out[k] = orc_e2m1_value(nibble(codes, k)) * orc_e4m3_value(sf[k / 16]) * global;
}

/* The layer input of one token as float64 values: its NVFP4 (mode 1) or MXFP8
 * (mode 3) quantisation decoded, or its BF16 values (mode 0). */
static void layer_input(int mode, const uint16_t* xt, int H, float act_global, double* xd) {
    if (mode == 3) {
        uint8_t* xq = (uint8_t*)malloc((size_t)H);
        uint8_t* xs = (uint8_t*)malloc((size_t)H / 32);
        orc_quantize_mxfp8_bf16(xt, 1, H, xq, xs);
        for (int h = 0; h < H; ++h) xd[h] = mxfp8_value(xq, xs, h);
        free(xq);
        free(xs);
    } else if (mode == 1) {
        uint8_t* xq = (uint8_t*)malloc((size_t)H / 2);
        uint8_t* xs = (uint8_t*)malloc((size_t)H / 16);
        orc_quantize_bf16(xt, 1, H, act_global, xq, xs);
        for (int h = 0; h < H; ++h)
            xd[h] = orc_e2m1_value(nibble(xq, h)) * orc_e4m3_value(xs[h / 16]) * (double)act_global;
        free(xq);
        free(xs);
    } else {
        for (int h = 0; h < H; ++h) xd[h] = (double)orc_bf16_to_float(xt[h]);
    }
}

/* The SwiGLU output a[I] of one (token, expert) pair as the down projection
 * sees it: requantised to MXFP8 (mode 3) or NVFP4 with act_global_mid (mode 1),
 * or rounded to BF16 (mode 0). */
static void down_input(int mode, int I, float act_global_mid, double* a) {
    float* a32 = (float*)malloc(sizeof(float) * (size_t)I);
    if (mode == 3) {
        uint8_t* mq = (uint8_t*)malloc((size_t)I);
        uint8_t* ms = (uint8_t*)malloc((size_t)I / 32);
        for (int i = 0; i < I; ++i) a32[i] = (float)a[i];
        orc_quantize_mxfp8_f32(a32, 1, I, mq, ms);
        for (int i = 0; i < I; ++i) a[i] = mxfp8_value(mq, ms, i);
        free(mq);
        free(ms);
    } else if (mode == 1) {
        uint8_t* aq = (uint8_t*)malloc((size_t)I / 2);
        uint8_t* as = (uint8_t*)malloc((size_t)I / 16);
        for (int i = 0; i < I; ++i) a32[i] = (float)a[i];
        orc_quantize_f32(a32, 1, I, act_global_mid, aq, as);
        for (int i = 0; i < I; ++i)
            a[i] = orc_e2m1_value(nibble(aq, i)) * orc_e4m3_value(as[i / 16]) * (double)act_global_mid;
        free(aq);
        free(as);
    } else {
        for (int i = 0; i < I; ++i) a[i] = (double)orc_bf16_to_float(orc_float_to_bf16((float)a[i]));
    }
    free(a32);
}

/* Dot products of one decoded weight row w[K] with the rows v[q * ld .. + K) of
 * n operands: out[q] = sum_k v[q][k] * w[k], each summed in k order (four
 * operands at a time, so their sums proceed side by side).  */
static void row_dots(const double* w, const double* const* v, int n, int64_t K, double* out) {
    int q = 0;
    for (; q + 4 <= n; q += 4) {
        double s0 = 0.0, s1 = 0.0, s2 = 0.0, s3 = 0.0;
        const double *v0 = v[q], *v1 = v[q + 1], *v2 = v[q + 2], *v3 = v[q + 3];
        for (int64_t k = 0; k < K; ++k) {
            s0 += v0[k] * w[k];
            s1 += v1[k] * w[k];
            s2 += v2[k] * w[k];
            s3 += v3[k] * w[k];
        }
        out[q] = s0, out[q + 1] = s1, out[q + 2] = s2, out[q + 3] = s3;
    }
    for (; q < n; ++q) {
        double s0 = 0.0;
        for (int64_t k = 0; k < K; ++k) s0 += v[q][k] * w[k];
        out[q] = s0;
    }
}

/* The layer with separate activation global scales for the layer input
 * (act_global) and the down-projection input (act_global_mid): [P1] "Why a unit
 * activation scale" compares calibrated per-layer scales, the down-projection
 * input's scale capped at 2688, and a unit scale everywhere.
 * Evaluation order: tokens are routed and their inputs quantised first; then,
 * expert by expert, every weight row is decoded once and applied to all of the
 * sample's pairs routed to that expert; each output element is the same float64
 * sum, in the same k order, as a token-by-token evaluation would form.  The
 * sample is processed in batches of at most 512 tokens (bounded memory). */
void orc_moe_layer2(int mode, const uint16_t* x, const float* logits, const float* bias, const uint8_t* gate_codes,
                    const uint8_t* gate_sf, const uint8_t* up_codes, const uint8_t* up_sf, const uint8_t* down_codes,
                    const uint8_t* down_sf, const float* w_global, float act_global, float act_global_mid, int T,
                    int H, int I, int E, int n_group, int topk_group, int top_k, float rsf, int renormalize,
                    const int32_t* tokens, int n_tokens, double* out) {
    (void)T;
    const int BATCH = 512;
    int32_t* ids = (int32_t*)malloc(sizeof(int32_t) * (size_t)BATCH * top_k);
    float* wts = (float*)malloc(sizeof(float) * (size_t)BATCH * top_k);
    double* xd = (double*)malloc(sizeof(double) * (size_t)BATCH * H);
    double* abuf = (double*)malloc(sizeof(double) * (size_t)BATCH * top_k * I);  /* per pair, SwiGLU output */
    double* ybuf = (double*)malloc(sizeof(double) * (size_t)BATCH * top_k * H);  /* per pair, expert output */
    int* pair_list = (int*)malloc(sizeof(int) * (size_t)BATCH * top_k);
    int* first = (int*)malloc(sizeof(int) * (size_t)(E + 1));
    for (int b0 = 0; b0 < n_tokens; b0 += BATCH) {
        const int nb = n_tokens - b0 < BATCH ? n_tokens - b0 : BATCH;
        const int np = nb * top_k;
#pragma omp parallel for schedule(dynamic, 1)
        for (int it = 0; it < nb; ++it) {
            const int t = tokens[b0 + it];
            orc_route(logits + (int64_t)t * E, bias, 1, E, n_group, topk_group, top_k, rsf, renormalize,
                      ids + (int64_t)it * top_k, wts + (int64_t)it * top_k);
            layer_input(mode, x + (int64_t)t * H, H, act_global, xd + (int64_t)it * H);
        }
        /* the batch's pairs (it * top_k + j) grouped by expert */
        for (int e = 0; e <= E; ++e) first[e] = 0;
        for (int q = 0; q < np; ++q) first[ids[q] + 1]++;
        for (int e = 0; e < E; ++e) first[e + 1] += first[e];
        {
            int* fill = (int*)malloc(sizeof(int) * (size_t)E);
            for (int e = 0; e < E; ++e) fill[e] = first[e];
            for (int q = 0; q < np; ++q) pair_list[fill[ids[q]]++] = q;
            free(fill);
        }
        for (int e = 0; e < E; ++e) {
            const int n = first[e + 1] - first[e];
            if (n == 0) continue;
            const int* pl = pair_list + first[e];
            const double gg = w_global[e * 3 + 0], gu = w_global[e * 3 + 1], gd = w_global[e * 3 + 2];
            const double** xv = (const double**)malloc(sizeof(double*) * (size_t)n);
            const double** av = (const double**)malloc(sizeof(double*) * (size_t)n);
            for (int q = 0; q < n; ++q) {
                xv[q] = xd + (int64_t)(pl[q] / top_k) * H;
                av[q] = abuf + (int64_t)pl[q] * I;
            }
#pragma omp parallel
            {
                double* wrow = (double*)malloc(sizeof(double) * (size_t)(H > I ? H : I));
                double* gv = (double*)malloc(sizeof(double) * (size_t)n);
                double* uv = (double*)malloc(sizeof(double) * (size_t)n);
#pragma omp for schedule(dynamic, 16)
                for (int i = 0; i < I; ++i) {
                    const int64_t r = (int64_t)e * I + i;
                    decode_row(gate_codes + r * (H / 2), gate_sf + r * (H / 16), gg, H, wrow);
                    row_dots(wrow, xv, n, H, gv);
                    decode_row(up_codes + r * (H / 2), up_sf + r * (H / 16), gu, H, wrow);
                    row_dots(wrow, xv, n, H, uv);
                    for (int q = 0; q < n; ++q) {
                        double* a = abuf + (int64_t)pl[q] * I;
                        const double g = gv[q], u = uv[q];
                        a[i] = silu(g) * u;
                    }
                }
#pragma omp for schedule(dynamic, 1)
                for (int q = 0; q < n; ++q) down_input(mode, I, act_global_mid, abuf + (int64_t)pl[q] * I);
#pragma omp for schedule(dynamic, 16)
                for (int h = 0; h < H; ++h) {
                    const int64_t r = (int64_t)e * H + h;
                    decode_row(down_codes + r * (I / 2), down_sf + r * (I / 16), gd, I, wrow);
                    row_dots(wrow, av, n, I, gv);
                    for (int q = 0; q < n; ++q) ybuf[(int64_t)pl[q] * H + h] = gv[q];
                }
                free(wrow);
                free(gv);
                free(uv);
            }
            free(xv);
            free(av);
        }
        /* out = sum_j g_{t,j} y_j, slot order */
#pragma omp parallel for schedule(static)
        for (int it = 0; it < nb; ++it) {
            double* o = out + (int64_t)(b0 + it) * H;
            for (int h = 0; h < H; ++h) o[h] = 0.0;
            for (int j = 0; j < top_k; ++j) {
                const int64_t q = (int64_t)it * top_k + j;
                for (int h = 0; h < H; ++h) {
                    const double y = ybuf[q * H + h];
                    o[h] += (double)wts[q] * y;
                }
            }
        }
    }
    free(ids);
    free(wts);
    free(xd);
    free(abuf);
    free(ybuf);
    free(pair_list);
    free(first);
}

/* The layer split at the down projection's input, for checks that hold each
 * half on its own.  orc_moe_intermediate: per sampled token its routing and,
 * per slot j, the SwiGLU output a = SiLU(g) * u (float64, as orc_moe_layer2
 * forms it) rounded to FP32 -- the values the intermediate quantisation takes
 * in.  a32 [n_tokens, top_k, I], ids / wts [n_tokens, top_k].
 * a_err (optional, same shape as a32): a bound on how far an FP32 evaluation of
 * the same a may lie from it, for a GEMM whose dot products g and u carry an
 * error of at most acc_rel * sum_h |x_h w_h| (the sum scaled like g and u):
 *   |da| <= 1.1 * eg * (|u| + eu) + |SiLU(g)| * eu + 2^-20 |a|,
 * with eg, eu those bounds, 1.1 the largest slope of SiLU and 2^-20 |a| the
 * rounding of SiLU and the product in FP32. */
static double silu_slope_bound(void) { return 1.1; }

static void row_abs_dots(const double* w, const double* const* v, int n, int64_t K, double* out) {
    for (int q = 0; q < n; ++q) {
        double s0 = 0.0;
        for (int64_t k = 0; k < K; ++k) s0 += fabs(v[q][k] * w[k]);
        out[q] = s0;
    }
}

void orc_moe_intermediate(int mode, const uint16_t* x, const float* logits, const float* bias,
                          const uint8_t* gate_codes, const uint8_t* gate_sf, const uint8_t* up_codes,
                          const uint8_t* up_sf, const float* w_global, float act_global, int H, int I, int E,
                          int n_group, int topk_group, int top_k, float rsf, int renormalize, const int32_t* tokens,
                          int n_tokens, float* a32, int32_t* ids, float* wts, double acc_rel, float* a_err) {
    double* xd = (double*)malloc(sizeof(double) * (size_t)n_tokens * H);
    const int np = n_tokens * top_k;
#pragma omp parallel for schedule(dynamic, 1)
    for (int it = 0; it < n_tokens; ++it) {
        const int t = tokens[it];
        orc_route(logits + (int64_t)t * E, bias, 1, E, n_group, topk_group, top_k, rsf, renormalize,
                  ids + (int64_t)it * top_k, wts + (int64_t)it * top_k);
        layer_input(mode, x + (int64_t)t * H, H, act_global, xd + (int64_t)it * H);
    }
    for (int e = 0; e < E; ++e) {
        int n = 0;
        for (int q = 0; q < np; ++q) n += ids[q] == e;
        if (n == 0) continue;
        int* pl = (int*)malloc(sizeof(int) * (size_t)n);
        const double** xv = (const double**)malloc(sizeof(double*) * (size_t)n);
        n = 0;
        for (int q = 0; q < np; ++q)
            if (ids[q] == e) {
                pl[n] = q;
                xv[n] = xd + (int64_t)(q / top_k) * H;
                ++n;
            }
        const double gg = w_global[e * 3 + 0], gu = w_global[e * 3 + 1];
#pragma omp parallel
        {
            double* wrow = (double*)malloc(sizeof(double) * (size_t)H);
            double* gv = (double*)malloc(sizeof(double) * (size_t)n);
            double* uv = (double*)malloc(sizeof(double) * (size_t)n);
            double* ga = (double*)malloc(sizeof(double) * (size_t)n);
            double* ua = (double*)malloc(sizeof(double) * (size_t)n);
#pragma omp for schedule(dynamic, 16)
            for (int i = 0; i < I; ++i) {
                const int64_t r = (int64_t)e * I + i;
                decode_row(gate_codes + r * (H / 2), gate_sf + r * (H / 16), gg, H, wrow);
                row_dots(wrow, xv, n, H, gv);
                if (a_err) row_abs_dots(wrow, xv, n, H, ga);
                decode_row(up_codes + r * (H / 2), up_sf + r * (H / 16), gu, H, wrow);
                row_dots(wrow, xv, n, H, uv);
                if (a_err) row_abs_dots(wrow, xv, n, H, ua);
                for (int q = 0; q < n; ++q) {
                    const double a = silu(gv[q]) * uv[q];
                    a32[(int64_t)pl[q] * I + i] = (float)a;
                    if (a_err) {
                        const double eg = acc_rel * ga[q], eu = acc_rel * ua[q];
                        a_err[(int64_t)pl[q] * I + i] = (float)(silu_slope_bound() * eg * (fabs(uv[q]) + eu) +
                                                                fabs(silu(gv[q])) * eu + ldexp(fabs(a), -20));
                    }
                }
            }
            free(wrow);
            free(gv);
            free(uv);
            free(ga);
            free(ua);
        }
        free(pl);
        free(xv);
    }
    free(xd);
}

/* orc_moe_down: the layer output from given down-projection inputs a [n_tokens,
 * top_k, I] (float64 values, already in the precision the mode uses) with the
 * tokens' routing ids / wts [n_tokens, top_k]: out[t] = sum_j w_{t,j} *
 * (W_down,e_j a_{t,j}) * global, in float64, slot order.  Fed the oracle's own
 * requantised intermediate it reproduces orc_moe_layer2 exactly. */
void orc_moe_down(const double* a, const int32_t* ids, const float* wts, const uint8_t* down_codes,
                  const uint8_t* down_sf, const float* w_global, int H, int I, int E, int top_k, int n_tokens,
                  double* out) {
    const int np = n_tokens * top_k;
    double* ybuf = (double*)malloc(sizeof(double) * (size_t)np * H);
    for (int e = 0; e < E; ++e) {
        int n = 0;
        for (int q = 0; q < np; ++q) n += ids[q] == e;
        if (n == 0) continue;
        int* pl = (int*)malloc(sizeof(int) * (size_t)n);
        const double** av = (const double**)malloc(sizeof(double*) * (size_t)n);
        n = 0;
        for (int q = 0; q < np; ++q)
            if (ids[q] == e) {
                pl[n] = q;
                av[n] = a + (int64_t)q * I;
                ++n;
            }
        const double gd = w_global[e * 3 + 2];
#pragma omp parallel
        {
            double* wrow = (double*)malloc(sizeof(double) * (size_t)I);
            double* yv = (double*)malloc(sizeof(double) * (size_t)n);
#pragma omp for schedule(dynamic, 16)
            for (int h = 0; h < H; ++h) {
                const int64_t r = (int64_t)e * H + h;
                decode_row(down_codes + r * (I / 2), down_sf + r * (I / 16), gd, I, wrow);
                row_dots(wrow, av, n, I, yv);
                for (int q = 0; q < n; ++q) ybuf[(int64_t)pl[q] * H + h] = yv[q];
            }
            free(wrow);
            free(yv);
        }
        free(pl);
        free(av);
    }
#pragma omp parallel for schedule(static)
    for (int it = 0; it < n_tokens; ++it) {
        double* o = out + (int64_t)it * H;
        for (int h = 0; h < H; ++h) o[h] = 0.0;
        for (int j = 0; j < top_k; ++j) {
            const int64_t q = (int64_t)it * top_k + j;
            for (int h = 0; h < H; ++h) o[h] += (double)wts[q] * ybuf[q * H + h];
        }
    }
    free(ybuf);
}

/* Values of MXFP8 rows: E4M3 element x 2^(E8M0 - 127) per 32, codes [M, K],
 * scales [M, K/32]. */
void orc_decode_mxfp8(const uint8_t* codes, const uint8_t* scales, int64_t M, int64_t K, double* out) {
    for (int64_t m = 0; m < M; ++m)
        for (int64_t k = 0; k < K; ++k) out[m * K + k] = mxfp8_value(codes + m * K, scales + m * (K / 32), k);
}

/* One activation global scale for both quantisations (the pages' unit scale). */
void orc_moe_layer(int mode, const uint16_t* x, const float* logits, const float* bias, const uint8_t* gate_codes,
                   const uint8_t* gate_sf, const uint8_t* up_codes, const uint8_t* up_sf, const uint8_t* down_codes,
                   const uint8_t* down_sf, const float* w_global, float act_global, int T, int H, int I, int E,
                   int n_group, int topk_group, int top_k, float rsf, int renormalize, const int32_t* tokens,
                   int n_tokens, double* out) {
    orc_moe_layer2(mode, x, logits, bias, gate_codes, gate_sf, up_codes, up_sf, down_codes, down_sf, w_global,
                   act_global, act_global, T, H, I, E, n_group, topk_group, top_k, rsf, renormalize, tokens, n_tokens,
                   out);
}

/* Routing weights/ids for a subset of tokens, for the sampled-token checks. */
int orc_num_threads(void) {
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
