/*
 * qmoe_oracle.c -- CPU oracle for the weight-only-quantized MoE forward.
 *
 * TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg may load this file's library. The CUDA path
 * shares no code, header, table or helper with it.
 *
 * It states the plain definition of the operator in fp64:
 *   - "QMoE" operator page (graiphic.io), input list and attributes: tensor
 *     layouts, pack_size = 8 / expert_weight_bits along K, per-column or
 *     per-K-block scales, swiglu_fusion layouts, activation attributes,
 *     k and normalize_routing_weights;
 *   - "MoE" page (clika_runtime.nn), class summary: a router picks the top-k
 *     experts per token, each runs its gated FFN, and the outputs are combined
 *     under the router weights;
 *   - "QLinearWoQ" page, class summary: each linear is
 *     y = x @ dequant(W).T + b;
 *   - "ClikaRT::nn::QMoEWoQ" page, forward(): [T, H] in, [T, H] out, and the
 *     optional shared_output folds into the routed combine.
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *   - codes are unsigned; the zero point is implicit and equals 2^(bits-1);
 *   - with 4 bits, even k sits in the low nibble of byte k/2;
 *   - selection is by raw logit, ties go to the lower expert id, the list is
 *     ordered by (logit descending, id ascending);
 *   - weights are the softmax over all E experts restricted to the selection,
 *     renormalised over the k when asked;
 *   - swiglu: g' = min(g, L), u' = clamp(u, -L, L),
 *     h = (u' + beta) * g' * sigmoid(alpha * g'); alpha == 0 means 1; a limit
 *     that is <= 0 or not finite means no clamp;
 *   - the expert output includes its fc2 bias and is then weighted;
 *   - fusion 1: gate = even rows, up = odd rows; fusion 2: gate = first I
 *     rows, up = last I rows; fusion 0 with fc3: gate = fc1, up = fc3.
 *
 * Routing options the "MoE" page names without formulas (n_group,
 * topk_group, routed_scaling_factor, apply_router_weight_on_input,
 * expert_output_scale, gelu_mode), read as:
 *   - grouped top-k: the E experts form n_group consecutive groups of
 *     E / n_group; a group's score is the largest raw logit among its
 *     experts; the topk_group groups with the highest scores are kept (ties
 *     to the lower group id) and the k experts are the top-k by logit among
 *     the kept groups' experts; n_group <= 1 means no grouping;
 *   - routed_scaling_factor multiplies the router-weighted sum of the expert
 *     outputs, not the shared output;
 *   - apply_router_weight_on_input: the router weight multiplies the
 *     expert's input row instead of its output;
 *   - expert_output_scale multiplies every expert's output (its fc2 bias
 *     included) before the router weighting;
 *   - gelu_mode "tanh" selects the tanh form of GELU (see plain_act).
 * e_score_correction_bias: see oracle_route.
 *
 * MXFP4 weights (the block format the QMoEWoQ page names for its gpt-oss
 * checkpoint), read as OCP microscaling FP4: a 4-bit code is e2m1 -- sign
 * bit 3, exponent bits 2-1, mantissa bit 0; exponent 0 is subnormal
 * (m * 0.5), otherwise 2^(e - 1) * (1 + m / 2) -- packed like int4 codes,
 * with one E8M0 scale 2^(x - 127) per 32 codes along K (the scales arrive
 * here already as fp64 values).
 *
 * Int8 block compute tier ("ClikaRT::nn::QMoEWoQ" page, class description:
 * a packed block weight on the int8 tier rounds the activation to per-block
 * int8 before the dot). The pages give no rounding rule; read as symmetric
 * absmax rounding over the weight's own K blocks, decided in fp32:
 *   s = absmax(block) / 127, q = clamp(rint(v / s), -127, 127), ties to even
 *   (s = 0 and q = 0 for an all-zero block);
 *   dot = sum_b s_w[n, b] * s[b] * sum_{k in b} (q_w[n, k] - 2^(bits-1)) * q[k].
 * The expert's input row is the activation as stored (the router-weighted row
 * rounded to the activation dtype when the weight scales the input), and
 * FC2's input is h rounded to the activation dtype.
 *
 * Every sum is a serial fp64 loop in index order, so the result does not
 * depend on the thread count.
 */
#define _GNU_SOURCE
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* O_GELU_TANH: GELU in its tanh form (gelu_mode "tanh"). */
enum { O_RELU = 0, O_GELU = 1, O_SILU = 2, O_SWIGLU = 3, O_IDENTITY = 4, O_GELU_TANH = 5 };

typedef struct oracle_cfg {
    int64_t T, H, I, E, k;
    int32_t bits;        /* 4 or 8 */
    int32_t block_size;  /* 0 = one scale per output row */
    int32_t act;         /* O_* above */
    int32_t fusion;      /* 0, 1, 2 */
    int32_t normalize;
    int32_t has_fc3;
    double alpha, beta, limit;
    int32_t n_group, topk_group;         /* grouped top-k; n_group <= 1: none */
    int32_t apply_router_weight_on_input;
    double routed_scaling_factor;
    int32_t mxfp4;                       /* codes are e2m1, no zero point */
    int32_t act_bf16;                    /* activation dtype: 1 bf16, 0 fp32 */
    int32_t int8_block;                  /* int8 block compute tier */
    int32_t pad_;
    double expert_output_scale;          /* multiplies every expert output (with its bias) */
    const double* score_bias;            /* e_score_correction_bias [E], or NULL */
} oracle_cfg;

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Code of element (n, k) of a packed [N, K/pack] stack (QMoE page, weights). */
static int32_t code_at(const uint8_t* packed, int64_t K, int bits, int64_t n, int64_t k) {
    if (bits == 8) return packed[n * K + k];
    const uint8_t byte = packed[n * (K / 2) + k / 2];
    return (k % 2 == 0) ? (byte & 0x0F) : (byte >> 4);
}

void oracle_unpack(const uint8_t* packed, int64_t N, int64_t K, int32_t bits, int32_t* q) {
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) q[n * K + k] = code_at(packed, K, bits, n, k);
}

/* Value of an e2m1 code (MXFP4). */
double oracle_e2m1(int32_t code) {
    const int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
    const double mag = e == 0 ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return s ? -mag : mag;
}

/* One dequantised row: w[k] = (q[n,k] - 2^(bits-1)) * s, s from the block of k
 * (QMoE page, fcX_scales and block_size); MXFP4: w[k] = e2m1(q[n,k]) * s. */
static void dequant_row(const uint8_t* packed, const double* scales, int64_t K, int bits,
                        int64_t bs, int32_t mxfp4, int64_t n, double* w) {
    const int32_t z = 1 << (bits - 1);
    for (int64_t k = 0; k < K; ++k) {
        const double s = bs > 0 ? scales[n * (K / bs) + k / bs] : scales[n];
        const int32_t q = code_at(packed, K, bits, n, k);
        w[k] = (mxfp4 ? oracle_e2m1(q) : (double)(q - z)) * s;
    }
}

void oracle_dequant(const uint8_t* packed, const double* scales, int64_t N, int64_t K,
                    int32_t bits, int64_t bs, int32_t mxfp4, double* w) {
    for (int64_t n = 0; n < N; ++n) dequant_row(packed, scales, K, bits, bs, mxfp4, n, w + n * K);
}

/* Routing ("MoE" page summary; QMoE page attributes k and
 * normalize_routing_weights). A NaN logit reads as -inf: it loses to every
 * number, and among equal values the lower id wins, so every selected index
 * names an expert.
 *
 * e_score_correction_bias (QMoEWoQ pages, a set_weights tensor without a
 * formula), read as: the bias moves the selection only. Experts (and groups)
 * are ranked by the key fp32(logit + bias[e]) -- one IEEE single-precision
 * addition of the stored logit and the fp32 bias, a NaN key reading as -inf
 * -- while the weights stay the softmax of the unbiased logits over all E,
 * restricted to the selection. */
void oracle_route(const double* logits, int64_t T, int64_t E, int64_t k, int32_t normalize,
                  int32_t n_group, int32_t topk_group, const double* score_bias, int32_t* idx, double* w) {
    char* taken = (char*)malloc((size_t)E);
    char* allowed = (char*)malloc((size_t)E);
    double* p = (double*)malloc(sizeof(double) * (size_t)E);
    double* lv = (double*)malloc(sizeof(double) * (size_t)E);  /* logits, NaN as -inf */
    double* l = (double*)malloc(sizeof(double) * (size_t)E);   /* selection keys */
    const int64_t G = n_group > 1 ? n_group : 1, gsize = E / G;
    char* kept = (char*)malloc((size_t)G);
    for (int64_t t = 0; t < T; ++t) {
        for (int64_t e = 0; e < E; ++e) {
            lv[e] = isnan(logits[t * E + e]) ? -INFINITY : logits[t * E + e];
            if (score_bias) {
                const float key = (float)lv[e] + (float)score_bias[e];
                l[e] = isnan(key) ? -INFINITY : (double)key;
            } else {
                l[e] = lv[e];
            }
        }
        /* groups: keep the topk_group groups of largest member logit */
        memset(kept, G == 1, (size_t)G);
        for (int64_t r = 0; G > 1 && r < topk_group; ++r) {
            int64_t bestg = -1;
            double bests = 0.0;
            for (int64_t g = 0; g < G; ++g) {
                if (kept[g]) continue;
                double sg = l[g * gsize];
                for (int64_t e = g * gsize + 1; e < (g + 1) * gsize; ++e)
                    if (l[e] > sg) sg = l[e];
                if (bestg < 0 || sg > bests) {
                    bestg = g;
                    bests = sg;
                }
            }
            kept[bestg] = 1;
        }
        for (int64_t e = 0; e < E; ++e) allowed[e] = kept[e / gsize];
        memset(taken, 0, (size_t)E);
        for (int64_t j = 0; j < k; ++j) {
            int64_t best = -1;
            for (int64_t e = 0; e < E; ++e)
                if (allowed[e] && !taken[e] && (best < 0 || l[e] > l[best])) best = e;
            taken[best] = 1;
            idx[t * k + j] = (int32_t)best;
        }
        double mx = lv[0];
        for (int64_t e = 1; e < E; ++e)
            if (lv[e] > mx) mx = lv[e];
        double z = 0.0;
        for (int64_t e = 0; e < E; ++e) z += exp(lv[e] - mx);
        for (int64_t e = 0; e < E; ++e) p[e] = exp(lv[e] - mx) / z;
        double sel = 0.0;
        for (int64_t j = 0; j < k; ++j) sel += p[idx[t * k + j]];
        for (int64_t j = 0; j < k; ++j)
            w[t * k + j] = normalize ? p[idx[t * k + j]] / sel : p[idx[t * k + j]];
    }
    free(taken);
    free(allowed);
    free(kept);
    free(p);
    free(l);
    free(lv);
}

/* Token -> expert permutation: segments in expert order, tokens ascending
 * inside a segment. offsets[E+1], perm_tok[T*k], inv[T*k]. */
void oracle_permute(const int32_t* idx, int64_t T, int64_t E, int64_t k, int32_t* offsets,
                    int32_t* perm_tok, int32_t* inv) {
    int64_t pos = 0;
    for (int64_t e = 0; e < E; ++e) {
        offsets[e] = (int32_t)pos;
        for (int64_t t = 0; t < T; ++t)
            for (int64_t j = 0; j < k; ++j)
                if (idx[t * k + j] == e) {
                    perm_tok[pos] = (int32_t)t;
                    inv[t * k + j] = (int32_t)pos;
                    ++pos;
                }
    }
    offsets[E] = (int32_t)pos;
}

static double sigmoid(double v) { return 1.0 / (1.0 + exp(-v)); }

/* activation_type of the QMoE page; GELU in its erf form, or (gelu_mode
 * "tanh", named by the MoE page's options without a formula) in the tanh
 * form of the GELU paper (Hendrycks and Gimpel):
 * 0.5 a (1 + tanh(sqrt(2/pi) (a + 0.044715 a^3))). */
static double plain_act(int act, double a) {
    switch (act) {
        case O_RELU: return a > 0.0 ? a : 0.0;
        case O_GELU: return 0.5 * a * (1.0 + erf(a / sqrt(2.0)));
        case O_GELU_TANH: return 0.5 * a * (1.0 + tanh(sqrt(2.0 / M_PI) * (a + 0.044715 * a * a * a)));
        case O_SILU: return a * sigmoid(a);
        default: return a; /* identity */
    }
}

/* Gated activation h = act(gate, up) (QMoE page: activation_type,
 * activation_alpha, activation_beta, swiglu_limit). */
double oracle_gated_act(int32_t act, double g, double u, double alpha, double beta, double limit) {
    if (act == O_SWIGLU) {
        const double a = (alpha == 0.0 || !isfinite(alpha)) ? 1.0 : alpha;
        if (isfinite(limit) && limit > 0.0) {
            g = g < limit ? g : limit;
            u = u < -limit ? -limit : (u > limit ? limit : u);
        }
        return (u + beta) * g * sigmoid(a * g);
    }
    return plain_act(act, g) * u;
}

double oracle_plain_act(int32_t act, double a) { return plain_act(act, a); }

/* Round to the activation dtype, to nearest with ties to even: fp32 by the
 * C conversion; bf16 (8 significant bits, fp32's exponent range) by scaling
 * the value so that its last kept bit is the unit and rounding to an integer
 * (exact in fp64). */
double oracle_round_act(double v, int32_t bf16) {
    if (!bf16) return (double)(float)v;
    if (v == 0.0 || !isfinite(v)) return v;
    int ex;
    frexp(v, &ex);                     /* |v| in [2^(ex-1), 2^ex) */
    int lsb = ex - 8;                  /* exponent of the last kept bit */
    if (lsb < -133) lsb = -133;        /* subnormal spacing of bf16 */
    return ldexp(nearbyint(ldexp(v, -lsb)), lsb);
}

/* Per-block int8 rounding of one activation row of K values (int8 tier, see
 * the header): q[K] codes, s[K / bs] scales. All decisions in fp32. */
void oracle_quantize_i8(const double* v, int64_t K, int64_t bs, int8_t* q, float* s) {
    for (int64_t b = 0; b < K / bs; ++b) {
        float amax = 0.0f;
        for (int64_t k = b * bs; k < (b + 1) * bs; ++k) {
            const float a = fabsf((float)v[k]);
            if (a > amax) amax = a;
        }
        const float sc = amax / 127.0f;
        s[b] = sc;
        for (int64_t k = b * bs; k < (b + 1) * bs; ++k) {
            float r = sc > 0.0f ? rintf((float)v[k] / sc) : 0.0f;
            if (r > 127.0f) r = 127.0f;
            if (r < -127.0f) r = -127.0f;
            q[k] = (int8_t)r;
        }
    }
}

/* One output of the int8 tier: sum over the K blocks of
 * s_w * s_x * (exact integer dot of centred weight codes and activation codes). */
static double dot_i8(const uint8_t* packed, const double* scales, int64_t K, int bits, int64_t bs,
                     int64_t n, const int8_t* q, const float* s) {
    const int32_t z = 1 << (bits - 1);
    double acc = 0.0;
    for (int64_t b = 0; b < K / bs; ++b) {
        int64_t d = 0;
        for (int64_t k = b * bs; k < (b + 1) * bs; ++k)
            d += (int64_t)(code_at(packed, K, bits, n, k) - z) * (int64_t)q[k];
        acc += scales[n * (K / bs) + b] * (double)s[b] * (double)d;
    }
    return acc;
}

/* y[r, n] = the int8-tier dot of activation row r with weight row n, for
 * rows x[rows, K] (no bias). */
void oracle_linear_i8(const double* x, int64_t rows, const uint8_t* packed, const double* scales,
                      int64_t N, int64_t K, int32_t bits, int64_t bs, double* y) {
    int8_t* q = (int8_t*)malloc((size_t)K);
    float* s = (float*)malloc(sizeof(float) * (size_t)(K / bs));
    for (int64_t r = 0; r < rows; ++r) {
        oracle_quantize_i8(x + r * K, K, bs, q, s);
        for (int64_t n = 0; n < N; ++n) y[r * N + n] = dot_i8(packed, scales, K, bits, bs, n, q, s);
    }
    free(q);
    free(s);
}

/*
 * The whole forward. Float inputs arrive as fp64 arrays holding the stored
 * values exactly. Outputs: y[T,H] (fp64, unrounded), topk_idx[T,k],
 * topk_w[T,k], and optionally h[T*k, I] (row t*k+j is the hidden activation of
 * token t under its j-th expert).
 */
int oracle_forward(const oracle_cfg* c, const double* x, const double* logits,
                   const uint8_t* fc1_w, const double* fc1_s, const double* fc1_b,
                   const uint8_t* fc2_w, const double* fc2_s, const double* fc2_b,
                   const uint8_t* fc3_w, const double* fc3_s, const double* fc3_b,
                   const double* shared, double* y, int32_t* topk_idx, double* topk_w,
                   double* h_out) {
    const int64_t T = c->T, H = c->H, I = c->I, E = c->E, k = c->k, R = T * k;
    const int fused = (c->fusion == 1 || c->fusion == 2);
    const int gated = fused || c->has_fc3;
    const int64_t N1 = (fused ? 2 : 1) * I;
    const int64_t bs = c->block_size;
    const int bits = c->bits;
    const int64_t pk1 = H * bits / 8, pk2 = I * bits / 8;
    const int64_t sc1 = bs > 0 ? H / bs : 1, sc2 = bs > 0 ? I / bs : 1;

    oracle_route(logits, T, E, k, c->normalize, c->n_group, c->topk_group, c->score_bias, topk_idx, topk_w);
    const double rsf = c->routed_scaling_factor;
    const double eos = c->expert_output_scale;

    double* a1 = (double*)calloc((size_t)(R * N1), sizeof(double)); /* fc1 pre-activation */
    double* a3 = c->has_fc3 ? (double*)calloc((size_t)(R * I), sizeof(double)) : NULL;
    double* h = (double*)calloc((size_t)(R * I), sizeof(double));
    double* o = (double*)calloc((size_t)(R * H), sizeof(double));
    int64_t* rows = (int64_t*)malloc(sizeof(int64_t) * (size_t)(R > 0 ? R : 1));
    if (!a1 || !h || !o || !rows || (c->has_fc3 && !a3)) return -1;

    for (int64_t e = 0; e < E; ++e) {
        int64_t m = 0; /* routed (t, j) pairs of expert e, as r = t*k + j */
        for (int64_t r = 0; r < R; ++r)
            if (topk_idx[r] == e) rows[m++] = r;
        if (m == 0) continue;

        /* FC1 (and FC3): a[r, n] = sum_k x[t, k] * W[n, k] + b[n] */
        const uint8_t* w1 = fc1_w + e * N1 * pk1;
        const double* s1 = fc1_s + e * N1 * sc1;
        /* int8 tier: the expert's input rows rounded per block to int8 */
        int8_t* q1 = NULL;
        float* qs1 = NULL;
        if (c->int8_block) {
            q1 = (int8_t*)malloc((size_t)(m * H));
            qs1 = (float*)malloc(sizeof(float) * (size_t)(m * sc1));
            double* v = (double*)malloc(sizeof(double) * (size_t)H);
            if (!q1 || !qs1 || !v) return -1;
            for (int64_t i = 0; i < m; ++i) {
                const int64_t r = rows[i], t = r / k;
                const double win = c->apply_router_weight_on_input ? topk_w[r] : 1.0;
                for (int64_t kk = 0; kk < H; ++kk) v[kk] = oracle_round_act(win * x[t * H + kk], c->act_bf16);
                oracle_quantize_i8(v, H, bs, q1 + i * H, qs1 + i * sc1);
            }
            free(v);
        }
#pragma omp parallel
        {
            double* wrow = (double*)malloc(sizeof(double) * (size_t)H);
#pragma omp for schedule(static)
            for (int64_t n = 0; n < N1; ++n) {
                dequant_row(w1, s1, H, bits, bs, c->mxfp4, n, wrow);
                for (int64_t i = 0; i < m; ++i) {
                    const int64_t r = rows[i], t = r / k;
                    /* the expert's input row: x[t], or w[r] * x[t] */
                    const double win = c->apply_router_weight_on_input ? topk_w[r] : 1.0;
                    double acc = 0.0;
                    if (c->int8_block)
                        acc = dot_i8(w1, s1, H, bits, bs, n, q1 + i * H, qs1 + i * sc1);
                    else
                        for (int64_t kk = 0; kk < H; ++kk) acc += (win * x[t * H + kk]) * wrow[kk];
                    if (fc1_b) acc += fc1_b[e * N1 + n];
                    a1[r * N1 + n] = acc;
                }
            }
            if (c->has_fc3) {
                const uint8_t* w3 = fc3_w + e * I * pk1;
                const double* s3 = fc3_s + e * I * sc1;
#pragma omp for schedule(static)
                for (int64_t n = 0; n < I; ++n) {
                    dequant_row(w3, s3, H, bits, bs, c->mxfp4, n, wrow);
                    for (int64_t i = 0; i < m; ++i) {
                        const int64_t r = rows[i], t = r / k;
                        const double win = c->apply_router_weight_on_input ? topk_w[r] : 1.0;
                        double acc = 0.0;
                        if (c->int8_block)
                            acc = dot_i8(w3, s3, H, bits, bs, n, q1 + i * H, qs1 + i * sc1);
                        else
                            for (int64_t kk = 0; kk < H; ++kk) acc += (win * x[t * H + kk]) * wrow[kk];
                        if (fc3_b) acc += fc3_b[e * I + n];
                        a3[r * I + n] = acc;
                    }
                }
            }
            free(wrow);
        }

        /* activation: split gate / up by the fusion layout */
        for (int64_t i = 0; i < m; ++i) {
            const int64_t r = rows[i];
            for (int64_t n = 0; n < I; ++n) {
                double v;
                if (!gated) {
                    v = plain_act(c->act, a1[r * N1 + n]);
                } else {
                    double g, u;
                    if (c->fusion == 1) {
                        g = a1[r * N1 + 2 * n];
                        u = a1[r * N1 + 2 * n + 1];
                    } else if (c->fusion == 2) {
                        g = a1[r * N1 + n];
                        u = a1[r * N1 + I + n];
                    } else {
                        g = a1[r * N1 + n];
                        u = a3[r * I + n];
                    }
                    v = oracle_gated_act(c->act, g, u, c->alpha, c->beta, c->limit);
                }
                h[r * I + n] = v;
            }
        }

        free(q1);
        free(qs1);

        /* FC2: o[r, m] = eos * (sum_i h[r, i] * W2[m, i] + b2[m]) */
        const uint8_t* w2 = fc2_w + e * H * pk2;
        const double* s2 = fc2_s + e * H * sc2;
        /* int8 tier: h rounded to the activation dtype, then per block to int8 */
        int8_t* q2 = NULL;
        float* qs2 = NULL;
        if (c->int8_block) {
            q2 = (int8_t*)malloc((size_t)(m * I));
            qs2 = (float*)malloc(sizeof(float) * (size_t)(m * sc2));
            double* v = (double*)malloc(sizeof(double) * (size_t)I);
            if (!q2 || !qs2 || !v) return -1;
            for (int64_t i = 0; i < m; ++i) {
                for (int64_t kk = 0; kk < I; ++kk) v[kk] = oracle_round_act(h[rows[i] * I + kk], c->act_bf16);
                oracle_quantize_i8(v, I, bs, q2 + i * I, qs2 + i * sc2);
            }
            free(v);
        }
#pragma omp parallel
        {
            double* wrow = (double*)malloc(sizeof(double) * (size_t)I);
#pragma omp for schedule(static)
            for (int64_t n = 0; n < H; ++n) {
                dequant_row(w2, s2, I, bits, bs, c->mxfp4, n, wrow);
                for (int64_t i = 0; i < m; ++i) {
                    const int64_t r = rows[i];
                    double acc = 0.0;
                    if (c->int8_block)
                        acc = dot_i8(w2, s2, I, bits, bs, n, q2 + i * I, qs2 + i * sc2);
                    else
                        for (int64_t kk = 0; kk < I; ++kk) acc += h[r * I + kk] * wrow[kk];
                    if (fc2_b) acc += fc2_b[e * H + n];
                    o[r * H + n] = eos * acc;
                }
            }
            free(wrow);
        }
        free(q2);
        free(qs2);
    }

    /* combine: y[t] = rsf * sum_j w[t, j] * o[t*k + j] + shared[t], j in list
     * order; the weight is 1 here when it already scaled the expert's input */
    for (int64_t t = 0; t < T; ++t)
        for (int64_t n = 0; n < H; ++n) {
            double acc = 0.0;
            for (int64_t j = 0; j < k; ++j) {
                const double wj = c->apply_router_weight_on_input ? 1.0 : topk_w[t * k + j];
                acc += wj * o[(t * k + j) * H + n];
            }
            acc *= rsf;
            if (shared) acc += shared[t * H + n];
            y[t * H + n] = acc;
        }

    if (h_out) memcpy(h_out, h, sizeof(double) * (size_t)(R * I));
    free(a1);
    free(a3);
    free(h);
    free(o);
    free(rows);
    return 0;
}
