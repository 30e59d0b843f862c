/*
 * oracle.c -- plain, slow fp64 CPU reference of the routed mixture-of-experts
 * expert layer (router/gate epilogue -> permute by expert -> grouped GEMM1 with
 * clamped, parameterised SwiGLU -> grouped GEMM2 -> routing-weighted combine).
 *
 * TEST INFRASTRUCTURE. Only the test suite, the smoke check and the bench's CPU
 * baseline leg load this library. The CUDA library never links it, shares no code,
 * header, table or helper with it, and must never fall back to it.
 *
 * Every function names the passage it follows:
 *   [P2] sglang PR #39920 "Fix flashinfer_trtllm silently dropping swiglu_limit",
 *        section "Modifications" (the TRT-LLM clamped SwiGLU formula) and
 *        "Motivation" (GLM clamp limit L = 10).
 *   [P3] sglang PR #36385 "Enable and fuse the Inkling MoE gate epilogue on Intel XPU",
 *        item 2 "Correctness" (exp(lp - logsumexp(lp)), lp = logsigmoid(x)),
 *        item 3 "Performance" (masked-max top-k, shared-sink columns, ties to the
 *        lower index through the ~index key, raw logit carried out of the top-k).
 *   [P4] DeepGEMM PR #445 "fix(sm90): support parameterized SwiGLU in FP8 MegaMoE",
 *        "Summary" (OAI-SwiGLU) and "Compatibility" (alpha=1, up_bias=0 reduces to
 *        gate*sigmoid(gate)*up).
 *   [P1] xorl-wheels "FlashInfer 0.6.18 SM100a+SM103a MoE-LoRA AOT", "Changes"
 *        (fused act-quant activation kernel; separate gate/up scales brought to true
 *        units before the activation; routing ids must lie in the expert range).
 *   [P5] batchgen PR #239 "sm100: Fused INT4 grouped + SiLU Triton kernel",
 *        commit notes (per-expert sorted-token dispatch; slot-specific routing-weight
 *        reduction with fp32 accumulation).
 *
 * Readings where the pages are silent (gate half first in W1, ranking on the raw
 * logit, slot order, fp32 quantisation decisions, no-clamp as L = +inf, ...) are
 * listed in the repository's design notes; each one used here is named in place.
 *
 * Build: gcc -O2 -fopenmp -shared -fPIC (no -ffast-math: float division and
 * comparisons must stay IEEE).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Mutation hooks for the oracle's own tests: a build with -DORACLE_MUTANT=n plants one
 * plausible mistake (numbered below) so the tests can show that a pin catches it. The
 * normal build (ORACLE_MUTANT = 0) plants none. */
#ifndef ORACLE_MUTANT
#define ORACLE_MUTANT 0
#endif
#define MUTANT(n) (ORACLE_MUTANT == (n))

/* ------------------------------------------------------------------------- */
/* Number formats                                                             */
/* ------------------------------------------------------------------------- */

/* bf16 is the upper half of an IEEE binary32; the conversion to double is exact. */
double oracle_bf16_to_double(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* E4M3 ("E4M3FN" of the OCP 8-bit floating point spec): 1 sign bit, 4 exponent
 * bits with bias 7, 3 mantissa bits, no infinities, S.1111.111 is NaN, largest
 * finite magnitude 448. Exponent field 0 encodes subnormals m/8 * 2^-6. */
double oracle_e4m3_decode(uint8_t b) {
    int s = b >> 7, e = (b >> 3) & 0xF, m = b & 7;
    double v;
    if (e == 0xF && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);           /* (m/8) * 2^-6   */
    else        v = ldexp((double)(8 + m), e - 10); /* (1+m/8) * 2^(e-7) */
    return s ? -v : v;
}

/* Round a float to E4M3, nearest with ties to the even code, saturating to +-448
 * (the "satfinite" behaviour). Brute force over the 127 non-negative finite codes,
 * so that the rounding rule can be read off directly. NaN maps to 0x7F. */
uint8_t oracle_e4m3_encode(float v) {
    if (isnan(v)) return 0x7F;
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double a = fabs((double)v);
    if (a >= 448.0) return sign | 0x7E;
    int best = 0;
    double best_err = a; /* distance to code 0 (value 0) */
    for (int c = 1; c <= 0x7E; ++c) {
        double err = fabs(a - oracle_e4m3_decode((uint8_t)c));
        if (err < best_err || (err == best_err && (MUTANT(10) || ((c & 1) == 0 && (best & 1) == 1)))) {
            best = c;
            best_err = err;
        }
    }
    return sign | (uint8_t)best;
}

/* 1x128 block quantisation of a row-major [rows][cols] float matrix (cols % 128 == 0)
 * to E4M3 with one fp32 scale per block: s = amax / 448 (s = 1 when amax = 0), code =
 * E4M3(v / s). Every decision is taken in fp32, the precision the kernels use, since
 * the pages fix the block shape (GLM 128x128 blockwise FP8 in [P2] "Motivation"; the
 * fused act-quant activation kernel in [P1] "Changes") but not the arithmetic.
 * Scales are written row-major [rows][cols/128]. */
void oracle_quant_1x128(const float* v, int64_t rows, int64_t cols, uint8_t* q, float* s) {
    int64_t nb = cols / 128;
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t b = 0; b < nb; ++b) {
            const float* blk = v + r * cols + b * 128;
            float amax = 0.0f;
            for (int j = 0; j < 128; ++j) {
                float a = fabsf(blk[j]);
                if (a > amax) amax = a;
            }
            float sc = (amax == 0.0f) ? 1.0f : amax / (MUTANT(11) ? 240.0f : 448.0f);
            s[r * nb + b] = sc;
            for (int j = 0; j < 128; ++j) {
                float t = blk[j] / sc;
                q[r * cols + b * 128 + j] = oracle_e4m3_encode(t);
            }
        }
    }
}

/* ------------------------------------------------------------------------- */
/* Activation                                                                 */
/* ------------------------------------------------------------------------- */

/* Clamped, parameterised SwiGLU ([P2] "Modifications"; [P4] "Summary"):
 *   g = min(gate, L), u = clamp(up, -L, L), out = g * sigmoid(alpha * g) * (u + beta).
 * The gate is clamped from above only. No clamp is L = +inf. alpha = 1, beta = 0 and
 * L = +inf is the standard silu(gate) * up ([P4] "Compatibility"). */
double oracle_swiglu(double gate, double up, double alpha, double beta, double limit) {
    double g = (gate < limit || MUTANT(3)) ? gate : limit;
    double u = up;
    if (u > limit) u = limit;
    if (u < -limit && !MUTANT(4)) u = -limit;
    double sig = 1.0 / (1.0 + exp((MUTANT(5) ? 1.0 : -1.0) * alpha * g));
    return g * sig * (u + (MUTANT(6) ? 0.0 : beta));
}

/* ------------------------------------------------------------------------- */
/* Router / gate epilogue                                                     */
/* ------------------------------------------------------------------------- */

/* log(sigmoid(x)) = min(x, 0) - log1p(exp(-|x|)); finite for every finite x. */
static double logsigmoid(double x) {
    return (x < 0.0 ? x : 0.0) - log1p(exp(-fabs(x)));
}

/* Route one gate row ([P3] items 2 and 3).
 *   row: N routed logits followed by S shared-sink logits (fp32).
 *   Selection: k passes of "largest remaining key"; equal keys go to the lower
 *   expert id (the ~index half of the sort key); a column is taken at most once
 *   (the "remaining" mask). Without a correction bias the key is the raw logit, which
 *   orders the routed columns exactly as sigmoid(logit) does. With a bias [N] the key
 *   is sigmoid(logit) + bias ([P3] item 3: ranking on sigmoid(logits) + bias, sink
 *   columns take no bias), here in fp64; the weights below still use the raw logits
 *   of the selected columns ("the value carried out of the top-k loop becomes the
 *   winner's RAW logit").
 *   Weights, score 0 (softmax renormalised over the selected k):
 *       w_j = exp(l_j - logsumexp(l_sel)).
 *   Weights, score 1 (sigmoid with logsigmoid-logsumexp renorm, sinks included):
 *       lp = logsigmoid(l), w_j = exp(lp_j - logsumexp(lp over sel and sinks)),
 *       the sink terms give the shared weights.
 *   All weights are multiplied by route_scale. Outputs in selection order. */
static double route_key(const float* row, const float* bias, int e) {
    double l = (double)row[e];
    if (!bias) return l;
    return 1.0 / (1.0 + exp(-l)) + (double)bias[e];
}

static void route_row(const float* row, const float* bias, int N, int S, int k, int score, double route_scale,
                      int32_t* ids, double* w, double* shared_w) {
    unsigned char* taken = (unsigned char*)calloc((size_t)N, 1);
    double* lsel = (double*)malloc(sizeof(double) * (size_t)(k + S));
    for (int j = 0; j < k; ++j) {
        int best = -1;
        for (int e = 0; e < N; ++e) {
            if (taken[e]) continue;
            /* strictly greater keeps the lower id on ties, since e increases */
            if (best < 0 || route_key(row, bias, e) > route_key(row, bias, best) ||
                (MUTANT(1) && route_key(row, bias, e) == route_key(row, bias, best)))
                best = e;
        }
        taken[best] = 1;
        ids[j] = best;
        lsel[j] = MUTANT(2) ? 1.0 / (1.0 + exp(-(double)row[best])) : (double)row[best];
        if (MUTANT(20) && bias) lsel[j] += (double)bias[best];
    }
    int n = k;
    if (score == 1) {
        for (int j = 0; j < k; ++j) lsel[j] = logsigmoid(lsel[j]);
        for (int s = 0; s < S; ++s) lsel[n++] = logsigmoid((double)row[N + s]);
    }
    const int n_lse = MUTANT(7) ? k : n;
    double m = lsel[0];
    for (int j = 1; j < n_lse; ++j) if (lsel[j] > m) m = lsel[j];
    double acc = 0.0;
    for (int j = 0; j < n_lse; ++j) acc += exp(lsel[j] - m);
    if (MUTANT(8) && score == 0)
        for (int e = 0; e < N; ++e) {
            int sel = 0;
            for (int j = 0; j < k; ++j) sel |= ids[j] == e;
            if (!sel) acc += exp((double)row[e] - m);
        }
    double lse = m + log(acc);
    const double rs = MUTANT(15) ? 1.0 : route_scale;
    for (int j = 0; j < k; ++j) w[j] = exp(lsel[j] - lse) * rs;
    if (score == 1)
        for (int s = 0; s < S; ++s) shared_w[s] = exp(lsel[k + s] - lse) * rs;
    free(taken);
    free(lsel);
}

/* Route T rows of logits [T][N+S] (bias [N] or NULL). Returns 0, or -1 on invalid
 * sizes or a bias with softmax scoring (the pages define the bias for the sigmoid
 * ranking only). */
int oracle_route(const float* logits, const float* bias, int T, int N, int S, int k, int score,
                 double route_scale, int32_t* ids, double* w, double* shared_w) {
    if (T < 0 || N <= 0 || k <= 0 || k > N || S < 0 || (score == 0 && S != 0)) return -1;
    if (bias && score != 1) return -1;
    for (int t = 0; t < T; ++t)
        route_row(logits + (int64_t)t * (N + S), bias, N, S, k, score, route_scale,
                  ids + (int64_t)t * k, w + (int64_t)t * k, shared_w ? shared_w + (int64_t)t * S : NULL);
    return 0;
}

/* Gate GEMV in front of the router ([P3]: the 258-column gate GEMM whose output the
 * epilogue routes, fused with it at <= 4 tokens): logits[t][c] = sum_h x[t][h] * w[c][h]
 * with bf16 inputs and fp64 sums. x [T][H], w [C][H] bf16 bits; out [T][C] fp64. */
int oracle_gate_logits(const uint16_t* x, const uint16_t* w, int T, int H, int C, double* out) {
    if (T < 0 || H <= 0 || C <= 0) return -1;
    for (int t = 0; t < T; ++t)
        for (int c = 0; c < C; ++c) {
            double acc = 0.0;
            for (int h = 0; h < H; ++h)
                acc += oracle_bf16_to_double(x[(int64_t)t * H + h]) * oracle_bf16_to_double(w[(int64_t)c * H + h]);
            out[(int64_t)t * C + c] = acc;
        }
    return 0;
}

/* ------------------------------------------------------------------------- */
/* Permutation by expert                                                      */
/* ------------------------------------------------------------------------- */

/* Per-expert sorted-token dispatch ([P5] commit notes): group g < E holds the
 * (token, slot) pairs routed to expert g, ordered by token then slot; groups
 * E .. E+n_shared-1 are the always-on shared experts and hold every token in order.
 *   offsets[g] = first row of group g (offsets[G] = A = T*k + T*n_shared),
 *   perm[r]    = source token of row r,
 *   inv[t*k+j] = row that holds slot j of token t.
 * Returns 0, or -1 if an id lies outside [0, E) ([P1] "Changes": ids outside the
 * expert range are an error, never read past the end). */
int oracle_permute(const int32_t* ids, int T, int k, int E, int n_shared,
                   int32_t* offsets, int32_t* perm, int32_t* inv) {
    int G = E + n_shared;
    int64_t* count = (int64_t*)calloc((size_t)G, sizeof(int64_t));
    for (int64_t i = 0; i < (int64_t)T * k; ++i) {
        if (ids[i] < 0 || ids[i] >= E) { free(count); return -1; }
        count[ids[i]]++;
    }
    for (int s = 0; s < n_shared; ++s) count[E + s] = T;
    offsets[0] = 0;
    for (int g = 0; g < G; ++g) offsets[g + 1] = offsets[g] + (int32_t)count[g];
    int32_t* cursor = (int32_t*)malloc(sizeof(int32_t) * (size_t)G);
    for (int g = 0; g < G; ++g) cursor[g] = offsets[g];
    for (int tt = 0; tt < T; ++tt) {
        const int t = MUTANT(9) ? T - 1 - tt : tt;
        for (int j = 0; j < k; ++j) {
            int e = ids[(int64_t)t * k + j];
            int32_t r = cursor[e]++;
            perm[r] = t;
            inv[(int64_t)t * k + j] = r;
        }
    }
    for (int s = 0; s < n_shared; ++s)
        for (int t = 0; t < T; ++t) perm[offsets[E + s] + t] = t;
    free(cursor);
    free(count);
    return 0;
}

/* ------------------------------------------------------------------------- */
/* Expert MLP and the whole layer                                             */
/* ------------------------------------------------------------------------- */

typedef struct {
    int32_t T, H, I, E, k, n_sink, n_shared;
    int32_t wdtype;               /* 0: bf16 weights; 1: E4M3 with 128x128 fp32 block scales;
                                     2: INT4 group-32 with bf16 scales (activations bf16);
                                     3: NVFP4, E2M1 with one E4M3 scale per 16 (activations bf16) */
    int32_t score;                /* 0: softmax renorm; 1: sigmoid + logsigmoid-LSE renorm */
    int32_t pad_;
    double alpha, beta, limit, route_scale;
    const float* logits;          /* [T][E + n_sink] fp32 */
    const uint16_t* x;            /* [T][H] bf16 bits */
    const void* w1;               /* [E+n_shared][2I][H]; rows [0,I) gate, [I,2I) up */
    const void* w1_scale;         /* wdtype 1: fp32 [E+n_shared][2I/128][H/128];
                                     wdtype 2: bf16 bits [E+n_shared][2I][H/32];
                                     wdtype 3: E4M3 codes [E+n_shared][2I][H/16] */
    const void* w2;               /* [E+n_shared][H][I] */
    const void* w2_scale;         /* wdtype 1: fp32 [E+n_shared][H/128][I/128];
                                     wdtype 2: bf16 bits [E+n_shared][H][I/32];
                                     wdtype 3: E4M3 codes [E+n_shared][H][I/16] */
    const float* gate_scale;      /* [E+n_shared] or NULL (1.0) */
    const float* up_scale;        /* [E+n_shared] or NULL (1.0) */
    const float* limits;          /* [E+n_shared] clamp per expert, or NULL (limit) */
    const float* router_bias;     /* [E] correction bias of the ranking, or NULL */
} oracle_layer;

/* Round to bf16, nearest even, a value exactly representable in binary32 (finite). */
static double round_bf16(double v) {
    float f = (float)v;
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    u += 0x7FFFu + ((u >> 16) & 1u);
    u &= 0xFFFF0000u;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* INT4 group-32 element (batchgen PR #239 commit notes): packed [rows][K/2] bytes, the
 * low nibble holding the even K index and the high nibble the odd one; scale [rows][K/32]
 * bf16; value (nibble - 8) * scale, taken in bf16 as the dot products consume it (the
 * product has at most 12 significant bits, so it is exact before that rounding). */
double oracle_int4_at(const uint8_t* packed, const uint16_t* scale, int64_t K, int64_t row, int64_t col) {
    uint8_t b = packed[row * (K / 2) + col / 2];
    int n = ((col & 1) != MUTANT(13)) ? (b >> 4) : (b & 0xF);
    double s = oracle_bf16_to_double(scale[row * (K / 32) + col / 32]);
    return round_bf16((double)(n - 8) * s);
}

/* E2M1 (the 4-bit element of NVFP4, named on the xorl-wheels FlashInfer 0.6.18 page,
 * "Changes": NVFP4 checkpoints): 1 sign bit, 2 exponent bits with bias 1, 1 mantissa bit,
 * no infinities or NaN. Exponent field 0 is subnormal: m * 2^-1; otherwise
 * (1 + m/2) * 2^(e - 1). */
double oracle_e2m1_decode(uint8_t code) {
    int sgn = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
    double mag = e == 0 ? 0.5 * m : (1.0 + 0.5 * m) * ldexp(1.0, e - (MUTANT(21) ? 2 : 1));
    return sgn ? -mag : mag;
}

/* NVFP4 weight element: packed [rows][K/2] bytes (low nibble = even K index, as for INT4),
 * one E4M3 scale per 16 consecutive K [rows][K/16]; value E2M1(nibble) * E4M3(scale). The
 * product has at most 6 significant bits and lies in bf16's range, so it enters the MMA
 * exactly (the rounding below is the identity). The per-expert global scales of NVFP4
 * checkpoints (gate and up halves separately) are the layer's gate_scale / up_scale. */
double oracle_fp4_at(const uint8_t* packed, const uint8_t* scale, int64_t K, int64_t row, int64_t col) {
    uint8_t b = packed[row * (K / 2) + col / 2];
    uint8_t n = (col & 1) ? (b >> 4) : (b & 0xF);
    double s = MUTANT(22) ? oracle_e4m3_decode(scale[row * (K / 16) + col / 32])
                          : oracle_e4m3_decode(scale[row * (K / 16) + col / 16]);
    return round_bf16(oracle_e2m1_decode(n) * s);
}

/* Dequantised weight element. */
static double w1_at(const oracle_layer* L, int e, int64_t row, int64_t col) {
    int64_t idx = ((int64_t)e * 2 * L->I + row) * L->H + col;
    if (L->wdtype == 0) return oracle_bf16_to_double(((const uint16_t*)L->w1)[idx]);
    if (L->wdtype == 2)
        return oracle_int4_at((const uint8_t*)L->w1, (const uint16_t*)L->w1_scale, L->H, (int64_t)e * 2 * L->I + row,
                              col);
    if (L->wdtype == 3)
        return oracle_fp4_at((const uint8_t*)L->w1, (const uint8_t*)L->w1_scale, L->H, (int64_t)e * 2 * L->I + row,
                             col);
    int64_t nbr = 2 * L->I / 128, nbc = L->H / 128;
    double s = ((const float*)L->w1_scale)[((int64_t)e * nbr + row / 128) * nbc + col / 128];
    return oracle_e4m3_decode(((const uint8_t*)L->w1)[idx]) * (MUTANT(12) ? 1.0 : s);
}

static double w2_at(const oracle_layer* L, int e, int64_t row, int64_t col) {
    int64_t idx = MUTANT(18) ? ((int64_t)e * L->I + col) * L->H + row : ((int64_t)e * L->H + row) * L->I + col;
    if (L->wdtype == 0) return oracle_bf16_to_double(((const uint16_t*)L->w2)[idx]);
    if (L->wdtype == 2)
        return oracle_int4_at((const uint8_t*)L->w2, (const uint16_t*)L->w2_scale, L->I, (int64_t)e * L->H + row, col);
    if (L->wdtype == 3)
        return oracle_fp4_at((const uint8_t*)L->w2, (const uint8_t*)L->w2_scale, L->I, (int64_t)e * L->H + row, col);
    int64_t nbr = L->H / 128, nbc = L->I / 128;
    double s = ((const float*)L->w2_scale)[((int64_t)e * nbr + row / 128) * nbc + col / 128];
    return oracle_e4m3_decode(((const uint8_t*)L->w2)[idx]) * s;
}

/* h = SwiGLU(s_g[e] * (xv . W_gate[e]), s_u[e] * (xv . W_up[e])) for one activation
 * row xv[H] (already dequantised). The per-expert scales bring both halves to their
 * own true units before the clamp and the activation ([P1] "Changes"). */
static void expert_gemm1(const oracle_layer* L, int e, const double* xv, double* h) {
    double sg = L->gate_scale ? (double)L->gate_scale[e] : 1.0;
    double su = L->up_scale ? (double)L->up_scale[e] : 1.0;
    if (MUTANT(17)) {
        const double t = sg;
        sg = su;
        su = t;
    }
    /* the clamp limit may be one fp32 value per expert (sglang PR #39920, "Speed Tests
     * and Profiling": a per-expert fp32 tensor materialised at weight-load time) */
    double lim = (L->limits && !MUTANT(16)) ? (double)L->limits[e] : L->limit;
    const int64_t gr = MUTANT(19) ? L->I : 0, ur = MUTANT(19) ? 0 : L->I;  /* gate / up row offsets */
    for (int64_t i = 0; i < L->I; ++i) {
        double gate = 0.0, up = 0.0;
        for (int64_t c = 0; c < L->H; ++c) {
            gate += xv[c] * w1_at(L, e, gr + i, c);
            up += xv[c] * w1_at(L, e, ur + i, c);
        }
        h[i] = oracle_swiglu(sg * gate, su * up, L->alpha, L->beta, lim);
    }
}

/* With FP8 weights the activations entering each GEMM are 1x128 E4M3 blocks
 * ([P1] fused act-quant kernel): quantise in fp32 and return the dequantised row. */
static void fp8_roundtrip_row(const double* v, int64_t n, double* out) {
    float* f = (float*)malloc(sizeof(float) * (size_t)n);
    uint8_t* q = (uint8_t*)malloc((size_t)n);
    float* s = (float*)malloc(sizeof(float) * (size_t)(n / 128));
    for (int64_t i = 0; i < n; ++i) f[i] = (float)v[i];
    oracle_quant_1x128(f, 1, n, q, s);
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_e4m3_decode(q[i]) * (double)s[i / 128];
    free(f); free(q); free(s);
}

/* y[H] = h . W2[e]^T. */
static void expert_gemm2(const oracle_layer* L, int e, const double* h, double* y) {
    for (int64_t o = 0; o < L->H; ++o) {
        double acc = 0.0;
        for (int64_t i = 0; i < L->I; ++i) acc += h[i] * w2_at(L, e, o, i);
        y[o] = acc;
    }
}

/* One expert's contribution for one activation row: y = W2[e](SwiGLU(W1[e] xv)). */
static void expert_mlp(const oracle_layer* L, int e, const double* xv, double* y) {
    double* h = (double*)malloc(sizeof(double) * (size_t)L->I);
    expert_gemm1(L, e, xv, h);
    if (L->wdtype == 1) fp8_roundtrip_row(h, L->I, h);
    expert_gemm2(L, e, h, y);
    free(h);
}

/* Whole layer for the listed tokens: route the token's gate row, run each selected
 * expert and each shared expert on it, and sum the routing-weighted outputs
 * ([P5] slot-specific routing-weight reduction):
 *   out[t] = sum_j w[t,j] * MLP_{id[t,j]}(x_t) + sum_s gamma[t,s] * MLP_{E+s}(x_t),
 * gamma = the sink weight of sink s when the row has sinks, else 1.
 * out is [n_tok][H] fp64. Tokens are independent, so they run in parallel. */
int oracle_moe_rows(const oracle_layer* L, const int32_t* tokens, int n_tok, double* out) {
    if (L->n_sink > 0 && L->n_shared > 0 && L->n_sink != L->n_shared) return -1;
    if (L->score == 0 && L->n_sink != 0) return -1;
    if (L->score == 0 && L->router_bias) return -1;
    int N = L->E, S = L->n_sink;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int it = 0; it < n_tok; ++it) {
        int t = tokens[it];
        if (t < 0 || t >= L->T) { bad = 1; continue; }
        int32_t* ids = (int32_t*)malloc(sizeof(int32_t) * (size_t)L->k);
        double* w = (double*)malloc(sizeof(double) * (size_t)L->k);
        double* sw = (double*)malloc(sizeof(double) * (size_t)(S > 0 ? S : 1));
        double* xv = (double*)malloc(sizeof(double) * (size_t)L->H);
        double* y = (double*)malloc(sizeof(double) * (size_t)L->H);
        double* o = out + (int64_t)it * L->H;
        route_row(L->logits + (int64_t)t * (N + S), L->router_bias, N, S, L->k, L->score, L->route_scale, ids, w,
                  sw);
        for (int64_t c = 0; c < L->H; ++c) xv[c] = oracle_bf16_to_double(L->x[(int64_t)t * L->H + c]);
        if (L->wdtype == 1) fp8_roundtrip_row(xv, L->H, xv);
        for (int64_t c = 0; c < L->H; ++c) o[c] = 0.0;
        for (int j = 0; j < L->k; ++j) {
            expert_mlp(L, ids[j], xv, y);
            for (int64_t c = 0; c < L->H; ++c) o[c] += w[j] * y[c];
        }
        for (int s = 0; s < L->n_shared; ++s) {
            double gamma = (S > 0 && !MUTANT(14)) ? sw[s] : 1.0;
            expert_mlp(L, L->E + s, xv, y);
            for (int64_t c = 0; c < L->H; ++c) o[c] += gamma * y[c];
        }
        free(ids); free(w); free(sw); free(xv); free(y);
    }
    return bad ? -1 : 0;
}

/* GEMM1 + SwiGLU alone, for rows of an already permuted activation matrix.
 *   xp: [A][H] bf16 bits (wdtype 0) or E4M3 codes (wdtype 1) with scales
 *   xs: [H/128][A] fp32 (block-major, one scale per row and 128-column block).
 *   row_expert[i]: the group (expert) of rows[i]. h: [n_rows][I] fp64.
 * The activation rows are inputs here, so they are dequantised, not re-quantised. */
int oracle_gemm1_rows(const oracle_layer* L, int64_t A, const void* xp, const float* xs,
                      const int32_t* rows, const int32_t* row_expert, int n_rows, double* h) {
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int it = 0; it < n_rows; ++it) {
        int64_t r = rows[it];
        if (r < 0 || r >= A) { bad = 1; continue; }
        double* xv = (double*)malloc(sizeof(double) * (size_t)L->H);
        for (int64_t c = 0; c < L->H; ++c) {
            if (L->wdtype != 1) xv[c] = oracle_bf16_to_double(((const uint16_t*)xp)[r * L->H + c]);
            else xv[c] = oracle_e4m3_decode(((const uint8_t*)xp)[r * L->H + c]) * (double)xs[(c / 128) * A + r];
        }
        expert_gemm1(L, row_expert[it], xv, h + (int64_t)it * L->I);
        free(xv);
    }
    return bad ? -1 : 0;
}

/* GEMM2 + weighted combine alone, for the listed tokens, from a given permuted
 * intermediate hp ([A][I] bf16 bits, or E4M3 codes with scales hs [I/128][A]):
 *   out[t] = sum_j row_w[inv[t,j]] * hp[inv[t,j]] . W2[g(inv[t,j])]^T
 *          + sum_s row_w[r_s] * hp[r_s] . W2[E+s]^T,  r_s = offsets[E+s] + t,
 * where g(r) is the group whose [offsets[g], offsets[g+1]) holds row r. */
int oracle_gemm2_rows(const oracle_layer* L, int64_t A, const void* hp, const float* hs,
                      const int32_t* offsets, const int32_t* inv, const float* row_w,
                      const int32_t* tokens, int n_tok, double* out) {
    int G = L->E + L->n_shared;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int it = 0; it < n_tok; ++it) {
        int t = tokens[it];
        double* hv = (double*)malloc(sizeof(double) * (size_t)L->I);
        double* y = (double*)malloc(sizeof(double) * (size_t)L->H);
        double* o = out + (int64_t)it * L->H;
        for (int64_t c = 0; c < L->H; ++c) o[c] = 0.0;
        int nslots = L->k + L->n_shared;
        for (int j = 0; j < nslots; ++j) {
            int64_t r = (j < L->k) ? inv[(int64_t)t * L->k + j] : (int64_t)offsets[L->E + (j - L->k)] + t;
            if (r < 0 || r >= A) { bad = 1; break; }
            int g = 0;
            while (g < G && !(offsets[g] <= r && r < offsets[g + 1])) ++g;
            if (g == G) { bad = 1; break; }
            for (int64_t i = 0; i < L->I; ++i) {
                if (L->wdtype != 1) hv[i] = oracle_bf16_to_double(((const uint16_t*)hp)[r * L->I + i]);
                else hv[i] = oracle_e4m3_decode(((const uint8_t*)hp)[r * L->I + i]) * (double)hs[(i / 128) * A + r];
            }
            expert_gemm2(L, g, hv, y);
            for (int64_t c = 0; c < L->H; ++c) o[c] += (double)row_w[r] * y[c];
        }
        free(hv); free(y);
    }
    return bad ? -1 : 0;
}

/* Number of threads the parallel loops use (reported with CPU timings). */
int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
