/*
 * oracle.c -- plain, slow CPU oracle for the Llama-4 style top-1 sigmoid-gated
 * mixture-of-experts feed-forward layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or calls
 * this file; only the test suite, the smoke check and the CPU-baseline leg of
 * the benchmark do.  It shares no code, header, table or helper with the CUDA
 * library.
 *
 * What it computes, token by token, in fp64 (every input widened exactly):
 *
 *   superteams.ai "Llama 4" glossary, section "Mixture of Experts: Why Total
 *   and Active Parameters Diverge" (the routing sketch): the router produces
 *   one score per expert, the single highest-scoring expert is selected, and
 *   the layer returns the shared expert's output plus the selected expert's
 *   output; the remaining experts do no work for that token.
 *   KerasFormers "Llama 4" page, "What is unusual about the block": the
 *   routed expert is applied to the input after it has been multiplied by a
 *   sigmoid gate, so the routed expert sees sigmoid(winning logit) * x while
 *   the shared expert sees the ungated x.
 *   llm-architectures-explained "Llama 4 Maverick", field table rows
 *   ffns.moe.gated / ffns.moe.d_expert / ffns.moe.d_shared: experts and the
 *   shared expert are gated MLPs (SwiGLU) of width 8192.
 *
 * With E = 0 the layer is the shared SwiGLU alone: the dense feed-forward of
 * the layers without experts (llm-architectures-explained "Llama 4
 * Maverick", field table: d_ffn 16384 for the dense layers).
 *
 * Readings where the pages are silent (each listed in the design notes):
 *   - logits are formed in fp64 and rounded once to fp32; the argmax runs on
 *     those fp32 values with a strict ">" so the lowest index wins a tie and a
 *     NaN never wins;
 *   - gate g = 1 / (1 + exp(-l*)) evaluated in fp64 on the fp32 logit;
 *   - the fused gate/up weight is [d, 2F] with gate columns [0, F) and up
 *     columns [F, 2F); the down weight is [F, d]; the router weight is [d, E];
 *   - silu(z) = z / (1 + exp(-z));
 *   - an optional fp32 router bias b[E] is added to the logits;
 *   - FP8 weights are OCP E4M3 (bias 7, no infinities, S.1111.111 = NaN,
 *     max 448) with one fp32 scale per output column; w = e4m3(q) * scale.
 *   - int8 weights (KerasFormers "Llama 4" page, "Lower memory": weight-only
 *     int8 loading) are two's-complement integers with one fp32 scale per
 *     output column, symmetric (no zero point); w = q * scale.
 *   - FP8 activations, an opt-in mode (superteams.ai glossary, "Running
 *     Llama 4 Yourself": Maverick served with FP8 quantisation): each
 *     contraction input row -- a token's x, and a token's hidden row of each
 *     expert it runs -- is quantised to E4M3 with its own scale:
 *     s = fp32(max|v| / 448) (at least 2^-126; 1 for an all-zero row), code =
 *     e4m3_rne_satfinite(fp32(v * fp32(1 / s))), value = code * s.  A hidden row is
 *     held in the layer's activation type before it is quantised: each
 *     value is rounded to fp32 and then, in layers with bf16 activations, to
 *     bf16 (round to nearest even).  The gate still scales the routed
 *     expert's (dequantised) input.
 *   - int4 weights (superteams.ai glossary, "The Llama 4 Herd": Scout fits on
 *     one H100 quantized to int4; aibase model card, "Quantization": on-the-fly
 *     int4) are two's-complement 4-bit integers packed two per byte along the
 *     output (column) dimension, the even column in the low nibble, with one
 *     fp32 scale per output column; w = q * scale.
 *
 * Parity pins (tests/test_oracle_pins.py): E = 1 with the gate forced to 1
 * reduces to two dense SwiGLU FFNs evaluated by a library matmul; a constant
 * logit gives the sigmoid closed form and pins input (not output) gating;
 * ties resolve to the lowest index like numpy.argmax; the permutation equals
 * numpy's stable argsort; zero input gives exactly zero output; the E4M3 and
 * bf16 decoders agree with torch's for every code; E4M3 and int8 weights
 * equal the dense layer on dequantised weights, int8 codes with unit scales
 * the bf16 layer on the same integers, int4 codes the int8 layer on the same
 * integers; top-k selection equals a lexsort of the logits, and with k = E
 * the layer equals a library evaluation over every expert; without experts
 * the layer is one library SwiGLU; the hidden-rounding output equals a
 * library evaluation that rounds the hidden values with torch's own
 * conversions; one expert's rows (oracle_expert_rows) equal a library
 * SwiGLU of the gated rows.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORACLE_F32 = 0, ORACLE_BF16 = 1, ORACLE_E4M3 = 2, ORACLE_INT8 = 3, ORACLE_INT4 = 4 };

/* bf16 is the upper half of an IEEE binary32; widening is exact. */
double oracle_bf16_to_double(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* OCP 8-bit floating point, E4M3 variant: 1 sign, 4 exponent (bias 7),
 * 3 mantissa bits; exponent field 0 is subnormal; S.1111.111 is NaN; there
 * is no infinity. */
double oracle_e4m3_to_double(uint8_t q) {
    int sign = (q >> 7) & 1;
    int e = (q >> 3) & 0xF;
    int m = q & 0x7;
    double v;
    if (e == 0xF && m == 0x7) return NAN;
    if (e == 0)
        v = ldexp((double)m / 8.0, 1 - 7);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -v : v;
}

/* OCP E4M3 encoding of a float: round to nearest even, values beyond the
 * largest finite one (448) saturate to +-448, NaN gives 0x7F.  Normal
 * numbers are 1.f * 2^E with E in [-6, 8] and 3 fraction bits (exponent
 * field E + 7); below 2^-6 the codes are multiples of 2^-9 (exponent field 0).
 * Every step below is exact in double except the one rint (round half to
 * even, the default rounding mode). */
uint8_t oracle_e4m3_encode(float v) {
    if (v != v) return 0x7F;
    const uint8_t sign = signbit(v) ? 0x80 : 0x00;
    const double a = fabs((double)v);
    if (a >= 448.0) return sign | 0x7E;
    if (a < ldexp(1.0, -6)) /* 0..8 multiples of 2^-9; 8 is 2^-6, code 0x08 */
        return sign | (uint8_t)rint(a * 512.0);
    int e2;
    frexp(a, &e2); /* a = m * 2^e2, m in [0.5, 1) */
    int E = e2 - 1;
    double f = rint((a / ldexp(1.0, E) - 1.0) * 8.0);
    if (f == 8.0) {
        f = 0.0;
        E += 1;
    }
    return sign | (uint8_t)(((E + 7) << 3) | (int)f);
}

/* FP8 activation mode, one row of fp32 values v[0..n): its scale
 * s = fp32(max|v| / 448), at least 2^-126 (the smallest normal fp32, so that
 * 1 / s is finite), and 1 for an all-zero row, is returned; codes[j] =
 * e4m3_rne_satfinite(fp32(v[j] * fp32(1 / s))) (see the header). */
float oracle_e4m3_row(int n, const float *v, uint8_t *codes) {
    float amax = 0.0f;
    for (int j = 0; j < n; ++j) {
        float a = fabsf(v[j]);
        if (a > amax) amax = a;
    }
    float s = amax / 448.0f;
    if (s < 0x1p-126f) s = 0x1p-126f;
    if (amax == 0.0f) s = 1.0f;
    const float rcp = 1.0f / s;
    for (int j = 0; j < n; ++j) codes[j] = oracle_e4m3_encode(v[j] * rcp);
    return s;
}

/* FP8 activation mode: v[0..n) (fp64 values, first rounded to fp32) replaced
 * by their E4M3 quantisation with one scale for the row: code * s. */
static void quantise_row_e4m3(int n, double *v) {
    float *f = (float *)calloc((size_t)(n > 0 ? n : 1), sizeof(float));
    uint8_t *c = (uint8_t *)malloc((size_t)(n > 0 ? n : 1));
    for (int j = 0; j < n; ++j) f[j] = (float)v[j];
    const float s = oracle_e4m3_row(n, f, c);
    for (int j = 0; j < n; ++j) v[j] = oracle_e4m3_to_double(c[j]) * (double)s;
    free(f);
    free(c);
}

static double load_elem(const void *p, int dtype, size_t i) {
    switch (dtype) {
    case ORACLE_F32: return (double)((const float *)p)[i];
    case ORACLE_BF16: return oracle_bf16_to_double(((const uint16_t *)p)[i]);
    case ORACLE_E4M3: return oracle_e4m3_to_double(((const uint8_t *)p)[i]);
    case ORACLE_INT8: return (double)((const int8_t *)p)[i];
    case ORACLE_INT4: { /* element i is nibble i: byte i / 2, low nibble first */
        const uint8_t b = ((const uint8_t *)p)[i >> 1];
        const int q = (i & 1) ? (b >> 4) : (b & 0xF);
        return (double)(q >= 8 ? q - 16 : q);
    }
    default: return NAN;
    }
}

/* A weight element of a [rows, cols] row-major matrix (int4: cols even,
 * packed along the row, so element (row, col) is nibble row * cols + col);
 * for E4M3, int8 and int4 the per-output-column scale is applied
 * (dequantisation). */
static double load_weight(const void *W, int dtype, const float *col_scale,
                          size_t row, size_t cols, size_t col) {
    double w = load_elem(W, dtype, row * cols + col);
    if (dtype == ORACLE_E4M3 || dtype == ORACLE_INT8 || dtype == ORACLE_INT4) w *= (double)col_scale[col];
    return w;
}

/* Hidden-row rounding of the reading where the GPU keeps the hidden rows in
 * a 16-bit type: the fp64 value is first rounded to fp32 (the GPU forms h in
 * fp32), then to bf16 or IEEE binary16 by round-to-nearest-even. */
enum { HROUND_NONE = 0, HROUND_BF16 = 1, HROUND_F16 = 2 };

/* fp32 -> bf16 (8-bit significand), round to nearest even: add half of the
 * dropped 16 bits' weight plus the kept lsb, then truncate (the carry moves
 * into the exponent when the significand overflows, as it should). */
static double round_bf16(double v) {
    float f = (float)v;
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7F800000u) == 0x7F800000u) return (double)f; /* inf / NaN */
    u += 0x7FFFu + ((u >> 16) & 1u);
    u &= 0xFFFF0000u;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* fp32 -> binary16 (11-bit significand, exponents -14..15, subnormals in
 * steps of 2^-24, largest finite 65504), round to nearest even; values that
 * round beyond 65504 become infinite. */
static double round_f16(double v) {
    double a = fabs((double)(float)v), q;
    if (a != a || a == INFINITY) return (double)(float)v;
    if (a < ldexp(1.0, -14)) {
        q = ldexp(rint(ldexp(a, 24)), -24);           /* subnormal grid */
    } else {
        int e2;
        frexp(a, &e2);                                /* a in [2^(e2-1), 2^e2) */
        q = ldexp(rint(ldexp(a, 11 - e2)), e2 - 11);  /* 11 significant bits */
        if (q > 65504.0) q = INFINITY;
    }
    return v < 0 ? -q : q;
}

static double round_hidden(double v, int h_round) {
    return h_round == HROUND_BF16 ? round_bf16(v) : h_round == HROUND_F16 ? round_f16(v) : v;
}

double oracle_round_hidden(double v, int h_round) { return round_hidden(v, h_round); }

/* FP8 activation mode, bf16 activations: how near a hidden row's scale is
 * to changing.  The scale comes from the largest |value| after the bf16
 * rounding; an implementation that forms the values in fp32 with a slightly
 * different rounding error rounds an element to the other bf16 neighbour
 * when the element lies near a rounding midpoint, and if that element is
 * (or becomes) the largest, the whole row gets another scale.  Returns the
 * smallest distance, relative to the row's largest |fp32 value|, from an
 * element within one bf16 spacing of that largest value to its nearest bf16
 * rounding midpoint (bf16 keeps 8 significant bits: spacing 2^(e-8) in the
 * binade [2^(e-1), 2^e), half that just below it); +inf for a zero row. */
static double hidden_scale_margin(int n, const double *h) {
    double m = 0.0;
    for (int j = 0; j < n; ++j) {
        double a = fabs((double)(float)h[j]);
        if (a > m) m = a;
    }
    if (m == 0.0) return INFINITY;
    double best = INFINITY;
    for (int j = 0; j < n; ++j) {
        double a = fabs((double)(float)h[j]);
        if (a < m * (1.0 - ldexp(1.0, -7)) || a == 0.0) continue;
        int e2;
        frexp(a, &e2); /* a in [2^(e2-1), 2^e2) */
        double ulp = ldexp(1.0, e2 - 8);
        double lo = floor(a / ulp) * ulp;
        double dist = fabs(a - (lo + 0.5 * ulp));
        if (lo == ldexp(1.0, e2 - 1)) { /* the midpoint below the binade is finer */
            double below = a - (lo - 0.25 * ulp);
            if (below < dist) dist = below;
        }
        if (dist / m < best) best = dist / m;
    }
    return best;
}

static double sigmoid(double z) { return 1.0 / (1.0 + exp(-z)); }
static double silu(double z) { return z / (1.0 + exp(-z)); }

/* Router for one token: fp32 logits, top-1 index (lowest index on ties),
 * winning logit and the margin to the runner-up (+inf when E == 1). */
static int route_token(int d, int E, const void *x_t, int x_dtype,
                       const void *Wr, int wr_dtype, const float *bias,
                       float *lmax_out, float *margin_out) {
    int best = 0;
    float lbest = -INFINITY, lsecond = -INFINITY;
    for (int e = 0; e < E; ++e) {
        double acc = 0.0;
        for (int k = 0; k < d; ++k)
            acc += load_elem(x_t, x_dtype, (size_t)k) *
                   load_elem(Wr, wr_dtype, (size_t)k * (size_t)E + (size_t)e);
        if (bias) acc += (double)bias[e];
        float l = (float)acc;
        if (l > lbest) {            /* strict: earlier index keeps a tie */
            lsecond = lbest;
            lbest = l;
            best = e;
        } else if (l > lsecond) {
            lsecond = l;
        }
    }
    if (lmax_out) *lmax_out = lbest;
    if (margin_out) *margin_out = (E > 1) ? (float)((double)lbest - (double)lsecond) : INFINITY;
    return best;
}

/* Top-k router for one token (k >= 1): the k largest fp32 logits, in
 * descending order, each pass taking the lowest index among the remaining
 * maxima (strict ">" in ascending order; NaN never wins); margin = k-th
 * selected logit minus the largest logit left out (+inf when k == E). */
static void route_token_topk(int d, int E, int k, const void *x_t, int x_dtype,
                             const void *Wr, int wr_dtype, const float *bias,
                             int32_t *sel, float *lsel, float *margin_out) {
    float *l = (float *)malloc(sizeof(float) * (size_t)E);
    char *taken = (char *)calloc((size_t)E, 1);
    for (int e = 0; e < E; ++e) {
        double acc = 0.0;
        for (int kk = 0; kk < d; ++kk)
            acc += load_elem(x_t, x_dtype, (size_t)kk) *
                   load_elem(Wr, wr_dtype, (size_t)kk * (size_t)E + (size_t)e);
        if (bias) acc += (double)bias[e];
        l[e] = (float)acc;
    }
    for (int j = 0; j < k; ++j) {
        int best = -1;
        float lb = -INFINITY;
        for (int e = 0; e < E; ++e) {
            if (taken[e] || l[e] != l[e]) continue;      /* NaN never wins */
            if (best < 0 || l[e] > lb) {                 /* ties keep the lower index */
                best = e;
                lb = l[e];
            }
        }
        for (int e = 0; best < 0 && e < E; ++e)          /* only NaN logits left */
            if (!taken[e]) best = e;
        taken[best] = 1;
        sel[j] = best;
        lsel[j] = l[best];
    }
    float rest = -INFINITY;
    for (int e = 0; e < E; ++e)
        if (!taken[e] && l[e] > rest) rest = l[e];
    if (margin_out) *margin_out = (k < E) ? (float)((double)lsel[k - 1] - (double)rest) : INFINITY;
    free(l);
    free(taken);
}

/* One SwiGLU FFN on one input row u[d]:
 *   a = u . Wgu  (2Fw values), h_j = silu(a_j) * a_{Fw+j},  y += h . Wd.
 * yh (optional): the same down projection with each h_j rounded as h_round
 * says, added into yh. */
static void swiglu_ffn_accumulate(int d, int Fw, const double *u,
                                  const void *Wgu, const void *Wd, int w_dtype,
                                  const float *s_gu, const float *s_d, int act_fp8,
                                  int act_bf16, double *a, double *h, double *y,
                                  int h_round, double *yh, double *scale_margin) {
    size_t two_f = 2 * (size_t)Fw;
    for (size_t j = 0; j < two_f; ++j) a[j] = 0.0;
    for (int k = 0; k < d; ++k) {
        double uk = u[k];
        for (size_t j = 0; j < two_f; ++j)
            a[j] += uk * load_weight(Wgu, w_dtype, s_gu, (size_t)k, two_f, j);
    }
    for (int j = 0; j < Fw; ++j) h[j] = silu(a[j]) * a[Fw + j];
    if (act_fp8) {
        /* the hidden row in the layer's activation type, then quantised; the
         * quantised values are what the down contraction reads, so the
         * hidden-rounding variant below has nothing left to round */
        if (act_bf16) {
            if (scale_margin) {
                double mg = hidden_scale_margin(Fw, h);
                if (mg < *scale_margin) *scale_margin = mg;
            }
            for (int j = 0; j < Fw; ++j) h[j] = round_bf16(h[j]);
        }
        quantise_row_e4m3(Fw, h);
        h_round = HROUND_NONE;
    }
    for (int j = 0; j < Fw; ++j) {
        double hj = h[j];
        for (int n = 0; n < d; ++n)
            y[n] += hj * load_weight(Wd, w_dtype, s_d, (size_t)j, (size_t)d, (size_t)n);
    }
    if (!yh) return;
    for (int j = 0; j < Fw; ++j) {
        double hj = round_hidden(h[j], h_round);
        for (int n = 0; n < d; ++n)
            yh[n] += hj * load_weight(Wd, w_dtype, s_d, (size_t)j, (size_t)d, (size_t)n);
    }
}

/* Routing for all T tokens. */
void oracle_route(int T, int d, int E, const void *x, int x_dtype,
                  const void *Wr, int wr_dtype, const float *bias,
                  int32_t *idx, float *lmax, float *margin) {
    size_t xs = (x_dtype == ORACLE_F32) ? 4 : 2;
#pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t) {
        const char *x_t = (const char *)x + (size_t)t * (size_t)d * xs;
        idx[t] = route_token(d, E, x_t, x_dtype, Wr, wr_dtype, bias,
                             lmax ? &lmax[t] : NULL, margin ? &margin[t] : NULL);
    }
}

/* Top-k routing for all T tokens: idx / lsel [T][k], margin [T]. */
void oracle_route_topk(int T, int d, int E, int k, const void *x, int x_dtype,
                       const void *Wr, int wr_dtype, const float *bias,
                       int32_t *idx, float *lsel, float *margin) {
    size_t xs = (x_dtype == ORACLE_F32) ? 4 : 2;
#pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t) {
        const char *x_t = (const char *)x + (size_t)t * (size_t)d * xs;
        route_token_topk(d, E, k, x_t, x_dtype, Wr, wr_dtype, bias, idx + (size_t)t * k,
                         lsel + (size_t)t * k, margin ? &margin[t] : NULL);
    }
}

/* Per-expert counts, exclusive offsets and the stable permutation
 * perm[p] = token at expert-sorted slot p (order by expert, then token). */
void oracle_permutation(int T, int E, const int32_t *idx, int32_t *counts,
                        int32_t *offsets, int32_t *perm) {
    for (int e = 0; e < E; ++e) counts[e] = 0;
    for (int t = 0; t < T; ++t) counts[idx[t]] += 1;
    offsets[0] = 0;
    for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
    int32_t *fill = (int32_t *)malloc(sizeof(int32_t) * (size_t)(E > 0 ? E : 1));
    for (int e = 0; e < E; ++e) fill[e] = offsets[e];
    for (int t = 0; t < T; ++t) perm[fill[idx[t]]++] = t;
    free(fill);
}

/* Full layer output for the tokens listed in sel[0..n_sel) (all tokens
 * when sel == NULL, n_sel == T).  out is [n_sel, d] fp64.  W_gate_up[e] /
 * W_down[e] may be NULL for experts that none of the selected tokens
 * reaches; returns -1 if a needed expert is missing, 0 on success.
 * sel_idx / sel_gate (optional) receive each selected token's expert and
 * gate.  scale_margin (optional, [n_sel]): in the FP8 activation mode with
 * bf16 activations, the smallest hidden_scale_margin over the token's hidden
 * rows (shared and routed), else +inf. */
int oracle_forward(int T, int d, int E, int k, int F, int Fs,
                   const void *x, int x_dtype,
                   const void *Wr, int wr_dtype, const float *bias,
                   const void *const *W_gate_up, const void *const *W_down,
                   const void *Ws_gate_up, const void *Ws_down, int w_dtype,
                   const float *const *s_gate_up, const float *const *s_down,
                   const float *ss_gate_up, const float *ss_down, int act_fp8,
                   int n_sel, const int32_t *sel, double *out,
                   int32_t *sel_idx, double *sel_gate, int h_round, double *out_h,
                   double *scale_margin) {
    size_t xs = (x_dtype == ORACLE_F32) ? 4 : 2;
    const int act_bf16 = x_dtype == ORACLE_BF16; /* the layer's activations are bf16 */
    int missing = 0;
    (void)T;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : missing)
    for (int i = 0; i < n_sel; ++i) {
        int t = sel ? sel[i] : i;
        const char *x_t = (const char *)x + (size_t)t * (size_t)d * xs;
        int Fmax = F > Fs ? F : Fs;
        double *u = (double *)malloc(sizeof(double) * (size_t)d);
        double *a = (double *)malloc(sizeof(double) * 2 * (size_t)Fmax);
        double *h = (double *)malloc(sizeof(double) * (size_t)Fmax);
        double *y = out + (size_t)i * (size_t)d;
        double *yh = out_h ? out_h + (size_t)i * (size_t)d : NULL;
        for (int n = 0; n < d; ++n) y[n] = 0.0;
        for (int n = 0; yh && n < d; ++n) yh[n] = 0.0;
        if (scale_margin) scale_margin[i] = INFINITY;
        /* shared expert on the ungated input (with E == 0 the whole layer:
         * the dense SwiGLU feed-forward of the layers without experts) */
        for (int k = 0; k < d; ++k) u[k] = load_elem(x_t, x_dtype, (size_t)k);
        if (act_fp8) quantise_row_e4m3(d, u); /* x_t as the contractions see it */
        double *xq = (double *)malloc(sizeof(double) * (size_t)d);
        for (int k = 0; k < d; ++k) xq[k] = u[k];
        swiglu_ffn_accumulate(d, Fs, u, Ws_gate_up, Ws_down, w_dtype,
                              ss_gate_up, ss_down, act_fp8, act_bf16, a, h, y, h_round, yh,
                              scale_margin ? &scale_margin[i] : NULL);
        if (E == 0) {
            if (sel_idx) sel_idx[i] = -1;
            if (sel_gate) sel_gate[i] = 0.0;
            free(u);
            free(xq);
            free(a);
            free(h);
            continue;
        }
        int32_t sel_e[8];
        float sel_l[8];
        if (k == 1) {
            sel_e[0] = route_token(d, E, x_t, x_dtype, Wr, wr_dtype, bias, &sel_l[0], NULL);
        } else {
            route_token_topk(d, E, k, x_t, x_dtype, Wr, wr_dtype, bias, sel_e, sel_l, NULL);
        }
        /* each selected expert on the input gated by its own sigmoid */
        for (int j = 0; j < k; ++j) {
            int e = sel_e[j];
            double g = sigmoid((double)sel_l[j]);
            if (sel_idx) sel_idx[(size_t)i * k + j] = e;
            if (sel_gate) sel_gate[(size_t)i * k + j] = g;
            if (!W_gate_up[e] || !W_down[e]) {
                missing |= 1;
                continue;
            }
            for (int kk = 0; kk < d; ++kk) u[kk] = g * xq[kk];
            swiglu_ffn_accumulate(d, F, u, W_gate_up[e], W_down[e], w_dtype,
                                  s_gate_up ? s_gate_up[e] : NULL,
                                  s_down ? s_down[e] : NULL, act_fp8, act_bf16, a, h, y, h_round, yh,
                                  scale_margin ? &scale_margin[i] : NULL);
        }
        free(u);
        free(xq);
        free(a);
        free(h);
    }
    return missing ? -1 : 0;
}

/* One expert's SwiGLU on n given rows: out[i] = SwiGLU_W(g[i] * x[i]) for
 * rows x[i] of width d (storage dtype x_dtype) with their gates g[i] -- the
 * routed part of the layer for each (token, expert) entry, as an expert
 * holding W_gate_up [d, 2F] / W_down [F, d] (and, for 8-bit or int4
 * weights, their column scales) computes it.  out is [n, d] fp64. */
void oracle_expert_rows(int n, int d, int F, const void *x, int x_dtype, const double *g,
                        const void *W_gate_up, const void *W_down, int w_dtype,
                        const float *s_gate_up, const float *s_down, double *out) {
    size_t xs = (x_dtype == ORACLE_F32) ? 4 : 2;
#pragma omp parallel for schedule(dynamic, 1)
    for (int i = 0; i < n; ++i) {
        const char *x_i = (const char *)x + (size_t)i * (size_t)d * xs;
        double *u = (double *)malloc(sizeof(double) * (size_t)d);
        double *a = (double *)malloc(sizeof(double) * 2 * (size_t)F);
        double *h = (double *)malloc(sizeof(double) * (size_t)F);
        double *y = out + (size_t)i * (size_t)d;
        for (int k = 0; k < d; ++k) u[k] = g[i] * load_elem(x_i, x_dtype, (size_t)k);
        for (int k = 0; k < d; ++k) y[k] = 0.0;
        swiglu_ffn_accumulate(d, F, u, W_gate_up, W_down, w_dtype, s_gate_up, s_down, 0, 0, a, h, y,
                              HROUND_NONE, NULL, NULL);
        free(u);
        free(a);
        free(h);
    }
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
