/*
 * Oracle for the MoE FFN forward pass -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow CPU restatement of what the layer computes, used to check the CUDA path.
 * Only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline / reference legs may load
 * it; the product library never does.  It shares no code, header or table generator with
 * the CUDA path.
 *
 * Sources (DeepSeek-V3.2-Exp model atlas pages):
 *   [NORM]   "MoE update" page, RMSNorm.forward excerpt: with a residual, s = x.float() +
 *            residual.float(); var = mean(s^2); s * rsqrt(var + eps); weight * s; both the
 *            normed value and the new residual are cast back to x's dtype.  eps = 1e-6, the
 *            gain is a float32 vector.
 *   [MOE]    "MoE update" / "Add shared output" pages, MoE.forward excerpt: the router returns
 *            (weights, indices); y (float32) accumulates expert(x[idx]) * weight for every
 *            (token, slot) routed to an expert; the shared expert is added to every token; the
 *            result is cast to x's dtype.  Equation: delta_ffn = y_routed + y_shared.
 *   [EXPERT] "Gate projection" page, expert excerpt: w2((silu(w1 x).float() * (w3 x).float())
 *            .type_as(x)); weights are held [out, in] without bias.
 *   [LINEAR] "Gate projection" page, Linear excerpt and "Direct evidence": a 1-byte weight
 *            carries a float32 scale of shape [ceil(out/128), ceil(in/128)], one per 128x128
 *            block.
 *
 * Readings where the pages are silent (each is listed in the design doc):
 *   - router: the gate body is not shown; scores = sigmoid(xn . Wg_e + bias_e) in float64,
 *     top-k by score with the lower expert index first on equal scores, weights = selected
 *     scores / their sum.
 *   - mean(s^2): the exact sum of the squares rounded to double, divided by d in double,
 *     rounded to float32.  rsqrt = 1 / sqrt with IEEE float32 sqrt and divide.
 *   - Linear outputs are in x's dtype (bf16): the expert excerpt's .float() casts imply it.
 *     g = bf16(W1 a), u = bf16(W3 a), y_e = bf16(W2 h); the sums themselves in float64.
 *     h = bf16(fp32(silu(g)) * fp32(u)): the excerpt fixes float32 for silu and the product;
 *     silu is taken correctly rounded to float32.
 *   - FP8 activations (performance mode): per token and per 128-column group,
 *     sc = amax / 448 (float32 divide), q = e4m3(v / sc) (float32 divide, round to nearest
 *     even, saturate to +-448); a = q * sc.  amax == 0 gives sc = 1, q = 0.  The same quant
 *     is applied to h before w2.
 *   - several shared experts are one SwiGLU with their hidden units concatenated.
 *
 * Everything is float64 unless a rounding point above says otherwise.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <float.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------------------------ */
/* number formats                                                                              */
/* ------------------------------------------------------------------------------------------ */

/* bfloat16: IEEE-754 binary32 with the low 16 mantissa bits dropped (1 sign, 8 exponent with
 * bias 127, 7 mantissa bits; subnormals below 2^-126, quantum 2^-133 there). */
double oracle_bf16_to_f64(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* Round a double to the nearest bfloat16, ties to even; overflow gives +-inf. */
uint16_t oracle_f64_to_bf16(double v)
{
    if (isnan(v)) return 0x7FC0;
    double a = fabs(v);
    double q;
    if (a == 0.0) {
        q = 0.0;
    } else {
        int e;
        frexp(a, &e);            /* a = m * 2^e, m in [0.5, 1): the binade's leading bit is 2^(e-1) */
        int lead = e - 1;
        if (lead < -126) lead = -126;          /* subnormal range shares the quantum 2^-133 */
        double quantum = ldexp(1.0, lead - 7); /* 7 stored mantissa bits */
        q = rint(a / quantum) * quantum;       /* rint: round half to even */
        if (q >= ldexp(1.0, 128)) q = INFINITY;
    }
    float f = (float)(signbit(v) ? -q : q);     /* exact: q is a bfloat16 value */
    uint32_t u;
    memcpy(&u, &f, 4);
    return (uint16_t)(u >> 16);
}

/* OCP 8-bit floating point, E4M3 ("fn" variant): 1 sign, 4 exponent bits with bias 7,
 * 3 mantissa bits; no infinities; S.1111.111 is NaN; largest finite 448; subnormals
 * m * 2^-9 for exponent field 0. */
double oracle_e4m3_to_f64(uint8_t b)
{
    int s = (b >> 7) & 1, ex = (b >> 3) & 15, m = b & 7;
    double v;
    if (ex == 15 && m == 7) return NAN;
    if (ex == 0) v = ldexp((double)m, -9);
    else v = ldexp(1.0 + m / 8.0, ex - 7);
    return s ? -v : v;
}

/* Round to the nearest E4M3 value, ties to even, saturating to +-448 (finite). */
uint8_t oracle_f64_to_e4m3(double v)
{
    if (isnan(v)) return 0x7F;
    int s = signbit(v) != 0;
    double a = fabs(v);
    double q;
    if (a == 0.0) {
        q = 0.0;
    } else {
        int e;
        frexp(a, &e);
        int lead = e - 1;
        if (lead < -6) lead = -6;              /* subnormals: quantum 2^-9 */
        double quantum = ldexp(1.0, lead - 3);
        q = rint(a / quantum) * quantum;
        if (q > 448.0) q = 448.0;
    }
    /* encode */
    uint8_t code;
    if (q == 0.0) {
        code = 0;
    } else if (q < ldexp(1.0, -6)) {
        code = (uint8_t)(q / ldexp(1.0, -9));  /* exponent field 0 */
    } else {
        int e;
        double m = frexp(q, &e);               /* q = m 2^e, m in [0.5,1) => q = (2m) 2^(e-1) */
        int ex = (e - 1) + 7;
        int mant = (int)((2.0 * m - 1.0) * 8.0);
        code = (uint8_t)((ex << 3) | mant);
    }
    return (uint8_t)(code | (s ? 0x80 : 0));
}

static double g_e4m3_table[256];
static int g_table_ready = 0;

static void build_table(void)
{
    if (g_table_ready) return;
    for (int c = 0; c < 256; ++c) g_e4m3_table[c] = oracle_e4m3_to_f64((uint8_t)c);
    g_table_ready = 1;
}

/* ------------------------------------------------------------------------------------------ */
/* exact sum of squares of float32 values                                                      */
/* ------------------------------------------------------------------------------------------ */
/* Each float32 s is M * 2^E with an integer |M| < 2^24 and E >= -149, so s^2 = M^2 2^(2E) with
 * M^2 < 2^48 and 2E >= -298.  The squares are added as integers in a fixed-point accumulator
 * (little-endian 32-bit limbs, unit 2^-298), which is exact in any order; the total is then
 * rounded once to double. */
#define SQ_LIMBS 24   /* 768 bits: 2^-298 .. 2^470 */

static void acc_add_square(uint32_t* acc, float s)
{
    if (s == 0.0f) return;
    int e;
    double m = frexp(fabs((double)s), &e);           /* |s| = m 2^e */
    /* integer mantissa M with |s| = M 2^(e-24); shift down for subnormals to keep E >= -149 */
    int E = e - 24;
    uint64_t M = (uint64_t)ldexp(m, 24);
    if (E < -149) { M >>= (-149 - E); E = -149; }    /* exact: low bits of a subnormal are 0 */
    uint64_t M2 = M * M;                              /* < 2^48 */
    int shift = 2 * E + 298;                          /* bit position of M2's lsb */
    int limb = shift / 32, bit = shift % 32;
    /* add M2 << bit at limb (spans at most 3 limbs), then propagate the carry */
    unsigned __int128 v = (unsigned __int128)M2 << bit;
    uint64_t carry = 0;
    for (int i = 0; i < 3 || carry; ++i) {
        uint64_t add = (i < 3) ? (uint64_t)((v >> (32 * i)) & 0xFFFFFFFFu) : 0;
        uint64_t t = (uint64_t)acc[limb + i] + add + carry;
        acc[limb + i] = (uint32_t)t;
        carry = t >> 32;
    }
}

/* Round the non-negative fixed-point value to the nearest double (ties to even). */
static double acc_to_double(const uint32_t* acc)
{
    int top = -1;
    for (int i = SQ_LIMBS - 1; i >= 0; --i)
        if (acc[i]) { top = i; break; }
    if (top < 0) return 0.0;
    /* collect the leading 64 bits and a sticky bit for everything below */
    int hb = 31;
    while (!((acc[top] >> hb) & 1)) --hb;
    int msb = top * 32 + hb;                          /* index of the leading one */
    /* take bits msb .. msb-53 (54 bits: 53 kept + 1 round), sticky = any lower bit */
    uint64_t head = 0;
    for (int b = 0; b < 54; ++b) {
        int pos = msb - b;
        int bitv = pos >= 0 ? (acc[pos / 32] >> (pos % 32)) & 1 : 0;
        head = (head << 1) | (uint64_t)bitv;
    }
    int sticky = 0;
    for (int pos = msb - 54; pos >= 0 && !sticky; --pos)
        if ((acc[pos / 32] >> (pos % 32)) & 1) sticky = 1;
    uint64_t keep = head >> 1;                        /* 53 bits */
    int rbit = head & 1;
    if (rbit && (sticky || (keep & 1))) keep += 1;    /* may carry into 2^53: still exact below */
    return ldexp((double)keep, msb - 52 - 298);
}

/* var = fp32( RN64(sum s_i^2) / d ), the reading of mean(s^2) adopted for [NORM]. */
float oracle_mean_square(int d, const float* s)
{
    uint32_t acc[SQ_LIMBS];
    memset(acc, 0, sizeof acc);
    for (int i = 0; i < d; ++i) acc_add_square(acc, s[i]);
    double ss = acc_to_double(acc);
    return (float)(ss / (double)d);
}

/* ------------------------------------------------------------------------------------------ */
/* [NORM] RMSNorm with the residual add                                                        */
/* ------------------------------------------------------------------------------------------ */
/* xn (bf16), residual_out (bf16), xn64 (the same value without any rounding, float64), xn32
 * (the float32 value just before the bf16 cast).  r may be NULL (no residual: s = x). */
void oracle_norm_token(int d, const uint16_t* x, const uint16_t* r, const float* g, float eps,
                       uint16_t* xn, uint16_t* resid_out, double* xn64, float* xn32)
{
    float* s = (float*)malloc(sizeof(float) * d);
    double ss64 = 0.0;
    for (int i = 0; i < d; ++i) {
        float xi = (float)oracle_bf16_to_f64(x[i]);
        float ri = r ? (float)oracle_bf16_to_f64(r[i]) : 0.0f;
        s[i] = r ? xi + ri : xi;                      /* float32 add */
        if (r && resid_out) resid_out[i] = oracle_f64_to_bf16((double)s[i]);
        ss64 += (double)s[i] * (double)s[i];
    }
    float var = oracle_mean_square(d, s);
    float v = var + eps;                              /* float32 */
    float sq = sqrtf(v);                              /* IEEE float32 sqrt */
    float rinv = 1.0f / sq;                           /* IEEE float32 divide */
    double rinv64 = 1.0 / sqrt(ss64 / d + (double)eps);
    for (int i = 0; i < d; ++i) {
        float t = s[i] * rinv;                        /* x * rsqrt(var + eps) */
        float y = g[i] * t;                           /* weight * x */
        if (xn32) xn32[i] = y;
        if (xn) xn[i] = oracle_f64_to_bf16((double)y);
        if (xn64) xn64[i] = (double)g[i] * (double)s[i] * rinv64;
    }
    free(s);
}

/* ------------------------------------------------------------------------------------------ */
/* FP8 activation quant (per 128-column group)                                                 */
/* ------------------------------------------------------------------------------------------ */
/* v: n bf16-valued doubles (n a multiple of 128).  q: e4m3 codes, sc: n/128 scales,
 * deq: q * sc (float64, exact). */
void oracle_act_quant(int n, const double* v, uint8_t* q, float* sc, double* deq)
{
    build_table();
    for (int g0 = 0; g0 < n; g0 += 128) {
        float amax = 0.0f;
        for (int i = g0; i < g0 + 128; ++i) {
            float a = (float)fabs(v[i]);
            if (a > amax) amax = a;
        }
        float s = amax > 0.0f ? amax / 448.0f : 1.0f;  /* float32 divide */
        if (sc) sc[g0 / 128] = s;
        for (int i = g0; i < g0 + 128; ++i) {
            uint8_t c = 0;
            if (amax > 0.0f) {
                float t = (float)v[i] / s;               /* float32 divide */
                c = oracle_f64_to_e4m3((double)t);
            }
            if (q) q[i] = c;
            if (deq) deq[i] = g_e4m3_table[c] * (double)s;
        }
    }
}

/* ------------------------------------------------------------------------------------------ */
/* weights                                                                                     */
/* ------------------------------------------------------------------------------------------ */
/* Element (o, i) of a [rows, cols] weight: bf16 as stored, or e4m3 code times the float32
 * scale of its 128x128 block ([LINEAR]: scale shape [ceil(rows/128), ceil(cols/128)]). */
static inline double weight_at(int fp8, const void* w, const float* scale, int cols, int o, int i)
{
    size_t idx = (size_t)o * cols + i;
    if (!fp8) return oracle_bf16_to_f64(((const uint16_t*)w)[idx]);
    int sc_cols = (cols + 127) / 128;
    return g_e4m3_table[((const uint8_t*)w)[idx]] * (double)scale[(size_t)(o / 128) * sc_cols + i / 128];
}

static double silu(double z) { return z / (1.0 + exp(-z)); }

/* [EXPERT] one SwiGLU on one activation vector a (length d, already the values the expert
 * sees).  w1, w3: [I, d]; w2: [d, I] (with scales when fp8).  act_fp8: quantize h before w2.
 * y: d outputs, each rounded to bf16 (held as double). */
void oracle_swiglu(int d, int I, int fp8, int act_fp8, const double* a,
                   const void* w1, const float* s1, const void* w3, const float* s3,
                   const void* w2, const float* s2, double* y)
{
    build_table();
    double* h = (double*)malloc(sizeof(double) * I);
    double* hq = (double*)malloc(sizeof(double) * I);
    for (int o = 0; o < I; ++o) {
        double gs = 0.0, us = 0.0;
        for (int i = 0; i < d; ++i) {
            gs += weight_at(fp8, w1, s1, d, o, i) * a[i];
            us += weight_at(fp8, w3, s3, d, o, i) * a[i];
        }
        double g = oracle_bf16_to_f64(oracle_f64_to_bf16(gs));   /* w1(x) in x's dtype */
        double u = oracle_bf16_to_f64(oracle_f64_to_bf16(us));   /* w3(x) in x's dtype */
        /* silu(g.float()) * u.float() is float32 arithmetic on the page: silu correctly rounded
         * to float32, an IEEE float32 multiply, then .type_as(x) */
        float sg = (float)silu(g);
        float hv = sg * (float)u;
        h[o] = oracle_bf16_to_f64(oracle_f64_to_bf16((double)hv));
    }
    if (act_fp8) oracle_act_quant(I, h, NULL, NULL, hq);
    else memcpy(hq, h, sizeof(double) * I);
    for (int o = 0; o < d; ++o) {
        double acc = 0.0;
        for (int i = 0; i < I; ++i) acc += weight_at(fp8, w2, s2, I, o, i) * hq[i];
        y[o] = oracle_bf16_to_f64(oracle_f64_to_bf16(acc));     /* w2(.) in x's dtype */
    }
    free(h);
    free(hq);
}

/* ------------------------------------------------------------------------------------------ */
/* router (reading: sigmoid scores, top-k, lower index first on ties, normalised weights)      */
/* ------------------------------------------------------------------------------------------ */
/* scores: E float64 scores (out).  idx/w: k selected experts in descending score order.
 * margin: score of the k-th minus score of the (k+1)-th (INFINITY when k == E). */
void oracle_gate_token(int d, int E, int k, const uint16_t* xn, const uint16_t* gate_w,
                       const float* bias, double* scores, int* idx, double* w, double* margin)
{
    double* sc = scores;
    for (int e = 0; e < E; ++e) {
        double z = 0.0;
        for (int i = 0; i < d; ++i)
            z += oracle_bf16_to_f64(xn[i]) * oracle_bf16_to_f64(gate_w[(size_t)e * d + i]);
        if (bias) z += (double)bias[e];
        sc[e] = 1.0 / (1.0 + exp(-z));
    }
    /* selection: k passes of "largest score, lowest index among equals" over the unchosen */
    char* taken = (char*)calloc(E, 1);
    double sum = 0.0;
    for (int j = 0; j < k; ++j) {
        int best = -1;
        for (int e = 0; e < E; ++e)
            if (!taken[e] && (best < 0 || sc[e] > sc[best])) best = e;
        taken[best] = 1;
        idx[j] = best;
        sum += sc[best];
    }
    for (int j = 0; j < k; ++j) w[j] = sc[idx[j]] / sum;
    if (margin) {
        if (k >= E) {
            *margin = INFINITY;
        } else {
            int next = -1;
            for (int e = 0; e < E; ++e)
                if (!taken[e] && (next < 0 || sc[e] > sc[next])) next = e;
            *margin = sc[idx[k - 1]] - sc[next];
        }
    }
    free(taken);
}

/* ------------------------------------------------------------------------------------------ */
/* the whole layer for a list of tokens                                                        */
/* ------------------------------------------------------------------------------------------ */
typedef struct {
    int T, d, I, E, k, Is;   /* Is: width of the (concatenated) shared SwiGLU; 0 = none */
    int fp8;                 /* weights are e4m3 + 128x128 float32 block scales */
    int act_fp8;             /* FP8 activations (per 1x128 group) into every expert GEMM */
    float eps;
} oracle_cfg;

typedef struct {
    const uint16_t *x, *residual;   /* [T, d] bf16; residual may be NULL */
    const float* norm_w;            /* [d] */
    const uint16_t* gate_w;         /* [E, d] bf16 */
    const float* gate_bias;         /* [E] or NULL */
    const void *w1, *w3, *w2;       /* [E, I, d], [E, I, d], [E, d, I] */
    const float *s1, *s3, *s2;      /* [E, I/128, d/128], [E, d/128, I/128] */
    const void *sw1, *sw3, *sw2;    /* [Is, d], [Is, d], [d, Is] */
    const float *ss1, *ss3, *ss2;
} oracle_inputs;

/* Outputs are indexed by position in the token list; any pointer may be NULL.
 * out, resid_out, xn: [n, d] bf16.  xn64: [n, d].  idx: [n, k].  w: [n, k].  margin: [n].
 * route_only != 0 skips the experts (norm + router only). */
void oracle_forward(const oracle_cfg* c, const oracle_inputs* in, int n, const int* tokens,
                    int route_only, uint16_t* out, uint16_t* resid_out, uint16_t* xn_out,
                    double* xn64_out, int* idx_out, double* w_out, double* margin_out, int nthreads)
{
    build_table();
    const int d = c->d, I = c->I, E = c->E, k = c->k, Is = c->Is;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (int p = 0; p < n; ++p) {
        const int t = tokens[p];
        uint16_t* xn = (uint16_t*)malloc(sizeof(uint16_t) * d);
        uint16_t* ro = (uint16_t*)malloc(sizeof(uint16_t) * d);
        double* xn64 = (double*)malloc(sizeof(double) * d);
        double* a = (double*)malloc(sizeof(double) * d);
        double* y = (double*)malloc(sizeof(double) * d);
        double* acc = (double*)calloc(d, sizeof(double));
        double* scores = (double*)malloc(sizeof(double) * E);
        int* idx = (int*)malloc(sizeof(int) * k);
        double* w = (double*)malloc(sizeof(double) * k);
        double margin;

        oracle_norm_token(d, in->x + (size_t)t * d, in->residual ? in->residual + (size_t)t * d : NULL,
                          in->norm_w, c->eps, xn, ro, xn64, NULL);
        /* a dense block ("MoE update" page, Block excerpt: the first n_dense_layers blocks use the
         * MLP instead of the MoE) has no router: E = 0, k = 0, and the MLP is the shared SwiGLU */
        if (E > 0) oracle_gate_token(d, E, k, xn, in->gate_w, in->gate_bias, scores, idx, w, &margin);
        else margin = INFINITY;

        if (!route_only) {
            /* the activation every expert sees: xn itself, or its FP8 quant */
            for (int i = 0; i < d; ++i) a[i] = oracle_bf16_to_f64(xn[i]);
            if (c->act_fp8) oracle_act_quant(d, a, NULL, NULL, a);
            /* [MOE] y = sum over the token's slots of expert(x) * weight */
            for (int j = 0; j < k; ++j) {
                const int e = idx[j];
                size_t o13 = (size_t)e * I * d, o2 = (size_t)e * d * I;
                size_t so13 = (size_t)e * (I / 128) * (d / 128), so2 = (size_t)e * (d / 128) * (I / 128);
                const void *w1 = c->fp8 ? (const void*)((const uint8_t*)in->w1 + o13) : (const void*)((const uint16_t*)in->w1 + o13);
                const void *w3 = c->fp8 ? (const void*)((const uint8_t*)in->w3 + o13) : (const void*)((const uint16_t*)in->w3 + o13);
                const void *w2 = c->fp8 ? (const void*)((const uint8_t*)in->w2 + o2) : (const void*)((const uint16_t*)in->w2 + o2);
                oracle_swiglu(d, I, c->fp8, c->act_fp8, a, w1, c->fp8 ? in->s1 + so13 : NULL,
                              w3, c->fp8 ? in->s3 + so13 : NULL, w2, c->fp8 ? in->s2 + so2 : NULL, y);
                for (int i = 0; i < d; ++i) acc[i] += y[i] * w[j];
            }
            /* + shared expert on every token ("Add shared output") */
            if (Is > 0) {
                oracle_swiglu(d, Is, c->fp8, c->act_fp8, a, in->sw1, in->ss1, in->sw3, in->ss3, in->sw2, in->ss2, y);
                for (int i = 0; i < d; ++i) acc[i] += y[i];
            }
            if (out)
                for (int i = 0; i < d; ++i) out[(size_t)p * d + i] = oracle_f64_to_bf16(acc[i]);
        }
        if (resid_out) memcpy(resid_out + (size_t)p * d, ro, sizeof(uint16_t) * d);
        if (xn_out) memcpy(xn_out + (size_t)p * d, xn, sizeof(uint16_t) * d);
        if (xn64_out) memcpy(xn64_out + (size_t)p * d, xn64, sizeof(double) * d);
        if (idx_out) memcpy(idx_out + (size_t)p * k, idx, sizeof(int) * k);
        if (w_out) memcpy(w_out + (size_t)p * k, w, sizeof(double) * k);
        if (margin_out) margin_out[p] = margin;
        free(xn); free(ro); free(xn64); free(a); free(y); free(acc); free(scores); free(idx); free(w);
    }
}

/* Scores of every expert for a list of tokens whose normed input is given (xn [n, d] bf16). */
void oracle_gate_scores(int n, int d, int E, const uint16_t* xn, const uint16_t* gate_w,
                        const float* bias, double* scores, int nthreads)
{
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(static)
#endif
    for (int p = 0; p < n; ++p) {
        for (int e = 0; e < E; ++e) {
            double z = 0.0;
            for (int i = 0; i < d; ++i)
                z += oracle_bf16_to_f64(xn[(size_t)p * d + i]) * oracle_bf16_to_f64(gate_w[(size_t)e * d + i]);
            if (bias) z += (double)bias[e];
            scores[(size_t)p * E + e] = 1.0 / (1.0 + exp(-z));
        }
    }
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
