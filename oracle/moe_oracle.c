/*
 * moe_oracle.c - plain, slow CPU oracle for the fused Mixture-of-Experts layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or call
 * this file: only the test-suite, the smoke check and the benchmark's CPU
 * baseline leg use it.  It shares no code, header, table or constant with the
 * CUDA library; the two meet only through the seeded input generator.
 *
 * What it computes (sources):
 *   - "Mixture-of-Experts kernel engineering on Amazon SageMaker AI" (abstract):
 *     a fused MoE layer is token routing + data shuffling + the experts' network
 *     math + expert aggregation, done as one batched operation.
 *   - "AWS раскрыла оптимизации ядер MoE на SageMaker AI", section
 *     "Зачем оптимизировать ядра MoE": the same decomposition.
 *   - The pages never give the gate function or the expert MLP.  The layer this
 *     library targets is the Mixtral / DeepSeek-V3 / Qwen2-MoE layer: top-k
 *     gating over router logits (softmax renormalised over the chosen k, or
 *     sigmoid renormalised and scaled), SwiGLU experts
 *         MLP_e(x) = W2[e] . ( SiLU(W1[e] x) * (W3[e] x) ),   SiLU(g) = g / (1 + e^-g)
 *     and an optional always-on shared expert with weight 1.
 *   - FP8: "tensor-quantized" FP8 (the AWS abstract, backend paragraph; the
 *     Russian summary, section "Triton вместо CUTLASS для FP8-квантования"):
 *     one fp32 scale per tensor.  Read here as one scale per expert weight
 *     matrix and one static scale per activation tensor; value = code * scale.
 *
 * Everything is computed per token, densely, in double precision, straight
 * from the definition
 *     out[t] = sum_j w[t,j] * MLP_{e_j}(x_t)  (+ MLP_shared(x_t))
 * without building any permutation.  The separate counting sort below is the
 * reference for the align/permute step only.
 *
 * Number formats are decoded from their definitions (bf16 = upper half of an
 * IEEE binary32; E4M3 "fn" = 1 sign, 4 exponent bits with bias 7, 3 mantissa
 * bits, subnormals, no infinities, S.1111.111 = NaN, largest finite 448).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_BF16 0
#define ORC_E4M3 1
#define ORC_SOFTMAX 0
#define ORC_SIGMOID 1

/* ------------------------------------------------------------------------ */
/* number formats                                                            */
/* ------------------------------------------------------------------------ */

double orc_bf16_decode(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

double orc_e4m3_decode(uint8_t c)
{
    int s = c >> 7, ex = (c >> 3) & 15, m = c & 7;
    double v;
    if (ex == 15 && m == 7) return NAN;
    if (ex == 0)
        v = ldexp((double)m, -9);              /* subnormal: m/8 * 2^(1-7) */
    else
        v = ldexp(1.0 + m / 8.0, ex - 7);
    return s ? -v : v;
}

/* Round v to nearest, ties to even, in a binary format with p significand
 * bits whose smallest normal has exponent emin; unbounded above. */
static double round_to_format(double v, int p, int emin)
{
    if (v == 0.0 || !isfinite(v)) return v;
    int e;
    frexp(fabs(v), &e);                 /* |v| = f * 2^e, f in [0.5, 1) */
    int lead = e - 1;
    if (lead < emin) lead = emin;
    double quantum = ldexp(1.0, lead - (p - 1));
    double q = fabs(v) / quantum;       /* exact: power-of-two scaling */
    double r = nearbyint(q);            /* default mode: ties to even */
    return copysign(r * quantum, v);
}

/* E4M3 with round-to-nearest-even and saturation to +-448 (no NaN output for
 * finite input). */
uint8_t orc_e4m3_encode(double v)
{
    if (isnan(v)) return 0x7F;
    uint8_t s = signbit(v) ? 0x80 : 0;
    double r = round_to_format(v, 4, -6);
    double a = fabs(r);
    if (a > 448.0) a = 448.0;
    if (a == 0.0) return s;
    int e;
    frexp(a, &e);
    int lead = e - 1;
    if (lead < -6) {                     /* subnormal: a = m * 2^-9 */
        int m = (int)(a / ldexp(1.0, -9));
        return (uint8_t)(s | m);
    }
    int m = (int)((a / ldexp(1.0, lead) - 1.0) * 8.0);
    return (uint8_t)(s | ((lead + 7) << 3) | m);
}

/* bf16 with round-to-nearest-even, overflow to infinity. */
uint16_t orc_bf16_encode(double v)
{
    if (isnan(v)) return 0x7FC0;
    uint16_t s = signbit(v) ? 0x8000 : 0;
    double r = round_to_format(v, 8, -126);
    double a = fabs(r);
    if (a == 0.0) return s;
    if (a >= ldexp(1.0, 128)) return (uint16_t)(s | 0x7F80);
    int e;
    frexp(a, &e);
    int lead = e - 1;
    if (lead < -126) {                   /* subnormal: a = m * 2^-133 */
        int m = (int)(a / ldexp(1.0, -133));
        return (uint16_t)(s | m);
    }
    int m = (int)((a / ldexp(1.0, lead) - 1.0) * 128.0);
    return (uint16_t)(s | ((lead + 127) << 7) | m);
}

/* Quantise fp32 values to E4M3 codes with a per-tensor scale.  The quotient
 * is formed in fp32 (IEEE division, correctly rounded) before the rounding to
 * E4M3, the precision the layer's activation quantiser works in, so that the
 * integer codes are decided in one precision on both sides. */
void orc_quant_e4m3_f32(const float *v, float scale, uint8_t *codes, long n)
{
    for (long i = 0; i < n; ++i) {
        float q = v[i] / scale;
        codes[i] = orc_e4m3_encode((double)q);
    }
}

static double decode_w(const void *base, int dtype, long idx)
{
    if (dtype == ORC_BF16) return orc_bf16_decode(((const uint16_t *)base)[idx]);
    return orc_e4m3_decode(((const uint8_t *)base)[idx]);
}

/* ------------------------------------------------------------------------ */
/* routing: top-k gating over router logits                                  */
/* ------------------------------------------------------------------------ */

/* Router logits, the step before top-k gating: l[t,e] = sum_h x[t,h] * Wg[e,h]
 * with x [T,H] and Wg [E,H] bf16.  The Chinese retelling (section
 * "2. 用于FP8量化的Triton后端路由") has the routing decided inside the fused
 * kernel, without host control flow; the pages give no summation order.  So
 * that routing is bit-exact between implementations, the order is fixed as
 * part of the definition:
 *   - in double precision (a product of two bf16 values is exact in double);
 *   - 32 partial sums s_l, l = 0..31: s_l sums, in ascending h, the products
 *     whose 8-element chunk index h / 8 is congruent to l mod 32;
 *   - then s_l <- s_l + s_(l xor o) for o = 16, 8, 4, 2, 1 (every s_l ends
 *     equal);
 *   - the result rounded once to fp32, to nearest even.
 * Requires H to be a multiple of 8. */
void orc_router_logits(int T, int E, int H, const uint16_t *x, const uint16_t *wg, float *logits)
{
    for (int t = 0; t < T; ++t)
        for (int e = 0; e < E; ++e) {
            double s[32], n[32];
            for (int l = 0; l < 32; ++l) s[l] = 0.0;
            for (int c = 0; c < H / 8; ++c)
                for (int i = 0; i < 8; ++i) {
                    const long h = 8L * c + i;
                    s[c % 32] += orc_bf16_decode(x[(long)t * H + h]) * orc_bf16_decode(wg[(long)e * H + h]);
                }
            for (int o = 16; o >= 1; o >>= 1) {
                for (int l = 0; l < 32; ++l) n[l] = s[l] + s[l ^ o];
                for (int l = 0; l < 32; ++l) s[l] = n[l];
            }
            logits[(long)t * E + e] = (float)s[0];
        }
}

/* Expert a ranks above expert b: larger logit, equal logits -> lower id.
 * NaN ranks below every number (and among NaNs the lower id first). */
static int ranks_above(const float *l, int a, int b)
{
    int na = isnan(l[a]), nb = isnan(l[b]);
    if (na || nb) {
        if (na && nb) return a < b;
        return nb;
    }
    if (l[a] != l[b]) return l[a] > l[b];
    return a < b;
}

/* For each token: the k experts of highest logit (ties -> lower id), in rank
 * order, and their weights.
 *   softmax, renorm : w_j = e^{l_j} / sum_{selected} e^{l_i}
 *   softmax, !renorm: w_j = e^{l_j} / sum_{all E} e^{l_i}
 *   sigmoid, renorm : w_j = s_j / sum_{selected} s_i,  s = 1/(1+e^-l)
 *   sigmoid, !renorm: w_j = s_j
 * then w_j *= routed_scale.  Selection is on the logit itself: both maps are
 * monotone, so the chosen set is the same as by score. */
void orc_route(int T, int E, int k, int gate, int renorm, double routed_scale,
               const float *logits, int32_t *ids, double *w)
{
    for (int t = 0; t < T; ++t) {
        const float *l = logits + (long)t * E;
        int32_t *id = ids + (long)t * k;
        double *wt = w + (long)t * k;
        unsigned char *taken = calloc((size_t)E, 1);
        for (int j = 0; j < k; ++j) {
            int best = -1;
            for (int e = 0; e < E; ++e)
                if (!taken[e] && (best < 0 || ranks_above(l, e, best))) best = e;
            taken[best] = 1;
            id[j] = best;
        }
        free(taken);
        if (gate == ORC_SOFTMAX) {
            double m = -INFINITY;
            if (renorm) {
                for (int j = 0; j < k; ++j) if (l[id[j]] > m) m = l[id[j]];
                double z = 0.0;
                for (int j = 0; j < k; ++j) z += exp((double)l[id[j]] - m);
                for (int j = 0; j < k; ++j) wt[j] = exp((double)l[id[j]] - m) / z;
            } else {
                for (int e = 0; e < E; ++e) if (l[e] > m) m = l[e];
                double z = 0.0;
                for (int e = 0; e < E; ++e) z += exp((double)l[e] - m);
                for (int j = 0; j < k; ++j) wt[j] = exp((double)l[id[j]] - m) / z;
            }
        } else {
            double z = 0.0;
            for (int j = 0; j < k; ++j) {
                wt[j] = 1.0 / (1.0 + exp(-(double)l[id[j]]));
                z += wt[j];
            }
            if (renorm)
                for (int j = 0; j < k; ++j) wt[j] /= z;
        }
        for (int j = 0; j < k; ++j) wt[j] *= routed_scale;
    }
}

/* ------------------------------------------------------------------------ */
/* align / permute: a plain stable counting sort                             */
/* ------------------------------------------------------------------------ */

/* Rows are the flat routed indices f = t*k + j (R = T*k of them) plus, for each
 * shared expert s, the codes R + s*T + t.  Expert segments are laid out in
 * expert order, each padded up to a multiple of `pad` rows; within a segment
 * rows appear in ascending code order; pad slots hold -1.
 *   counts[e]     rows routed to e (T for a shared expert)
 *   offsets[e]    first slot of e's segment, offsets[E_tot] = total slots
 *   sorted_rows[] slot -> row code (or -1)
 *   inv[f]        routed row f -> its slot
 * Returns the total number of slots. */
long orc_align(int T, int k, int E, int n_shared, int pad, const int32_t *ids,
               int32_t *counts, int32_t *offsets, int32_t *sorted_rows,
               int32_t *inv)
{
    long R = (long)T * k;
    int Et = E + n_shared;
    for (int e = 0; e < Et; ++e) counts[e] = 0;
    for (long f = 0; f < R; ++f) counts[ids[f]] += 1;
    for (int s = 0; s < n_shared; ++s) counts[E + s] = T;
    offsets[0] = 0;
    for (int e = 0; e < Et; ++e) {
        long padded = ((long)counts[e] + pad - 1) / pad * pad;
        offsets[e + 1] = (int32_t)(offsets[e] + padded);
    }
    long total = offsets[Et];
    for (long q = 0; q < total; ++q) sorted_rows[q] = -1;
    int32_t *fill = calloc((size_t)Et, sizeof(int32_t));
    for (long f = 0; f < R; ++f) {
        int e = ids[f];
        long slot = offsets[e] + fill[e]++;
        sorted_rows[slot] = (int32_t)f;
        inv[f] = (int32_t)slot;
    }
    for (int s = 0; s < n_shared; ++s)
        for (int t = 0; t < T; ++t)
            sorted_rows[offsets[E + s] + t] = (int32_t)(R + (long)s * T + t);
    free(fill);
    return total;
}

/* ------------------------------------------------------------------------ */
/* per-row expert math (the references for the two grouped GEMM calls)      */
/* ------------------------------------------------------------------------ */

static int expert_of_slot(const int32_t *offsets, int Et, long slot)
{
    for (int e = 0; e < Et; ++e)
        if (slot >= offsets[e] && slot < offsets[e + 1]) return e;
    return -1;
}

/* Row-wise value of an activation matrix: bf16 bits, or E4M3 codes * scale. */
static double act_val(const void *a, int adtype, double ascale, long idx)
{
    if (adtype == ORC_BF16) return orc_bf16_decode(((const uint16_t *)a)[idx]);
    return orc_e4m3_decode(((const uint8_t *)a)[idx]) * ascale;
}

static double silu(double g) { return g / (1.0 + exp(-g)); }

/* h[s][i] = SiLU(g) * u with g = sum_h xp[s][h] W1[e][i][h] * sw[e],
 * u = sum_h xp[s][h] W3[e][i][h] * sw[e] for every slot s of expert e's
 * segment; W13[e] holds the I gate rows (W1) then the I up rows (W3), each a
 * K-major row of H values.  Slots outside every segment are left untouched. */
void orc_expert_swiglu(int H, int I, int Et, const int32_t *offsets,
                       const void *xp, int adtype, double a1,
                       const void *w13, int wdtype, const float *w13_scale,
                       double *h)
{
    long total = offsets[Et];
#pragma omp parallel for schedule(dynamic, 1)
    for (long s = 0; s < total; ++s) {
        int e = expert_of_slot(offsets, Et, s);
        double sw = w13_scale ? (double)w13_scale[e] : 1.0;
        double *x = malloc(sizeof(double) * (size_t)H);
        for (int c = 0; c < H; ++c) x[c] = act_val(xp, adtype, a1, s * H + c);
        long wb = (long)e * 2 * I * H;
        for (int i = 0; i < I; ++i) {
            double g = 0.0, u = 0.0;
            for (int c = 0; c < H; ++c) {
                g += x[c] * decode_w(w13, wdtype, wb + (long)i * H + c);
                u += x[c] * decode_w(w13, wdtype, wb + (long)(I + i) * H + c);
            }
            g *= sw;
            u *= sw;
            h[s * I + i] = silu(g) * u;
        }
        free(x);
    }
}

/* y[s][o] = sum_i h[s][i] W2[e][o][i] * sw[e] for every slot s of expert e. */
void orc_expert_down(int H, int I, int Et, const int32_t *offsets,
                     const void *hin, int adtype, double a2,
                     const void *w2, int wdtype, const float *w2_scale,
                     double *y)
{
    long total = offsets[Et];
#pragma omp parallel for schedule(dynamic, 1)
    for (long s = 0; s < total; ++s) {
        int e = expert_of_slot(offsets, Et, s);
        double sw = w2_scale ? (double)w2_scale[e] : 1.0;
        double *hv = malloc(sizeof(double) * (size_t)I);
        for (int c = 0; c < I; ++c) hv[c] = act_val(hin, adtype, a2, s * I + c);
        long wb = (long)e * H * I;
        for (int o = 0; o < H; ++o) {
            double acc = 0.0;
            for (int c = 0; c < I; ++c)
                acc += hv[c] * decode_w(w2, wdtype, wb + (long)o * I + c);
            y[s * H + o] = acc * sw;
        }
        free(hv);
    }
}

/* out[t][o] = sum_j w[t][j] * y[inv[t*k+j]][o] + sum_s y[offsets[E+s]+t][o] */
void orc_combine(int T, int H, int k, int E, int n_shared, const int32_t *offsets,
                 const double *y, const double *w, const int32_t *inv, double *out)
{
    for (int t = 0; t < T; ++t)
        for (int o = 0; o < H; ++o) {
            double acc = 0.0;
            for (int j = 0; j < k; ++j)
                acc += w[(long)t * k + j] * y[(long)inv[(long)t * k + j] * H + o];
            for (int s = 0; s < n_shared; ++s)
                acc += y[((long)offsets[E + s] + t) * H + o];
            out[(long)t * H + o] = acc;
        }
}

/* ------------------------------------------------------------------------ */
/* the whole layer, per token, from the definition                          */
/* ------------------------------------------------------------------------ */

/* One expert's SwiGLU MLP on one token vector x (already in double).
 * The hidden vector h is an activation of the layer and is stored in the
 * layer's activation dtype before the down projection reads it, as the token
 * vector is: adtype == BF16 rounds h to bf16 (nearest even); adtype == E4M3
 * (the token vector was quantised with a1 by the caller) quantises it,
 * h_q = e4m3(h / a2) * a2.  Everything else is double. */
static void expert_mlp(int H, int I, int e, const double *x,
                       const void *w13, const void *w2, int wdtype,
                       const float *w13_scale, const float *w2_scale,
                       int adtype, double a2, double *hbuf, double *y)
{
    double s1 = w13_scale ? (double)w13_scale[e] : 1.0;
    double s2 = w2_scale ? (double)w2_scale[e] : 1.0;
    long b13 = (long)e * 2 * I * H, b2 = (long)e * H * I;
    for (int i = 0; i < I; ++i) {
        double g = 0.0, u = 0.0;
        for (int c = 0; c < H; ++c) {
            g += x[c] * decode_w(w13, wdtype, b13 + (long)i * H + c);
            u += x[c] * decode_w(w13, wdtype, b13 + (long)(I + i) * H + c);
        }
        double hv = silu(g * s1) * (u * s1);
        if (adtype == ORC_E4M3) hv = orc_e4m3_decode(orc_e4m3_encode(hv / a2)) * a2;
        else hv = orc_bf16_decode(orc_bf16_encode(hv));
        hbuf[i] = hv;
    }
    for (int o = 0; o < H; ++o) {
        double acc = 0.0;
        for (int c = 0; c < I; ++c) acc += hbuf[c] * decode_w(w2, wdtype, b2 + (long)o * I + c);
        y[o] = acc * s2;
    }
}

/* out[n][:] for the tokens listed in toks[0..n_tok): the routed experts of
 * token t weighted by its gate weights, plus every shared expert with weight
 * 1.  Shared experts are stored after the E routed ones in w13/w2/scales.
 * x is bf16 bits [T,H]; adtype == E4M3 quantises x with a1 (fp32 quotient,
 * as in orc_quant_e4m3_f32) before the experts. */
void orc_forward(int T, int H, int I, int E, int k, int n_shared, int gate,
                 int renorm, double routed_scale, int wdtype, int adtype,
                 const uint16_t *x, const float *logits,
                 const void *w13, const float *w13_scale,
                 const void *w2, const float *w2_scale,
                 double a1, double a2, const int32_t *toks, long n_tok,
                 double *out)
{
    (void)T;
#pragma omp parallel for schedule(dynamic, 1)
    for (long n = 0; n < n_tok; ++n) {
        int t = toks[n];
        int32_t *ids = malloc(sizeof(int32_t) * (size_t)k);
        double *w = malloc(sizeof(double) * (size_t)k);
        double *xv = malloc(sizeof(double) * (size_t)H);
        double *hb = malloc(sizeof(double) * (size_t)I);
        double *yv = malloc(sizeof(double) * (size_t)H);
        double *acc = out + n * H;
        orc_route(1, E, k, gate, renorm, routed_scale, logits + (long)t * E, ids, w);
        for (int c = 0; c < H; ++c) {
            double v = orc_bf16_decode(x[(long)t * H + c]);
            if (adtype == ORC_E4M3) {
                float q = (float)v / (float)a1;
                v = orc_e4m3_decode(orc_e4m3_encode((double)q)) * a1;
            }
            xv[c] = v;
        }
        for (int o = 0; o < H; ++o) acc[o] = 0.0;
        for (int j = 0; j < k; ++j) {
            expert_mlp(H, I, ids[j], xv, w13, w2, wdtype, w13_scale, w2_scale,
                       adtype, a2, hb, yv);
            for (int o = 0; o < H; ++o) acc[o] += w[j] * yv[o];
        }
        for (int s = 0; s < n_shared; ++s) {
            expert_mlp(H, I, E + s, xv, w13, w2, wdtype, w13_scale, w2_scale,
                       adtype, a2, hb, yv);
            for (int o = 0; o < H; ++o) acc[o] += yv[o];
        }
        free(ids); free(w); free(xv); free(hb); free(yv);
    }
}

/* max |h| over the listed tokens' routed and shared experts, the quantity a
 * static activation scale for the hidden vector is calibrated from. */
double orc_hidden_amax(int H, int I, int E, int k, int n_shared, int gate,
                       int renorm, double routed_scale, int wdtype, int adtype,
                       const uint16_t *x, const float *logits,
                       const void *w13, const float *w13_scale, double a1,
                       const int32_t *toks, long n_tok)
{
    double amax = 0.0;
#pragma omp parallel for schedule(dynamic, 1) reduction(max : amax)
    for (long n = 0; n < n_tok; ++n) {
        int t = toks[n];
        int32_t *ids = malloc(sizeof(int32_t) * (size_t)(k + n_shared));
        double *w = malloc(sizeof(double) * (size_t)k);
        double *xv = malloc(sizeof(double) * (size_t)H);
        orc_route(1, E, k, gate, renorm, routed_scale, logits + (long)t * E, ids, w);
        for (int s = 0; s < n_shared; ++s) ids[k + s] = E + s;
        for (int c = 0; c < H; ++c) {
            double v = orc_bf16_decode(x[(long)t * H + c]);
            if (adtype == ORC_E4M3) {
                float q = (float)v / (float)a1;
                v = orc_e4m3_decode(orc_e4m3_encode((double)q)) * a1;
            }
            xv[c] = v;
        }
        for (int j = 0; j < k + n_shared; ++j) {
            int e = ids[j];
            double s1 = w13_scale ? (double)w13_scale[e] : 1.0;
            long b13 = (long)e * 2 * I * H;
            for (int i = 0; i < I; ++i) {
                double g = 0.0, u = 0.0;
                for (int c = 0; c < H; ++c) {
                    g += xv[c] * decode_w(w13, wdtype, b13 + (long)i * H + c);
                    u += xv[c] * decode_w(w13, wdtype, b13 + (long)(I + i) * H + c);
                }
                double hv = fabs(silu(g * s1) * (u * s1));
                if (hv > amax) amax = hv;
            }
        }
        free(ids); free(w); free(xv);
    }
    return amax;
}

/* ------------------------------------------------------------------------ */
/* inverse rotary embedding + per-head E4M3 quantisation (attention side)    */
/* ------------------------------------------------------------------------ */

/* The Russian summary, section "Убрать лишние JIT-перекомпиляции Triton",
 * names a kernel that fuses rotary position embedding with FP8 quantisation
 * per head and must take the token count as a run-time value.  The pages say
 * nothing more, so the plain reading is:
 *   - x [T, n_heads, head_dim] bf16 holds vectors that carry the rotary
 *     rotation of their token's position p (forward RoPE: each pair (a, b)
 *     became (a c - b s, b c + a s) with c = cos(p w_i), s = sin(p w_i));
 *   - the inverse rotation undoes it: a = a' c + b' s, b = b' c - a' s;
 *   - pairs are (i, i + rot_dim/2) (the "neox" layout) or (2i, 2i+1)
 *     (interleaved), over the first rot_dim elements; the rest pass through;
 *   - c and s come from a table cos_sin [max_pos, rot_dim]: row p holds
 *     cos(p w_i) for i < rot_dim/2, then sin(p w_i);
 *   - each (token, head) vector r is then quantised to E4M3 with its own
 *     scale = amax(|r|)/448 (1 when r is all zero): code = e4m3(r / scale).
 * Every code is an integer decided by floating point, so the arithmetic is
 * fixed in fp32 as the kernel does it: each product rounded, then the sum or
 * difference rounded (no fused multiply-add), the scale and the quotient by
 * IEEE fp32 division, then round-to-nearest-even with saturation to +-448.
 * A position outside [0, max_pos) gives zero codes and scale 0. */
void orc_inv_rope_quant(int T, int n_heads, int head_dim, int rot_dim, int interleaved,
                        const uint16_t *x, const int32_t *pos, const float *cos_sin, int max_pos,
                        uint8_t *q, float *scale)
{
    const int half = rot_dim / 2;
#pragma omp parallel for schedule(static)
    for (long th = 0; th < (long)T * n_heads; ++th) {
        const long t = th / n_heads;
        const uint16_t *xh = x + th * head_dim;
        uint8_t *qh = q + th * head_dim;
        const int p = pos[t];
        if (p < 0 || p >= max_pos) {
            for (int j = 0; j < head_dim; ++j) qh[j] = 0;
            scale[th] = 0.0f;
            continue;
        }
        const float *cs = cos_sin + (long)p * rot_dim;
        float *r = malloc(sizeof(float) * (size_t)head_dim);
        float amax = 0.0f;
        for (int j = 0; j < head_dim; ++j) {
            const float y = (float)orc_bf16_decode(xh[j]);
            float v = y;
            if (j < rot_dim) {
                int i, partner, first;
                if (interleaved) {
                    i = j / 2;
                    first = (j % 2) == 0;
                    partner = first ? j + 1 : j - 1;
                } else {
                    first = j < half;
                    i = first ? j : j - half;
                    partner = first ? j + half : j - half;
                }
                const float yp = (float)orc_bf16_decode(xh[partner]);
                const float a = y * cs[i];
                const float b = yp * cs[half + i];
                v = first ? a + b : a - b;
            }
            r[j] = v;
            if (fabsf(v) > amax) amax = fabsf(v);
        }
        const float sc = amax > 0.0f ? amax / 448.0f : 1.0f;
        scale[th] = sc;
        for (int j = 0; j < head_dim; ++j) {
            const float quot = r[j] / sc;
            qh[j] = orc_e4m3_encode((double)quot);
        }
        free(r);
    }
}

int orc_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
