/*
 * moe_oracle.c -- the plain, slow, fp64 CPU oracle of the fused MoE forward.
 *
 * TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only tests/, __graft_entry__.smoke()
 * and bench.py's cpu_baseline / reference arm may load or run this file.  It
 * shares no code, header, table or helper with the CUDA library and includes
 * nothing from it.
 *
 * What it computes (sources: the web pages this project restates):
 *   - "tpu_inference/kernels/fused_moe/v1/kernel.py" (tpu-inference 0.11.1),
 *     function ref_moe: softmax over the router logits, lax.top_k, then for
 *     every token and each chosen expert x.[W_gate | W_up] -> act(gate)*up ->
 *     .W2, and the top-k-weighted sum over the chosen experts.
 *   - the same file at tpu-inference 0.13.2, ref_moe: optional division of
 *     the k chosen weights by their sum (renormalize_topk_logits).
 *   - atrex-bench operator #009 "fused_moe", reference.py Model.forward: the
 *     same function written as a loop over experts with a token mask, the
 *     vLLM weight layout w1 [E, 2I, H] (rows 0..I-1 gate, I..2I-1 up) and
 *     w2 [E, H, I] applied as F.linear, and an fp32 [T, H] output that starts
 *     at zero.
 *
 * Everything is computed in double precision from the bf16 inputs (bf16 ->
 * double is exact).  Nothing is blocked, fused or reordered beyond what the
 * definitions state; OpenMP only splits independent tokens across threads.
 *
 * Readings taken where the pages are silent or leave a choice open:
 *   - top-k order: largest logit first; equal logits go to the lowest expert
 *     index (the in-kernel argmax on the TPU page returns the lowest index).
 *     Ranking logits is ranking the exact softmax, since exp is monotone.
 *   - logits of -inf get probability 0 and can still fill the remaining
 *     slots, lowest untaken index first; an expert is never chosen twice.
 *   - expert ids outside [0, E) in the forward input are skipped (the
 *     per-expert loop of Model.forward only visits 0..E-1).
 *   - silu(z) = z / (1 + exp(-z)).
 *   - the variants of the 0.13.2 page (activation_fn, swigluoai, b1/b2 in
 *     ref_moe): gelu is the tanh form, which is what jax.nn.gelu computes
 *     when called as activation_fn calls it (approximate defaults to true);
 *     swigluoai(g, u) = (clip(u, -7, 7) + 1) * g' * sigmoid(1.702 g') with
 *     g' = min(g, 7); b1 (fp32 [E, 2I]: gate bias, then up bias) is added to
 *     the two projections before the activation, b2 (fp32 [E, H]) to the
 *     expert output before the top-k weighting.
 *   - sub-channel quantised weights (0.13.2 page: w1_scale, w2_scale,
 *     subc_quant_wsz; ref_moe multiplies each weight, widened to f32, by the
 *     scale of its block of subc_quant_wsz contraction elements): the codes
 *     are OCP FP8 E4M3 ("e4m3fn": exponent bias 7, no infinities, 0x7f and
 *     0xff are NaN), w1 [E, 2I, H] and w2 [E, H, I] in the layout above; a
 *     scale belongs to one output row and one block of `block` consecutive
 *     contraction elements: w1_scale [E, 2I, H / block], w2_scale
 *     [E, H, I / block].  The dequantised weight is code * scale, exact in
 *     double.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Planted-mistake builds: tests compile this file with -DORACLE_MUTATION=n to
 * check that the pins catch each plausible mistake.  The normal build leaves
 * ORACLE_MUTATION at 0 and every MUTATED(n) is false. */
#ifndef ORACLE_MUTATION
#define ORACLE_MUTATION 0
#endif
#define MUTATED(n) (ORACLE_MUTATION == (n))

static double bf16_to_double(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* OCP FP8 E4M3 ("e4m3fn"): sign, 4 exponent bits (bias 7), 3 mantissa
 * bits; exponent 0 is subnormal (m/8 * 2^-6); S.1111.111 is NaN; there are
 * no infinities.  Planted mistake 10 uses bias 8. */
static double e4m3_to_double(uint8_t c)
{
    const int s = c >> 7, e = (c >> 3) & 15, m = c & 7;
    const int bias = MUTATED(10) ? 8 : 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0)
        v = ldexp((double)m / 8.0, 1 - bias);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - bias);
    return s ? -v : v;
}

double oracle_e4m3_to_double(uint8_t c) { return e4m3_to_double(c); }

static double silu(double z) { return z / (1.0 + exp(-z)); }

enum { ACT_SILU = 0, ACT_GELU_TANH = 1, ACT_SWIGLUOAI = 2 };

/* 0.5 z (1 + tanh(sqrt(2/pi) (z + 0.044715 z^3))) */
static double gelu_tanh(double z)
{
    const double c = sqrt(2.0 / 3.14159265358979323846);
    if (MUTATED(8)) return 0.5 * z * (1.0 + erf(z / sqrt(2.0)));  /* the erf form */
    return 0.5 * z * (1.0 + tanh(c * (z + 0.044715 * z * z * z)));
}

/* the gated activation of activation_fn: act(gate) * up, or swigluoai */
static double gated(int act, double g, double u)
{
    if (act == ACT_GELU_TANH) return gelu_tanh(g) * u;
    if (act == ACT_SWIGLUOAI) {
        const double alpha = 1.702, limit = 7.0;
        double gc = g < limit ? g : limit;
        double uc = u < -limit ? -limit : (u > limit ? limit : u);
        return (uc + 1.0) * gc / (1.0 + exp(-alpha * gc));
    }
    return silu(g) * u;
}

int oracle_mutation(void) { return ORACLE_MUTATION; }

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/*
 * Routing: per token, p_e = exp(l_e - m) / sum_e' exp(l_e' - m) with
 * m = max_e l_e; the k experts with the largest logits in (logit desc,
 * index asc) order; w_j = p_{id_j}; with renorm, w_j /= sum_j w_j.
 * Pages: ref_moe (softmax, lax.top_k), ref_moe of 0.13.2 (renormalisation),
 * atrex-bench #009 input.py (softmax -> topk -> divide by the sum).
 * logits [T, E] fp32 row-major -> ids [T, k] int32, weights [T, k] double.
 * Returns 0, or -1 for bad arguments.
 */
int oracle_route(const float *logits, int64_t T, int E, int k, int renorm,
                 int32_t *ids, double *weights)
{
    if (T < 0 || E < 1 || k < 1 || k > E) return -1;
    char *taken = (char *)malloc((size_t)E);
    if (!taken) return -1;
    for (int64_t t = 0; t < T; ++t) {
        const float *l = logits + t * E;
        double m = -INFINITY;
        for (int e = 0; e < E; ++e)
            if ((double)l[e] > m) m = (double)l[e];
        double s = 0.0;
        for (int e = 0; e < E; ++e) s += exp((double)l[e] - m);

        memset(taken, 0, (size_t)E);
        double wsum = 0.0;
        for (int j = 0; j < k; ++j) {
            int best = -1;
            for (int e = 0; e < E; ++e) {
                if (taken[e]) continue;
                if (best < 0) { best = e; continue; }
                if (MUTATED(4) ? (l[e] >= l[best]) : (l[e] > l[best])) best = e;
            }
            taken[best] = 1;
            ids[t * k + j] = best;
            double p = exp((double)l[best] - m) / s;
            weights[t * k + j] = p;
            wsum += p;
        }
        if (renorm && !MUTATED(3))
            for (int j = 0; j < k; ++j) weights[t * k + j] /= wsum;
    }
    free(taken);
    return 0;
}

/*
 * Permutation of the flat (token, slot) indices i = t*k + j by expert: a
 * stable counting sort.  counts[e] = #{i : ids[i] == e}; offsets is the
 * exclusive prefix sum (offsets[0] = 0, offsets[E] = number of valid ids);
 * sorted_rows[offsets[e] + r] is the r-th smallest i with ids[i] == e.
 * This is the (token, k) visiting order in which the TPU kernel's scatter
 * hands rows to each expert (start_a2a_scatter) and the ascending token
 * order of Model.forward's nonzero() per expert.  Ids outside [0, E) are
 * left out.  sorted_rows must hold n entries; entries past offsets[E] are
 * set to -1.
 */
int oracle_permute(const int32_t *ids, int64_t n, int E,
                   int32_t *sorted_rows, int32_t *offsets)
{
    if (n < 0 || E < 1) return -1;
    int64_t *cursor = (int64_t *)calloc((size_t)E + 1, sizeof(int64_t));
    if (!cursor) return -1;
    for (int64_t i = 0; i < n; ++i) {
        int e = ids[i];
        if (e >= 0 && e < E) cursor[e + 1] += 1;
    }
    for (int e = 0; e < E; ++e) cursor[e + 1] += cursor[e];
    for (int e = 0; e <= E; ++e) offsets[e] = (int32_t)cursor[e];
    for (int64_t i = 0; i < n; ++i) sorted_rows[i] = -1;
    if (MUTATED(5)) {
        /* planted mistake: visit the indices from the back (unstable order) */
        for (int64_t i = n - 1; i >= 0; --i) {
            int e = ids[i];
            if (e >= 0 && e < E) sorted_rows[cursor[e]++] = (int32_t)i;
        }
    } else {
        for (int64_t i = 0; i < n; ++i) {
            int e = ids[i];
            if (e >= 0 && e < E) sorted_rows[cursor[e]++] = (int32_t)i;
        }
    }
    free(cursor);
    return 0;
}

/*
 * The expert weights: bf16 (w1, w2) or FP8 E4M3 codes with per-block scales
 * (q1, s1, q2, s2, block).  W1(e, r, h) is row r of w1[e] at contraction
 * index h, W2(e, h, i) likewise for w2[e].
 */
typedef struct {
    const uint16_t *w1, *w2;
    const uint8_t *q1, *q2;
    const float *s1, *s2;
    int64_t block;
} Weights;

static double W1(const Weights *W, int e, int64_t r, int64_t h, int64_t H, int64_t I)
{
    const size_t row = (size_t)e * 2 * I + (size_t)r;
    if (W->w1) return bf16_to_double(W->w1[row * H + h]);
    /* planted mistake 9 picks the scale block by h modulo the block count */
    const int64_t nb = H / W->block;
    const int64_t b = MUTATED(9) ? h % nb : h / W->block;
    return e4m3_to_double(W->q1[row * H + h]) * (double)W->s1[row * nb + b];
}

static double W2(const Weights *W, int e, int64_t h, int64_t i, int64_t H, int64_t I)
{
    const size_t row = (size_t)e * H + (size_t)h;
    if (W->w2) return bf16_to_double(W->w2[row * I + i]);
    const int64_t nb = I / W->block;
    const int64_t b = MUTATED(9) ? i % nb : i / W->block;
    return e4m3_to_double(W->q2[row * I + i]) * (double)W->s2[row * nb + b];
}

/*
 * One expert's gated FFN on one token, in double:
 *   g_i = W1[e][i,:] . x + b1[e][i], u_i = W1[e][I+i,:] . x + b1[e][I+i],
 *   a_i = act(g_i, u_i), y_h = W2[e][h,:] . a + b2[e][h]
 * (absent biases count as zero; act is silu(g)*u unless a variant is asked).
 * Layout of atrex-bench #009: F.linear(x, w1_e) is x . w1_e^T with w1_e of
 * shape [2I, H]; the first I outputs are gate, the next I are up;
 * F.linear(act, w2_e) with w2_e of shape [H, I].
 */
static void expert_ffn(const Weights *W, const float *b1,
                       const float *b2, int act, int e, int64_t H, int64_t I,
                       const double *x, double *a, double *y)
{
    for (int64_t i = 0; i < I; ++i) {
        int64_t rg = i, ru = I + i;
        if (MUTATED(1)) { int64_t tmp = rg; rg = ru; ru = tmp; }
        double g = 0.0, u = 0.0;
        for (int64_t h = 0; h < H; ++h) {
            g += W1(W, e, rg, h, H, I) * x[h];
            u += W1(W, e, ru, h, H, I) * x[h];
        }
        if (b1) {
            double bg = (double)b1[(size_t)e * 2 * I + i];
            double bu = (double)b1[(size_t)e * 2 * I + I + i];
            if (MUTATED(6)) { double tmp = bg; bg = bu; bu = tmp; }
            g += bg;
            u += bu;
        }
        a[i] = gated(act, g, u);
    }
    for (int64_t h = 0; h < H; ++h) {
        double acc = 0.0;
        for (int64_t i = 0; i < I; ++i) {
            /* planted mistake 2 reads W2 as if it were stored [I, H]
             * (only meaningful when H == I, which the test uses) */
            double wv = MUTATED(2) ? W2(W, e, i, h, I, H) : W2(W, e, h, i, H, I);
            acc += wv * a[i];
        }
        y[h] = acc + (b2 && !MUTATED(7) ? (double)b2[(size_t)e * H + h] : 0.0);
    }
}

/* planted mistake 7: b2 added once per chosen expert after the weighting */
static void add_b2_unweighted(const float *b2, int e, int64_t H, double *o)
{
    if (MUTATED(7) && b2)
        for (int64_t h = 0; h < H; ++h) o[h] += (double)b2[(size_t)e * H + h];
}

/*
 * Formulation A, the per-token loop of ref_moe: for every token t (or only
 * the tokens listed in `rows`, when nrows >= 0), out[t] = sum over j of
 * w[t,j] * FFN_{ids[t,j]}(x_t), with j ascending.  Ids outside [0, E) are
 * skipped.  hidden [T,H], w1 [E,2I,H], w2 [E,H,I] are bf16 bit patterns;
 * topk_w [T,k] double; out is [nrows or T, H] double, overwritten.
 */
static int token_loop(const uint16_t *hidden, const Weights *W, const float *b1,
                      const float *b2, int act, const double *topk_w, const int32_t *ids,
                      int64_t T, int64_t H, int64_t I, int E, int k,
                      const int64_t *rows, int64_t nrows, double *out)
{
    if (act < ACT_SILU || act > ACT_SWIGLUOAI) return -1;
    if (T < 0 || H < 1 || I < 1 || E < 1 || k < 1) return -1;
    int64_t n = nrows >= 0 ? nrows : T;
    int err = 0;
#pragma omp parallel
    {
        double *x = (double *)malloc(sizeof(double) * (size_t)H);
        double *a = (double *)malloc(sizeof(double) * (size_t)I);
        double *y = (double *)malloc(sizeof(double) * (size_t)H);
        if (!x || !a || !y) {
#pragma omp atomic write
            err = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t r = 0; r < n; ++r) {
                int64_t t = nrows >= 0 ? rows[r] : r;
                double *o = out + (size_t)r * H;
                for (int64_t h = 0; h < H; ++h) o[h] = 0.0;
                if (t < 0 || t >= T) continue;
                for (int64_t h = 0; h < H; ++h) x[h] = bf16_to_double(hidden[(size_t)t * H + h]);
                for (int j = 0; j < k; ++j) {
                    int e = ids[t * k + j];
                    if (e < 0 || e >= E) continue;
                    expert_ffn(W, b1, b2, act, e, H, I, x, a, y);
                    double wj = topk_w[t * k + j];
                    for (int64_t h = 0; h < H; ++h) o[h] += wj * y[h];
                    add_b2_unweighted(b2, e, H, o);
                }
            }
        }
        free(x); free(a); free(y);
    }
    return err ? -1 : 0;
}

int oracle_moe_token_loop_ex(const uint16_t *hidden, const uint16_t *w1,
                             const uint16_t *w2, const float *b1, const float *b2,
                             int act, const double *topk_w, const int32_t *ids,
                             int64_t T, int64_t H, int64_t I, int E, int k,
                             const int64_t *rows, int64_t nrows, double *out)
{
    const Weights W = {w1, w2, NULL, NULL, NULL, NULL, 0};
    return token_loop(hidden, &W, b1, b2, act, topk_w, ids, T, H, I, E, k, rows, nrows, out);
}

/*
 * Formulation A on FP8 E4M3 weights with per-block scales (silu, no
 * biases): q1 [E, 2I, H] codes, s1 [E, 2I, H / block]; q2 [E, H, I] codes,
 * s2 [E, H, I / block].  block must divide H and I.
 */
int oracle_moe_token_loop_fp8(const uint16_t *hidden, const uint8_t *q1, const float *s1,
                              const uint8_t *q2, const float *s2, int64_t block,
                              const double *topk_w, const int32_t *ids, int64_t T,
                              int64_t H, int64_t I, int E, int k, const int64_t *rows,
                              int64_t nrows, double *out)
{
    if (block < 1 || H % block != 0 || I % block != 0) return -1;
    const Weights W = {NULL, NULL, q1, q2, s1, s2, block};
    return token_loop(hidden, &W, NULL, NULL, ACT_SILU, topk_w, ids, T, H, I, E, k, rows,
                      nrows, out);
}

int oracle_moe_token_loop(const uint16_t *hidden, const uint16_t *w1,
                          const uint16_t *w2, const double *topk_w,
                          const int32_t *ids, int64_t T, int64_t H, int64_t I,
                          int E, int k, const int64_t *rows, int64_t nrows,
                          double *out)
{
    return oracle_moe_token_loop_ex(hidden, w1, w2, NULL, NULL, ACT_SILU, topk_w, ids,
                                    T, H, I, E, k, rows, nrows, out);
}

/*
 * Formulation B, the per-expert mask loop of Model.forward: out = 0; for
 * e = 0..E-1: w_hat[t] = sum_j w[t,j] * [ids[t,j] == e]; for every token
 * with w_hat[t] != 0 (ascending t): out[t] += w_hat[t] * FFN_e(x_t).
 * A token routed twice to e thus gets the summed weight.  Same argument
 * layout as formulation A (all T rows).
 */
static int expert_loop(const uint16_t *hidden, const Weights *W, const float *b1,
                       const float *b2, int act, const double *topk_w, const int32_t *ids,
                       int64_t T, int64_t H, int64_t I, int E, int k, double *out)
{
    if (T < 0 || H < 1 || I < 1 || E < 1 || k < 1) return -1;
    if (act < ACT_SILU || act > ACT_SWIGLUOAI) return -1;
    double *what = (double *)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
    if (!what) return -1;
    for (int64_t i = 0; i < T * H; ++i) out[i] = 0.0;
    int err = 0;
    for (int e = 0; e < E; ++e) {
        for (int64_t t = 0; t < T; ++t) {
            double s = 0.0;
            for (int j = 0; j < k; ++j)
                if (ids[t * k + j] == e) s += topk_w[t * k + j];
            what[t] = s;
        }
#pragma omp parallel
        {
            double *x = (double *)malloc(sizeof(double) * (size_t)H);
            double *a = (double *)malloc(sizeof(double) * (size_t)I);
            double *y = (double *)malloc(sizeof(double) * (size_t)H);
            if (!x || !a || !y) {
#pragma omp atomic write
                err = 1;
            } else {
#pragma omp for schedule(dynamic, 1)
                for (int64_t t = 0; t < T; ++t) {
                    if (what[t] == 0.0) continue;
                    for (int64_t h = 0; h < H; ++h) x[h] = bf16_to_double(hidden[(size_t)t * H + h]);
                    expert_ffn(W, b1, b2, act, e, H, I, x, a, y);
                    double *o = out + (size_t)t * H;
                    for (int64_t h = 0; h < H; ++h) o[h] += what[t] * y[h];
                }
            }
            free(x); free(a); free(y);
        }
    }
    free(what);
    return err ? -1 : 0;
}

int oracle_moe_expert_loop_ex(const uint16_t *hidden, const uint16_t *w1,
                              const uint16_t *w2, const float *b1, const float *b2,
                              int act, const double *topk_w, const int32_t *ids,
                              int64_t T, int64_t H, int64_t I, int E, int k, double *out)
{
    const Weights W = {w1, w2, NULL, NULL, NULL, NULL, 0};
    return expert_loop(hidden, &W, b1, b2, act, topk_w, ids, T, H, I, E, k, out);
}

/* Formulation B on FP8 E4M3 weights with per-block scales (as above). */
int oracle_moe_expert_loop_fp8(const uint16_t *hidden, const uint8_t *q1, const float *s1,
                               const uint8_t *q2, const float *s2, int64_t block,
                               const double *topk_w, const int32_t *ids, int64_t T,
                               int64_t H, int64_t I, int E, int k, double *out)
{
    if (block < 1 || H % block != 0 || I % block != 0) return -1;
    const Weights W = {NULL, NULL, q1, q2, s1, s2, block};
    return expert_loop(hidden, &W, NULL, NULL, ACT_SILU, topk_w, ids, T, H, I, E, k, out);
}

int oracle_moe_expert_loop(const uint16_t *hidden, const uint16_t *w1,
                           const uint16_t *w2, const double *topk_w,
                           const int32_t *ids, int64_t T, int64_t H, int64_t I,
                           int E, int k, double *out)
{
    return oracle_moe_expert_loop_ex(hidden, w1, w2, NULL, NULL, ACT_SILU, topk_w, ids, T, H,
                                     I, E, k, out);
}
