/*
 * moe_oracle.c -- plain, slow, fp64 CPU oracle for the sparse MoE layer forward.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file; only the tests, the smoke check and the benchmark's CPU
 * baseline leg use it.  It shares no code, header or table with the CUDA
 * library.
 *
 * What it computes (the layer equation of "Mixtral of Experts", section 2.1
 * "Sparse Mixture of Experts", as restated on the learn.ifs.name flash-card
 * page; the three routing lines and Steps 1-4 of Part 3 of "Mixture of
 * Experts: Why Mixtral Only Wakes Up Two Specialists"):
 *
 *   y = sum_{i=0}^{n-1} Softmax(TopK(x . W_g))_i * SwiGLU_i(x)
 *   SwiGLU_i(x) = (silu(x . w1_i) (*) (x . w3_i)) . w2_i,  silu(z) = z * sigmoid(z)
 *
 * Every value is read from its stored type (fp32, bf16 bits, or fp64) and
 * widened exactly to double; all arithmetic is in double.  Loops follow the
 * definitions directly: no blocking, no fusion, no reordering beyond the plain
 * ascending-index sums.
 *
 * Readings of points the pages leave open:
 *   - top-K order: descending logit; equal logits -> lower expert index first
 *     (torch.topk, which the pages quote, fixes neither);
 *   - the softmax runs over the K kept logits only (the others are -inf);
 *   - the three expert matrices: w1, w3 [d][ffn] (gate and up), w2 [ffn][d]
 *     (down), no biases;
 *   - dispatch order: rows grouped by expert ascending, tokens ascending within
 *     an expert (the pages say only that unchosen experts are skipped).
 *
 * Error behaviour: functions return 0 on success and -1 on a bad argument
 * (null pointer, non-positive size, K > n); they never abort.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { OR_F32 = 0, OR_BF16 = 1, OR_F64 = 2 };

/* Element i of a stored array, widened exactly to double. */
static double elem(const void *base, int dt, size_t i)
{
    if (dt == OR_F64)
        return ((const double *)base)[i];
    if (dt == OR_F32)
        return (double)((const float *)base)[i];
    /* bf16: the 16 stored bits are the upper half of an IEEE binary32 value */
    uint32_t u = (uint32_t)((const uint16_t *)base)[i] << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static int dt_ok(int dt) { return dt == OR_F32 || dt == OR_BF16 || dt == OR_F64; }

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n > 0)
        omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* silu(z) = z * sigmoid(z) = z / (1 + e^{-z}) */
double oracle_silu(double z) { return z / (1.0 + exp(-z)); }

/*
 * Router for one token: logits L_e = sum_j x_j W_g[j][e] (the bias-free
 * linear gate, Step 1), keep the K largest (Step 2), softmax over the kept K
 * (Step 3).  idx gets the K expert indices in selection order; gate the K
 * weights; logits (n values) is optional.
 */
static void route_one(int d, int n, int K, const void *x, int x_dt, size_t xoff,
                      const void *Wg, int wg_dt, int32_t *idx, double *gate,
                      double *L, unsigned char *taken)
{
    for (int e = 0; e < n; ++e) {
        double s = 0.0;
        for (int j = 0; j < d; ++j)
            s += elem(x, x_dt, xoff + (size_t)j) * elem(Wg, wg_dt, (size_t)j * n + e);
        L[e] = s;
        taken[e] = 0;
    }
    /* Top-K: K rounds of "largest remaining logit"; scanning e upwards with a
     * strict '>' keeps the lower index on equal logits. */
    for (int k = 0; k < K; ++k) {
        int best = -1;
        for (int e = 0; e < n; ++e)
            if (!taken[e] && (best < 0 || L[e] > L[best]))
                best = e;
        taken[best] = 1;
        idx[k] = best;
    }
    /* Softmax over the kept logits (the others are -inf and contribute 0). */
    double m = L[idx[0]];
    double z = 0.0;
    for (int k = 0; k < K; ++k)
        z += exp(L[idx[k]] - m);
    for (int k = 0; k < K; ++k)
        gate[k] = exp(L[idx[k]] - m) / z;
}

int oracle_router(int64_t T, int d, int n, int K, const void *x, int x_dt,
                  const void *Wg, int wg_dt, int32_t *idx, double *gate, double *logits)
{
    if (T < 0 || d <= 0 || n <= 0 || K <= 0 || K > n || !dt_ok(x_dt) || !dt_ok(wg_dt))
        return -1;
    if (T == 0)
        return 0;
    if (!x || !Wg || !idx || !gate)
        return -1;
    int bad = 0;
#pragma omp parallel
    {
        double *L = (double *)malloc(sizeof(double) * (size_t)n);
        unsigned char *taken = (unsigned char *)malloc((size_t)n);
        if (!L || !taken) {
#pragma omp atomic write
            bad = 1;
        } else {
#pragma omp for schedule(static)
            for (int64_t t = 0; t < T; ++t) {
                route_one(d, n, K, x, x_dt, (size_t)t * d, Wg, wg_dt, idx + t * K, gate + t * K, L, taken);
                if (logits)
                    memcpy(logits + t * n, L, sizeof(double) * (size_t)n);
            }
        }
        free(L);
        free(taken);
    }
    return bad ? -1 : 0;
}

/*
 * One expert e on one token: out[d] = (silu(x.w1_e) * (x.w3_e)) . w2_e.
 * a, b, h are caller scratch of ffn doubles.
 */
static void expert_one(int d, int F, const void *x, int x_dt, size_t xoff,
                       const void *w1, const void *w3, const void *w2, int w_dt, int e,
                       double *a, double *b, double *out)
{
    size_t ebase1 = (size_t)e * (size_t)d * (size_t)F; /* w1[e], w3[e]: [d][F] */
    size_t ebase2 = (size_t)e * (size_t)F * (size_t)d; /* w2[e]: [F][d] */
    for (int f = 0; f < F; ++f) {
        a[f] = 0.0;
        b[f] = 0.0;
    }
    for (int j = 0; j < d; ++j) {
        double xj = elem(x, x_dt, xoff + (size_t)j);
        size_t row = ebase1 + (size_t)j * F;
        for (int f = 0; f < F; ++f) {
            a[f] += xj * elem(w1, w_dt, row + f);
            b[f] += xj * elem(w3, w_dt, row + f);
        }
    }
    for (int f = 0; f < F; ++f)
        a[f] = oracle_silu(a[f]) * b[f]; /* a now holds h */
    for (int i = 0; i < d; ++i)
        out[i] = 0.0;
    for (int f = 0; f < F; ++f) {
        size_t row = ebase2 + (size_t)f * d;
        for (int i = 0; i < d; ++i)
            out[i] += a[f] * elem(w2, w_dt, row + i);
    }
}

/* Gates in the activations' dtype: the routing code quoted in Part 3 of the
 * neobadger page computes the softmax in fp32 and then casts the weights to
 * the inputs' dtype.  For bf16 inputs each gate becomes: the fp64 gate rounded
 * to fp32 (round to nearest even), then that float rounded to bf16 (its upper
 * 16 bits, round to nearest even on the 16 dropped bits). */
int oracle_gates_to_bf16(int64_t count, const double *gate, double *out)
{
    if (count < 0 || (count > 0 && (!gate || !out)))
        return -1;
    for (int64_t i = 0; i < count; ++i) {
        float f = (float)gate[i];
        uint32_t u;
        memcpy(&u, &f, sizeof u);
        if ((u & 0x7f800000u) == 0x7f800000u) { /* inf or nan: keep (not reached by gates) */
            out[i] = (double)f;
            continue;
        }
        uint32_t low = u & 0xffffu;
        uint32_t hi = u >> 16;
        if (low > 0x8000u || (low == 0x8000u && (hi & 1u)))
            hi += 1u; /* carries into the exponent when the mantissa overflows */
        uint32_t r = hi << 16;
        float g;
        memcpy(&g, &r, sizeof g);
        out[i] = (double)g;
    }
    return 0;
}

int oracle_expert(int d, int F, int n, int e, const void *x_row, int x_dt,
                  const void *w1, const void *w3, const void *w2, int w_dt, double *out)
{
    if (d <= 0 || F <= 0 || n <= 0 || e < 0 || e >= n || !x_row || !w1 || !w3 || !w2 || !out ||
        !dt_ok(x_dt) || !dt_ok(w_dt))
        return -1;
    double *a = (double *)malloc(sizeof(double) * (size_t)F);
    double *b = (double *)malloc(sizeof(double) * (size_t)F);
    if (!a || !b) {
        free(a);
        free(b);
        return -1;
    }
    expert_one(d, F, x_row, x_dt, 0, w1, w3, w2, w_dt, e, a, b, out);
    free(a);
    free(b);
    return 0;
}

/*
 * y[t] = sum_k gate[t][k] * SwiGLU_{idx[t][k]}(x[t]) under a routing given
 * from outside (the gate-weighted additive combine of Step 4).
 */
int oracle_forward_with_routing(int64_t T, int d, int F, int n, int K,
                                const void *x, int x_dt, const int32_t *idx, const double *gate,
                                const void *w1, const void *w3, const void *w2, int w_dt, double *y)
{
    if (T < 0 || d <= 0 || F <= 0 || n <= 0 || K <= 0 || K > n || !dt_ok(x_dt) || !dt_ok(w_dt))
        return -1;
    if (T == 0)
        return 0;
    if (!x || !idx || !gate || !w1 || !w3 || !w2 || !y)
        return -1;
    for (int64_t i = 0; i < T * K; ++i)
        if (idx[i] < 0 || idx[i] >= n)
            return -1;
    int bad = 0;
#pragma omp parallel
    {
        double *a = (double *)malloc(sizeof(double) * (size_t)F);
        double *b = (double *)malloc(sizeof(double) * (size_t)F);
        double *o = (double *)malloc(sizeof(double) * (size_t)d);
        if (!a || !b || !o) {
#pragma omp atomic write
            bad = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t t = 0; t < T; ++t) {
                double *yt = y + t * d;
                for (int i = 0; i < d; ++i)
                    yt[i] = 0.0;
                for (int k = 0; k < K; ++k) {
                    expert_one(d, F, x, x_dt, (size_t)t * d, w1, w3, w2, w_dt, idx[t * K + k], a, b, o);
                    double g = gate[t * K + k];
                    for (int i = 0; i < d; ++i)
                        yt[i] += g * o[i];
                }
            }
        }
        free(a);
        free(b);
        free(o);
    }
    return bad ? -1 : 0;
}

/* The whole layer: route, then combine the chosen experts. */
int oracle_moe_forward(int64_t T, int d, int F, int n, int K,
                       const void *x, int x_dt, const void *Wg, int wg_dt,
                       const void *w1, const void *w3, const void *w2, int w_dt,
                       double *y, int32_t *idx, double *gate)
{
    int rc = oracle_router(T, d, n, K, x, x_dt, Wg, wg_dt, idx, gate, NULL);
    if (rc)
        return rc;
    return oracle_forward_with_routing(T, d, F, n, K, x, x_dt, idx, gate, w1, w3, w2, w_dt, y);
}

/*
 * Dispatch: the (token, slot) pairs grouped into per-expert segments.  The
 * method only says that experts with a zero gate are skipped; this lays the
 * chosen pairs out expert by expert (ascending), tokens ascending inside an
 * expert.  counts[n], offsets[n+1], row_token[T*K] (token of each row),
 * token_row[T*K] (row of each (token, slot) pair).
 */
int oracle_dispatch(int64_t T, int n, int K, const int32_t *idx, int64_t *counts,
                    int64_t *offsets, int64_t *row_token, int64_t *token_row)
{
    if (T < 0 || n <= 0 || K <= 0 || K > n || !counts || !offsets)
        return -1;
    if (T > 0 && (!idx || !row_token || !token_row))
        return -1;
    for (int64_t i = 0; i < T * K; ++i)
        if (idx[i] < 0 || idx[i] >= n)
            return -1;
    int64_t row = 0;
    for (int e = 0; e < n; ++e) {
        offsets[e] = row;
        for (int64_t t = 0; t < T; ++t)
            for (int k = 0; k < K; ++k)
                if (idx[t * K + k] == e) {
                    row_token[row] = t;
                    token_row[t * K + k] = row;
                    ++row;
                }
        counts[e] = row - offsets[e];
    }
    offsets[n] = row;
    return 0;
}

/*
 * Load-balancing statistics of the router ("Mixture of Experts: Why Mixtral
 * Only Wakes Up Two Specialists", Part 5, "Tool 2: a fine for favouritism",
 * after the Switch Transformers paper):
 *   f_i = share of the routed (token, slot) pairs sent to expert i
 *         (count_i / (T*K); with K = 1 this is the share of tokens);
 *   P_i = average over the tokens of the router's probability for expert i,
 *         the softmax over ALL n logits;
 *   aux = alpha * n * sum_i f_i * P_i.
 * idx are the routed experts ([T][K], e.g. from oracle_router); the logits
 * are recomputed here from x and W_g.
 */
int oracle_router_stats(int64_t T, int d, int n, int K, const void *x, int x_dt, const void *Wg,
                        int wg_dt, const int32_t *idx, double alpha, double *f, double *P,
                        double *aux)
{
    if (T <= 0 || d <= 0 || n <= 0 || K <= 0 || K > n || !x || !Wg || !idx || !f || !P || !aux ||
        !dt_ok(x_dt) || !dt_ok(wg_dt))
        return -1;
    for (int64_t i = 0; i < T * K; ++i)
        if (idx[i] < 0 || idx[i] >= n)
            return -1;
    double *L = (double *)malloc(sizeof(double) * (size_t)n);
    if (!L)
        return -1;
    for (int e = 0; e < n; ++e) {
        f[e] = 0.0;
        P[e] = 0.0;
    }
    for (int64_t t = 0; t < T; ++t) {
        double m = 0.0;
        for (int e = 0; e < n; ++e) {
            double s = 0.0;
            for (int j = 0; j < d; ++j)
                s += elem(x, x_dt, (size_t)t * d + j) * elem(Wg, wg_dt, (size_t)j * n + e);
            L[e] = s;
            if (e == 0 || s > m)
                m = s;
        }
        double z = 0.0;
        for (int e = 0; e < n; ++e)
            z += exp(L[e] - m);
        for (int e = 0; e < n; ++e)
            P[e] += exp(L[e] - m) / z;
        for (int k = 0; k < K; ++k)
            f[idx[t * K + k]] += 1.0;
    }
    double acc = 0.0;
    for (int e = 0; e < n; ++e) {
        f[e] /= (double)(T * K);
        P[e] /= (double)T;
        acc += f[e] * P[e];
    }
    *aux = alpha * (double)n * acc;
    free(L);
    return 0;
}

/*
 * Dispatch with an expert capacity (the Switch paper's capacity, Part 5 of
 * the neobadger page: "the tokens in the batch divided by the number of
 * experts, times a capacity factor"; the pairs that overflow are dropped and
 * skip the expert).  capacity = the most (token, slot) pairs one expert takes;
 * the first ones in dispatch order (tokens ascending) are kept.  Dropped pairs
 * get token_row = -1 and are not counted.  Outputs as oracle_dispatch.
 */
int oracle_dispatch_capacity(int64_t T, int n, int K, const int32_t *idx, int64_t capacity,
                             int64_t *counts, int64_t *offsets, int64_t *row_token,
                             int64_t *token_row)
{
    if (T < 0 || n <= 0 || K <= 0 || K > n || capacity < 0 || !counts || !offsets)
        return -1;
    if (T > 0 && (!idx || !row_token || !token_row))
        return -1;
    for (int64_t i = 0; i < T * K; ++i)
        if (idx[i] < 0 || idx[i] >= n)
            return -1;
    int64_t row = 0;
    for (int e = 0; e < n; ++e) {
        offsets[e] = row;
        for (int64_t t = 0; t < T; ++t)
            for (int k = 0; k < K; ++k)
                if (idx[t * K + k] == e) {
                    if (row - offsets[e] < capacity) {
                        row_token[row] = t;
                        token_row[t * K + k] = row;
                        ++row;
                    } else {
                        token_row[t * K + k] = -1;
                    }
                }
        counts[e] = row - offsets[e];
    }
    offsets[n] = row;
    return 0;
}

/*
 * Expert-choice routing ("Mixtral of Experts? Mixture of Experts? Try to
 * explain Mixtral 8x7B", section "How Experts Are Chosen", item 2: experts
 * choose which tokens to process, each with a fixed capacity).  Reading taken:
 *   S[t][e] = softmax over the n experts of the logits x_t . W_g;
 *   expert e keeps the C tokens with the largest S[.][e] (equal scores: lower
 *   token index first), listed in sel_token[e][0..C) by ascending token, with
 *   sel_gate[e][j] = S[token][e];
 *   y[t] = sum over the experts e that kept t (ascending e) of S[t][e] * SwiGLU_e(x_t);
 *   a token no expert kept gets y[t] = 0.
 * Requires 1 <= C <= T.
 */
static const double *g_sort_S; /* qsort context: one expert's column */
static int g_sort_n, g_sort_e;

static int cmp_score_desc_token_asc(const void *a, const void *b)
{
    int64_t ta = *(const int64_t *)a, tb = *(const int64_t *)b;
    double sa = g_sort_S[ta * g_sort_n + g_sort_e], sb = g_sort_S[tb * g_sort_n + g_sort_e];
    if (sa > sb) return -1;
    if (sa < sb) return 1;
    return (ta < tb) ? -1 : (ta > tb);
}

static int cmp_i64(const void *a, const void *b)
{
    int64_t x = *(const int64_t *)a, y = *(const int64_t *)b;
    return (x < y) ? -1 : (x > y);
}

int oracle_expert_choice(int64_t T, int d, int F, int n, int64_t C, const void *x, int x_dt,
                         const void *Wg, int wg_dt, const void *w1, const void *w3, const void *w2,
                         int w_dt, double *y, int64_t *sel_token, double *sel_gate)
{
    if (T <= 0 || d <= 0 || F <= 0 || n <= 0 || C < 1 || C > T || !x || !Wg || !w1 || !w3 || !w2 ||
        !y || !sel_token || !sel_gate || !dt_ok(x_dt) || !dt_ok(wg_dt) || !dt_ok(w_dt))
        return -1;
    double *S = (double *)malloc(sizeof(double) * (size_t)T * n);
    int64_t *order = (int64_t *)malloc(sizeof(int64_t) * (size_t)T);
    double *a = (double *)malloc(sizeof(double) * (size_t)F);
    double *b = (double *)malloc(sizeof(double) * (size_t)F);
    double *o = (double *)malloc(sizeof(double) * (size_t)d);
    if (!S || !order || !a || !b || !o) {
        free(S); free(order); free(a); free(b); free(o);
        return -1;
    }
    /* router probabilities: softmax over all n logits of each token */
    for (int64_t t = 0; t < T; ++t) {
        double m = 0.0;
        for (int e = 0; e < n; ++e) {
            double s = 0.0;
            for (int j = 0; j < d; ++j)
                s += elem(x, x_dt, (size_t)t * d + j) * elem(Wg, wg_dt, (size_t)j * n + e);
            S[t * n + e] = s;
            if (e == 0 || s > m) m = s;
        }
        double z = 0.0;
        for (int e = 0; e < n; ++e)
            z += exp(S[t * n + e] - m);
        for (int e = 0; e < n; ++e)
            S[t * n + e] = exp(S[t * n + e] - m) / z;
    }
    /* each expert keeps its C best tokens */
    for (int e = 0; e < n; ++e) {
        for (int64_t t = 0; t < T; ++t)
            order[t] = t;
        g_sort_S = S;
        g_sort_n = n;
        g_sort_e = e;
        qsort(order, (size_t)T, sizeof(int64_t), cmp_score_desc_token_asc);
        qsort(order, (size_t)C, sizeof(int64_t), cmp_i64);
        for (int64_t j = 0; j < C; ++j) {
            sel_token[e * C + j] = order[j];
            sel_gate[e * C + j] = S[order[j] * n + e];
        }
    }
    /* y: the chosen experts' outputs, weighted by the router probability */
    for (int64_t i = 0; i < T * (int64_t)d; ++i)
        y[i] = 0.0;
    for (int e = 0; e < n; ++e)
        for (int64_t j = 0; j < C; ++j) {
            int64_t t = sel_token[e * C + j];
            expert_one(d, F, x, x_dt, (size_t)t * d, w1, w3, w2, w_dt, e, a, b, o);
            for (int i = 0; i < d; ++i)
                y[t * d + i] += sel_gate[e * C + j] * o[i];
        }
    free(S); free(order); free(a); free(b); free(o);
    return 0;
}

/*
 * FP8 E4M3 expert weights and activations (the "load it in 4-bit" option of
 * Part 4 of the neobadger page, here at 8 bits).  E4M3 as the OCP 8-bit
 * floating point specification defines it: 1 sign bit, 4 exponent bits (bias
 * 7), 3 mantissa bits, subnormals, no infinities, largest finite 448, NaN =
 * S.1111.111.  Encoding rounds to nearest, ties to even, and saturates finite
 * values beyond 448 to +-448.
 */
double oracle_e4m3_decode(int code)
{
    int s = (code >> 7) & 1, e = (code >> 3) & 15, m = code & 7;
    double v;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);           /* subnormal: m/8 * 2^-6 */
    else
        v = ldexp(1.0 + m / 8.0, e - 7);
    return s ? -v : v;
}

static double round_half_even(double v)
{
    double f = floor(v), r = v - f;
    if (r > 0.5) return f + 1.0;
    if (r < 0.5) return f;
    return (fmod(f, 2.0) == 0.0) ? f : f + 1.0;
}

int oracle_e4m3_encode(double v)
{
    if (isnan(v))
        return 0x7F;
    int s = signbit(v) ? 1 : 0;
    double a = fabs(v), q;
    if (a >= 448.0) {
        q = 448.0;
    } else if (a < ldexp(1.0, -6)) {
        q = ldexp(round_half_even(ldexp(a, 9)), -9);     /* multiples of 2^-9 */
    } else {
        int E;
        frexp(a, &E);                                     /* a = f * 2^E, 0.5 <= f < 1 */
        double step = ldexp(1.0, E - 1 - 3);              /* 3 mantissa bits below 2^(E-1) */
        q = round_half_even(a / step) * step;
        if (q > 448.0) q = 448.0;
    }
    /* q is representable: find its code */
    int code;
    if (q < ldexp(1.0, -6)) {
        code = (int)ldexp(q, 9);                          /* e = 0, m = q / 2^-9 */
    } else {
        int E;
        double f = frexp(q, &E);                          /* q = f * 2^E, f in [0.5, 1) */
        int e = E - 1 + 7;
        int m = (int)((f * 2.0 - 1.0) * 8.0 + 0.5);
        code = (e << 3) | m;
    }
    return (s << 7) | code;
}

/* Scale of a group of values: max |v| / 448 in fp32 (1 when the group is all
 * zero), the same precision the GPU uses, so both sides pick the same codes. */
static float e4m3_scale_f32(float amax) { return amax > 0.0f ? amax / 448.0f : 1.0f; }

/* Codes of v / scale, the quotient taken in fp32. */
static int e4m3_code_f32(float v, float scale) { return oracle_e4m3_encode((double)(v / scale)); }

/*
 * Per-channel weight quantization: w [n][rows][cols] (bf16 bits or fp32) ->
 * codes [n][rows][cols] (uint8) and scales [n][cols] (fp32): one scale per
 * output column over all rows (the reduction dimension).
 */
int oracle_quantize_weights_e4m3(int n, int rows, int cols, const void *w, int w_dt, uint8_t *codes,
                                 float *scales)
{
    if (n <= 0 || rows <= 0 || cols <= 0 || !w || !codes || !scales || !dt_ok(w_dt))
        return -1;
#pragma omp parallel for collapse(2) schedule(static)
    for (int e = 0; e < n; ++e)
        for (int c = 0; c < cols; ++c) {
            float amax = 0.0f;
            for (int r = 0; r < rows; ++r) {
                float v = (float)elem(w, w_dt, ((size_t)e * rows + r) * cols + c);
                if (fabsf(v) > amax) amax = fabsf(v);
            }
            float s = e4m3_scale_f32(amax);
            scales[(size_t)e * cols + c] = s;
            for (int r = 0; r < rows; ++r) {
                size_t i = ((size_t)e * rows + r) * cols + c;
                codes[i] = (uint8_t)e4m3_code_f32((float)elem(w, w_dt, i), s);
            }
        }
    return 0;
}

/* bf16 rounding (nearest, ties to even) of a float, as a float */
static float round_bf16(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    u = (u + 0x7FFFu + ((u >> 16) & 1u)) & 0xFFFF0000u;
    float r;
    memcpy(&r, &u, 4);
    return r;
}

/*
 * The layer with E4M3 experts under a given routing (idx, gate as for
 * oracle_forward_with_routing), each step in the order and precision of the
 * quantized path:
 *   x row -> per-row scale sx = max|x| / 448 (fp32), codes qx;
 *   a = sum_j qx_j * q1_jf (exact products, summed in double) * sx * s1_f,
 *   b likewise with w3; h = silu(a) * b, rounded to fp32 then bf16 (the
 *   stored hidden layer);
 *   h row -> sh = max|h| / 448, codes qh;
 *   o_i = sum_f qh_f * q2_fi * sh * s2_i;  y = sum_k gate_k * o (double).
 * q1, q3: [n][d][F] codes with scales s1, s3 [n][F]; q2: [n][F][d] with s2 [n][d].
 */
int oracle_forward_e4m3(int64_t T, int d, int F, int n, int K, const void *x, int x_dt,
                        const int32_t *idx, const double *gate, const uint8_t *q1, const float *s1,
                        const uint8_t *q3, const float *s3, const uint8_t *q2, const float *s2,
                        double *y)
{
    if (T <= 0 || d <= 0 || F <= 0 || n <= 0 || K <= 0 || !x || !idx || !gate || !q1 || !s1 || !q3 ||
        !s3 || !q2 || !s2 || !y || !dt_ok(x_dt))
        return -1;
    for (int64_t i = 0; i < T * K; ++i)
        if (idx[i] < 0 || idx[i] >= n)
            return -1;
    double lut[256];
    for (int c = 0; c < 256; ++c)
        lut[c] = oracle_e4m3_decode(c);
    int bad = 0;
#pragma omp parallel
    {
        double *qx = (double *)malloc(sizeof(double) * (size_t)d);
        double *a = (double *)malloc(sizeof(double) * (size_t)F);
        double *b = (double *)malloc(sizeof(double) * (size_t)F);
        float *hf = (float *)malloc(sizeof(float) * (size_t)F);
        double *qh = (double *)malloc(sizeof(double) * (size_t)F);
        if (!qx || !a || !b || !hf || !qh) {
#pragma omp atomic write
            bad = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t t = 0; t < T; ++t) {
                float amax = 0.0f;
                for (int j = 0; j < d; ++j) {
                    float v = (float)elem(x, x_dt, (size_t)t * d + j);
                    if (fabsf(v) > amax) amax = fabsf(v);
                }
                float sx = e4m3_scale_f32(amax);
                for (int j = 0; j < d; ++j)
                    qx[j] = lut[e4m3_code_f32((float)elem(x, x_dt, (size_t)t * d + j), sx)];
                double *yt = y + t * d;
                for (int i = 0; i < d; ++i)
                    yt[i] = 0.0;
                for (int k = 0; k < K; ++k) {
                    int e = idx[t * K + k];
                    size_t base1 = (size_t)e * d * F, base2 = (size_t)e * F * d;
                    for (int f = 0; f < F; ++f)
                        a[f] = b[f] = 0.0;
                    for (int j = 0; j < d; ++j)
                        for (int f = 0; f < F; ++f) {
                            a[f] += qx[j] * lut[q1[base1 + (size_t)j * F + f]];
                            b[f] += qx[j] * lut[q3[base1 + (size_t)j * F + f]];
                        }
                    float hmax = 0.0f;
                    for (int f = 0; f < F; ++f) {
                        double av = a[f] * sx * s1[(size_t)e * F + f];
                        double bv = b[f] * sx * s3[(size_t)e * F + f];
                        hf[f] = round_bf16((float)(oracle_silu(av) * bv));
                        if (fabsf(hf[f]) > hmax) hmax = fabsf(hf[f]);
                    }
                    float sh = e4m3_scale_f32(hmax);
                    for (int f = 0; f < F; ++f)
                        qh[f] = lut[e4m3_code_f32(hf[f], sh)];
                    double g = gate[t * K + k];
                    for (int i = 0; i < d; ++i) {
                        double o = 0.0;
                        for (int f = 0; f < F; ++f)
                            o += qh[f] * lut[q2[base2 + (size_t)f * d + i]];
                        yt[i] += g * o * sh * s2[(size_t)e * d + i];
                    }
                }
            }
        }
        free(qx); free(a); free(b); free(hf); free(qh);
    }
    return bad ? -1 : 0;
}

/*
 * 4-bit expert weights.  "Mixture of Experts: Why Mixtral Only Wakes Up Two
 * Specialists", Part 4 ("Why total and active both matter"), sizes the
 * weights at 16 bits and at 4 bits and names no format; this oracle fixes one:
 * E2M1 values (1 sign, 2 exponent bits with bias 1, 1 mantissa bit: 0, 0.5,
 * 1, 1.5, 2, 3, 4, 6; no infinities or NaN) with an E4M3 scale per block of
 * 16 consecutive reduction rows of one output column and one fp32 scale per
 * expert matrix:
 *   st = amax(matrix) / (6 * 448)                 (1 for an all-zero matrix)
 *   sb = E4M3( fp32(fp32(amax(block) / 6) / st) )  (round to nearest even)
 *   code = E2M1( fp32(v / fp32(sb * st)) )        (round to nearest even,
 *          saturating at +-6; 0 when sb is 0)
 *   w ~= E2M1(code) * sb * st
 * E2M1(code) * sb has at most 6 significant bits, so it is exact in bf16.
 */
double oracle_e2m1_decode(int code)
{
    int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
    double v = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return s ? -v : v;
}

int oracle_e2m1_encode(double v)
{
    static const double grid[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
    if (isnan(v))
        return 0x7; /* not produced by finite inputs; maps to +6 */
    int s = signbit(v) ? 1 : 0;
    double a = fabs(v), q;
    /* the grid is uniform inside [0, 2), [2, 4) and [4, 6]: count steps of
     * 0.5, 1 and 2 and round half to even (an even step count = an even
     * mantissa bit) */
    if (a >= 6.0)
        q = 6.0;
    else if (a < 2.0)
        q = 0.5 * round_half_even(a / 0.5);
    else if (a < 4.0)
        q = round_half_even(a);
    else
        q = 2.0 * round_half_even(a / 2.0);
    int mag = 0;
    for (int c = 0; c < 8; ++c)
        if (grid[c] == q)
            mag = c;
    return (s << 3) | mag;
}

/*
 * w [n][rows][cols] (bf16 bits or fp32), rows % 16 == 0, cols even ->
 *   codes [n][rows][cols / 2]: column 2j in the low nibble of byte j, 2j + 1
 *   in the high nibble; bscale [n][rows / 16][cols]: E4M3 codes; tscale [n].
 */
int oracle_quantize_weights_fp4(int n, int rows, int cols, const void *w, int w_dt, uint8_t *codes,
                                uint8_t *bscale, float *tscale)
{
    if (n <= 0 || rows <= 0 || cols <= 0 || rows % 16 != 0 || cols % 2 != 0 || !w || !codes ||
        !bscale || !tscale || !dt_ok(w_dt))
        return -1;
    for (int e = 0; e < n; ++e) {
        float amax = 0.0f;
        for (size_t i = 0; i < (size_t)rows * cols; ++i) {
            float v = (float)elem(w, w_dt, (size_t)e * rows * cols + i);
            if (fabsf(v) > amax)
                amax = fabsf(v);
        }
        float st = amax > 0.0f ? amax / 2688.0f : 1.0f;
        tscale[e] = st;
        uint8_t *ce = codes + (size_t)e * rows * (cols / 2);
        memset(ce, 0, (size_t)rows * (cols / 2));
        /* a thread owns the column pair (2j, 2j + 1) and so whole code bytes */
#pragma omp parallel for schedule(static)
        for (int j = 0; j < cols / 2; ++j)
            for (int h = 0; h < 2; ++h) {
                const int c = 2 * j + h;
                for (int b = 0; b < rows / 16; ++b) {
                    float amax_b = 0.0f;
                    for (int r = 16 * b; r < 16 * b + 16; ++r) {
                        float v = (float)elem(w, w_dt, ((size_t)e * rows + r) * cols + c);
                        if (fabsf(v) > amax_b)
                            amax_b = fabsf(v);
                    }
                    float qb = (amax_b / 6.0f) / st;
                    int sb_code = oracle_e4m3_encode((double)qb);
                    bscale[((size_t)e * (rows / 16) + b) * cols + c] = (uint8_t)sb_code;
                    float sb = (float)oracle_e4m3_decode(sb_code);
                    float denom = sb * st;
                    for (int r = 16 * b; r < 16 * b + 16; ++r) {
                        float v = (float)elem(w, w_dt, ((size_t)e * rows + r) * cols + c);
                        int code = (sb == 0.0f) ? 0 : oracle_e2m1_encode((double)(v / denom));
                        ce[(size_t)r * (cols / 2) + j] |= (uint8_t)(code << (4 * h));
                    }
                }
            }
    }
    return 0;
}

/* codes, bscale, tscale as produced above -> w [n][rows][cols] (fp64). */
int oracle_dequantize_fp4(int n, int rows, int cols, const uint8_t *codes, const uint8_t *bscale,
                          const float *tscale, double *w)
{
    if (n <= 0 || rows <= 0 || cols <= 0 || rows % 16 != 0 || cols % 2 != 0 || !codes || !bscale ||
        !tscale || !w)
        return -1;
    for (int e = 0; e < n; ++e)
        for (int r = 0; r < rows; ++r)
            for (int c = 0; c < cols; ++c) {
                int byte = codes[((size_t)e * rows + r) * (cols / 2) + c / 2];
                int code = (byte >> (4 * (c & 1))) & 0xF;
                double sb = oracle_e4m3_decode(bscale[((size_t)e * (rows / 16) + r / 16) * cols + c]);
                w[((size_t)e * rows + r) * cols + c] = oracle_e2m1_decode(code) * sb * (double)tscale[e];
            }
    return 0;
}

/* Decoded E2M1 and E4M3 codes (filled before any parallel region reads them). */
static double fp4_lut[16], e4m3_lut[256];

static void fp4_luts(void)
{
    for (int c = 0; c < 16; ++c)
        fp4_lut[c] = oracle_e2m1_decode(c);
    for (int c = 0; c < 256; ++c)
        e4m3_lut[c] = oracle_e4m3_decode(c);
}

/* One dequantised 4-bit weight: matrix e of [n][rows][cols]. */
static double fp4_weight(const uint8_t *codes, const uint8_t *bscale, const float *tscale, int rows, int cols,
                         int e, int r, int c)
{
    int byte = codes[((size_t)e * rows + r) * (cols / 2) + c / 2];
    int code = (byte >> (4 * (c & 1))) & 0xF;
    double sb = e4m3_lut[bscale[((size_t)e * (rows / 16) + r / 16) * cols + c]];
    return fp4_lut[code] * sb * (double)tscale[e];
}

/*
 * The layer of the dequantised 4-bit weights (the same loops as
 * oracle_forward_with_routing, each weight dequantised where it is read):
 * c1/b1/t1, c3/b3/t3 for w1, w3 [n][d][F]; c2/b2/t2 for w2 [n][F][d].
 */
int oracle_forward_fp4(int64_t T, int d, int F, int n, int K, const void *x, int x_dt, const int32_t *idx,
                       const double *gate, const uint8_t *c1, const uint8_t *b1, const float *t1,
                       const uint8_t *c3, const uint8_t *b3, const float *t3, const uint8_t *c2,
                       const uint8_t *b2, const float *t2, double *y)
{
    if (T <= 0 || d <= 0 || F <= 0 || n <= 0 || K <= 0 || d % 16 != 0 || F % 16 != 0 || !x || !idx || !gate ||
        !c1 || !b1 || !t1 || !c3 || !b3 || !t3 || !c2 || !b2 || !t2 || !y || !dt_ok(x_dt))
        return -1;
    for (int64_t i = 0; i < T * K; ++i)
        if (idx[i] < 0 || idx[i] >= n)
            return -1;
    fp4_luts();
    int bad = 0;
#pragma omp parallel
    {
        double *a = (double *)malloc(sizeof(double) * (size_t)F);
        double *b = (double *)malloc(sizeof(double) * (size_t)F);
        if (!a || !b) {
#pragma omp atomic write
            bad = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t t = 0; t < T; ++t) {
                double *yt = y + t * d;
                for (int i = 0; i < d; ++i)
                    yt[i] = 0.0;
                for (int k = 0; k < K; ++k) {
                    int e = idx[t * K + k];
                    for (int f = 0; f < F; ++f)
                        a[f] = b[f] = 0.0;
                    for (int j = 0; j < d; ++j) {
                        double xj = elem(x, x_dt, (size_t)t * d + j);
                        for (int f = 0; f < F; ++f) {
                            a[f] += xj * fp4_weight(c1, b1, t1, d, F, e, j, f);
                            b[f] += xj * fp4_weight(c3, b3, t3, d, F, e, j, f);
                        }
                    }
                    for (int f = 0; f < F; ++f)
                        a[f] = oracle_silu(a[f]) * b[f];
                    double g = gate[t * K + k];
                    for (int i = 0; i < d; ++i) {
                        double o = 0.0;
                        for (int f = 0; f < F; ++f)
                            o += a[f] * fp4_weight(c2, b2, t2, F, d, e, f, i);
                        yt[i] += g * o;
                    }
                }
            }
        }
        free(a);
        free(b);
    }
    return bad ? -1 : 0;
}

/*
 * 4-bit activations, the other operand of the 4-bit tensor-core path: each row
 * of x [T][d] is quantised like one 4-bit weight matrix whose blocks run
 * along the row -- rs = max|row| / (6 * 448) (1 for a zero row), an E4M3
 * scale per 16 consecutive elements, E2M1 codes; codes [T][d/2] (element 2j
 * in the low nibble of byte j), bscale [T][d/16], rscale [T].
 */
int oracle_quantize_rows_fp4(int64_t T, int d, const void *x, int x_dt, uint8_t *codes, uint8_t *bscale,
                             float *rscale)
{
    if (T <= 0 || d <= 0 || d % 16 != 0 || !x || !codes || !bscale || !rscale || !dt_ok(x_dt))
        return -1;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        float amax = 0.0f;
        for (int j = 0; j < d; ++j) {
            float v = (float)elem(x, x_dt, (size_t)t * d + j);
            if (fabsf(v) > amax)
                amax = fabsf(v);
        }
        float rs = amax > 0.0f ? amax / 2688.0f : 1.0f;
        rscale[t] = rs;
        uint8_t *ct = codes + (size_t)t * (d / 2);
        memset(ct, 0, (size_t)d / 2);
        for (int b = 0; b < d / 16; ++b) {
            float amax_b = 0.0f;
            for (int j = 16 * b; j < 16 * b + 16; ++j) {
                float v = (float)elem(x, x_dt, (size_t)t * d + j);
                if (fabsf(v) > amax_b)
                    amax_b = fabsf(v);
            }
            int sb_code = oracle_e4m3_encode((double)((amax_b / 6.0f) / rs));
            bscale[(size_t)t * (d / 16) + b] = (uint8_t)sb_code;
            float denom = (float)oracle_e4m3_decode(sb_code) * rs;
            for (int j = 16 * b; j < 16 * b + 16; ++j) {
                float v = (float)elem(x, x_dt, (size_t)t * d + j);
                int code = (denom == 0.0f) ? 0 : oracle_e2m1_encode((double)(v / denom));
                ct[j / 2] |= (uint8_t)(code << (4 * (j & 1)));
            }
        }
    }
    return 0;
}

static double fp4_act(const uint8_t *codes, const uint8_t *bscale, float rs, int j)
{
    int code = (codes[j / 2] >> (4 * (j & 1))) & 0xF;
    return fp4_lut[code] * e4m3_lut[bscale[j / 16]] * (double)rs;
}

/*
 * The layer with 4-bit weights AND 4-bit activations: per token, x is
 * quantised per row as above; a, b = the dot products of the dequantised
 * x row with the dequantised w1, w3 columns; h = bf16(silu(a) * b); h is
 * quantised per row the same way; o = the dequantised h row times the
 * dequantised w2; y = sum_k gate_k * o_k.  Weights as oracle_quantize_weights_fp4
 * writes them (c*, b*, t*).
 */
int oracle_forward_w4a4(int64_t T, int d, int F, int n, int K, const void *x, int x_dt, const int32_t *idx,
                        const double *gate, const uint8_t *c1, const uint8_t *b1, const float *t1,
                        const uint8_t *c3, const uint8_t *b3, const float *t3, const uint8_t *c2,
                        const uint8_t *b2, const float *t2, double *y)
{
    if (T <= 0 || d <= 0 || F <= 0 || n <= 0 || K <= 0 || d % 16 != 0 || F % 16 != 0 || !x || !idx || !gate ||
        !c1 || !b1 || !t1 || !c3 || !b3 || !t3 || !c2 || !b2 || !t2 || !y || !dt_ok(x_dt))
        return -1;
    for (int64_t i = 0; i < T * K; ++i)
        if (idx[i] < 0 || idx[i] >= n)
            return -1;
    fp4_luts();
    int bad = 0;
#pragma omp parallel
    {
        double *a = (double *)malloc(sizeof(double) * (size_t)F);
        double *b = (double *)malloc(sizeof(double) * (size_t)F);
        float *hf = (float *)malloc(sizeof(float) * (size_t)F);
        uint8_t *qx = (uint8_t *)malloc((size_t)d / 2), *sx = (uint8_t *)malloc((size_t)d / 16);
        uint8_t *qh = (uint8_t *)malloc((size_t)F / 2), *sh = (uint8_t *)malloc((size_t)F / 16);
        if (!a || !b || !hf || !qx || !sx || !qh || !sh) {
#pragma omp atomic write
            bad = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t t = 0; t < T; ++t) {
                float rx = 0.0f, rh = 0.0f;
                double *yt = y + t * d;
                /* quantise this token's row (bf16 bits or fp32, read as stored) */
                const size_t es = x_dt == OR_BF16 ? 2 : (x_dt == OR_F32 ? 4 : 8);
                if (oracle_quantize_rows_fp4(1, d, (const uint8_t *)x + (size_t)t * d * es, x_dt, qx, sx, &rx) != 0) {
#pragma omp atomic write
                    bad = 1;
                    continue;
                }
                for (int i = 0; i < d; ++i)
                    yt[i] = 0.0;
                for (int k = 0; k < K; ++k) {
                    int e = idx[t * K + k];
                    for (int f = 0; f < F; ++f)
                        a[f] = b[f] = 0.0;
                    for (int j = 0; j < d; ++j) {
                        double xj = fp4_act(qx, sx, rx, j);
                        for (int f = 0; f < F; ++f) {
                            a[f] += xj * fp4_weight(c1, b1, t1, d, F, e, j, f);
                            b[f] += xj * fp4_weight(c3, b3, t3, d, F, e, j, f);
                        }
                    }
                    for (int f = 0; f < F; ++f)
                        hf[f] = round_bf16((float)(oracle_silu(a[f]) * b[f]));
                    if (oracle_quantize_rows_fp4(1, F, hf, OR_F32, qh, sh, &rh) != 0) {
#pragma omp atomic write
                        bad = 1;
                        break;
                    }
                    double g = gate[t * K + k];
                    for (int i = 0; i < d; ++i) {
                        double o = 0.0;
                        for (int f = 0; f < F; ++f)
                            o += fp4_act(qh, sh, rh, f) * fp4_weight(c2, b2, t2, F, d, e, f, i);
                        yt[i] += g * o;
                    }
                }
            }
        }
        free(a); free(b); free(hf); free(qx); free(sx); free(qh); free(sh);
    }
    return bad ? -1 : 0;
}
