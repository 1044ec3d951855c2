/*
 * dspark_oracle.c -- plain, slow CPU oracle of the DSpark drafter-head path.
 *
 * TEST INFRASTRUCTURE.  Only the tests, the smoke check and the benchmark's
 * CPU-baseline leg may load this library.  The product path (the CUDA library
 * and its Python binding) never calls it and shares no code with it.
 *
 * Every quantity is formed in fp64 from the bf16/fp32 inputs, in the order the
 * definitions state, with no blocking, fusion or reordering.  Requests are
 * independent, so an OpenMP loop runs them on several host cores; inside one
 * request the loops are the definitions written out.
 *
 * Sources (web pages on DSpark):
 *   [G]  gdymind.com, "DSpark: DeepSeek's new speculative decoding work
 *        (Video + Blog)", sections 0-6.
 *   [W]  wispaper.ai, "DSpark: Overcoming the Efficiency Wall in LLM
 *        Speculative Decoding", section "The Hardware-Aware Prefix Scheduler".
 *   [S]  seventnews.com, "DeepSeek's DSpark just fixed the two things that
 *        held back faster AI inference".
 *
 * Readings taken where the pages are silent (each one is shared with the GPU
 * path as a stated convention, not as code):
 *   - draft distribution: p_k(v) proportional to exp(U_k(v) + B(x_{k-1}, v)),
 *     the transition bias added to the backbone's base logit, with x_0 the
 *     anchor ([G] section 4; the formula itself is missing from the page);
 *   - greedy selection takes the smallest vocabulary index among equal maxima;
 *   - Gumbel-max noise: Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel
 *     random numbers: as easy as 1, 2, 3", SC'11), key = (seed low word, seed
 *     high word), counter = (v / 4, k - 1, b, 0), output word v mod 4,
 *     u = ((w >> 9) + 0.5) 2^-23, g = -ln(-ln u), score = l / tau + g;
 *   - confidence: c_k = sigmoid(z_k / T_k) with
 *     z_k = w . [h_k ; W1[x_{k-1}]] + b  ([G] section 5, "Sequential
 *     Temperature Scaling" applied to the whole logit);
 *   - prefix survival: P_k = prod_{j <= k} c_j  ([W], [S]: the survival probability
 *     of each prefix; [G] section 5: a cumulative product);
 *   - scheduler objective: expected tokens per second
 *     F = (B + sum_b sum_{k <= L_b} P_{b,k}) / Tstep(B + sum_b L_b), scores
 *     fixed-point q = floor(P 2^46), order (P desc, b asc, k asc), first
 *     maximum over N ([W]; [G] section 6);
 *   - verification: accepted = index of the first mismatch among the first L_b
 *     drafts (or L_b), bonus = target token at that position ([S]).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_INVALID 1

static double bf16_to_f64(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* --------------------------------------------------------------------------
 * Philox4x32-10 (SC'11): ten rounds of the 4-word Philox S-box.  Each round
 * multiplies words 0 and 2 by the two round multipliers, swaps the halves of
 * the products into place and XORs the high halves with words 1 and 3 and the
 * round key; the key is bumped by the two Weyl constants between rounds.
 * ------------------------------------------------------------------------ */
void oracle_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4])
{
    uint32_t x0 = ctr[0], x1 = ctr[1], x2 = ctr[2], x3 = ctr[3];
    uint32_t k0 = key[0], k1 = key[1];
    for (int round = 0; round < 10; ++round) {
        if (round > 0) {
            k0 += 0x9E3779B9u;
            k1 += 0xBB67AE85u;
        }
        uint64_t p0 = (uint64_t)0xD2511F53u * (uint64_t)x0;
        uint64_t p1 = (uint64_t)0xCD9E8D57u * (uint64_t)x2;
        uint32_t y0 = (uint32_t)(p1 >> 32) ^ x1 ^ k0;
        uint32_t y1 = (uint32_t)p1;
        uint32_t y2 = (uint32_t)(p0 >> 32) ^ x3 ^ k1;
        uint32_t y3 = (uint32_t)p0;
        x0 = y0; x1 = y1; x2 = y2; x3 = y3;
    }
    out[0] = x0; out[1] = x1; out[2] = x2; out[3] = x3;
}

/* Uniform in (0, 1), exact in fp32 and fp64, from one 32-bit Philox word. */
double oracle_uniform_from_word(uint32_t w)
{
    return ((double)(w >> 9) + 0.5) * 0x1p-23;
}

/* Gumbel noise g(b, k, v) for request b (global index), position k (1-based). */
double oracle_gumbel(uint64_t seed, int b, int k, int v)
{
    uint32_t ctr[4] = {(uint32_t)v / 4u, (uint32_t)(k - 1), (uint32_t)b, 0u};
    uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    uint32_t out[4];
    oracle_philox4x32_10(ctr, key, out);
    double u = oracle_uniform_from_word(out[v % 4]);
    return -log(-log(u));
}

/* --------------------------------------------------------------------------
 * Markov-head drafting ([G] section 4, "Sequential stage" and "Markov head").
 *
 * For each listed request i (global id b_index[i]) and k = 1..gamma:
 *   bias(v)  = sum_{j<r} W1[x_{k-1}, j] W2[j, v]            (j ascending)
 *   l(v)     = U[i, k-1, v] + bias(v)
 *   s(v)     = l(v)                      (greedy, mode 0)
 *            = l(v) / tau + g(b, k, v)   (Gumbel-max, mode 1)
 *   x_k      = smallest v with s(v) = max s
 *   logit[k] = l(x_k);  gap[k] = max s - second largest s (0 on an exact tie)
 * with x_0 = anchor[i].  U holds only the listed requests: [nb, gamma, V].
 *
 * Teacher-forced use (forced_prev non-NULL, [nb, gamma]): position k conditions on
 * x_{k-1} = forced_prev[i, k-1] instead of the token this call picked at k - 1, so
 * every position is the one-step Markov transition from a given previous token (the
 * same arithmetic; only where x_{k-1} comes from differs).
 * ------------------------------------------------------------------------ */
int oracle_draft(const uint16_t *U, const int32_t *anchor, const uint16_t *W1,
                 const uint16_t *W2, int nb, int gamma, int V, int r, int mode, double tau,
                 uint64_t seed, const int32_t *b_index, int32_t *x_out, double *logit_out,
                 double *gap_out, const int32_t *forced_prev, int nthreads)
{
    if (nb < 0 || gamma < 1 || V < 2 || r < 1 || (mode != 0 && mode != 1))
        return ORACLE_INVALID;
    if (mode == 1 && !(tau > 0.0))
        return ORACLE_INVALID;
    for (int i = 0; i < nb; ++i)
        if (anchor[i] < 0 || anchor[i] >= V)
            return ORACLE_INVALID;
    if (forced_prev)
        for (size_t o = 0; o < (size_t)nb * (size_t)gamma; ++o)
            if (forced_prev[o] < 0 || forced_prev[o] >= V)
                return ORACLE_INVALID;
    if (nthreads < 1)
        nthreads = oracle_num_threads();

    int status = ORACLE_OK;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
    for (int i = 0; i < nb; ++i) {
        double *bias = (double *)malloc(sizeof(double) * (size_t)V);
        if (!bias) {
#pragma omp atomic write
            status = ORACLE_INVALID;
            continue;
        }
        int prev = anchor[i];
        for (int k = 1; k <= gamma; ++k) {
            if (forced_prev)
                prev = forced_prev[(size_t)i * (size_t)gamma + (size_t)(k - 1)];
            const uint16_t *row = W1 + (size_t)prev * (size_t)r;
            for (int v = 0; v < V; ++v)
                bias[v] = 0.0;
            for (int j = 0; j < r; ++j) {
                const double a = bf16_to_f64(row[j]);
                const uint16_t *w2j = W2 + (size_t)j * (size_t)V;
                for (int v = 0; v < V; ++v)
                    bias[v] += a * bf16_to_f64(w2j[v]);
            }
            const uint16_t *Uk = U + ((size_t)i * (size_t)gamma + (size_t)(k - 1)) * (size_t)V;
            double best = -INFINITY, second = -INFINITY, best_l = 0.0;
            int best_v = -1;
            for (int v = 0; v < V; ++v) {
                const double l = bf16_to_f64(Uk[v]) + bias[v];
                double s = l;
                if (mode == 1)
                    s = l / tau + oracle_gumbel(seed, b_index ? b_index[i] : i, k, v);
                if (s > best) {
                    second = best;
                    best = s;
                    best_v = v;
                    best_l = l;
                } else if (s > second) {
                    second = s;
                }
            }
            const size_t o = (size_t)i * (size_t)gamma + (size_t)(k - 1);
            x_out[o] = best_v;
            if (logit_out)
                logit_out[o] = best_l;
            if (gap_out)
                gap_out[o] = best - second;
            prev = best_v;
        }
        free(bias);
    }
    return status;
}

/* --------------------------------------------------------------------------
 * RNN head ([G] section 4, "Two instantiations of the sequential block": a
 * recurrent state that accumulates the whole prefix of the block).  The pages
 * give no equations; this is the plain Elman reading over the Markov head's
 * factors (PARITY UNPINNED against the pages):
 *   s_0 = 0,   s_k = tanh(W1[x_{k-1}] + s_{k-1} Whh)       (r-vector, fp64)
 *   a_k = bf16(fp32(s_k))                                   (the GEMM operand)
 *   l_k(v) = U[b, k-1, v] + sum_j a_k[j] W2[j, v]
 * and x_k is chosen as in oracle_draft (greedy or Gumbel-max).  With Whh = 0
 * the bias is that of a Markov head whose table is bf16(fp32(tanh(W1))).
 * forced_prev (optional, [nb, gamma]) gives x_{k-1} for every position as in
 * oracle_draft; the state then runs along the given tokens.
 * ------------------------------------------------------------------------ */
static uint16_t f32_to_bf16_rne(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu))
        return (uint16_t)((u >> 16) | 0x40u);                  /* quiet NaN */
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

int oracle_draft_rnn(const uint16_t *U, const int32_t *anchor, const uint16_t *W1,
                     const uint16_t *W2, const uint16_t *Whh, int nb, int gamma, int V, int r,
                     int mode, double tau, uint64_t seed, const int32_t *b_index,
                     int32_t *x_out, double *logit_out, double *gap_out,
                     const int32_t *forced_prev, int nthreads)
{
    if (nb < 0 || gamma < 1 || V < 2 || r < 1 || (mode != 0 && mode != 1))
        return ORACLE_INVALID;
    if (mode == 1 && !(tau > 0.0))
        return ORACLE_INVALID;
    for (int i = 0; i < nb; ++i)
        if (anchor[i] < 0 || anchor[i] >= V)
            return ORACLE_INVALID;
    if (forced_prev)
        for (size_t o = 0; o < (size_t)nb * (size_t)gamma; ++o)
            if (forced_prev[o] < 0 || forced_prev[o] >= V)
                return ORACLE_INVALID;
    if (nthreads < 1)
        nthreads = oracle_num_threads();

    int status = ORACLE_OK;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
    for (int i = 0; i < nb; ++i) {
        double *bias = (double *)malloc(sizeof(double) * (size_t)V);
        double *st = (double *)calloc((size_t)r, sizeof(double));
        double *nx = (double *)malloc(sizeof(double) * (size_t)r);
        if (!bias || !st || !nx) {
            free(bias);
            free(st);
            free(nx);
#pragma omp atomic write
            status = ORACLE_INVALID;
            continue;
        }
        int prev = anchor[i];
        for (int k = 1; k <= gamma; ++k) {
            if (forced_prev)
                prev = forced_prev[(size_t)i * (size_t)gamma + (size_t)(k - 1)];
            const uint16_t *row = W1 + (size_t)prev * (size_t)r;
            for (int j = 0; j < r; ++j) {
                double acc = bf16_to_f64(row[j]);
                for (int q = 0; q < r; ++q)
                    acc += st[q] * bf16_to_f64(Whh[(size_t)q * (size_t)r + (size_t)j]);
                nx[j] = tanh(acc);
            }
            for (int j = 0; j < r; ++j)
                st[j] = nx[j];
            for (int v = 0; v < V; ++v)
                bias[v] = 0.0;
            for (int j = 0; j < r; ++j) {
                const double a = bf16_to_f64(f32_to_bf16_rne((float)st[j]));
                const uint16_t *w2j = W2 + (size_t)j * (size_t)V;
                for (int v = 0; v < V; ++v)
                    bias[v] += a * bf16_to_f64(w2j[v]);
            }
            const uint16_t *Uk = U + ((size_t)i * (size_t)gamma + (size_t)(k - 1)) * (size_t)V;
            double best = -INFINITY, second = -INFINITY, best_l = 0.0;
            int best_v = -1;
            for (int v = 0; v < V; ++v) {
                const double l = bf16_to_f64(Uk[v]) + bias[v];
                double sc = l;
                if (mode == 1)
                    sc = l / tau + oracle_gumbel(seed, b_index ? b_index[i] : i, k, v);
                if (sc > best) {
                    second = best;
                    best = sc;
                    best_v = v;
                    best_l = l;
                } else if (sc > second) {
                    second = sc;
                }
            }
            const size_t o = (size_t)i * (size_t)gamma + (size_t)(k - 1);
            x_out[o] = best_v;
            if (logit_out)
                logit_out[o] = best_l;
            if (gap_out)
                gap_out[o] = best - second;
            prev = best_v;
        }
        free(bias);
        free(st);
        free(nx);
    }
    return status;
}

/* --------------------------------------------------------------------------
 * Confidence head, Sequential Temperature Scaling and prefix survival
 * ([G] section 5; [S] "Confidence-scheduled verification").
 *
 *   z_{b,k} = sum_{i<d} w[i] h[b, k-1, i] + sum_{j<r} w[d+j] W1[x_{k-1}, j] + b_conf
 *   c_{b,k} = 1 / (1 + exp(-z_{b,k} / T_k))
 *   P64_{b,k} = P64_{b,k-1} c_{b,k},  P64_{b,0} = 1
 *   P32_{b,k} = fl32(P32_{b,k-1} * fl32(c_{b,k})),  P32_{b,0} = 1
 * with x_0 = anchor[b] and x_{k-1} = x[b, k-2] for k >= 2.  P32 is the fp32
 * rendering of the same product (one fp32 rounding per factor and per step),
 * used to feed the scheduler identical fp32 scores on both sides.
 * ------------------------------------------------------------------------ */
int oracle_confidence(const uint16_t *h, const int32_t *anchor, const int32_t *x,
                      const uint16_t *W1, const uint16_t *w, double b_conf, const float *T,
                      int B, int gamma, int d, int r, int V, double *z_out, double *c_out,
                      double *P64_out, float *P32_out, int nthreads)
{
    if (B < 0 || gamma < 1 || d < 0 || r < 1)
        return ORACLE_INVALID;
    for (int b = 0; b < B; ++b) {
        if (anchor[b] < 0 || anchor[b] >= V)
            return ORACLE_INVALID;
        for (int k = 0; k + 1 < gamma; ++k)
            if (x[(size_t)b * gamma + k] < 0 || x[(size_t)b * gamma + k] >= V)
                return ORACLE_INVALID;
    }
    for (int k = 0; k < gamma; ++k)
        if (!(T[k] > 0.0f))
            return ORACLE_INVALID;
    if (nthreads < 1)
        nthreads = oracle_num_threads();

#pragma omp parallel for schedule(static) num_threads(nthreads)
    for (int b = 0; b < B; ++b) {
        double P64 = 1.0;
        float P32 = 1.0f;
        for (int k = 1; k <= gamma; ++k) {
            const int prev = (k == 1) ? anchor[b] : x[(size_t)b * gamma + (k - 2)];
            const uint16_t *hk = h + ((size_t)b * gamma + (size_t)(k - 1)) * (size_t)d;
            const uint16_t *e = W1 + (size_t)prev * (size_t)r;
            double z = 0.0;
            for (int i = 0; i < d; ++i)
                z += bf16_to_f64(w[i]) * bf16_to_f64(hk[i]);
            for (int j = 0; j < r; ++j)
                z += bf16_to_f64(w[d + j]) * bf16_to_f64(e[j]);
            z += b_conf;
            const double c = 1.0 / (1.0 + exp(-z / (double)T[k - 1]));
            P64 *= c;
            P32 = (float)((double)P32 * (double)(float)c);
            const size_t o = (size_t)b * gamma + (size_t)(k - 1);
            if (z_out)
                z_out[o] = z;
            if (c_out)
                c_out[o] = c;
            if (P64_out)
                P64_out[o] = P64;
            if (P32_out)
                P32_out[o] = P32;
        }
    }
    return ORACLE_OK;
}

/* --------------------------------------------------------------------------
 * Hardware-aware prefix scheduler ([W] "The Hardware-Aware Prefix Scheduler";
 * [G] section 6, the batch-wide throughput maximisation).
 *
 * Scores P[b, k-1] (fp32) are ordered by (P desc, b asc, k asc).  With
 * q = floor(P 2^46) (exact integers) and S_N the sum of the first N of them,
 *   F(N) = double(B 2^46 + S_N) / Tstep[B + N],     N = 0 .. B gamma,
 * N* is the smallest N with the largest F, and L_b counts the entries of
 * request b among the first N*.  Tstep[n] is the wall time of one target step
 * that verifies n tokens (each request feeds its anchor plus L_b drafts).
 * The reported objective is F 2^-46 (an exact rescaling): expected accepted
 * tokens per unit of Tstep's time.  The scale 2^46 keeps the largest numerator,
 * (B + B gamma) 2^46 <= 98304 2^46 < 2^63, inside int64 for every supported size
 * (B <= 32768, B gamma <= 65536).
 * ------------------------------------------------------------------------ */
typedef struct {
    float p;
    int b;
    int k;
} oracle_score_t;

static int score_order(const void *pa, const void *pb)
{
    const oracle_score_t *a = (const oracle_score_t *)pa, *c = (const oracle_score_t *)pb;
    if (a->p > c->p)
        return -1;
    if (a->p < c->p)
        return 1;
    if (a->b != c->b)
        return a->b < c->b ? -1 : 1;
    return (a->k > c->k) - (a->k < c->k);
}

int oracle_schedule(const float *P, int B, int gamma, const double *Tstep, int32_t *L_out,
                    int32_t *N_out, double *F_out, double *F_all)
{
    if (B < 1 || gamma < 1)
        return ORACLE_INVALID;
    const int n = B * gamma;
    for (int i = 0; i < n; ++i)
        if (!(P[i] >= 0.0f && P[i] <= 1.0f))
            return ORACLE_INVALID;
    for (int m = B; m <= B + n; ++m)
        if (!(Tstep[m] > 0.0))
            return ORACLE_INVALID;

    oracle_score_t *s = (oracle_score_t *)malloc(sizeof(oracle_score_t) * (size_t)n);
    if (!s)
        return ORACLE_INVALID;
    for (int b = 0; b < B; ++b)
        for (int k = 1; k <= gamma; ++k) {
            s[b * gamma + (k - 1)].p = P[b * gamma + (k - 1)];
            s[b * gamma + (k - 1)].b = b;
            s[b * gamma + (k - 1)].k = k;
        }
    qsort(s, (size_t)n, sizeof(oracle_score_t), score_order);

    const int64_t base = (int64_t)B << 46;
    int64_t S = 0;
    double bestF = (double)base / Tstep[B];
    int bestN = 0;
    if (F_all)
        F_all[0] = ldexp(bestF, -46);
    for (int N = 1; N <= n; ++N) {
        S += (int64_t)floor(ldexp((double)s[N - 1].p, 46));
        const double F = (double)(base + S) / Tstep[B + N];
        if (F_all)
            F_all[N] = ldexp(F, -46);
        if (F > bestF) {
            bestF = F;
            bestN = N;
        }
    }
    for (int b = 0; b < B; ++b)
        L_out[b] = 0;
    for (int i = 0; i < bestN; ++i)
        L_out[s[i].b] += 1;
    if (N_out)
        *N_out = bestN;
    if (F_out)
        *F_out = ldexp(bestF, -46);
    free(s);
    return ORACLE_OK;
}

/* --------------------------------------------------------------------------
 * Strict prefix-match verification ([S], "the first rejected token and
 * everything after it get dropped").  target[b] holds the target model's tokens
 * for positions 1..gamma+1.
 *   accepted_b = (smallest k-1 with 1 <= k <= L_b and x[b,k-1] != target[b,k-1]), else L_b
 *   bonus_b    = target[b, accepted_b]
 * ------------------------------------------------------------------------ */
int oracle_verify(const int32_t *x, const int32_t *L, const int32_t *target, int B, int gamma,
                  int32_t *accepted_out, int32_t *bonus_out)
{
    if (B < 0 || gamma < 1)
        return ORACLE_INVALID;
    for (int b = 0; b < B; ++b)
        if (L[b] < 0 || L[b] > gamma)
            return ORACLE_INVALID;
    for (int b = 0; b < B; ++b) {
        int a = L[b];
        for (int k = 1; k <= L[b]; ++k) {
            if (x[(size_t)b * gamma + (k - 1)] != target[(size_t)b * (gamma + 1) + (k - 1)]) {
                a = k - 1;
                break;
            }
        }
        accepted_out[b] = a;
        bonus_out[b] = target[(size_t)b * (gamma + 1) + a];
    }
    return ORACLE_OK;
}

/* --------------------------------------------------------------------------
 * Sequential Temperature Scaling: fitting ([G] section 5, "Sequential
 * Temperature Scaling"): position by position, left to right, a 1-D grid
 * search picks the temperature that minimises the expected calibration error
 * (ECE) of the cumulative product, with the temperatures of all earlier
 * positions already fixed.
 *
 * Calibration set: N blocks with raw confidence logits z[n, k-1] and accepted
 * lengths acc[n] (number of drafts the target accepted).  Survival label at
 * position k: y = 1 if acc[n] >= k.  For a candidate T:
 *   P_k[n]   = P_{k-1}[n] * sigmoid(z[n, k-1] / T),   P_0 = 1
 *   bin(p)   = min(floor(p * n_bins), n_bins - 1)     (equal-width bins on [0, 1])
 *   ECE(T)   = sum_m |sum_{n in m} y - sum_{n in m} P_k| / N
 * (the count-weighted mean gap |B_m|/N |mean y - mean P| written as a sum).
 * Grid: T_i = t_min + i * t_step, i = 0 .. n_t - 1; the smallest i with the
 * smallest ECE wins.  Outputs the chosen T per position and its ECE, and, when
 * ece_grid is given, every candidate's ECE [gamma][n_t].  When T_fixed is given,
 * position k is frozen at T_fixed[k-1] instead of the chosen T (so that another
 * implementation's choices can be scored), while T_out still reports the choice.
 * ------------------------------------------------------------------------ */
double oracle_ece(const double *P, const int32_t *acc, int N, int k, int n_bins)
{
    double *sy = (double *)calloc((size_t)n_bins, sizeof(double));
    double *sp = (double *)calloc((size_t)n_bins, sizeof(double));
    if (!sy || !sp) {
        free(sy);
        free(sp);
        return -1.0;
    }
    for (int n = 0; n < N; ++n) {
        int m = (int)floor(P[n] * n_bins);
        if (m > n_bins - 1)
            m = n_bins - 1;
        if (m < 0)
            m = 0;
        sy[m] += (acc[n] >= k) ? 1.0 : 0.0;
        sp[m] += P[n];
    }
    double e = 0.0;
    for (int m = 0; m < n_bins; ++m)
        e += fabs(sy[m] - sp[m]);
    free(sy);
    free(sp);
    return e / N;
}

int oracle_sts_fit(const float *z, const int32_t *acc, int N, int gamma, double t_min,
                   double t_step, int n_t, int n_bins, const double *T_fixed, double *T_out,
                   double *ece_out, double *ece_grid, int nthreads)
{
    if (N < 1 || gamma < 1 || n_t < 1 || n_bins < 1 || !(t_min > 0.0) || !(t_step >= 0.0))
        return ORACLE_INVALID;
    if (nthreads < 1)
        nthreads = oracle_num_threads();
    double *P = (double *)malloc(sizeof(double) * (size_t)N);
    double *ece = (double *)malloc(sizeof(double) * (size_t)n_t);
    if (!P || !ece) {
        free(P);
        free(ece);
        return ORACLE_INVALID;
    }
    for (int n = 0; n < N; ++n)
        P[n] = 1.0;
    for (int k = 1; k <= gamma; ++k) {
#pragma omp parallel for schedule(static) num_threads(nthreads)
        for (int i = 0; i < n_t; ++i) {
            const double T = t_min + i * t_step;
            double *Pk = (double *)malloc(sizeof(double) * (size_t)N);
            for (int n = 0; n < N; ++n)
                Pk[n] = P[n] / (1.0 + exp(-(double)z[(size_t)n * gamma + (k - 1)] / T));
            ece[i] = oracle_ece(Pk, acc, N, k, n_bins);
            free(Pk);
        }
        int best = 0;
        for (int i = 1; i < n_t; ++i)
            if (ece[i] < ece[best])
                best = i;
        if (ece_grid)
            for (int i = 0; i < n_t; ++i)
                ece_grid[(size_t)(k - 1) * n_t + i] = ece[i];
        T_out[k - 1] = t_min + best * t_step;
        ece_out[k - 1] = ece[best];
        const double T = T_fixed ? T_fixed[k - 1] : T_out[k - 1];
        for (int n = 0; n < N; ++n)
            P[n] = P[n] / (1.0 + exp(-(double)z[(size_t)n * gamma + (k - 1)] / T));
    }
    free(P);
    free(ece);
    return ORACLE_OK;
}
