/*
 * sv_oracle.c -- plain, slow, double-precision CPU oracle for batched
 * speculative-sampling verification.
 *
 * TEST INFRASTRUCTURE.  Only the tests, the smoke check and the benchmark's
 * CPU-baseline leg use this file.  It shares no code, header or constant with
 * the CUDA library; the product path never calls it.
 *
 * What it computes, per sequence b (sources named in brackets):
 *
 *  1. Temperature before log-softmax, in log space [FlashSpec, Metodologia 1,
 *     "Estabilidade Numerica"; Significancia, engineering lessons]:
 *        lse(row) = M/T + log sum_v exp((l_v - M)/T),  M = max_v l_v
 *     for every target row j in [0, gamma] and draft row j in [0, gamma).
 *  2. The per-candidate test on two log-probability scalars [FlashSpec,
 *     Metodologia 1, "Mecanismo"]:
 *        log p_j(x_j) = lt[j][x_j]/T - lse_t[j],  log q_j(x_j) = ld[j][x_j]/T - lse_d[j]
 *        accept j  iff  log u_j < log p_j(x_j) - log q_j(x_j)
 *     The accepted prefix ends at the first rejection n; the rest is dropped
 *     [Speculative Speculative Decoding, "O Essencial", step 3].
 *  3. The verification outcome is (number accepted, one more token)
 *     [Speculative Speculative Decoding, Metodologia 2, "Conceito Central" 1].
 *     After a rejection at n the extra token comes from the residual
 *     distribution norm(max(0, p_n - q_n)) [same page, Desafios 2, "Amostragem
 *     Saguaro"]; when all gamma drafts are accepted it is the bonus token drawn
 *     from the target's (gamma+1)-th distribution p_gamma.
 *     Inverse CDF: the token is the smallest k with C_k > u * S, where C_k is the
 *     running sum of the weights and S their total; if rounding leaves no such k,
 *     the last k with a positive weight.  If the residual mass S is below
 *     2^-18 the residual counts as vanished and the draw falls back to p_n
 *     (row-status bit 8).  S = 0 needs p_n <= q_n at every token, which with
 *     both summing to one leaves only rounding-level differences; a mass this
 *     small is also below what fp32 weights resolve, and in the cases that
 *     reach it (q_n equal to p_n up to a shift of the normaliser) the residual
 *     is proportional to p_n anyway.
 *  4. T == 0 is greedy verification: accept j iff x_j is the first argmax of
 *     target row j; the extra token is the first argmax of target row n.  The
 *     draft logits and the uniforms are not used.
 *
 * The pages print neither min(1, p/q), the residual nor the bonus rule; the
 * formulas above are the standard speculative-sampling rule whose output
 * distribution equals the target's, which is the property the pages require
 * [FlashSpec, Metodologia 2, "Garantia Teorica"; Significancia, Teorema 1].
 *
 * Contract details that the pages leave open (library readings):
 *   - valid temperature: T == 0, or T finite and >= 1e-6; otherwise status 4;
 *   - status 1: some draft token outside [0, V);
 *   - status 16 (T > 0 only): some uniform u_accept[j] or u_resample outside
 *     [0, 1) or NaN (the uniforms stand for draws of U[0, 1));
 *   - status 2: a row that is read holds NaN or +inf, or is all -inf
 *     (T > 0: all 2*gamma+1 rows; T == 0: the gamma+1 target rows);
 *   - with status 1, 2, 4 or 16 the sequence emits n = 0 and all tokens -1;
 *   - tokens past the extra one are -1;
 *   - log_norm is NaN for greedy sequences, invalid T and bad rows.
 *
 * Near-tie report (for comparing an implementation that rounds differently):
 *   bit 1: |log u_j - delta_j| < 1e-6 at some tested position j;
 *   bit 2: at the chosen token k, min(|C_{k-1} - uS|, |C_k - uS|) < 1e-6, the
 *          weights being probabilities (p_v, or max(0, p_v - q_v)), so the gap
 *          is in units of probability mass; or, after a rejection, the residual
 *          mass S lies within 1e-6 of the 2^-18 fallback threshold.
 *
 * Inputs: logits are float32, or bf16 given as uint16 bit patterns; every
 * value is widened exactly to double before any arithmetic.
 */
#define _GNU_SOURCE
#include <math.h>
#include <stdint.h>
#include <string.h>
#include <stdlib.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_T_MIN 1e-6
#define ORACLE_NEAR 1e-6
#define ORACLE_RESIDUAL_MIN 0x1p-18 /* residual mass below this counts as vanished */

enum { ST_TOKEN = 1, ST_ROW = 2, ST_TEMP = 4, ST_RESID0 = 8, ST_UNIFORM = 16 };
enum { NEAR_ACCEPT = 1, NEAR_CDF = 2 };

static double widen(const void* base, int is_bf16, size_t i)
{
    if (!is_bf16) return (double)((const float*)base)[i];
    uint32_t bits = (uint32_t)((const uint16_t*)base)[i] << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/* One row's log-normaliser of l/T.  Returns 0 if the row is bad. */
static int row_lse(const void* base, int is_bf16, size_t off, int V, double T, double* lse)
{
    double M = -INFINITY;
    for (int v = 0; v < V; ++v) {
        double l = widen(base, is_bf16, off + (size_t)v);
        if (isnan(l)) return 0;
        if (l > M) M = l;
    }
    if (isinf(M)) return 0; /* +inf present, or every entry -inf */
    double s = 0.0;
    for (int v = 0; v < V; ++v) s += exp((widen(base, is_bf16, off + (size_t)v) - M) / T);
    *lse = M / T + log(s);
    return 1;
}

/* First index of the largest value.  Returns -1 if the row is bad. */
static int row_argmax(const void* base, int is_bf16, size_t off, int V)
{
    double best = -INFINITY;
    int arg = -1;
    for (int v = 0; v < V; ++v) {
        double l = widen(base, is_bf16, off + (size_t)v);
        if (isnan(l)) return -1;
        if (l > best) { best = l; arg = v; }
    }
    if (arg < 0 || isinf(best)) return -1;
    return arg;
}

/* Smallest k with running sum C_k > u*S; if none, the last k with w_k > 0. */
static int inverse_cdf(const double* w, int V, double u, int* near, double* gap)
{
    double S = 0.0;
    for (int v = 0; v < V; ++v) S += w[v];
    double target = u * S;
    double C = 0.0, prev = 0.0;
    int k = -1;
    for (int v = 0; v < V; ++v) {
        prev = C;
        C += w[v];
        if (C > target) { k = v; break; }
    }
    if (k < 0) {
        for (int v = V - 1; v >= 0; --v)
            if (w[v] > 0.0) { k = v; break; }
        *near |= NEAR_CDF;
        *gap = 0.0;
        return k;
    }
    *gap = fmin(fabs(prev - target), fabs(C - target));
    if (*gap < ORACLE_NEAR) *near |= NEAR_CDF;
    return k;
}

static void verify_one(const void* tgt, const void* dft, int is_bf16, const int32_t* tok,
                       double T, const float* u_acc, double u_res, int gamma, int V, size_t b,
                       int32_t* out_tok, int32_t* out_n, double* lnorm, int32_t* status,
                       int32_t* near, double* agap, double* cgap, double* wbuf)
{
    const int R = 2 * gamma + 1;
    int st = 0, nr = 0;
    *agap = INFINITY;
    *cgap = INFINITY;
    for (int j = 0; j <= gamma; ++j) out_tok[j] = -1;
    for (int r = 0; r < R; ++r) lnorm[r] = NAN;
    *out_n = 0;

    if (!(T == 0.0 || (isfinite(T) && T >= ORACLE_T_MIN))) {
        *status = ST_TEMP;
        *near = 0;
        return;
    }
    for (int j = 0; j < gamma; ++j)
        if (tok[j] < 0 || tok[j] >= V) st |= ST_TOKEN;
    if (T > 0.0) { /* a greedy sequence reads no uniform */
        for (int j = 0; j < gamma; ++j)
            if (!(u_acc[j] >= 0.0f && u_acc[j] < 1.0f)) st |= ST_UNIFORM;
        if (!(u_res >= 0.0 && u_res < 1.0)) st |= ST_UNIFORM;
    }

    const size_t trow0 = b * (size_t)(gamma + 1) * (size_t)V;
    const size_t drow0 = b * (size_t)gamma * (size_t)V;

    if (T == 0.0) {
        int arg[64];
        for (int j = 0; j <= gamma; ++j) {
            arg[j] = row_argmax(tgt, is_bf16, trow0 + (size_t)j * V, V);
            if (arg[j] < 0) st |= ST_ROW;
        }
        if (st) { *status = st; *near = 0; return; }
        int n = gamma;
        for (int j = 0; j < gamma; ++j)
            if (tok[j] != arg[j]) { n = j; break; }
        for (int j = 0; j < n; ++j) out_tok[j] = tok[j];
        out_tok[n] = arg[n];
        *out_n = n;
        *status = 0;
        *near = 0;
        return;
    }

    double lse_t[33], lse_d[32];
    for (int j = 0; j <= gamma; ++j) {
        if (row_lse(tgt, is_bf16, trow0 + (size_t)j * V, V, T, &lse_t[j])) lnorm[j] = lse_t[j];
        else st |= ST_ROW;
    }
    for (int j = 0; j < gamma; ++j) {
        if (row_lse(dft, is_bf16, drow0 + (size_t)j * V, V, T, &lse_d[j])) lnorm[gamma + 1 + j] = lse_d[j];
        else st |= ST_ROW;
    }
    if (st) { /* good rows keep their log_norm; the sequence emits nothing */
        *status = st;
        *near = 0;
        return;
    }

    /* accept scan in log space */
    int n = gamma;
    for (int j = 0; j < gamma; ++j) {
        double lp = widen(tgt, is_bf16, trow0 + (size_t)j * V + (size_t)tok[j]) / T - lse_t[j];
        double lq = widen(dft, is_bf16, drow0 + (size_t)j * V + (size_t)tok[j]) / T - lse_d[j];
        double delta = lp - lq;
        double lu = log((double)u_acc[j]);
        if (fabs(lu - delta) < *agap) *agap = fabs(lu - delta);
        if (fabs(lu - delta) < ORACLE_NEAR) nr |= NEAR_ACCEPT;
        if (!(lu < delta)) { n = j; break; }
    }

    int k;
    if (n < gamma) {
        double S = 0.0;
        for (int v = 0; v < V; ++v) {
            double p = exp(widen(tgt, is_bf16, trow0 + (size_t)n * V + v) / T - lse_t[n]);
            double q = exp(widen(dft, is_bf16, drow0 + (size_t)n * V + v) / T - lse_d[n]);
            wbuf[v] = fmax(0.0, p - q);
            S += wbuf[v];
        }
        if (!(S >= ORACLE_RESIDUAL_MIN)) {
            st |= ST_RESID0;
            for (int v = 0; v < V; ++v)
                wbuf[v] = exp(widen(tgt, is_bf16, trow0 + (size_t)n * V + v) / T - lse_t[n]);
        }
        k = inverse_cdf(wbuf, V, u_res, &nr, cgap);
        /* the fallback decision itself is a near tie when S is close to the threshold */
        if (fabs(S - ORACLE_RESIDUAL_MIN) < *cgap) *cgap = fabs(S - ORACLE_RESIDUAL_MIN);
        if (*cgap < ORACLE_NEAR) nr |= NEAR_CDF;
    } else {
        for (int v = 0; v < V; ++v)
            wbuf[v] = exp(widen(tgt, is_bf16, trow0 + (size_t)gamma * V + v) / T - lse_t[gamma]);
        k = inverse_cdf(wbuf, V, u_res, &nr, cgap);
    }
    for (int j = 0; j < n; ++j) out_tok[j] = tok[j];
    out_tok[n] = k;
    *out_n = n;
    *status = st;
    *near = nr;
}

/*
 * target: [B][gamma+1][V], draft: [B][gamma][V]; is_bf16 selects uint16 bf16 bits.
 * Outputs: out_tokens [B][gamma+1], out_n [B], log_norm [B][2*gamma+1],
 * row_status [B], near_tie [B], accept_gap [B] (smallest |log u_j - delta_j| over
 * the tested positions), cdf_gap [B] (the inverse-CDF gap above, or |S - 2^-18|
 * after a rejection if that is smaller; +inf when no draw was made).  Returns 0,
 * or -1 on a bad shape.
 */
int sv_oracle_verify(const void* target, const void* draft, int is_bf16,
                     const int32_t* draft_tokens, const float* temperature,
                     const float* u_accept, const float* u_resample,
                     int B, int gamma, int V,
                     int32_t* out_tokens, int32_t* out_n, double* log_norm,
                     int32_t* row_status, int32_t* near_tie, double* accept_gap,
                     double* cdf_gap, int n_threads)
{
    if (B < 0 || gamma < 1 || gamma > 32 || V < 1) return -1;
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#else
    (void)n_threads;
#endif
    int failed = 0;
#pragma omp parallel
    {
        double* wbuf = (double*)malloc(sizeof(double) * (size_t)V);
        if (!wbuf) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(dynamic, 1)
        for (int b = 0; b < B; ++b) {
            if (!wbuf) continue;
            verify_one(target, draft, is_bf16, draft_tokens + (size_t)b * gamma,
                       (double)temperature[b], u_accept + (size_t)b * gamma,
                       (double)u_resample[b], gamma, V, (size_t)b,
                       out_tokens + (size_t)b * (gamma + 1), out_n + b,
                       log_norm + (size_t)b * (2 * gamma + 1), row_status + b, near_tie + b,
                       accept_gap + b, cdf_gap + b, wbuf);
        }
        free(wbuf);
    }
    return failed ? -2 : 0;
}

/* Number of threads an OpenMP region would use (for reporting). */
int sv_oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * The speculation cache's side of the outcome [Speculative Speculative Decoding,
 * Metodologia 2, "Conceito Central" (the verification outcome is the number
 * accepted plus one more token, and the cache holds speculations for likely
 * outcomes); Desafios 1 (a geometric fan-out over the accepted lengths within a
 * budget) and 2 (the extra token after a rejection comes from the residual, and
 * Saguaro sampling puts residual mass on the cached top-F tokens)].
 *
 * sv_oracle_fanout: F_n for n in [0, gamma] from an acceptance rate alpha in
 * [0, 1] and a budget of cache slots.  P(n) = alpha^n (1 - alpha) for n < gamma and
 * alpha^gamma for n = gamma -- the law of the accepted length when every position
 * accepts with probability alpha; F_n = floor(budget * P(n)), then one more slot
 * to each n in decreasing order of budget * P(n) - F_n (ties: smaller n) until the
 * F_n add up to the budget.
 *
 * sv_oracle_topf: for sequence b and outcome n, the distribution the extra token
 * is drawn from after that outcome -- norm(max(0, p_n - q_n)) for n < gamma (p_n
 * when the residual mass is below 2^-18, as the draw does), p_gamma for n =
 * gamma; with T == 0 a point mass on the first argmax of target row n -- and its
 * F_n most probable tokens in decreasing probability (equal probabilities:
 * smaller token first), with their probabilities.  Slots past the tokens of
 * positive probability hold -1 and 0.  Sequences with an invalid temperature or
 * a bad row (status 4 or 2 as in sv_oracle_verify) hold -1 and 0 everywhere.
 * Outcome n's slots are [off_n, off_n + F_n), off_n = F_0 + ... + F_{n-1}.
 *
 * sv_oracle_cache_lookup: for sequence b with outcome n = out_n[b] and extra
 * token out_tokens[b][n], the slot s in [off_n, off_n + F_n) with
 * cache[b][s] == that token (the first one), else -1; -1 too when the sequence
 * emitted no extra token (-1).
 */
int sv_oracle_fanout(double alpha, int gamma, int budget, int32_t* F)
{
    if (gamma < 1 || gamma > 32 || budget < 0 || !(alpha >= 0.0 && alpha <= 1.0)) return -1;
    double want[33];
    int total = 0;
    for (int n = 0; n <= gamma; ++n) {
        const double P = n < gamma ? pow(alpha, n) * (1.0 - alpha) : pow(alpha, gamma);
        want[n] = (double)budget * P;
        F[n] = (int32_t)floor(want[n]);
        total += F[n];
    }
    while (total < budget) { /* largest remainder first, smaller n on ties */
        int best = 0;
        double br = -1.0;
        for (int n = 0; n <= gamma; ++n) {
            const double rem = want[n] - (double)F[n];
            if (rem > br) { br = rem; best = n; }
        }
        F[best] += 1;
        want[best] -= 1.0; /* its remainder is used up */
        total += 1;
    }
    return 0;
}

typedef struct { double w; int v; } WTok;

static int wtok_cmp(const void* a, const void* b)
{
    const WTok* x = (const WTok*)a;
    const WTok* y = (const WTok*)b;
    if (x->w > y->w) return -1;
    if (x->w < y->w) return 1;
    return (x->v > y->v) - (x->v < y->v);
}

static void topf_one(const void* tgt, const void* dft, int is_bf16, double T, int gamma, int V, size_t b,
                     const int32_t* F, int Ftot, int32_t* out_tok, double* out_p, WTok* buf)
{
    for (int s = 0; s < Ftot; ++s) { out_tok[s] = -1; out_p[s] = 0.0; }
    if (!(T == 0.0 || (isfinite(T) && T >= ORACLE_T_MIN))) return;
    const size_t trow0 = b * (size_t)(gamma + 1) * (size_t)V;
    const size_t drow0 = b * (size_t)gamma * (size_t)V;
    if (T == 0.0) {
        int arg[33];
        for (int j = 0; j <= gamma; ++j) {
            arg[j] = row_argmax(tgt, is_bf16, trow0 + (size_t)j * V, V);
            if (arg[j] < 0) return;
        }
        int off = 0;
        for (int n = 0; n <= gamma; ++n) {
            if (F[n] > 0) { out_tok[off] = arg[n]; out_p[off] = 1.0; }
            off += F[n];
        }
        return;
    }
    double lse_t[33], lse_d[32];
    for (int j = 0; j <= gamma; ++j)
        if (!row_lse(tgt, is_bf16, trow0 + (size_t)j * V, V, T, &lse_t[j])) return;
    for (int j = 0; j < gamma; ++j)
        if (!row_lse(dft, is_bf16, drow0 + (size_t)j * V, V, T, &lse_d[j])) return;
    int off = 0;
    for (int n = 0; n <= gamma; ++n) {
        double S = 0.0;
        for (int v = 0; v < V; ++v) {
            const double pt = exp(widen(tgt, is_bf16, trow0 + (size_t)n * V + v) / T - lse_t[n]);
            const double qd = n < gamma ? exp(widen(dft, is_bf16, drow0 + (size_t)n * V + v) / T - lse_d[n]) : 0.0;
            buf[v].w = n < gamma ? fmax(0.0, pt - qd) : pt;
            buf[v].v = v;
            S += buf[v].w;
        }
        if (n < gamma && !(ORACLE_RESIDUAL_MIN <= S)) { /* the residual vanished: p_n, as the draw */
            S = 0.0;
            for (int v = 0; v < V; ++v) {
                buf[v].w = exp(widen(tgt, is_bf16, trow0 + (size_t)n * V + v) / T - lse_t[n]);
                S += buf[v].w;
            }
        }
        qsort(buf, (size_t)V, sizeof(WTok), wtok_cmp);
        for (int s = 0; s < F[n] && s < V; ++s) {
            if (!(buf[s].w > 0.0)) break;
            out_tok[off + s] = buf[s].v;
            out_p[off + s] = buf[s].w / S;
        }
        off += F[n];
    }
}

/*
 * target: [B][gamma+1][V], draft: [B][gamma][V] (is_bf16 selects uint16 bf16 bits);
 * F: [gamma+1] slots per outcome.  Outputs: out_tokens [B][sum F] int32 and out_prob
 * [B][sum F] double.  Returns 0, or -1 on a bad shape.
 */
int sv_oracle_topf(const void* target, const void* draft, int is_bf16, const float* temperature, int B,
                   int gamma, int V, const int32_t* F, int32_t* out_tokens, double* out_prob, int n_threads)
{
    if (B < 0 || gamma < 1 || gamma > 32 || V < 1) return -1;
    int Ftot = 0;
    for (int n = 0; n <= gamma; ++n) {
        if (F[n] < 0) return -1;
        Ftot += F[n];
    }
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#else
    (void)n_threads;
#endif
    int failed = 0;
#pragma omp parallel
    {
        WTok* buf = (WTok*)malloc(sizeof(WTok) * (size_t)V);
        if (!buf) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(dynamic, 1)
        for (int b = 0; b < B; ++b) {
            if (!buf) continue;
            topf_one(target, draft, is_bf16, (double)temperature[b], gamma, V, (size_t)b, F, Ftot,
                     out_tokens + (size_t)b * Ftot, out_prob + (size_t)b * Ftot, buf);
        }
        free(buf);
    }
    return failed ? -2 : 0;
}

int sv_oracle_cache_lookup(const int32_t* out_tokens, const int32_t* out_n, const int32_t* cache, int B,
                           int gamma, const int32_t* F, int32_t* out_slot)
{
    if (B < 0 || gamma < 1 || gamma > 32) return -1;
    int off[34];
    off[0] = 0;
    for (int n = 0; n <= gamma; ++n) off[n + 1] = off[n] + F[n];
    const int Ftot = off[gamma + 1];
    for (int b = 0; b < B; ++b) {
        out_slot[b] = -1;
        const int n = out_n[b];
        if (n < 0 || n > gamma) continue;
        const int x = out_tokens[(size_t)b * (gamma + 1) + n];
        if (x < 0) continue;
        for (int s = off[n]; s < off[n + 1]; ++s)
            if (cache[(size_t)b * Ftot + s] == x) { out_slot[b] = s; break; }
    }
    return 0;
}

/*
 * Draft selection as a K-armed bandit [FlashSpec, Metodologia 2, "Selecao de
 * Rascunho via Bandit Online": each decoding step picks one draft model (an arm)
 * from past acceptances only; the reward is the fraction of draft tokens
 * accepted; UCB1 and Thompson sampling].
 *
 * State (K arms): t = number of rewards seen, arm = the arm chosen last (-1:
 * none yet), N[k] = rewards seen for arm k, R[k] = their sum.
 *
 * sv_oracle_bandit_step: (1) if an arm was chosen before, its reward is the
 * batch's fraction of accepted drafts, sum_b n_b / (B * gamma); N[arm] += 1,
 * R[arm] += reward, t += 1.  (2) The next arm: any arm never rewarded, the
 * smallest first; otherwise
 *   UCB1 (Auer, Cesa-Bianchi and Fischer, 2002): argmax_k R_k/N_k + sqrt(2 ln t / N_k);
 *   Thompson sampling with Gaussian posteriors (Agrawal and Goyal, 2013):
 *     argmax_k R_k/N_k + z_k / sqrt(N_k + 1), z_k = sqrt(-2 ln(1 - u1_k)) cos(2 pi u2_k)
 *     (Box-Muller), u1, u2 the caller's uniforms in [0, 1) for this step;
 *   Thompson sampling with the Beta posterior's moments (rewards in [0, 1]; a
 *     uniform prior, so after N_k rewards summing to R_k the posterior is
 *     Beta(R_k + 1, N_k - R_k + 1)): a normal draw with its mean and variance,
 *     argmax_k m_k + z_k sqrt(m_k (1 - m_k) / (N_k + 3)), m_k = (R_k + 1)/(N_k + 2);
 * ties go to the smaller k.  (3) arm = the chosen k.
 */
enum { BANDIT_UCB1 = 0, BANDIT_THOMPSON = 1, BANDIT_THOMPSON_BETA = 2 };

int sv_oracle_bandit_step(const int32_t* n_accepted, int B, int gamma, double* t, int32_t* arm, double* N,
                          double* R, int K, int policy, const float* u1, const float* u2)
{
    if (K < 1 || K > 16 || B < 0 || gamma < 1) return -1;
    if (*arm >= 0 && *arm < K && B > 0) {
        long long acc = 0;
        for (int b = 0; b < B; ++b) acc += n_accepted[b];
        const double reward = (double)acc / ((double)B * (double)gamma);
        N[*arm] += 1.0;
        R[*arm] += reward;
        *t += 1.0;
    }
    int pick = -1;
    for (int k = 0; k < K; ++k)
        if (N[k] == 0.0) { pick = k; break; }
    if (pick < 0) {
        double best = -INFINITY;
        for (int k = 0; k < K; ++k) {
            double score;
            if (policy == BANDIT_UCB1) {
                score = R[k] / N[k] + sqrt(2.0 * log(*t) / N[k]);
            } else {
                const double z = sqrt(-2.0 * log(1.0 - (double)u1[k])) * cos(2.0 * M_PI * (double)u2[k]);
                if (policy == BANDIT_THOMPSON_BETA) {
                    const double m = (R[k] + 1.0) / (N[k] + 2.0);
                    score = m + z * sqrt(m * (1.0 - m) / (N[k] + 3.0));
                } else {
                    score = R[k] / N[k] + z / sqrt(N[k] + 1.0);
                }
            }
            if (score > best) { best = score; pick = k; }
        }
    }
    *arm = pick;
    return 0;
}

/*
 * The regret simulation [FlashSpec, Resultados Principais, "Desempenho do
 * Bandit": T rounds against K arms whose rewards are Bernoulli].  Each run
 * composes sv_oracle_bandit_step with one sequence and gamma = 1, so a reward is
 * 0 or 1 accepted drafts.  uniforms[run][s][2K+1], s in [0, T]: row s holds the
 * step's u1 (K), u2 (K) and the round's reward draw r.  Step 0 (no reward yet)
 * makes the first choice from row 0; round s = 1..T adds the gap mu_max -
 * mu[arm] of the arm in play to the run's regret, then draws its reward
 * (r_s < mu[arm]) and steps with row s.  out_regret[run]; out_state, if not
 * null, gets each run's final [t, arm, N[K], R[K]].
 */
int sv_oracle_bandit_simulate(const double* mu, int K, int T, int policy, int runs, const float* uniforms,
                              double* out_regret, double* out_state)
{
    if (K < 1 || K > 16 || T < 0 || runs < 0) return -1;
    double mu_max = mu[0];
    for (int k = 1; k < K; ++k)
        if (mu[k] > mu_max) mu_max = mu[k];
    const long long row = 2 * K + 1;
    for (int r = 0; r < runs; ++r) {
        const float* u = uniforms + (long long)r * (T + 1) * row;
        double t = 0.0, N[16] = {0}, Rs[16] = {0}, regret = 0.0;
        int32_t arm = -1;
        sv_oracle_bandit_step(NULL, 0, 1, &t, &arm, N, Rs, K, policy, u, u + K);
        for (int s = 1; s <= T; ++s) {
            const float* us = u + (long long)s * row;
            int32_t reward = 0;
            if (arm >= 0) {
                regret += mu_max - mu[arm];
                reward = (double)us[2 * K] < mu[arm] ? 1 : 0;
            }
            sv_oracle_bandit_step(&reward, 1, 1, &t, &arm, N, Rs, K, policy, us, us + K);
        }
        out_regret[r] = regret;
        if (out_state) {
            double* o = out_state + (long long)r * (2 + 2 * K);
            o[0] = t;
            o[1] = (double)arm;
            for (int k = 0; k < K; ++k) {
                o[2 + k] = N[k];
                o[2 + K + k] = Rs[k];
            }
        }
    }
    return 0;
}

/*
 * Tree verification [SpecLA, Metodologia 1, "Kernels de Verificacao de Topologia
 * Conscientes": drafts shaped as chains or as branching trees; Speculative
 * Speculative Decoding, "Significado e Impacto": compatible with token trees].
 * The pages give no acceptance rule for several candidates; this follows the
 * multi-candidate form of the same speculative-sampling rule (the form whose
 * output law equals the target's when the children of a node are independent
 * draws from q at that node):
 *
 *   At node c (first the root), P starts as the target's p at c.  The children of
 *   c are tested in increasing index: child x is accepted iff
 *       log u_x < log P(tok_x) - log q(tok_x),
 *   q the draft's distribution at c.  After a rejection P becomes
 *   norm(max(0, P - q)) -- or stays P when that mass is below 2^-18 (status bit 8,
 *   the rule of sv_oracle_verify) -- and the next child is tested.  An accepted
 *   child becomes c.  When no child of c is accepted, or c has none, the extra
 *   token is drawn from P by the inverse CDF with u_resample, and the walk ends.
 *   T == 0 (greedy): the first child whose token is the first argmax of target
 *   row c is accepted; otherwise that argmax is the extra token.
 *
 * A chain (node i's parent i - 1) gives exactly sv_oracle_verify's result.
 *
 * Layout, sequence b with N nodes: node 0 is the root (the context verified so
 * far); node i >= 1 carries the draft token tok[i] and its parent par[i] in
 * [0, i); par[0] = -1.  target [B][N][V]: the target's next-token logits at node
 * i's context (the path to i, tok[i] included); draft [B][N][V]: the draft's,
 * the distribution node i's children were drawn from.  keep [B][N], optional:
 * node i >= 1 takes part iff keep[i] != 0 and its parent takes part.
 * u_accept [B][N]: the uniform of node i's test (entry 0 unused).
 *
 * P is held as weights w with P = w / S_w: w = p and S_w = 1 at first, then w =
 * max(0, P - q) and S_w = its sum, so the first residual and its draw are
 * sv_oracle_verify's bit for bit.
 *
 * Status: 4 bad temperature; 32 a parent index out of range; 1 a token of a
 * node that takes part outside [0, V); 16 (T > 0) u_accept of a node that takes
 * part, or u_resample, outside [0, 1) or NaN; 2 a row the walk reads (target row
 * of every node visited; T > 0: the draft row of every visited node that has
 * children taking part) is bad.  With 1, 2, 4, 16 or 32 nothing is emitted.
 * Near ties: bit 1 at a test with |log u - delta| below 1e-6 (the first child
 * of a node) or below 1e-6 + the relative error bound of P(tok) (later
 * children: fp32 weights carry about 4e-6 relative error per rounding, tracked
 * through the residual levels); bit 2 at a draw whose inverse-CDF gap is below
 * 1e-6, plus the tracked error of the weights after two or more rejections, or
 * whose residual mass lies within that of the 2^-18 threshold.
 */
#define ST_TREE 32
#define ORACLE_EPS_W 4e-6

static int tree_child_after(const int32_t* par, const int* in, int N, int c, int from)
{
    for (int i = from; i < N; ++i)
        if (in[i] && par[i] == c) return i;
    return -1;
}

static void tree_one(const void* tgt, const void* dft, int is_bf16, const int32_t* par, const int32_t* tok,
                     const int32_t* keep, double T, const float* u_acc, double u_res, int N, int V, size_t b,
                     int32_t* out_nodes, int32_t* out_tok, int32_t* out_n, double* lnorm, int32_t* status,
                     int32_t* near, double* agap, double* cgap, double* wbuf, double* ebuf)
{
    int st = 0, nr = 0, in[64];
    *agap = INFINITY;
    *cgap = INFINITY;
    for (int i = 0; i < N; ++i) { out_nodes[i] = -1; out_tok[i] = -1; }
    for (int r = 0; r < 2 * N; ++r) lnorm[r] = NAN;
    *out_n = 0;
    *near = 0;
    if (!(T == 0.0 || (isfinite(T) && T >= ORACLE_T_MIN))) { *status = ST_TEMP; return; }
    if (par[0] != -1) st |= ST_TREE;
    in[0] = 1;
    for (int i = 1; i < N; ++i) {
        if (par[i] < 0 || par[i] >= i) { st |= ST_TREE; in[i] = 0; continue; }
        in[i] = in[par[i]] && (keep == NULL || keep[i] != 0);
    }
    for (int i = 1; i < N; ++i)
        if (in[i] && (tok[i] < 0 || tok[i] >= V)) st |= ST_TOKEN;
    if (T > 0.0) {
        for (int i = 1; i < N; ++i)
            if (in[i] && !(u_acc[i] >= 0.0f && u_acc[i] < 1.0f)) st |= ST_UNIFORM;
        if (!(u_res >= 0.0 && u_res < 1.0)) st |= ST_UNIFORM;
    }
    if (st) { *status = st; return; }

    const size_t base = b * (size_t)N * (size_t)V;
    int c = 0, n = 0, k = -1;
    if (T == 0.0) {
        for (;;) {
            const int a = row_argmax(tgt, is_bf16, base + (size_t)c * V, V);
            if (a < 0) { st |= ST_ROW; break; }
            int next = -1;
            for (int i = tree_child_after(par, in, N, c, c + 1); i >= 0; i = tree_child_after(par, in, N, c, i + 1))
                if (tok[i] == a) { next = i; break; }
            if (next < 0) { k = a; break; }
            out_nodes[n] = next;
            ++n;
            c = next;
        }
    } else {
        for (;;) {
            double lse_t, lse_d = 0.0;
            const size_t trow = base + (size_t)c * V;
            if (!row_lse(tgt, is_bf16, trow, V, T, &lse_t)) { st |= ST_ROW; break; }
            lnorm[c] = lse_t;
            const int first = tree_child_after(par, in, N, c, c + 1);
            if (first >= 0) {
                if (!row_lse(dft, is_bf16, trow, V, T, &lse_d)) { st |= ST_ROW; break; }
                lnorm[N + c] = lse_d;
            }
            /* P = w / Sw, first the target's p at c */
            double Sw = 1.0;
            int level = 0;
            for (int v = 0; v < V; ++v) {
                wbuf[v] = exp(widen(tgt, is_bf16, trow + (size_t)v) / T - lse_t);
                ebuf[v] = ORACLE_EPS_W * wbuf[v];
            }
            int next = -1;
            double resid_gap = INFINITY;
            for (int i = first; i >= 0; i = tree_child_after(par, in, N, c, i + 1)) {
                const int x = tok[i];
                const double lq = widen(dft, is_bf16, trow + (size_t)x) / T - lse_d;
                const double lp = level == 0 ? widen(tgt, is_bf16, trow + (size_t)x) / T - lse_t
                                             : log(wbuf[x]) - log(Sw);
                const double delta = lp - lq;
                const double lu = log((double)u_acc[i]);
                /* a weight of exactly 0 rejects whatever u is: no band */
                const double band = level == 0 ? ORACLE_NEAR
                                    : (wbuf[x] > 0.0 ? ORACLE_NEAR + ebuf[x] / wbuf[x] + ORACLE_EPS_W : 0.0);
                const double g = fabs(lu - delta);
                if (g < *agap) *agap = g;
                if (!(g >= band)) nr |= NEAR_ACCEPT;
                if (lu < delta) { next = i; break; }
                /* rejected: the next child is tested against norm(max(0, P - q)) */
                double S = 0.0, E = 0.0;
                for (int v = 0; v < V; ++v) {
                    const double q = exp(widen(dft, is_bf16, trow + (size_t)v) / T - lse_d);
                    const double P = wbuf[v] / Sw;
                    S += fmax(0.0, P - q);
                    if (P + ebuf[v] / Sw + ORACLE_EPS_W * q > q) E += ebuf[v] / Sw + ORACLE_EPS_W * q;
                }
                const double thr_band = level == 0 ? ORACLE_NEAR : ORACLE_NEAR + E;
                if (fabs(S - ORACLE_RESIDUAL_MIN) < resid_gap) resid_gap = fabs(S - ORACLE_RESIDUAL_MIN);
                if (fabs(S - ORACLE_RESIDUAL_MIN) < thr_band) nr |= NEAR_CDF;
                if (S < ORACLE_RESIDUAL_MIN || S != S) {
                    st = st | ST_RESID0; /* the residual vanished: P stays */
                    continue;
                }
                for (int v = 0; v < V; ++v) {
                    const double q = exp(widen(dft, is_bf16, trow + (size_t)v) / T - lse_d);
                    const double P = wbuf[v] / Sw;
                    const double e = ebuf[v] / Sw + ORACLE_EPS_W * q;
                    wbuf[v] = fmax(0.0, P - q);
                    ebuf[v] = (P + ebuf[v] / Sw + ORACLE_EPS_W * q > q) ? e : 0.0;
                }
                Sw = S;
                ++level;
            }
            if (next >= 0) {
                out_nodes[n] = next;
                ++n;
                c = next;
                continue;
            }
            /* the extra token: from P (p itself when nothing was rejected) */
            k = inverse_cdf(wbuf, V, u_res, &nr, cgap);
            if (resid_gap < *cgap) *cgap = resid_gap;
            if (level >= 2) {
                double Et = 0.0;
                for (int v = 0; v < V; ++v) Et += ebuf[v];
                if (*cgap < ORACLE_NEAR + Et) nr |= NEAR_CDF;
            }
            break;
        }
    }
    if (st & (ST_ROW | ST_TOKEN | ST_UNIFORM | ST_TEMP | ST_TREE)) {
        for (int i = 0; i < N; ++i) { out_nodes[i] = -1; out_tok[i] = -1; }
        *out_n = 0;
        *status = st;
        *near = 0;
        return;
    }
    for (int j = 0; j < n; ++j) out_tok[j] = tok[out_nodes[j]];
    out_tok[n] = k;
    *out_n = n;
    *status = st;
    *near = nr;
}

/*
 * target, draft: [B][N][V]; parent, tokens, u_accept: [B][N]; keep: [B][N] or
 * NULL.  Outputs: out_nodes, out_tokens [B][N]; out_n [B]; log_norm [B][2N]
 * (target rows, then draft rows; NaN for rows not read); row_status, near_tie
 * [B]; accept_gap, cdf_gap [B] as in sv_oracle_verify.  Returns 0, -1 on a bad
 * shape (N outside [1, 64], V < 1), -2 if memory ran out.
 */
int sv_oracle_tree_verify(const void* target, const void* draft, int is_bf16, const int32_t* parent,
                          const int32_t* tokens, const int32_t* keep, const float* temperature,
                          const float* u_accept, const float* u_resample, int B, int N, int V,
                          int32_t* out_nodes, int32_t* out_tokens, int32_t* out_n, double* log_norm,
                          int32_t* row_status, int32_t* near_tie, double* accept_gap, double* cdf_gap,
                          int n_threads)
{
    if (B < 0 || N < 1 || N > 64 || V < 1) return -1;
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#else
    (void)n_threads;
#endif
    int failed = 0;
#pragma omp parallel
    {
        double* wbuf = (double*)malloc(sizeof(double) * 2 * (size_t)V);
        if (!wbuf) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(dynamic, 1)
        for (int b = 0; b < B; ++b) {
            if (!wbuf) continue;
            const size_t o = (size_t)b * N;
            tree_one(target, draft, is_bf16, parent + o, tokens + o, keep ? keep + o : NULL,
                     (double)temperature[b], u_accept + o, (double)u_resample[b], N, V, (size_t)b,
                     out_nodes + o, out_tokens + o, out_n + b, log_norm + 2 * o, row_status + b, near_tie + b,
                     accept_gap + b, cdf_gap + b, wbuf, wbuf + V);
        }
        free(wbuf);
    }
    return failed ? -2 : 0;
}

/*
 * Pruning by cumulative path probability [SpecLA, Metodologia 3, "Poda Guiada
 * por Confianca": paths of low cumulative draft log-probability are removed
 * before verification].  For node i >= 1 with parent c:
 *     cum[i] = cum[c] + log q_c(tok[i]),  cum[0] = 0,
 * log q_c = ld[c]/T - lse(ld[c]/T) for T > 0; for T == 0 the draft is greedy and
 * log q_c(x) is 0 at the first argmax of draft row c, -inf elsewhere.
 * keep[0] = 1; keep[i] = keep[c] and not (cum[i] < threshold).  Where cum cannot
 * be formed (bad temperature or tree: every node of the sequence; a token
 * outside [0, V) or a bad draft row c: the node) it is NaN and the node is kept,
 * so the verification reports the fault.  out_keep [B][N] int32, out_cum [B][N].
 */
int sv_oracle_tree_prune(const void* draft, int is_bf16, const int32_t* parent, const int32_t* tokens,
                         const float* temperature, double threshold, int B, int N, int V, int32_t* out_keep,
                         double* out_cum)
{
    if (B < 0 || N < 1 || N > 64 || V < 1) return -1;
    for (int b = 0; b < B; ++b) {
        const size_t o = (size_t)b * N;
        const int32_t* par = parent + o;
        const int32_t* tok = tokens + o;
        const double T = (double)temperature[b];
        int ok = (T == 0.0 || (isfinite(T) && T >= ORACLE_T_MIN)) && par[0] == -1;
        for (int i = 1; i < N; ++i)
            if (par[i] < 0 || par[i] >= i) ok = 0;
        out_keep[o] = 1;
        out_cum[o] = ok ? 0.0 : NAN;
        for (int i = 1; i < N; ++i) {
            if (!ok) { out_keep[o + i] = 1; out_cum[o + i] = NAN; continue; }
            const int c = par[i];
            const size_t row = (o + (size_t)c) * (size_t)V;
            double lq = NAN;
            if (tok[i] >= 0 && tok[i] < V) {
                if (T == 0.0) {
                    const int a = row_argmax(draft, is_bf16, row, V);
                    if (a >= 0) lq = (tok[i] == a) ? 0.0 : -INFINITY;
                } else {
                    double lse;
                    if (row_lse(draft, is_bf16, row, V, T, &lse))
                        lq = widen(draft, is_bf16, row + (size_t)tok[i]) / T - lse;
                }
            }
            out_cum[o + i] = out_cum[o + c] + lq;
            out_keep[o + i] = out_keep[o + c] && !(out_cum[o + i] < threshold);
        }
    }
    return 0;
}

/*
 * The low-rank draft head [SlimSpec, Metodologia, "Arquitetura": z = W_up W_down h
 * with W_down in R^{r x d}, W_up in R^{V x r}, r << d, instead of W_full h].
 *
 * Inputs are bf16 (uint16 bit patterns): h [M][d] (one row per draft position),
 * W_down [r][d], W_up [V][r].  The product is taken in two contractions, the
 * intermediate stored in bf16 (this library's reading: the second contraction
 * takes bf16 operands like the first):
 *     u[m][i] = bf16( sum_k W_down[i][k] h[m][k] )       (round to nearest even)
 *     z[m][v] = sum_i W_up[v][i] u[m][i]                  (exact here, fp64)
 * and the draft row's log-normaliser at temperature T_m of the logits as the
 * verifier reads them, bf16(z):
 *     lse[m] = M/T + log sum_v exp((bf16(z[m][v]) - M)/T),  M = max_v bf16(z[m][v])
 * (NaN for T_m = 0).  Sums of products are accumulated in fp64.
 */
/* x rounded to the nearest bf16 value (8 significant bits, the exponent range of
 * float32), ties to even; +-inf past the largest finite bf16. */
static double bf16_round(double x)
{
    if (!isfinite(x) || x == 0.0) return x;
    const double tiny = 0x1p-126; /* below it bf16 values are spaced 2^-133 */
    double r;
    if (fabs(x) < tiny) {
        r = ldexp(nearbyint(ldexp(x, 133)), -133);
    } else {
        int e;
        const double f = frexp(x, &e);                /* x = f 2^e, 0.5 <= |f| < 1 */
        r = ldexp(nearbyint(ldexp(f, 8)), e - 8);     /* default mode: nearest, ties to even */
    }
    if (fabs(r) > 0x1.fep127) r = copysign(INFINITY, r);
    return r;
}

static double bf16_value(const uint16_t* p, size_t i)
{
    uint32_t bits = (uint32_t)p[i] << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/* out[m][n] = sum_k A[m][k] B[n][k] over bf16 inputs, in fp64. */
int sv_oracle_gemm_bf16(const uint16_t* A, const uint16_t* B, int M, int N, int K, double* out)
{
    if (M < 0 || N < 0 || K < 0) return -1;
    for (int m = 0; m < M; ++m)
        for (int n = 0; n < N; ++n) {
            double s = 0.0;
            for (int k = 0; k < K; ++k) s += bf16_value(A, (size_t)m * K + k) * bf16_value(B, (size_t)n * K + k);
            out[(size_t)m * N + n] = s;
        }
    return 0;
}

/* bf16 of a double, ties to even, as the bit pattern. */
static uint16_t bf16_bits(double x)
{
    const float f = (float)bf16_round(x); /* exact: 8 significant bits fit in float */
    uint32_t bits;
    memcpy(&bits, &f, sizeof bits);
    return (uint16_t)(bits >> 16);
}

int sv_oracle_lowrank_head(const uint16_t* h, const uint16_t* w_down, const uint16_t* w_up, int M, int d, int r,
                           int V, const float* temperature, uint16_t* out_u, double* out_z, double* out_lse)
{
    if (M < 0 || d < 1 || r < 1 || V < 1) return -1;
    double* tmp = (double*)malloc(sizeof(double) * (size_t)(M > 0 ? M : 1) * (size_t)r);
    if (!tmp) return -2;
    sv_oracle_gemm_bf16(h, w_down, M, r, d, tmp);
    for (size_t i = 0; i < (size_t)M * r; ++i) out_u[i] = bf16_bits(tmp[i]);
    free(tmp);
    sv_oracle_gemm_bf16(out_u, w_up, M, V, r, out_z);
    for (int m = 0; m < M; ++m) {
        const double T = temperature ? (double)temperature[m] : 1.0;
        if (!(T > 0.0) || !isfinite(T)) { out_lse[m] = NAN; continue; }
        const double* z = out_z + (size_t)m * V;
        double mx = -INFINITY;
        for (int v = 0; v < V; ++v) mx = fmax(mx, bf16_round(z[v]));
        double s = 0.0;
        for (int v = 0; v < V; ++v) s += exp((bf16_round(z[v]) - mx) / T);
        out_lse[m] = mx / T + log(s);
    }
    return 0;
}
