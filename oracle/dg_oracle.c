/*
 * dg_oracle.c -- plain, slow, single-threaded CPU oracle for the DiffusionGemma
 * per-step sampler and its training-side companions.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the CUDA library and
 * its Python binding) may link, load or call this file.  Only the tests, the
 * smoke check and the benchmark's CPU-baseline leg use it.  It shares no code,
 * header, table or constant generator with the CUDA path.
 *
 * Precision: every floating-point quantity is computed in double.  Logits and
 * embeddings arrive as float (bf16 inputs are widened exactly by the caller).
 *
 * Sources ("the pages") and how they are cited:
 *   [TR-Method] DiffusionGemma Technical Report, hyper.ai paper summary,
 *               section "Method" (方法): forward probability path equation,
 *               noise schedule kappa_t, Step reverse-transition equation,
 *               the per-iteration update (Softmax / FFW(p0 E) / Step) and the
 *               canvas cross-entropy loss equation.
 *   [TR-Data]   same page, section "Dataset" (数据集): the P + K*C sequence
 *               layout, the decoder loss on one uniformly chosen canvas.
 *   [Philox]    J. K. Salmon, M. A. Moraes, R. O. Dror, D. E. Shaw,
 *               "Parallel random numbers: as easy as 1, 2, 3", SC'11:
 *               Philox4x32 round function, multipliers and Weyl key bumps.
 *
 * Readings where the pages leave a step open are listed in the header of each
 * function; the same list is kept in the repository's design notes.
 *
 * Parity pins: every function here is checked by a CPU test against something
 * other than itself (published known-answer vectors, closed forms, brute-force
 * Bayes, chi-square against the defining distribution, library routines).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* Philox4x32-10 [Philox]: a 10-round bijection of a 128-bit counter keyed   */
/* by a 64-bit key.  Round: two 32x32->64 products of counter words 0 and 2  */
/* with the published multipliers; the high halves are xored with the other  */
/* counter words and the key; the key is bumped by the published Weyl        */
/* constants between rounds.                                                 */
/* ------------------------------------------------------------------------ */
#define PHILOX_MUL_A 0xD2511F53u
#define PHILOX_MUL_B 0xCD9E8D57u
#define PHILOX_WEYL_A 0x9E3779B9u
#define PHILOX_WEYL_B 0xBB67AE85u

void dgo_philox4x32_10(const uint32_t ctr_in[4], const uint32_t key_in[2], uint32_t out[4])
{
    uint32_t c[4] = {ctr_in[0], ctr_in[1], ctr_in[2], ctr_in[3]};
    uint32_t k0 = key_in[0], k1 = key_in[1];
    for (int round = 0; round < 10; ++round) {
        if (round > 0) {
            k0 += PHILOX_WEYL_A;
            k1 += PHILOX_WEYL_B;
        }
        uint64_t p0 = (uint64_t)PHILOX_MUL_A * (uint64_t)c[0];
        uint64_t p1 = (uint64_t)PHILOX_MUL_B * (uint64_t)c[2];
        uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
        uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
        uint32_t n0 = hi1 ^ c[1] ^ k0;
        uint32_t n2 = hi0 ^ c[3] ^ k1;
        c[0] = n0;
        c[1] = lo1;
        c[2] = n2;
        c[3] = lo0;
    }
    memcpy(out, c, sizeof(c));
}

/* Counter domains (word 3 of the counter) -- a layout of our own, fixed
 * before any GPU code: the pages name no random-number generator. */
enum {
    DOM_GUMBEL_TOKEN = 0, DOM_STEP = 1, DOM_NOISE = 2, DOM_CANVAS = 3, DOM_GUMBEL_CHUNK = 4,
    DOM_RENOISE = 5, DOM_SC_DROP = 6
};

static void philox_word4(uint64_t seed, uint32_t c0, uint32_t c1, uint32_t c2, uint32_t dom,
                         uint32_t out[4])
{
    uint32_t ctr[4] = {c0, c1, c2, dom};
    uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    dgo_philox4x32_10(ctr, key, out);
}

/* Uniform on (0,1) from a 32-bit word: the top 23 bits give the odd
 * multiple (2k+1) * 2^-24, exact in float and double, never 0 or 1. */
double dgo_open_uniform(uint32_t w)
{
    return (double)(2u * (w >> 9) + 1u) * (1.0 / 16777216.0);
}

/* Standard Gumbel variate -log(-log u). */
double dgo_gumbel(uint32_t w)
{
    double u = dgo_open_uniform(w);
    return -log(-log(u));
}

/* floor(w * n / 2^32): a uniform index in [0, n) from one word. */
static int32_t word_to_index(uint32_t w, int32_t n)
{
    return (int32_t)(((uint64_t)w * (uint64_t)(uint32_t)n) >> 32);
}

/* w * 2^-32 as a double in [0, 1): exact. */
static double word_to_unit(uint32_t w)
{
    return (double)w * (1.0 / 4294967296.0);
}

/* ------------------------------------------------------------------------ */
/* Noise schedule [TR-Method]: kappa decreases monotonically and smoothly    */
/* from kappa_0 = 1 to kappa_1 = 0.  The pages give no functional form; the  */
/* two forms here are the workloads' (linear 1 - t, cosine cos^2(pi t / 2)). */
/* ------------------------------------------------------------------------ */
double dgo_kappa(int schedule, double t)
{
    if (schedule == 0) return 1.0 - t;
    double c = cos(M_PI * t / 2.0);
    return c * c;
}

/* ------------------------------------------------------------------------ */
/* Softmax statistics of one row of tempered logits l' = l * inv_tau         */
/* [TR-Method, p0 = Softmax(L_t / tau_t)].                                   */
/*   m = max l',  S = sum exp(l' - m),  lse = m + ln S,                     */
/*   max-prob = exp(m - lse) = 1/S,  entropy = -sum p ln p.                  */
/* Entropy is accumulated directly as -sum p_v ln p_v with p_v formed        */
/* explicitly (no shortcut formula), so the pins test the definition.        */
/* ------------------------------------------------------------------------ */
void dgo_row_stats(const float* l, int32_t V, double inv_tau, double* lse_out,
                   double* maxprob_out, double* entropy_out)
{
    double m = -INFINITY;
    for (int32_t v = 0; v < V; ++v) {
        double x = (double)l[v] * inv_tau;
        if (x > m) m = x;
    }
    double S = 0.0;
    for (int32_t v = 0; v < V; ++v) S += exp((double)l[v] * inv_tau - m);
    double lse = m + log(S);
    double H = 0.0, pmax = 0.0;
    for (int32_t v = 0; v < V; ++v) {
        double lp = (double)l[v] * inv_tau - lse; /* log p_v */
        double p = exp(lp);
        if (p > 0.0) H -= p * lp;
        if (p > pmax) pmax = p;
    }
    *lse_out = lse;
    *maxprob_out = pmax;
    *entropy_out = H;
}

/* Probabilities of one row (for pins: they must sum to one). */
void dgo_row_probs(const float* l, int32_t V, double inv_tau, double* p_out)
{
    double lse, pm, H;
    dgo_row_stats(l, V, inv_tau, &lse, &pm, &H);
    for (int32_t v = 0; v < V; ++v) p_out[v] = exp((double)l[v] * inv_tau - lse);
}

/* Deterministic prediction: the lowest index attaining the maximum of the
 * raw logits (the "deterministic sequence prediction" that adaptive stopping
 * compares across steps [TR-Method]; ties go to the lowest index). */
int32_t dgo_argmax(const float* l, int32_t V)
{
    int32_t best = 0;
    for (int32_t v = 1; v < V; ++v)
        if (l[v] > l[best]) best = v;
    return best;
}

/* ------------------------------------------------------------------------ */
/* Draw x0_hat ~ p0 = softmax(l') by two-level Gumbel-max.                   */
/*                                                                           */
/* Reading: the pages say only that the approximate posterior is used to     */
/* sample the next state [TR-Method].  The draw is Gumbel-max, keyed by      */
/* (seed, step, row, position), applied in two levels:                       */
/*   level 1: the vocabulary is cut into chunks of Q consecutive ids (the    */
/*            last one ragged).  Chunk c scores lse_c + G_c, with lse_c the  */
/*            log-sum-exp of l' over the chunk and G_c a Gumbel variate from */
/*            counter (c>>2, row, step, DOM_GUMBEL_CHUNK), word c&3.  The    */
/*            chunk with the highest score wins (lowest c on ties).          */
/*   level 2: inside the winning chunk, x0_hat = argmax_v l'_v + G_v, G_v    */
/*            from counter (v>>2, row, step, DOM_GUMBEL_TOKEN), word v&3     */
/*            (lowest v on ties).                                            */
/* The maximum of independent Gumbel-perturbed log-weights over a set is     */
/* Gumbel-distributed at the set's log-sum-exp, and the winner is softmax-   */
/* distributed, so the two levels together draw exactly from softmax(l').   */
/* With V <= Q there is one chunk and this is plain Gumbel-max.              */
/*                                                                           */
/* gap1 / gap2: (best - second best) / max(|best|, 1) at each level, or      */
/* +inf where a level has a single candidate; small gaps mark near-ties.     */
/* ------------------------------------------------------------------------ */
int32_t dgo_draw_x0(const float* l, int32_t V, double inv_tau, uint64_t seed, uint32_t step,
                    uint32_t row, int32_t Q, double* gap1, double* gap2)
{
    int32_t n_chunks = (V + Q - 1) / Q;
    double best1 = -INFINITY, second1 = -INFINITY;
    int32_t best_chunk = 0;
    uint32_t w[4];
    for (int32_t c = 0; c < n_chunks; ++c) {
        int32_t lo = c * Q, hi = lo + Q < V ? lo + Q : V;
        double m = -INFINITY;
        for (int32_t v = lo; v < hi; ++v) {
            double x = (double)l[v] * inv_tau;
            if (x > m) m = x;
        }
        double S = 0.0;
        for (int32_t v = lo; v < hi; ++v) S += exp((double)l[v] * inv_tau - m);
        double lse_c = m + log(S);
        philox_word4(seed, (uint32_t)c >> 2, row, step, DOM_GUMBEL_CHUNK, w);
        double score = lse_c + dgo_gumbel(w[c & 3]);
        if (score > best1) {
            second1 = best1;
            best1 = score;
            best_chunk = c;
        } else if (score > second1) {
            second1 = score;
        }
    }
    *gap1 = n_chunks > 1 ? (best1 - second1) / fmax(fabs(best1), 1.0) : INFINITY;

    int32_t lo = best_chunk * Q, hi = lo + Q < V ? lo + Q : V;
    double best2 = -INFINITY, second2 = -INFINITY;
    int32_t winner = lo;
    for (int32_t v = lo; v < hi; ++v) {
        philox_word4(seed, (uint32_t)v >> 2, row, step, DOM_GUMBEL_TOKEN, w);
        double score = (double)l[v] * inv_tau + dgo_gumbel(w[v & 3]);
        if (score > best2) {
            second2 = best2;
            best2 = score;
            winner = v;
        } else if (score > second2) {
            second2 = score;
        }
    }
    *gap2 = hi - lo > 1 ? (best2 - second2) / fmax(fabs(best2), 1.0) : INFINITY;
    return winner;
}

/* ------------------------------------------------------------------------ */
/* Draw x0_hat ~ p0 = softmax(l') by plain (flat) Gumbel-max over the whole  */
/* vocabulary: x0_hat = argmax_v l'_v + G_v, one Gumbel variate per id from  */
/* counter (v>>2, row, step, DOM_GUMBEL_TOKEN), word v&3 -- the same words   */
/* the two-level draw uses inside its winning chunk.  This is the textbook   */
/* Gumbel-max definition, with no chunking; the tests compare the two-level  */
/* draw above with it in distribution at the full vocabulary size.  Ties go  */
/* to the lowest id.  gap: (best - second best) / max(|best|, 1).            */
/* ------------------------------------------------------------------------ */
int32_t dgo_draw_x0_flat(const float* l, int32_t V, double inv_tau, uint64_t seed, uint32_t step,
                         uint32_t row, double* gap)
{
    double best = -INFINITY, second = -INFINITY;
    int32_t winner = 0;
    uint32_t w[4];
    for (int32_t v = 0; v < V; ++v) {
        if ((v & 3) == 0) philox_word4(seed, (uint32_t)v >> 2, row, step, DOM_GUMBEL_TOKEN, w);
        double score = (double)l[v] * inv_tau + dgo_gumbel(w[v & 3]);
        if (score > best) {
            second = best;
            best = score;
            winner = v;
        } else if (score > second) {
            second = score;
        }
    }
    *gap = V > 1 ? (best - second) / fmax(fabs(best), 1.0) : INFINITY;
    return winner;
}

/* Many draws of one row, one per (seed[k], step[k]) key, for the statistical */
/* pins: flat != 0 runs dgo_draw_x0_flat per key; otherwise the two-level     */
/* draw of dgo_draw_x0 with chunk width Q, whose per-chunk log-sum-exps do    */
/* not depend on the key and are computed once (with the same arithmetic as   */
/* dgo_draw_x0, so every draw equals that function's).                        */
void dgo_draw_x0_keys(const float* l, int32_t V, double inv_tau, const uint64_t* seeds,
                      const uint32_t* steps, int32_t n, uint32_t row, int32_t Q, int32_t flat,
                      int32_t* out)
{
    double gap;
    if (flat) {
        for (int32_t k = 0; k < n; ++k)
            out[k] = dgo_draw_x0_flat(l, V, inv_tau, seeds[k], steps[k], row, &gap);
        return;
    }
    int32_t n_chunks = (V + Q - 1) / Q;
    double* lse_c = (double*)malloc(sizeof(double) * (size_t)n_chunks);
    for (int32_t c = 0; c < n_chunks; ++c) {
        int32_t lo = c * Q, hi = lo + Q < V ? lo + Q : V;
        double m = -INFINITY;
        for (int32_t v = lo; v < hi; ++v) {
            double x = (double)l[v] * inv_tau;
            if (x > m) m = x;
        }
        double S = 0.0;
        for (int32_t v = lo; v < hi; ++v) S += exp((double)l[v] * inv_tau - m);
        lse_c[c] = m + log(S);
    }
    uint32_t w[4];
    for (int32_t k = 0; k < n; ++k) {
        double best1 = -INFINITY;
        int32_t best_chunk = 0;
        for (int32_t c = 0; c < n_chunks; ++c) {
            philox_word4(seeds[k], (uint32_t)c >> 2, row, steps[k], DOM_GUMBEL_CHUNK, w);
            double score = lse_c[c] + dgo_gumbel(w[c & 3]);
            if (score > best1) {
                best1 = score;
                best_chunk = c;
            }
        }
        int32_t lo = best_chunk * Q, hi = lo + Q < V ? lo + Q : V;
        double best2 = -INFINITY;
        int32_t winner = lo;
        for (int32_t v = lo; v < hi; ++v) {
            philox_word4(seeds[k], (uint32_t)v >> 2, row, steps[k], DOM_GUMBEL_TOKEN, w);
            double score = (double)l[v] * inv_tau + dgo_gumbel(w[v & 3]);
            if (score > best2) {
                best2 = score;
                winner = v;
            }
        }
        out[k] = winner;
    }
    free(lse_c);
}

/* ------------------------------------------------------------------------ */
/* The Step reverse transition [TR-Method, Step equation], read as ancestral */
/* sampling: x0_hat ~ p0 (above), then the exact posterior of the uniform    */
/* mixture path                                                              */
/*     P(X_s = . | X_t = x_t, X_0 = x0_hat),  s = max(t - dt, 0),            */
/* built from the forward marginal kappa_t delta(x, x0) + (1 - kappa_t)/V    */
/* [TR-Method, forward path equation].  Between s < t the only uniform-      */
/* mixture kernel consistent with those marginals is                         */
/*     P(x_t | x_s) = alpha delta(x_t, x_s) + (1 - alpha)/V,                 */
/*     alpha = kappa_t / kappa_s,                                            */
/* and Bayes' rule gives, with a = x_t and b = x0_hat,                       */
/*   b != a:  P(x_s = a) = (alpha + (1-alpha)/V)(1-kappa_s)/(1-kappa_t)      */
/*            P(x_s = b) = (1-alpha)(kappa_s + (1-kappa_s)/V)/(1-kappa_t)    */
/*            P(x_s = c) = (1-alpha)(1-kappa_s)/(V (1-kappa_t)), c not a, b  */
/*   b == a:  D = kappa_t + (1-kappa_t)/V,                                   */
/*            P(x_s = c) = (1-alpha)(1-kappa_s)/(V^2 D) for c != a, rest a.  */
/* Written as a three-way mixture "stay at a" / "jump to b" / "uniform over  */
/* V" (the uniform part covers every token once, a and b included):          */
/*   b != a: stay = alpha(1-kappa_s)/(1-kappa_t),                            */
/*           jump = (1-alpha) kappa_s/(1-kappa_t),  uniform = the rest.      */
/*   b == a: uniform = (1-alpha)(1-kappa_s)/(V D), stay = the rest.          */
/* One Philox draw, counter (0, row, step, DOM_STEP): word 0 picks the       */
/* branch (u = w0 * 2^-32 against the cumulative masses), word 1 the uniform */
/* token floor(w1 V / 2^32).                                                 */
/* If kappa_s <= kappa_t (dt = 0 in effect) the state stays at x_t.          */
/* Branch codes: 0 stay, 1 jump to x0_hat, 2 uniform.                        */
/* ------------------------------------------------------------------------ */
int32_t dgo_step(int32_t x_t, int32_t x0_hat, double kappa_t, double kappa_s, int32_t V,
                 uint64_t seed, uint32_t step, uint32_t row, uint8_t* branch)
{
    if (kappa_s <= kappa_t) {
        *branch = 0;
        return x_t;
    }
    uint32_t w[4];
    philox_word4(seed, 0u, row, step, DOM_STEP, w);
    double u = word_to_unit(w[0]);
    double alpha = kappa_t / kappa_s;
    if (x0_hat != x_t) {
        double stay = alpha * (1.0 - kappa_s) / (1.0 - kappa_t);
        double jump = (1.0 - alpha) * kappa_s / (1.0 - kappa_t);
        if (u < stay) {
            *branch = 0;
            return x_t;
        }
        if (u < stay + jump) {
            *branch = 1;
            return x0_hat;
        }
        *branch = 2;
        return word_to_index(w[1], V);
    }
    double D = kappa_t + (1.0 - kappa_t) / (double)V;
    double uniform = (1.0 - alpha) * (1.0 - kappa_s) / ((double)V * D);
    if (u < 1.0 - uniform) {
        *branch = 0;
        return x_t;
    }
    *branch = 2;
    return word_to_index(w[1], V);
}

/* Exact posterior probabilities P(x_s = v | x_t, x0) for all v (pins). */
void dgo_step_posterior(int32_t x_t, int32_t x0, double kappa_t, double kappa_s, int32_t V,
                        double* p_out)
{
    if (kappa_s <= kappa_t) {
        for (int32_t v = 0; v < V; ++v) p_out[v] = v == x_t ? 1.0 : 0.0;
        return;
    }
    double alpha = kappa_t / kappa_s;
    if (x0 != x_t) {
        double stay = alpha * (1.0 - kappa_s) / (1.0 - kappa_t);
        double jump = (1.0 - alpha) * kappa_s / (1.0 - kappa_t);
        double each = (1.0 - stay - jump) / (double)V;
        for (int32_t v = 0; v < V; ++v)
            p_out[v] = each + (v == x_t ? stay : 0.0) + (v == x0 ? jump : 0.0);
        return;
    }
    double D = kappa_t + (1.0 - kappa_t) / (double)V;
    double uniform = (1.0 - alpha) * (1.0 - kappa_s) / ((double)V * D);
    for (int32_t v = 0; v < V; ++v)
        p_out[v] = uniform / (double)V + (v == x_t ? 1.0 - uniform : 0.0);
}

/* ------------------------------------------------------------------------ */
/* One whole sampler step over B canvases of C rows [TR-Method, per-         */
/* iteration update].  logits: float [B*C, ld]; per-canvas host scalars t,   */
/* dt, inv_tau (inv_tau may be NULL: 1).  mode 0 = sample (two-level Gumbel- */
/* max), 1 = greedy (x0_hat = argmax).  Outputs are per row.                 */
/* ------------------------------------------------------------------------ */
void dgo_sampler_step(const float* logits, int64_t ld, const int32_t* x_t, int32_t B, int32_t C,
                      int32_t V, int32_t schedule, const double* t, const double* dt,
                      const float* inv_tau, uint64_t seed, uint32_t step, int32_t mode, int32_t Q,
                      int32_t* x_next, int32_t* x0_hat, int32_t* argmax, double* max_prob,
                      double* lse, double* entropy, uint8_t* branch, double* gap1, double* gap2)
{
    for (int32_t b = 0; b < B; ++b) {
        double s = t[b] - dt[b];
        if (s < 0.0) s = 0.0;
        double kt = dgo_kappa(schedule, t[b]);
        double ks = dgo_kappa(schedule, s);
        double it = inv_tau ? (double)inv_tau[b] : 1.0;
        for (int32_t i = 0; i < C; ++i) {
            int64_t r = (int64_t)b * C + i;
            const float* l = logits + r * ld;
            dgo_row_stats(l, V, it, &lse[r], &max_prob[r], &entropy[r]);
            argmax[r] = dgo_argmax(l, V);
            if (mode == 1) {
                x0_hat[r] = argmax[r];
                gap1[r] = INFINITY;
                gap2[r] = INFINITY;
            } else {
                x0_hat[r] = dgo_draw_x0(l, V, it, seed, step, (uint32_t)r, Q, &gap1[r], &gap2[r]);
            }
            x_next[r] = dgo_step(x_t[r], x0_hat[r], kt, ks, V, seed, step, (uint32_t)r, &branch[r]);
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Self-conditioning input [TR-Method]: z = p0 E with p0 = softmax(l'),      */
/* E [V, d] row-major.  The trained FFW that follows on the pages is left   */
/* out (no weights exist); the expected embedding p0 E is computed as is.    */
/* Only the listed rows are computed (rows[n]); z_out is [n, d].             */
/* ------------------------------------------------------------------------ */
void dgo_selfcond_rows(const float* logits, int64_t ld, int32_t V, const float* E, int32_t d,
                       const float* inv_tau_rows, const int32_t* rows, int32_t n, double* z_out)
{
    double* p = (double*)malloc(sizeof(double) * (size_t)V);
    for (int32_t k = 0; k < n; ++k) {
        int64_t r = rows[k];
        double it = inv_tau_rows ? (double)inv_tau_rows[r] : 1.0;
        dgo_row_probs(logits + r * ld, V, it, p);
        double* z = z_out + (int64_t)k * d;
        for (int32_t j = 0; j < d; ++j) z[j] = 0.0;
        for (int32_t v = 0; v < V; ++v) {
            const float* e = E + (int64_t)v * d;
            double pv = p[v];
            for (int32_t j = 0; j < d; ++j) z[j] += pv * (double)e[j];
        }
    }
    free(p);
}

/* ------------------------------------------------------------------------ */
/* Training-side forward corruption [TR-Method, forward path equation and    */
/* "noisy tokens are sampled uniformly from the vocabulary"; TR-Data layout  */
/* P prompt tokens + K canvases of C tokens].  Sequence b has time t_b and   */
/* kappa_b = kappa(t_b).  Prompt tokens are copied (the decoder conditions   */
/* on a clean prompt).  Every canvas token j is kept with probability        */
/* kappa_b (u = w0 * 2^-32 < kappa_b, counter (j, b, 0, DOM_NOISE)) and      */
/* otherwise replaced by floor(w1 V / 2^32).  The loss canvas k_b is         */
/* floor(w0 K / 2^32) from counter (0, b, 0, DOM_CANVAS) [TR-Data: one       */
/* canvas per sequence, chosen uniformly].                                    */
/* ------------------------------------------------------------------------ */
void dgo_forward_noise(const int32_t* x0, int32_t n_seq, int32_t P, int32_t K, int32_t C,
                       int32_t V, int32_t schedule, const double* t, uint64_t seed, int32_t* x_t,
                       int32_t* canvas_idx)
{
    int64_t L = (int64_t)P + (int64_t)K * C;
    uint32_t w[4];
    for (int32_t b = 0; b < n_seq; ++b) {
        double kappa = dgo_kappa(schedule, t[b]);
        for (int64_t j = 0; j < L; ++j) {
            int32_t tok = x0[(int64_t)b * L + j];
            if (j >= P) {
                philox_word4(seed, (uint32_t)j, (uint32_t)b, 0u, DOM_NOISE, w);
                if (!(word_to_unit(w[0]) < kappa)) tok = word_to_index(w[1], V);
            }
            x_t[(int64_t)b * L + j] = tok;
        }
        philox_word4(seed, 0u, (uint32_t)b, 0u, DOM_CANVAS, w);
        canvas_idx[b] = word_to_index(w[0], K);
    }
}

/* ------------------------------------------------------------------------ */
/* Canvas cross-entropy [TR-Method, loss equation L = -sum_i log p(x0^i|..)] */
/* on the chosen canvas of each sequence [TR-Data].  logits: float           */
/* [n_seq*C, ld], row b*C + i predicts x0[b, P + k_b*C + i].  Outputs the    */
/* per-row loss lse_i - l_i[target], the per-row lse, and the per-sequence   */
/* sum over the C rows (the equation's sum).  Forward only.                  */
/* ------------------------------------------------------------------------ */
void dgo_canvas_ce(const float* logits, int64_t ld, const int32_t* x0, const int32_t* canvas_idx,
                   int32_t n_seq, int32_t P, int32_t K, int32_t C, int32_t V, double* loss_rows,
                   double* loss_seq, double* lse_rows)
{
    int64_t L = (int64_t)P + (int64_t)K * C;
    for (int32_t b = 0; b < n_seq; ++b) {
        double sum = 0.0;
        for (int32_t i = 0; i < C; ++i) {
            int64_t r = (int64_t)b * C + i;
            const float* l = logits + r * ld;
            double m = -INFINITY;
            for (int32_t v = 0; v < V; ++v)
                if ((double)l[v] > m) m = (double)l[v];
            double S = 0.0;
            for (int32_t v = 0; v < V; ++v) S += exp((double)l[v] - m);
            double lse = m + log(S);
            int32_t target = x0[(int64_t)b * L + P + (int64_t)canvas_idx[b] * C + i];
            double loss = lse - (double)l[target];
            loss_rows[r] = loss;
            lse_rows[r] = lse;
            sum += loss;
        }
        loss_seq[b] = sum;
    }
}

/* ------------------------------------------------------------------------ */
/* Temperature schedule [TR-Method, sampler paragraph: the temperature       */
/* tau_t < 1 is annealed linearly over the denoising time scale from         */
/* tau_max = 0.8 to tau_min = 0.4].  Reading: linear in t with tau(1) =      */
/* tau_max (denoising starts at t = 1) and tau(0) = tau_min; t is clamped    */
/* to [0, 1].                                                                */
/* ------------------------------------------------------------------------ */
double dgo_tau_linear(double t, double tau_max, double tau_min)
{
    if (t < 0.0) t = 0.0;
    if (t > 1.0) t = 1.0;
    return tau_min + (tau_max - tau_min) * t;
}

/* Fixed-point entropy used by the acceptance and stopping decisions:        */
/* q = floor(H * 2^32) with H clamped to [0, 64] and NaN counted as 64.      */
/* (Reading: the decisions compare sums of entropies against thresholds; in  */
/* fixed point the sums are exact and independent of summation order.)      */
static int64_t entropy_q(float h)
{
    double x = (double)h;
    if (!(x >= 0.0)) x = isnan(x) ? 64.0 : 0.0;
    if (x > 64.0) x = 64.0;
    return (int64_t)floor(x * 4294967296.0);
}

/* Threshold ceil(x * 2^32) for a sum of fixed-point entropies ("sum < x").  */
static int64_t entropy_threshold(double x)
{
    double y = ceil(x * 4294967296.0);
    if (y > 9.0e18) return INT64_MAX;
    if (y < 0.0) return 0;
    return (int64_t)y;
}

typedef struct {
    int64_t q;
    int32_t i;
} qpos;

static int qpos_cmp(const void* a, const void* b)
{
    const qpos* x = (const qpos*)a;
    const qpos* y = (const qpos*)b;
    if (x->q != y->q) return x->q < y->q ? -1 : 1;
    return x->i < y->i ? -1 : (x->i > y->i);
}

/* ------------------------------------------------------------------------ */
/* Entropy-bounded acceptance with uniform re-noising [TR-Method, sampler    */
/* paragraph: tokens are accepted in ascending order of entropy so that a    */
/* mutual-information bound stays strictly below an error tolerance; once    */
/* the tolerance is reached, every other token is re-noised uniformly at     */
/* random].  Reading (the pages give no formula for the bound): the bound of */
/* an accepted set is the sum of its entropies, which bounds its total       */
/* correlation from above.  Per canvas of C positions, positions are ordered */
/* by ascending (q, position) and the k-th of that order is accepted iff     */
/* q_1 + ... + q_k < ceil(eps * 2^32); a canvas whose lowest entropy is      */
/* already >= eps accepts nothing.  Accepted positions take x0_hat, the      */
/* others floor(w0 V / 2^32) from counter (0, row, step, DOM_RENOISE).       */
/* H, x0_hat: [B*C]; outputs x_next [B*C], accepted [B*C] (0/1) and the      */
/* number accepted per canvas n_acc [B].                                     */
/* ------------------------------------------------------------------------ */
void dgo_entropy_accept(const float* H, const int32_t* x0_hat, int32_t B, int32_t C, int32_t V,
                        double eps, uint64_t seed, uint32_t step, int32_t* x_next,
                        uint8_t* accepted, int32_t* n_acc)
{
    qpos* order = (qpos*)malloc(sizeof(qpos) * (size_t)C);
    int64_t limit = entropy_threshold(eps);
    uint32_t w[4];
    for (int32_t b = 0; b < B; ++b) {
        int64_t r0 = (int64_t)b * C;
        for (int32_t i = 0; i < C; ++i) {
            order[i].q = entropy_q(H[r0 + i]);
            order[i].i = i;
            accepted[r0 + i] = 0;
        }
        qsort(order, (size_t)C, sizeof(qpos), qpos_cmp);
        int64_t sum = 0;
        int32_t n = 0;
        for (int32_t k = 0; k < C; ++k) {
            sum += order[k].q;
            if (!(sum < limit)) break;
            accepted[r0 + order[k].i] = 1;
            ++n;
        }
        n_acc[b] = n;
        for (int32_t i = 0; i < C; ++i) {
            int64_t r = r0 + i;
            if (accepted[r]) {
                x_next[r] = x0_hat[r];
            } else {
                philox_word4(seed, 0u, (uint32_t)r, step, DOM_RENOISE, w);
                x_next[r] = word_to_index(w[0], V);
            }
        }
    }
    free(order);
}

/* ------------------------------------------------------------------------ */
/* Adaptive stopping [TR-Method, sampler paragraph: early termination when   */
/* the mean predicted entropy over the whole canvas falls below a threshold  */
/* and the deterministic sequence predictions of two consecutive steps are   */
/* identical].  Reading: the deterministic prediction is the argmax token of */
/* each position; the mean uses the fixed-point entropies above, so the      */
/* first condition is sum_i q_i < ceil(theta * C * 2^32).  Without a         */
/* previous step (argmax_prev NULL) the second condition is false.           */
/* Outputs stop [B] (0/1) and mean_H [B] = (sum_i q_i) 2^-32 / C.            */
/* ------------------------------------------------------------------------ */
void dgo_adaptive_stop(const float* H, const int32_t* am, const int32_t* am_prev, int32_t B,
                       int32_t C, double theta, uint8_t* stop, double* mean_H)
{
    int64_t limit = entropy_threshold(theta * (double)C);
    for (int32_t b = 0; b < B; ++b) {
        int64_t r0 = (int64_t)b * C;
        int64_t sum = 0;
        int same = am_prev != NULL;
        for (int32_t i = 0; i < C; ++i) {
            sum += entropy_q(H[r0 + i]);
            if (am_prev && am[r0 + i] != am_prev[r0 + i]) same = 0;
        }
        mean_H[b] = (double)sum * (1.0 / 4294967296.0) / (double)C;
        stop[b] = (uint8_t)(sum < limit && same);
    }
}

/* ------------------------------------------------------------------------ */
/* Canvas cross-entropy backward [TR-Method, loss equation].  For row r with */
/* target id y_r the derivative of loss_r = lse_r - l_r[y_r] is               */
/*     d loss_r / d l_r[v] = softmax(l_r)_v - [v == y_r],                     */
/* scaled by the upstream gradient g_seq[b] of the sequence's summed loss    */
/* (rows b*C .. b*C+C-1).  lse is recomputed here in double.  A row whose    */
/* target is out of range gets a zero gradient.                               */
/* ------------------------------------------------------------------------ */
void dgo_canvas_ce_backward(const float* logits, int64_t ld, const int32_t* x0,
                            const int32_t* canvas_idx, int32_t n_seq, int32_t P, int32_t K,
                            int32_t C, int32_t V, const double* g_seq, double* grad)
{
    int64_t L = (int64_t)P + (int64_t)K * C;
    for (int32_t b = 0; b < n_seq; ++b) {
        int32_t k = canvas_idx[b];
        for (int32_t i = 0; i < C; ++i) {
            int64_t r = (int64_t)b * C + i;
            const float* l = logits + r * ld;
            double* g = grad + r * (int64_t)V;
            int32_t y = (k >= 0 && k < K) ? x0[(int64_t)b * L + P + (int64_t)k * C + i] : -1;
            if (y < 0 || y >= V) {
                for (int32_t v = 0; v < V; ++v) g[v] = 0.0;
                continue;
            }
            double m = -INFINITY;
            for (int32_t v = 0; v < V; ++v)
                if ((double)l[v] > m) m = (double)l[v];
            double S = 0.0;
            for (int32_t v = 0; v < V; ++v) S += exp((double)l[v] - m);
            double lse = m + log(S);
            for (int32_t v = 0; v < V; ++v)
                g[v] = g_seq[b] * (exp((double)l[v] - lse) - (v == y ? 1.0 : 0.0));
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Self-conditioning drop for training [TR-Data: for 50% of the batch the    */
/* decoder uses the self-conditioning state of a previous forward pass, for  */
/* the other 50% that state is zero].  Reading: an independent fair coin per */
/* sequence, keep iff w0 < 2^31 from counter (0, b, step, DOM_SC_DROP); the  */
/* C rows of a dropped sequence are set to zero.  z: [n_seq*C, d] in place;   */
/* keep [n_seq] (0/1).                                                       */
/* ------------------------------------------------------------------------ */
void dgo_selfcond_drop(double* z, int32_t n_seq, int32_t C, int32_t d, uint64_t seed,
                       uint32_t step, uint8_t* keep)
{
    uint32_t w[4];
    for (int32_t b = 0; b < n_seq; ++b) {
        philox_word4(seed, 0u, (uint32_t)b, step, DOM_SC_DROP, w);
        keep[b] = (uint8_t)(w[0] < 0x80000000u);
        if (!keep[b])
            for (int64_t j = (int64_t)b * C * d; j < ((int64_t)b + 1) * C * d; ++j) z[j] = 0.0;
    }
}

/* ------------------------------------------------------------------------ */
/* Feed-forward block on the self-conditioning input [TR-Method:            */
/* z = FFW(p0 E), FFW a standard feed-forward network].  Reading (the pages */
/* name no architecture and no trained weights exist): a two-layer          */
/* perceptron without biases, out = gelu(z W1) W2, with the tanh form of    */
/* GELU (Hendrycks and Gimpel, "Gaussian Error Linear Units", 2016):        */
/*     gelu(x) = x/2 (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3))).             */
/* z [R, d], W1 [d, dff], W2 [dff, d] row-major (float, widened from bf16   */
/* by the caller); out [R, d] in double, no rounding between the layers.    */
/* ------------------------------------------------------------------------ */
double dgo_gelu_tanh(double x)
{
    const double k = sqrt(2.0 / 3.14159265358979323846);
    return 0.5 * x * (1.0 + tanh(k * (x + 0.044715 * x * x * x)));
}

void dgo_ffw(const float* z, const float* W1, const float* W2, int32_t R, int32_t d, int32_t dff,
             double* out)
{
    double* h = (double*)malloc(sizeof(double) * (size_t)dff);
    for (int32_t r = 0; r < R; ++r) {
        for (int32_t j = 0; j < dff; ++j) h[j] = 0.0;
        for (int32_t k = 0; k < d; ++k) {
            double zk = (double)z[(int64_t)r * d + k];
            const float* w = W1 + (int64_t)k * dff;
            for (int32_t j = 0; j < dff; ++j) h[j] += zk * (double)w[j];
        }
        for (int32_t j = 0; j < dff; ++j) h[j] = dgo_gelu_tanh(h[j]);
        double* o = out + (int64_t)r * d;
        for (int32_t c = 0; c < d; ++c) o[c] = 0.0;
        for (int32_t j = 0; j < dff; ++j) {
            double hj = h[j];
            const float* w = W2 + (int64_t)j * d;
            for (int32_t c = 0; c < d; ++c) o[c] += hj * (double)w[c];
        }
    }
    free(h);
}
