/*
 * fp64 CPU oracle for the RWKV-4 WKV operator and the token-shift lerp.
 *
 * TEST INFRASTRUCTURE.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load or run this code.  The CUDA library
 * never links, includes or calls it, and the two share no code, headers,
 * tables or constants.  Plain, slow and obviously correct on purpose: every
 * loop follows the formula it cites, term by term, in double precision.
 * OpenMP only distributes independent channels over threads; it changes no
 * arithmetic.
 *
 * Sources (web pages on RWKV; cited by page and section):
 *   [MATH]  "RWKV" transformer-math page (aicassindra.com, tm_rwkv_math):
 *           section "The WKV operator: attention with a fixed decay" (the
 *           wkv_t equation, w = exp(omega) > 0, u the current-token bonus);
 *           section "Why it collapses into a recurrence" (the a_t, b_t
 *           recurrence with a_0 = b_0 = 0); section "Numerical stability:
 *           carry the exponent" (the (p, a, b) form); section "Token shift:
 *           a two-tap causal convolution" (the lerp).
 *   [WIKI]  "RWKV" (aiwiki.thehackersbrain.dev): eq. 1 and the one-token
 *           decode step in the stabilised form.
 *           Also section "Receptance: the gate on the way out" (the output is
 *           sigma(r) times wkv, channel by channel) and, in section "Token shift",
 *           the separate mu_r, mu_k, mu_v of the three projections.
 *   [VANOS] "RWKV (Attention-RNN Hybrid)" (vanos001.github.io): section
 *           "Versions: RWKV-4 -> Eagle -> Finch" (the Eagle matrix-state
 *           recurrence S_t = diag(d) S_{t-1} + k_t v_t^T read out as
 *           y_t = r_t^T S_t, one 64 x 64 state per head) and section
 *           "O(N) Inference Characteristics" (decode is one matrix-vector
 *           product against the state).
 *   [MULTI] "RWKV and Recurrent Models With Transformer Quality"
 *           (multigrid.ai): section "Prefill, decode, and where each form is
 *           used" (prefill yields the state after the last prompt token;
 *           decode steps from it).
 *
 * Indexing: 0-based t in [0, T).  eq. 1 at position t sums the past i < t with
 * weight exp(-(t-1-i) w + k_i) and the current token with exp(u + k_t); the
 * most recent past token (i = t-1) is not decayed.
 *
 * Layouts: k, v, y, s are [B][T][C] row-major; w, u are [C]; a state is
 * [3][B][C] holding (a, b, p) with true accumulators A = a e^p, B = b e^p.
 *
 * Every function also returns the "magnitude scale" s: the same weighted
 * average with |v| in place of v.  It is what the tests divide errors by
 * (|y| can be near zero while the terms that produced it are not).
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Initial running maximum for an empty state: finite, so p - w never forms
 * inf - inf, and far below any exponent the data can produce. */
#define ORACLE_P_EMPTY (-1e38)

static inline size_t at3(int64_t b, int64_t t, int64_t c, int64_t T, int64_t C)
{
    return ((size_t)b * (size_t)T + (size_t)t) * (size_t)C + (size_t)c;
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Threads for the parallel loops that follow (timing only: every loop distributes independent
 * channels, so the results do not depend on it). */
void oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/*
 * Direct evaluation of the wkv_t equation ([MATH] "The WKV operator: attention
 * with a fixed decay"; [WIKI] eq. 1), O(T^2) per channel, no stabilisation.
 * Valid while every exponent -(t-1-i) w + k_i and u + k_t stays below ~709.
 *   y[b,t,c] = (sum_{i<t} e^{-(t-1-i)w + k_i} v_i + e^{u + k_t} v_t)
 *            / (sum_{i<t} e^{-(t-1-i)w + k_i}     + e^{u + k_t})
 * s (may be NULL) is the same ratio with |v| in place of v.
 */
void oracle_wkv_direct(int64_t B, int64_t T, int64_t C, const double* w, const double* u,
                       const double* k, const double* v, double* y, double* s)
{
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t b = 0; b < B; ++b)
        for (int64_t c = 0; c < C; ++c)
            for (int64_t t = 0; t < T; ++t) {
                double num = 0.0, den = 0.0, mag = 0.0;
                for (int64_t i = 0; i < t; ++i) {
                    double e = exp(-(double)(t - 1 - i) * w[c] + k[at3(b, i, c, T, C)]);
                    num += e * v[at3(b, i, c, T, C)];
                    mag += e * fabs(v[at3(b, i, c, T, C)]);
                    den += e;
                }
                double e = exp(u[c] + k[at3(b, t, c, T, C)]);
                num += e * v[at3(b, t, c, T, C)];
                mag += e * fabs(v[at3(b, t, c, T, C)]);
                den += e;
                y[at3(b, t, c, T, C)] = num / den;
                if (s) s[at3(b, t, c, T, C)] = mag / den;
            }
}

/*
 * The running-maximum form ([MATH] "Numerical stability: carry the exponent";
 * [WIKI] decode step), applied token after token.  Per channel, with state
 * (a, b, p):
 *   output:  q = max(p, u + k_t)
 *            y_t = (e^{p-q} a + e^{u+k_t-q} v_t) / (e^{p-q} b + e^{u+k_t-q})
 *   update:  p' = max(p - w, k_t)
 *            a' = e^{p-w-p'} a + e^{k_t-p'} v_t
 *            b' = e^{p-w-p'} b + e^{k_t-p'}
 * The empty state is a = b = 0 with p = ORACLE_P_EMPTY.
 *
 * state_in  [3][B][C] (a, b, p) or NULL for the empty state.
 * sacc_in   [B][C] magnitude accumulator (a with |v|) or NULL for zeros.
 * y, s      [B][T][C]; s may be NULL.
 * state_out [3][B][C] or NULL; sacc_out [B][C] or NULL.
 * T may be 0 (state is copied through).  With T = 1 this is exactly one decode
 * step from a given state ([MULTI] "Prefill, decode, and where each form is
 * used").
 */
void oracle_wkv_recurrent(int64_t B, int64_t T, int64_t C, const double* w, const double* u,
                          const double* k, const double* v, const double* state_in,
                          const double* sacc_in, double* y, double* s, double* state_out,
                          double* sacc_out)
{
    const size_t BC = (size_t)B * (size_t)C;
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t b = 0; b < B; ++b)
        for (int64_t c = 0; c < C; ++c) {
            size_t bc = (size_t)b * (size_t)C + (size_t)c;
            double a = 0.0, bb = 0.0, p = ORACLE_P_EMPTY, sa = 0.0;
            if (state_in) {
                a = state_in[bc];
                bb = state_in[BC + bc];
                p = state_in[2 * BC + bc];
            }
            if (sacc_in) sa = sacc_in[bc];
            for (int64_t t = 0; t < T; ++t) {
                double kt = k[at3(b, t, c, T, C)];
                double vt = v[at3(b, t, c, T, C)];
                /* output */
                double q = fmax(p, u[c] + kt);
                double w_past = exp(p - q);         /* weight of the carried history */
                double w_now = exp(u[c] + kt - q);  /* weight of the current token */
                double den = w_past * bb + w_now;
                y[at3(b, t, c, T, C)] = (w_past * a + w_now * vt) / den;
                if (s) s[at3(b, t, c, T, C)] = (w_past * sa + w_now * fabs(vt)) / den;
                /* update */
                double p_new = fmax(p - w[c], kt);
                double keep = exp(p - w[c] - p_new); /* decayed history, rescaled */
                double add = exp(kt - p_new);        /* the new token, rescaled */
                a = keep * a + add * vt;
                bb = keep * bb + add;
                sa = keep * sa + add * fabs(vt);
                p = p_new;
            }
            if (state_out) {
                state_out[bc] = a;
                state_out[BC + bc] = bb;
                state_out[2 * BC + bc] = p;
            }
            if (sacc_out) sacc_out[bc] = sa;
        }
}

/*
 * The plain two-accumulator recurrence ([MATH] "Why it collapses into a
 * recurrence"), no exponent carried:
 *   y_t = (a_{t-1} + e^{u+k_t} v_t) / (b_{t-1} + e^{u+k_t})
 *   a_t = e^{-w} a_{t-1} + e^{k_t} v_t,   b_t = e^{-w} b_{t-1} + e^{k_t},   a = b = 0 at start.
 * Overflows for large keys; used only as an in-range cross-check.
 */
void oracle_wkv_naive(int64_t B, int64_t T, int64_t C, const double* w, const double* u,
                      const double* k, const double* v, double* y)
{
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t b = 0; b < B; ++b)
        for (int64_t c = 0; c < C; ++c) {
            double a = 0.0, bb = 0.0;
            double decay = exp(-w[c]);
            for (int64_t t = 0; t < T; ++t) {
                double kt = k[at3(b, t, c, T, C)];
                double vt = v[at3(b, t, c, T, C)];
                double cur = exp(u[c] + kt);
                y[at3(b, t, c, T, C)] = (a + cur * vt) / (bb + cur);
                a = decay * a + exp(kt) * vt;
                bb = decay * bb + exp(kt);
            }
        }
}

/*
 * Token shift ([MATH] "Token shift: a two-tap causal convolution"):
 *   xbar_t = mu * x_t + (1 - mu) * x_{t-1},  per channel.
 * x [B][T][C], mu [C], x_last [B][C] is the token before t = 0 (NULL: zeros,
 * the causal zero padding), xbar [B][T][C].  With T = 1 and x_last the
 * previous token this is the single decode-step lerp.
 */
void oracle_token_shift(int64_t B, int64_t T, int64_t C, const double* mu, const double* x,
                        const double* x_last, double* xbar)
{
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t b = 0; b < B; ++b)
        for (int64_t t = 0; t < T; ++t)
            for (int64_t c = 0; c < C; ++c) {
                double prev;
                if (t > 0)
                    prev = x[at3(b, t - 1, c, T, C)];
                else
                    prev = x_last ? x_last[(size_t)b * (size_t)C + (size_t)c] : 0.0;
                xbar[at3(b, t, c, T, C)] = mu[c] * x[at3(b, t, c, T, C)] + (1.0 - mu[c]) * prev;
            }
}

/*
 * Receptance gate ([MATH] "Receptance: the gate on the way out"): each channel of
 * wkv_t passes through the logistic sigmoid of r_t,
 *   out[i] = wkv[i] * sigma(r[i]),   sigma(r) = 1 / (1 + e^{-r}),
 * elementwise over n values (the W_o projection that follows is not part of it).
 * For r -> -inf, e^{-r} overflows to +inf and the quotient is the limit 0.
 */
void oracle_gate(int64_t n, const double* r, const double* wkv, double* out)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        const double sigma = 1.0 / (1.0 + exp(-r[i]));
        out[i] = wkv[i] * sigma;
    }
}

/*
 * Gradient of the wkv_t equation ([MATH] "The WKV operator: attention with a fixed decay";
 * [WIKI] eq. 1), differentiated as written; the pages give no gradient.  For a loss
 * L = sum_{b,t,c} gy[b,t,c] * y[b,t,c], with y_t = N_t / D_t,
 *   N_t = sum_{i<t} beta_{t,i} v_i + alpha_t v_t,   D_t = sum_{i<t} beta_{t,i} + alpha_t,
 *   beta_{t,i} = e^{-(t-1-i) w + k_i},   alpha_t = e^{u + k_t},
 * each term contributes (dy_t/dN_t = 1/D_t, dy_t/dD_t = -y_t/D_t):
 *   current token:  dy_t/dv_t = alpha_t / D_t;   dy_t/dk_t = dy_t/du = alpha_t (v_t - y_t) / D_t
 *   past token i:   dy_t/dv_i = beta_{t,i} / D_t;  dy_t/dk_i = beta_{t,i} (v_i - y_t) / D_t;
 *                   dy_t/dw  += -(t-1-i) beta_{t,i} (v_i - y_t) / D_t
 * gk, gv are [B][T][C]; gw, gu are [C], summed over b and t.  O(T^2) per channel, valid
 * while every exponent stays below ~709.  The optional s* outputs add up the same terms'
 * magnitudes with |gy| in place of gy and |v| + |y| in place of v - y: the scales the tests
 * divide by (y_t is only known to its own rounding, so v - y_t is only known to within a
 * fraction of |v| + |y_t|, whatever the arithmetic that follows).
 */
void oracle_wkv_backward_direct(int64_t B, int64_t T, int64_t C, const double* w, const double* u,
                                const double* k, const double* v, const double* gy, double* gk, double* gv,
                                double* gw, double* gu, double* sk, double* sv, double* sw, double* su)
{
#pragma omp parallel for schedule(static)
    for (int64_t c = 0; c < C; ++c) {
        double gwc = 0.0, guc = 0.0, swc = 0.0, suc = 0.0;
        for (int64_t b = 0; b < B; ++b) {
            for (int64_t t = 0; t < T; ++t) {
                gk[at3(b, t, c, T, C)] = 0.0;
                gv[at3(b, t, c, T, C)] = 0.0;
                if (sk) sk[at3(b, t, c, T, C)] = 0.0;
                if (sv) sv[at3(b, t, c, T, C)] = 0.0;
            }
            for (int64_t t = 0; t < T; ++t) {
                /* forward value of position t */
                double num = 0.0, den = 0.0;
                for (int64_t i = 0; i < t; ++i) {
                    double beta = exp(-(double)(t - 1 - i) * w[c] + k[at3(b, i, c, T, C)]);
                    num += beta * v[at3(b, i, c, T, C)];
                    den += beta;
                }
                double alpha = exp(u[c] + k[at3(b, t, c, T, C)]);
                num += alpha * v[at3(b, t, c, T, C)];
                den += alpha;
                double yt = num / den;
                double g = gy[at3(b, t, c, T, C)] / den;
                double gm = fabs(gy[at3(b, t, c, T, C)]) / den;
                /* current token */
                double vt = v[at3(b, t, c, T, C)];
                gv[at3(b, t, c, T, C)] += g * alpha;
                gk[at3(b, t, c, T, C)] += g * alpha * (vt - yt);
                guc += g * alpha * (vt - yt);
                if (sv) sv[at3(b, t, c, T, C)] += gm * alpha;
                if (sk) sk[at3(b, t, c, T, C)] += gm * alpha * (fabs(vt) + fabs(yt));
                suc += gm * alpha * (fabs(vt) + fabs(yt));
                /* past tokens */
                for (int64_t i = 0; i < t; ++i) {
                    double beta = exp(-(double)(t - 1 - i) * w[c] + k[at3(b, i, c, T, C)]);
                    double vi = v[at3(b, i, c, T, C)];
                    gv[at3(b, i, c, T, C)] += g * beta;
                    gk[at3(b, i, c, T, C)] += g * beta * (vi - yt);
                    gwc += -g * (double)(t - 1 - i) * beta * (vi - yt);
                    if (sv) sv[at3(b, i, c, T, C)] += gm * beta;
                    if (sk) sk[at3(b, i, c, T, C)] += gm * beta * (fabs(vi) + fabs(yt));
                    swc += gm * (double)(t - 1 - i) * beta * (fabs(vi) + fabs(yt));
                }
            }
        }
        gw[c] = gwc;
        gu[c] = guc;
        if (sw) sw[c] = swc;
        if (su) su[c] = suc;
    }
}

/*
 * Eagle (RWKV-5) matrix-state WKV ([VANOS] "Versions: RWKV-4 -> Eagle -> Finch"),
 * per sequence b and head h of N channels, token after token:
 *   S_t = diag(d) S_{t-1} + k_t v_t^T     S is N x N: row m a key channel, column j a value channel
 *   y_t = r_t^T S_t                       y_t[j] = sum_m r_t[m] S_t[m][j]
 * with d[m] = exp(-w[h N + m]) (w > 0: the per-channel decay rate, as in RWKV-4)
 * and S_{-1} = state_in (zero when NULL).
 *
 * r, k, v, y, s: [B][T][C] with C = H N, head h owning channels h N .. h N + N - 1.
 * w: [C].  state_in, state_out: [B][H][N][N] (m, j), either may be NULL.
 * s (may be NULL): the same read-out with |r|, |k|, |v| and |state_in|, the
 * magnitude scale that errors are measured against.
 * With T = 1 this is one decode step from the given state ([VANOS] "O(N) Inference
 * Characteristics").
 */
void oracle_eagle_recurrent(int64_t B, int64_t T, int64_t H, int64_t N, const double* w,
                            const double* r, const double* k, const double* v,
                            const double* state_in, double* y, double* s, double* state_out)
{
    const int64_t C = H * N;
    const size_t NN = (size_t)N * (size_t)N;
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t b = 0; b < B; ++b)
        for (int64_t h = 0; h < H; ++h) {
            const size_t sb = ((size_t)b * (size_t)H + (size_t)h) * NN;
            double* S = (double*)malloc(NN * sizeof(double));
            double* Sa = (double*)malloc(NN * sizeof(double));
            for (size_t e = 0; e < NN; ++e) {
                S[e] = state_in ? state_in[sb + e] : 0.0;
                Sa[e] = fabs(S[e]);
            }
            for (int64_t t = 0; t < T; ++t) {
                /* update: S <- diag(d) S + k_t v_t^T */
                for (int64_t m = 0; m < N; ++m) {
                    const double d = exp(-w[h * N + m]);
                    const double km = k[at3(b, t, h * N + m, T, C)];
                    for (int64_t j = 0; j < N; ++j) {
                        const double vj = v[at3(b, t, h * N + j, T, C)];
                        S[m * N + j] = d * S[m * N + j] + km * vj;
                        Sa[m * N + j] = d * Sa[m * N + j] + fabs(km) * fabs(vj);
                    }
                }
                /* read-out: y_t = r_t^T S_t */
                for (int64_t j = 0; j < N; ++j) {
                    double acc = 0.0, acc_s = 0.0;
                    for (int64_t m = 0; m < N; ++m) {
                        const double rm = r[at3(b, t, h * N + m, T, C)];
                        acc += rm * S[m * N + j];
                        acc_s += fabs(rm) * Sa[m * N + j];
                    }
                    y[at3(b, t, h * N + j, T, C)] = acc;
                    if (s) s[at3(b, t, h * N + j, T, C)] = acc_s;
                }
            }
            if (state_out)
                for (size_t e = 0; e < NN; ++e) state_out[sb + e] = S[e];
            free(S);
            free(Sa);
        }
}

/*
 * The same outputs summed directly instead of carried: unrolling the recurrence gives
 * S_t = sum_{i<=t} diag(d)^{t-i} k_i v_i^T + diag(d)^{t+1} S_{-1}, so
 *   y_t[j] = sum_{i<=t} sum_m r_t[m] exp(-(t-i) w[m]) k_i[m] v_i[j]
 *          + sum_m r_t[m] exp(-(t+1) w[m]) state_in[m][j].
 * O(T^2 N^2) per head: for small cases only.
 */
void oracle_eagle_direct(int64_t B, int64_t T, int64_t H, int64_t N, const double* w,
                         const double* r, const double* k, const double* v,
                         const double* state_in, double* y)
{
    const int64_t C = H * N;
    const size_t NN = (size_t)N * (size_t)N;
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t b = 0; b < B; ++b)
        for (int64_t h = 0; h < H; ++h) {
            const size_t sb = ((size_t)b * (size_t)H + (size_t)h) * NN;
            for (int64_t t = 0; t < T; ++t)
                for (int64_t j = 0; j < N; ++j) {
                    double acc = 0.0;
                    for (int64_t m = 0; m < N; ++m) {
                        const double rm = r[at3(b, t, h * N + m, T, C)];
                        for (int64_t i = 0; i <= t; ++i)
                            acc += rm * exp(-(double)(t - i) * w[h * N + m]) * k[at3(b, i, h * N + m, T, C)] *
                                   v[at3(b, i, h * N + j, T, C)];
                        if (state_in) acc += rm * exp(-(double)(t + 1) * w[h * N + m]) * state_in[sb + m * N + j];
                    }
                    y[at3(b, t, h * N + j, T, C)] = acc;
                }
        }
}
