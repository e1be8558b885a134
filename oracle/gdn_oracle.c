/*
 * gdn_oracle.c -- fp64 CPU oracle for the Gated DeltaNet layer mixer.
 *
 * TEST INFRASTRUCTURE. Only the tests, the package's smoke check and the
 * benchmark's CPU-baseline leg may load this file's library. The CUDA path
 * shares no code with it and never calls it.
 *
 * What it computes (Gated DeltaNet mixer, as used to verify a speculative
 * block; source pages: "Lithos-metal: Qwen3.8-27B on 40-core M5 Max", table
 * "GDN mixer" and the runtime paragraph on recurrent-state commit/rollback;
 * "Qwen 3.8 27B mac m5: 200 tok/s, audited", sections "How does lithos-metal
 * fuse layer mixers on Metal?" (32-bit recurrent state with a key side and a
 * value side) and "How does DSpark speculative decoding create more than one
 * token per read?" (7 drafts + 1 anchor = 8 rows; rewind after acceptance)):
 *
 *   per sequence b and value head h, with key head g = h / (H_v / H_k):
 *     khat_t = k_t / sqrt(sum k_t^2 + eps)
 *     qhat_t = scale * q_t / sqrt(sum q_t^2 + eps)
 *     log_alpha_t = -exp(A_log[h]) * softplus(a_t + dt_bias[h])
 *     alpha_t = exp(log_alpha_t),  beta_t = 1 / (1 + exp(-b_t))
 *     S_t = alpha_t * S_{t-1} (I - beta_t khat_t khat_t^T) + beta_t v_t khat_t^T
 *     o_t = S_t qhat_t
 *   S is d_v x d_k (row i = value index, column j = key index); the
 *   committed state is S_L, L = accept_len[b] in 0..T (L = 0: the state
 *   before the block, unchanged).
 *
 * Everything is fp64, one (b, h) pair at a time, in the order written above.
 * The product S (I - beta k k^T) is expanded by distributivity into
 * S - beta (S k) k^T; the d x d matrix is formed literally only by the
 * brute-force NumPy form in brute.py, which the tests compare against this.
 *
 * The chunked form (oracle_chunked) is a second, independent route to the
 * same numbers (the WY / UT-transform form for long prompts): within a chunk
 * the per-token updates are collected into a unit lower-triangular solve.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* softplus(x) = log(1 + e^x), written so that neither branch overflows. */
static double sp(double x) { return fmax(x, 0.0) + log1p(exp(-fabs(x))); }

static double sigm(double x) { return 1.0 / (1.0 + exp(-x)); }

static void set_threads(int nthreads) {
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
}

int oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * Rows of x ([n][d]) scaled to unit L2 norm: y = scale * x / sqrt(sum x^2 + eps).
 */
void oracle_l2norm(int64_t n, int d, const double* x, double eps, double scale, double* y) {
    for (int64_t r = 0; r < n; ++r) {
        const double* xr = x + r * d;
        double ss = 0.0;
        for (int j = 0; j < d; ++j) ss += xr[j] * xr[j];
        double inv = 1.0 / sqrt(ss + eps);
        for (int j = 0; j < d; ++j) y[r * d + j] = scale * xr[j] * inv;
    }
}

/*
 * Gates for n rows of H_v heads: a, b are [n][H_v]; A_log, dt_bias are [H_v].
 * log_alpha = -exp(A_log) * softplus(a + dt_bias), beta = sigmoid(b).
 */
void oracle_gates(int64_t n, int Hv, const double* a, const double* b, const double* A_log,
                  const double* dt_bias, double* log_alpha, double* beta) {
    for (int64_t r = 0; r < n; ++r) {
        for (int h = 0; h < Hv; ++h) {
            int64_t idx = r * Hv + h;
            log_alpha[idx] = -exp(A_log[h]) * sp(a[idx] + dt_bias[h]);
            beta[idx] = sigm(b[idx]);
        }
    }
}

/*
 * The per-token recurrence on already-normalised keys/queries and given gates.
 *
 *   qhat, khat : [B][T][Hk][dk]      v : [B][T][Hv][dv]
 *   alpha, beta: [B][T][Hv]          S0: [B][Hv][dv][dk]
 *   accept_len : [B] or NULL (NULL = commit after all T tokens)
 *   o          : [B][T][Hv][dv]      S_commit: [B][Hv][dv][dk]
 *   bad_accept : optional [B] out-flag, 1 where accept_len[b] is outside 0..T
 *                (then S_commit = S0, i.e. nothing is committed)
 *
 * Returns 0, or -1 for an inconsistent shape.
 */
int oracle_recurrence(int B, int T, int Hk, int Hv, int dk, int dv,
                      const double* qhat, const double* khat, const double* v,
                      const double* alpha, const double* beta, const double* S0,
                      const int32_t* accept_len, double* o, double* S_commit,
                      int32_t* bad_accept, int nthreads) {
    if (B < 0 || T < 0 || Hk <= 0 || Hv <= 0 || dk <= 0 || dv <= 0 || Hv % Hk != 0) return -1;
    const int G = Hv / Hk;
    const int64_t hs = (int64_t)dv * dk;
    set_threads(nthreads);

#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int bb = 0; bb < B; ++bb) {
        for (int h = 0; h < Hv; ++h) {
            const int g = h / G;
            int L = accept_len ? accept_len[bb] : T;
            int bad = (L < 0 || L > T);
            if (bad) L = 0;
            if (bad_accept && h == 0) bad_accept[bb] = bad;

            double* S = (double*)malloc(sizeof(double) * hs);
            double* p = (double*)malloc(sizeof(double) * dv);
            const double* s0 = S0 + ((int64_t)bb * Hv + h) * hs;
            double* sc = S_commit + ((int64_t)bb * Hv + h) * hs;
            memcpy(S, s0, sizeof(double) * hs);
            if (L == 0) memcpy(sc, s0, sizeof(double) * hs);

            for (int t = 0; t < T; ++t) {
                const double* kt = khat + (((int64_t)bb * T + t) * Hk + g) * dk;
                const double* qt = qhat + (((int64_t)bb * T + t) * Hk + g) * dk;
                const double* vt = v + (((int64_t)bb * T + t) * Hv + h) * dv;
                const double al = alpha[((int64_t)bb * T + t) * Hv + h];
                const double be = beta[((int64_t)bb * T + t) * Hv + h];
                double* ot = o + (((int64_t)bb * T + t) * Hv + h) * dv;

                /* p = S_{t-1} khat_t */
                for (int i = 0; i < dv; ++i) {
                    double acc = 0.0;
                    for (int j = 0; j < dk; ++j) acc += S[(int64_t)i * dk + j] * kt[j];
                    p[i] = acc;
                }
                /* S_t = alpha (S - beta p khat^T) + beta v khat^T */
                for (int i = 0; i < dv; ++i) {
                    for (int j = 0; j < dk; ++j) {
                        double s = S[(int64_t)i * dk + j];
                        S[(int64_t)i * dk + j] = al * (s - be * p[i] * kt[j]) + be * vt[i] * kt[j];
                    }
                }
                /* o_t = S_t qhat_t */
                for (int i = 0; i < dv; ++i) {
                    double acc = 0.0;
                    for (int j = 0; j < dk; ++j) acc += S[(int64_t)i * dk + j] * qt[j];
                    ot[i] = acc;
                }
                if (t + 1 == L) memcpy(sc, S, sizeof(double) * hs);
            }
            free(p);
            free(S);
        }
    }
    return 0;
}

/*
 * The whole mixer from raw inputs: normalisation, gates, recurrence, commit.
 *   q, k: [B][T][Hk][dk]; v: [B][T][Hv][dv]; a, b: [B][T][Hv];
 *   A_log, dt_bias: [Hv]; S0: [B][Hv][dv][dk]; accept_len: [B] or NULL.
 */
int oracle_verify(int B, int T, int Hk, int Hv, int dk, int dv,
                  const double* q, const double* k, const double* v,
                  const double* a, const double* b, const double* A_log, const double* dt_bias,
                  const double* S0, const int32_t* accept_len, double l2_eps, double scale,
                  double* o, double* S_commit, int32_t* bad_accept, int nthreads) {
    if (B < 0 || T < 0 || Hk <= 0 || Hv <= 0 || dk <= 0 || dv <= 0 || Hv % Hk != 0) return -1;
    const int64_t nk = (int64_t)B * T * Hk;
    const int64_t ng = (int64_t)B * T * Hv;
    double* qh = (double*)malloc(sizeof(double) * (nk * dk + 1));
    double* kh = (double*)malloc(sizeof(double) * (nk * dk + 1));
    double* la = (double*)malloc(sizeof(double) * (ng + 1));
    double* al = (double*)malloc(sizeof(double) * (ng + 1));
    double* be = (double*)malloc(sizeof(double) * (ng + 1));
    oracle_l2norm(nk, dk, q, l2_eps, scale, qh);
    oracle_l2norm(nk, dk, k, l2_eps, 1.0, kh);
    oracle_gates((int64_t)B * T, Hv, a, b, A_log, dt_bias, la, be);
    for (int64_t i = 0; i < ng; ++i) al[i] = exp(la[i]);
    int rc = oracle_recurrence(B, T, Hk, Hv, dk, dv, qh, kh, v, al, be, S0, accept_len, o,
                               S_commit, bad_accept, nthreads);
    free(qh); free(kh); free(la); free(al); free(be);
    return rc;
}

/*
 * Chunked (WY / UT-transform) form of the same recurrence, chunk length C
 * (the last chunk may be shorter). Inputs are normalised keys/queries and
 * log-gates. Within a chunk of n tokens starting from state S, with
 * G_t = sum_{m<=t} log_alpha_m (chunk-local, inclusive):
 *   A[t][s]  = beta_t exp(G_t - G_s) (khat_t . khat_s),  s < t
 *   (I + A) Utilde = diag(beta) V,   (I + A) W = diag(beta exp(G)) K
 *   U        = Utilde - W S^T                          (the u_t of the recurrence)
 *   o_t      = exp(G_t) S qhat_t + sum_{s<=t} exp(G_t - G_s) (qhat_t . khat_s) u_s
 *   S_next   = exp(G_{n-1}) S + sum_s exp(G_{n-1} - G_s) u_s khat_s^T
 * Decays are only ever formed as exp of a difference, never as a ratio.
 *   S0 may be NULL (zero initial state). S_final: [B][Hv][dv][dk].
 */
int oracle_chunked(int B, int T, int Hk, int Hv, int dk, int dv, int C,
                   const double* qhat, const double* khat, const double* v,
                   const double* log_alpha, const double* beta, const double* S0,
                   double* o, double* S_final, int nthreads) {
    if (B < 0 || T < 0 || Hk <= 0 || Hv <= 0 || dk <= 0 || dv <= 0 || Hv % Hk != 0 || C <= 0 ||
        C > 1024)
        return -1;
    const int G = Hv / Hk;
    const int64_t hs = (int64_t)dv * dk;
    set_threads(nthreads);

#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int bb = 0; bb < B; ++bb) {
        for (int h = 0; h < Hv; ++h) {
            const int g = h / G;
            double* S = (double*)malloc(sizeof(double) * hs);
            double* Gc = (double*)malloc(sizeof(double) * C);
            double* A = (double*)malloc(sizeof(double) * C * C);
            double* Ut = (double*)malloc(sizeof(double) * C * dv);
            double* W = (double*)malloc(sizeof(double) * C * dk);
            double* U = (double*)malloc(sizeof(double) * C * dv);
            double* dec = (double*)malloc(sizeof(double) * C);
            if (S0) memcpy(S, S0 + ((int64_t)bb * Hv + h) * hs, sizeof(double) * hs);
            else memset(S, 0, sizeof(double) * hs);

            for (int c0 = 0; c0 < T; c0 += C) {
                const int n = (T - c0 < C) ? (T - c0) : C;
#define KH(t) (khat + (((int64_t)bb * T + (c0 + (t))) * Hk + g) * dk)
#define QH(t) (qhat + (((int64_t)bb * T + (c0 + (t))) * Hk + g) * dk)
#define VV(t) (v + (((int64_t)bb * T + (c0 + (t))) * Hv + h) * dv)
#define GI(t) (((int64_t)bb * T + (c0 + (t))) * Hv + h)
                double run = 0.0;
                for (int t = 0; t < n; ++t) { run += log_alpha[GI(t)]; Gc[t] = run; }

                for (int t = 0; t < n; ++t) {
                    for (int s = 0; s < t; ++s) {
                        double kk = 0.0;
                        for (int j = 0; j < dk; ++j) kk += KH(t)[j] * KH(s)[j];
                        A[t * C + s] = beta[GI(t)] * exp(Gc[t] - Gc[s]) * kk;
                    }
                }
                /* forward substitution for (I + A) X = RHS, row by row */
                for (int t = 0; t < n; ++t) {
                    const double bt = beta[GI(t)];
                    const double ebt = bt * exp(Gc[t]);
                    for (int i = 0; i < dv; ++i) {
                        double x = bt * VV(t)[i];
                        for (int s = 0; s < t; ++s) x -= A[t * C + s] * Ut[s * dv + i];
                        Ut[t * dv + i] = x;
                    }
                    for (int j = 0; j < dk; ++j) {
                        double x = ebt * KH(t)[j];
                        for (int s = 0; s < t; ++s) x -= A[t * C + s] * W[s * dk + j];
                        W[t * dk + j] = x;
                    }
                }
                /* U = Utilde - W S^T */
                for (int t = 0; t < n; ++t) {
                    for (int i = 0; i < dv; ++i) {
                        double ws = 0.0;
                        for (int j = 0; j < dk; ++j) ws += W[t * dk + j] * S[(int64_t)i * dk + j];
                        U[t * dv + i] = Ut[t * dv + i] - ws;
                    }
                }
                /* outputs */
                for (int t = 0; t < n; ++t) {
                    double* ot = o + (((int64_t)bb * T + (c0 + t)) * Hv + h) * dv;
                    const double eg = exp(Gc[t]);
                    double qk[1024];
                    for (int s = 0; s <= t; ++s) {
                        double d = 0.0;
                        for (int j = 0; j < dk; ++j) d += QH(t)[j] * KH(s)[j];
                        qk[s] = exp(Gc[t] - Gc[s]) * d;
                    }
                    for (int i = 0; i < dv; ++i) {
                        double sq = 0.0;
                        for (int j = 0; j < dk; ++j) sq += S[(int64_t)i * dk + j] * QH(t)[j];
                        double acc = eg * sq;
                        for (int s = 0; s <= t; ++s) acc += qk[s] * U[s * dv + i];
                        ot[i] = acc;
                    }
                }
                /* state hand-off to the next chunk */
                const double eglast = exp(Gc[n - 1]);
                for (int s = 0; s < n; ++s) dec[s] = exp(Gc[n - 1] - Gc[s]);
                for (int i = 0; i < dv; ++i) {
                    for (int j = 0; j < dk; ++j) {
                        double acc = eglast * S[(int64_t)i * dk + j];
                        for (int s = 0; s < n; ++s) acc += dec[s] * U[s * dv + i] * KH(s)[j];
                        S[(int64_t)i * dk + j] = acc;
                    }
                }
#undef KH
#undef QH
#undef VV
#undef GI
            }
            memcpy(S_final + ((int64_t)bb * Hv + h) * hs, S, sizeof(double) * hs);
            free(S); free(Gc); free(A); free(Ut); free(W); free(U); free(dec);
        }
    }
    return 0;
}

/*
 * Causal short convolution with its history, rewound to the accepted prefix. The source
 * ("Qwen 3.8 27B mac m5: 200 tok/s, audited", section "How does DSpark speculative decoding
 * create more than one token per read?") names the short history that a small filter layer
 * keeps as one of the three structures brought back in line with the accepted tokens after a
 * verify block (with the key-value cache and the recurrent state). It gives no width or
 * activation; this is the plain reading: one filter of K taps per channel over that channel's
 * last K inputs, SiLU applied to the sum, no bias.
 *
 *   per sequence b and channel c, xc = [hist_0 .. hist_{K-2}, x_0 .. x_{T-1}] (oldest first):
 *     y_t = silu( sum_{i<K} w[c][i] * xc[t + i] ),   silu(z) = z / (1 + e^-z)
 *     so w[c][K-1] weighs the current input x_t and w[c][0] the oldest;
 *     new history = xc[L .. L + K - 2],   L = accept_len[b] (L = T when accept_len is NULL).
 *   An L outside 0..T keeps the old history and is counted in the return value.
 *
 * x, y: [B][T][C]; w: [C][K]; hist, hist_out: [B][K-1][C] (hist_out may be NULL).
 */
int oracle_short_conv(int B, int T, int C, int K, const double* x, const double* w, const double* hist,
                      const int32_t* accept_len, double* y, double* hist_out) {
    int bad = 0;
    const int H = K - 1;
    double* xc = (double*)malloc(sizeof(double) * (size_t)(H + T));
    for (int b = 0; b < B; ++b) {
        int L = accept_len ? accept_len[b] : T;
        const int ok = L >= 0 && L <= T;
        if (!ok) ++bad;
        for (int c = 0; c < C; ++c) {
            for (int r = 0; r < H; ++r) xc[r] = hist[((int64_t)b * H + r) * C + c];
            for (int t = 0; t < T; ++t) xc[H + t] = x[((int64_t)b * T + t) * C + c];
            for (int t = 0; t < T; ++t) {
                double z = 0.0;
                for (int i = 0; i < K; ++i) z += w[(int64_t)c * K + i] * xc[t + i];
                y[((int64_t)b * T + t) * C + c] = z / (1.0 + exp(-z));
            }
            if (hist_out) {
                const int from = ok ? L : 0;
                for (int r = 0; r < H; ++r) hist_out[((int64_t)b * H + r) * C + c] = xc[from + r];
            }
        }
    }
    free(xc);
    return bad;
}

/*
 * Gated RMS normalisation of the mixer's output. The source ("Lithos-metal: Qwen3.8-27B on
 * 40-core M5 Max", table "GDN mixer") lists gating and normalisation among the mixer's jobs,
 * after the recurrence, without the formula; this is the plain reading, per output row
 * (one token of one value head, d values):
 *   y_j = o_j / sqrt( (1/d) sum_j o_j^2 + eps ) * w_j * silu(z_j),   silu(z) = z / (1 + e^-z)
 * o, z, y: [n][d]; w: [d] (shared by all rows).
 */
void oracle_gated_rmsnorm(int64_t n, int d, const double* o, const double* z, const double* w, double eps,
                          double* y) {
    for (int64_t r = 0; r < n; ++r) {
        const double* orow = o + r * d;
        const double* zrow = z + r * d;
        double ss = 0.0;
        for (int j = 0; j < d; ++j) ss += orow[j] * orow[j];
        const double inv = 1.0 / sqrt(ss / d + eps);
        for (int j = 0; j < d; ++j) {
            const double g = zrow[j] / (1.0 + exp(-zrow[j]));
            y[r * d + j] = orow[j] * inv * w[j] * g;
        }
    }
}

/*
 * Acceptance of a verify block ("Qwen 3.8 27B mac m5: 200 tok/s, audited", section "How does
 * DSpark speculative decoding create more than one token per read?": up to seven guesses plus
 * the anchor, exact speculative sampling; greedy mode keeps a guess only if it matches the
 * large model's token; sampled mode accepts it with probability p / q capped at one, then a
 * correction token, or a bonus token when every guess was right).
 *
 * Per sequence b, tokens[b][0] is the anchor and tokens[b][t] (t = 1 .. T-1) the drafts. Target
 * row t (logits over V) is the large model's prediction of the token after row t; draft row t
 * (sampled mode) is the drafter's distribution that proposed tokens[b][t + 1]. With
 * p_t = softmax(target_t / tau), q_t = softmax(draft_t / tau):
 *   greedy:  draft t+1 survives iff tokens[t+1] == argmax p_t (lowest index among equal maxima);
 *   sampled: draft t+1 survives iff u[t+1] * q_t(tokens[t+1]) < p_t(tokens[t+1])
 *            (u < min(1, p / q) without a division);
 *   n = the number of leading survivors (0 .. T-1); accept_len = n + 1 (the anchor and the
 *   surviving drafts: the rows whose state the mixer commits);
 *   next token: greedy argmax p_n; sampled, n < T-1: drawn from the residual max(0, p_n - q_n)
 *   (normalised), n = T-1: drawn from p_{T-1}; a draw with u[0] takes the first index j whose
 *   cumulative mass exceeds u[0] times the total.
 * target: [B][T][V]; draft: [B][T-1][V] or NULL (greedy); tokens: [B][T]; u: [B][T] or NULL.
 * Diagnostics (may be NULL): pd, qd [B][T-1] = p_t and q_t at the draft token.
 */
static void softmax_row(const double* l, int V, double tau, double* p) {
    double m = l[0];
    for (int j = 1; j < V; ++j) m = fmax(m, l[j]);
    double s = 0.0;
    for (int j = 0; j < V; ++j) s += exp((l[j] - m) / tau);
    for (int j = 0; j < V; ++j) p[j] = exp((l[j] - m) / tau) / s;
}

static int draw(const double* w, int V, double u) {
    double tot = 0.0;
    for (int j = 0; j < V; ++j) tot += w[j];
    const double target = u * tot;
    double c = 0.0;
    for (int j = 0; j < V; ++j) {
        c += w[j];
        if (c > target && w[j] > 0.0) return j;
    }
    for (int j = V - 1; j >= 0; --j)
        if (w[j] > 0.0) return j;
    return 0;
}

int oracle_accept(int B, int T, int V, const double* target, const double* draft, const int32_t* tokens,
                  const double* u, double tau, int sampled, int32_t* accept_len, int32_t* next_token, double* pd,
                  double* qd) {
    if (T < 1 || V < 1 || (sampled && (!draft || !u)) || !(tau > 0.0)) return -1;
    double* p = (double*)malloc(sizeof(double) * (size_t)V);
    double* q = (double*)malloc(sizeof(double) * (size_t)V);
    for (int b = 0; b < B; ++b) {
        const int32_t* tok = tokens + (int64_t)b * T;
        int n = 0;
        int stopped = 0;
        for (int t = 0; t + 1 < T; ++t) {
            const double* lt = target + ((int64_t)b * T + t) * V;
            const int d = tok[t + 1];
            int ok;
            if (!sampled) {
                int am = 0;
                for (int j = 1; j < V; ++j)
                    if (lt[j] > lt[am]) am = j;
                ok = (d == am);
                if (pd) pd[(int64_t)b * (T - 1) + t] = (double)am;
            } else {
                softmax_row(lt, V, tau, p);
                softmax_row(draft + ((int64_t)b * (T - 1) + t) * V, V, tau, q);
                const double pv = (d >= 0 && d < V) ? p[d] : 0.0;
                const double qv = (d >= 0 && d < V) ? q[d] : 0.0;
                if (pd) pd[(int64_t)b * (T - 1) + t] = pv;
                if (qd) qd[(int64_t)b * (T - 1) + t] = qv;
                ok = u[(int64_t)b * T + t + 1] * qv < pv;
            }
            if (!stopped && ok) {
                ++n;
            } else {
                stopped = 1;
            }
        }
        accept_len[b] = n + 1;
        const double* ln = target + ((int64_t)b * T + n) * V;
        if (!sampled) {
            int am = 0;
            for (int j = 1; j < V; ++j)
                if (ln[j] > ln[am]) am = j;
            next_token[b] = am;
        } else {
            softmax_row(ln, V, tau, p);
            if (n < T - 1) {
                softmax_row(draft + ((int64_t)b * (T - 1) + n) * V, V, tau, q);
                for (int j = 0; j < V; ++j) q[j] = fmax(p[j] - q[j], 0.0);
                double tot = 0.0;
                for (int j = 0; j < V; ++j) tot += q[j];
                next_token[b] = draw(tot > 0.0 ? q : p, V, u[(int64_t)b * T]);
            } else {
                next_token[b] = draw(p, V, u[(int64_t)b * T]);
            }
        }
    }
    free(p);
    free(q);
    return 0;
}
