/*
 * lattice_oracle.c -- plain fp64 CPU oracle of the Lattice compression-layer
 * state recurrence.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product path links, loads or calls
 * this file; only the tests, the smoke check and the benchmark's CPU-baseline
 * leg use it. It shares no code, header or constant with the CUDA library.
 *
 * Source: "Lattice: Learning to Efficiently Compress the Memory" (Karami,
 * Pascanu, Mirrokni; arXiv 2504.05646).
 *   - §3.1.1, eq. (similarity_recurrence) and eq. (OSR): the online gradient
 *     step of the dot-product objective writes, into slot i, the part of the
 *     input orthogonal to that slot, P(s_i) x / ||s_i||, scaled by the writing
 *     intensity c_i (h_t = -v_t for the similarity objective).
 *   - §3.2, eq. (normalized_recurrence): each slot is projected back onto the
 *     unit sphere after the write.
 *   - §3.3, eq. (dacay_recurrence) and the "General Form": the forget gate mu
 *     scales the previous state; the normaliser applies to mu*s + write.
 *   - §3.4, Eq. 14 (recurrence_detailed): P(s) h = h - s (s.h)/||s||^2 costs one
 *     dot product and one axpy per slot.
 *   - §3.4.1 eq. (recurrence_linear1) and eq. (chunkwise_OSR): the other
 *     linearisation keeps the h~ k^ term on the chunk-start state:
 *     S_t = G_t (.) S_{t-1} + 1 (h~_t (.) k^_t)^T (.) S_{t'} - h_t k^_t^T, G_t = mu_t 1 beta_t^T.
 *   - §3.4.1 / Appendix B.1, Eq. 17 (recurrence_linear2) and eq. (beta_chunk):
 *     within a chunk the projection uses the chunk-start state; the update
 *     becomes the gated linear recurrence S_t = G_t (.) S_{t-1} - h_t k_t^T.
 *   - Appendix D (Implementation): argument shapes and the read-out y = q S_t
 *     with the updated state.
 *
 *   - backward pass (oracle_scan_bwd): the paper prints none; the adjoint of the
 *     similarity-objective forward above, exact and Eq. 17, derived step by step
 *     and pinned by finite differences of the forward.
 *   - §3.1.1 eq. (decoding_stateNorm_loss) and eq. (decoding_recurrence): the
 *     reconstruction objective writes the part of the reconstruction error
 *     e = phi(S) c - x orthogonal to each slot (h_t = e_t in eq. OSR).
 *
 * Readings of points the paper leaves open (each is listed in the design notes):
 *   - slots are rows of S ([m][d]), as in the Appendix D listing;
 *   - the normaliser targets the unit sphere (§3.2), with no epsilon;
 *   - the normaliser of the chunked form is n/sqrt(mu^2 n^2 + |Delta|^2) with
 *     n = |s0| the chunk-start norm: the Appendix D listing (compress_chunk)
 *     scales its rsqrt by s_norm, so a slot keeps its chunk-start norm; §B.1's
 *     (1 + D_S)^(-1/2) is the same value for n = 1. Without the n factor the
 *     chunked recurrence diverges (slot norms leave O(1) within a few chunks
 *     and the gates of small-norm slots explode). The printed eta^2 in front
 *     of s_norm^2 reads as a typo for mu^2: only mu^2 makes chunk size 1 equal
 *     the exact recurrence (for unit-norm states);
 *   - D_S uses "minus" (Pythagoras, §3.2), clipped at zero;
 *   - a slot whose update has zero norm (mu = 0 and no orthogonal write) is
 *     left unchanged and counted;
 *   - the reconstruction objective's step is -eta (c_i/|s_i|) P(s_i) e, the
 *     gradient of eq. (decoding_recurrence) as printed (that of |phi(S) c - x|^2 / 2);
 *     its error e is taken from the state the token's projection uses: the
 *     current state (exact recurrence) or the chunk-start state (Eq. 17), as in
 *     the Appendix D listing.
 *
 * Layouts (row-major):  x[B][T][H][d]  c,q[B][T][H][m]  mu,eta[B][T][H]
 *                       S[B][H][m][d]  y[B][T][H][d].   eta == NULL means 1.
 */
#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>

#define IDX_TOK(b, t, h, T, H) ((((size_t)(b) * (T)) + (t)) * (H) + (h))

/* ------------------------------------------------------------------------ */
/* One slot, one token (exact recurrence).                                   */
/* ------------------------------------------------------------------------ */

/* Unnormalised write w = mu*s + eta*(c/||s||) * P(s) x  (§3.1.1 eq. OSR with
 * h = -x, the forget gate of §3.3, the projection of §3.4 Eq. 14).
 * Returns ||s||^2 via *n2_out. */
void oracle_osr_write(int d, const double *s, const double *x, double c, double mu,
                      double eta, double *w, double *n2_out)
{
    double n2 = 0.0, p = 0.0;
    for (int k = 0; k < d; ++k) {
        n2 += s[k] * s[k];
        p += s[k] * x[k];
    }
    double n = sqrt(n2);
    for (int k = 0; k < d; ++k) {
        double x_perp = x[k] - (p / n2) * s[k]; /* P(s) x */
        w[k] = mu * s[k] + eta * (c / n) * x_perp;
    }
    if (n2_out) *n2_out = n2;
}

/* The negated write direction of one token, x_eff = -h_t (§3.1.1 eq. OSR).
 *   similarity objective (mode 0): h = -x, so x_eff = x;
 *   reconstruction objective (mode 1, §3.1.1 eq. decoding_stateNorm_loss and
 *   eq. decoding_recurrence): h = e = phi(S) c - x, the reconstruction error of
 *   the token with the normalised slots phi(s_i) = s_i/|s_i| (the listing's
 *   h = k @ Phi - v), so x_eff = x - sum_i c_i s_i/|s_i|.
 * S is the state the token's projection uses (the current state for the exact
 * recurrence, the chunk-start state for Eq. 17). A zero slot has no direction
 * and contributes nothing. */
void oracle_write_input(int mode, int m, int d, const double *S, const double *c,
                        const double *x, double *x_eff)
{
    for (int k = 0; k < d; ++k) x_eff[k] = x[k];
    if (mode != 1) return;
    for (int i = 0; i < m; ++i) {
        const double *s = S + (size_t)i * d;
        double n2 = 0.0;
        for (int k = 0; k < d; ++k) n2 += s[k] * s[k];
        if (n2 == 0.0) continue;
        double f = c[i] / sqrt(n2);
        for (int k = 0; k < d; ++k) x_eff[k] -= f * s[k];
    }
}

/* One exact step of the whole state (all m slots) followed by the read-out.
 * Updates S in place; writes y if non-NULL; counts zero-norm updates. */
static void exact_token(int m, int d, double *S, const double *x, const double *c,
                        const double *q, double mu, double eta, double *y, double *w,
                        long long *degenerate)
{
    for (int i = 0; i < m; ++i) {
        double *s = S + (size_t)i * d;
        double n2;
        oracle_osr_write(d, s, x, c[i], mu, eta, w, &n2);
        double nw2 = 0.0;
        for (int k = 0; k < d; ++k) nw2 += w[k] * w[k];
        if (n2 == 0.0 || nw2 == 0.0) { /* undefined projection: keep the slot */
            ++*degenerate;
            continue;
        }
        double nw = sqrt(nw2);
        for (int k = 0; k < d; ++k) s[k] = w[k] / nw; /* §3.2 unit sphere */
    }
    if (y) {
        for (int k = 0; k < d; ++k) y[k] = 0.0;
        for (int i = 0; i < m; ++i)
            for (int k = 0; k < d; ++k) y[k] += q[i] * S[(size_t)i * d + k];
    }
}

/* ------------------------------------------------------------------------ */
/* Chunked recurrence, Eq. 17: per-token gates from the chunk-start state.   */
/* ------------------------------------------------------------------------ */

/* Gates of one token against the chunk-start state S0 (Eq. 17 and eq.
 * beta_chunk, Appendix B.1; normaliser as in the Appendix D listing):
 *   h = -x;  hhat_i = (h.s0_i)/n_i^2;  khat_i = c_i/n_i;
 *   dsq_i  = eta^2 * max(0, khat_i^2 |h|^2 - n_i^2 hhat_i^2 khat_i^2)
 *   beta_i = n_i/sqrt(mu^2 n_i^2 + dsq_i)
 *   g_i    = beta_i (mu + eta hhat_i khat_i),   kt_i = -beta_i eta khat_i
 * so that the token's update is s_i <- g_i s_i + kt_i h. */
void oracle_chunk_token_gates2(int m, int d, const double *S0, const double *n2,
                               const double *x, const double *c, double mu, double eta,
                               double *g, double *kt, double *dsq_out, long long *degenerate,
                               double *gs, double *g0, int nobeta);
void oracle_chunk_token_gates(int m, int d, const double *S0, const double *n2,
                              const double *x, const double *c, double mu, double eta,
                              double *g, double *kt, double *dsq_out, long long *degenerate)
{
    oracle_chunk_token_gates2(m, d, S0, n2, x, c, mu, eta, g, kt, dsq_out, degenerate, NULL, NULL, 0);
}

/* As above, and the two parts of g: gs_i = beta_i mu (what scales the running slot
 * in eq. recurrence_linear1, the G_t of §3.4.1) and g0_i = beta_i eta hhat_i khat_i
 * (what scales the chunk-start slot there); g = gs + g0. nobeta != 0 drops the
 * per-token normaliser (beta = 1), for normalisation at chunk boundaries only
 * (Appendix C, "Per-token vs. Per-chunk Normalization"). */
void oracle_chunk_token_gates2(int m, int d, const double *S0, const double *n2,
                               const double *x, const double *c, double mu, double eta,
                               double *g, double *kt, double *dsq_out, long long *degenerate,
                               double *gs, double *g0, int nobeta)
{
    double hh = 0.0;
    for (int k = 0; k < d; ++k) hh += x[k] * x[k]; /* |h|^2, h = -x */
    for (int i = 0; i < m; ++i) {
        const double *s0 = S0 + (size_t)i * d;
        double hdot = 0.0;
        for (int k = 0; k < d; ++k) hdot += (-x[k]) * s0[k];
        double hhat = hdot / n2[i];
        double khat = c[i] / sqrt(n2[i]);
        double t = khat * khat * hh - n2[i] * hhat * hhat * khat * khat;
        double dsq = eta * eta * (t > 0.0 ? t : 0.0);
        double den = mu * mu * n2[i] + dsq;
        if (dsq_out) dsq_out[i] = dsq;
        if (nobeta) {
            g[i] = mu + eta * hhat * khat;
            kt[i] = -eta * khat;
            if (gs) { gs[i] = mu; g0[i] = eta * hhat * khat; }
            continue;
        }
        if (den == 0.0) { /* zero-norm update: keep the slot */
            g[i] = 1.0;
            kt[i] = 0.0;
            if (gs) { gs[i] = 1.0; g0[i] = 0.0; }
            if (degenerate) ++*degenerate;
            continue;
        }
        double beta = sqrt(n2[i]) / sqrt(den);
        g[i] = beta * (mu + eta * hhat * khat);
        kt[i] = -beta * eta * khat;
        if (gs) { gs[i] = beta * mu; g0[i] = beta * eta * hhat * khat; }
    }
}

/* ------------------------------------------------------------------------ */
/* Whole-sequence drivers, one (b,h) sequence at a time.                     */
/* ------------------------------------------------------------------------ */

typedef struct {
    int B, T, H, m, d, C, form; /* form: 0 exact, 1 chunked token-wise, 2 chunked matrix form */
    int mode;                   /* 0 similarity objective, 1 reconstruction objective */
    int lin;                    /* chunked forms: 2 Eq. 17 (recurrence_linear2), 1 recurrence_linear1 */
    int cnorm;                  /* chunked forms: 0 per-token normaliser, 1 normalise at chunk ends */
    const double *x, *c, *q, *mu, *eta, *S0;
    double *S_out, *y;
    long long degenerate;
    int next;
    pthread_mutex_t lock;
} job_t;

static void run_exact(job_t *J, int b, int h, double *S, double *w, double *xe, long long *deg)
{
    const int T = J->T, H = J->H, m = J->m, d = J->d;
    for (int t = 0; t < T; ++t) {
        size_t tok = IDX_TOK(b, t, h, T, H);
        double eta = J->eta ? J->eta[tok] : 1.0;
        oracle_write_input(J->mode, m, d, S, J->c + tok * m, J->x + tok * d, xe); /* before the update */
        exact_token(m, d, S, xe, J->c + tok * m, J->q + tok * m, J->mu[tok], eta, J->y + tok * d, w,
                    deg);
    }
}

/* Projection of every slot onto the unit sphere (§3.2), at a chunk boundary. */
static void normalise_slots(int m, int d, double *S)
{
    for (int i = 0; i < m; ++i) {
        double *s = S + (size_t)i * d, n2 = 0.0;
        for (int k = 0; k < d; ++k) n2 += s[k] * s[k];
        if (n2 == 0.0) continue;
        double n = sqrt(n2);
        for (int k = 0; k < d; ++k) s[k] /= n;
    }
}

static void run_chunked_tokenwise(job_t *J, int b, int h, double *S, double *S0, double *n2,
                                  double *g, double *kt, double *xe, double *gs, double *g0,
                                  long long *deg)
{
    const int T = J->T, H = J->H, m = J->m, d = J->d, C = J->C;
    for (int t0 = 0; t0 < T; t0 += C) {
        int t1 = t0 + C < T ? t0 + C : T;
        memcpy(S0, S, sizeof(double) * (size_t)m * d); /* chunk-start state S_{t'} */
        for (int i = 0; i < m; ++i) {
            double a = 0.0;
            for (int k = 0; k < d; ++k) a += S0[(size_t)i * d + k] * S0[(size_t)i * d + k];
            n2[i] = a;
        }
        for (int t = t0; t < t1; ++t) {
            size_t tok = IDX_TOK(b, t, h, T, H);
            oracle_write_input(J->mode, m, d, S0, J->c + tok * m, J->x + tok * d, xe); /* chunk start */
            const double *x = xe;
            double eta = J->eta ? J->eta[tok] : 1.0;
            oracle_chunk_token_gates2(m, d, S0, n2, x, J->c + tok * m, J->mu[tok], eta, g, kt,
                                      NULL, deg, gs, g0, J->cnorm);
            if (J->lin == 1) { /* eq. recurrence_linear1: s_i <- gs_i s_i + g0_i s0_i + kt_i h */
                for (int i = 0; i < m; ++i)
                    for (int k = 0; k < d; ++k)
                        S[(size_t)i * d + k] = gs[i] * S[(size_t)i * d + k] +
                                               g0[i] * S0[(size_t)i * d + k] + kt[i] * (-x[k]);
            } else { /* Eq. 17: s_i <- g_i s_i + kt_i h,  h = -x */
                for (int i = 0; i < m; ++i)
                    for (int k = 0; k < d; ++k)
                        S[(size_t)i * d + k] = g[i] * S[(size_t)i * d + k] + kt[i] * (-x[k]);
            }
            double *y = J->y + tok * d;
            const double *q = J->q + tok * m;
            for (int k = 0; k < d; ++k) y[k] = 0.0;
            for (int i = 0; i < m; ++i)
                for (int k = 0; k < d; ++k) y[k] += q[i] * S[(size_t)i * d + k];
        }
        if (J->cnorm) normalise_slots(m, d, S); /* after the chunk's last read-out */
    }
}

/* Chunk-level closed form of the gated linear recurrence of Eq. 17 (the form
 * that a chunk-parallel evaluation computes, §3.4.1 / Appendix B.1):
 *   y_tau = sum_i q_tau,i A_tau,i s0_i + sum_{j<=tau} P_tau,j h_j,
 *   P_tau,j = sum_i q_tau,i kt_j,i prod_{l=j+1..tau} g_l,i,
 *   S_C,i   = A_C,i s0_i + sum_j kt_j,i prod_{l=j+1..C} g_l,i h_j,
 * with A_tau = prod_{l<=tau} g_l. Products are formed directly (no division).
 * Used to check the token-wise form; both share the per-token gates. */
static void run_chunked_matrix(job_t *J, int b, int h, double *S, double *S0, double *n2,
                               double *G, double *KT, double *XE, double *GS, double *G0,
                               long long *deg)
{
    /* eq. recurrence_linear1's chunk form (eq. chunkwise_OSR) multiplies by the running
     * gates gs and adds f / F terms for g0 s0; Eq. 17's multiplies by g = gs + g0. */
    const int lin1 = J->lin == 1;
    const int T = J->T, H = J->H, m = J->m, d = J->d, C = J->C;
    for (int t0 = 0; t0 < T; t0 += C) {
        int L = (t0 + C < T ? t0 + C : T) - t0;
        memcpy(S0, S, sizeof(double) * (size_t)m * d);
        for (int i = 0; i < m; ++i) {
            double a = 0.0;
            for (int k = 0; k < d; ++k) a += S0[(size_t)i * d + k] * S0[(size_t)i * d + k];
            n2[i] = a;
        }
        for (int tau = 0; tau < L; ++tau) {
            size_t tok = IDX_TOK(b, t0 + tau, h, T, H);
            double eta = J->eta ? J->eta[tok] : 1.0;
            oracle_write_input(J->mode, m, d, S0, J->c + tok * m, J->x + tok * d, XE + (size_t)tau * d);
            oracle_chunk_token_gates2(m, d, S0, n2, XE + (size_t)tau * d, J->c + tok * m, J->mu[tok],
                                      eta, G + (size_t)tau * m, KT + (size_t)tau * m, NULL, deg,
                                      GS + (size_t)tau * m, G0 + (size_t)tau * m, J->cnorm);
            if (lin1) /* the products run over the running gates */
                memcpy(G + (size_t)tau * m, GS + (size_t)tau * m, sizeof(double) * (size_t)m);
        }
        for (int tau = 0; tau < L; ++tau) {
            size_t tok = IDX_TOK(b, t0 + tau, h, T, H);
            const double *q = J->q + tok * m;
            double *y = J->y + tok * d;
            for (int k = 0; k < d; ++k) y[k] = 0.0;
            for (int i = 0; i < m; ++i) { /* inter-chunk term (Q (.) (A + F)) S0 */
                double A = 1.0;
                for (int l = 0; l <= tau; ++l) A *= G[(size_t)l * m + i];
                if (lin1) { /* F_tau,i = sum_{j<=tau} g0_j,i prod_{l=j+1..tau} gs_l,i */
                    for (int j = 0; j <= tau; ++j) {
                        double prod = 1.0;
                        for (int l = j + 1; l <= tau; ++l) prod *= G[(size_t)l * m + i];
                        A += G0[(size_t)j * m + i] * prod;
                    }
                }
                for (int k = 0; k < d; ++k) y[k] += q[i] * A * S0[(size_t)i * d + k];
            }
            for (int j = 0; j <= tau; ++j) { /* intra-chunk term P H */
                double P = 0.0;
                for (int i = 0; i < m; ++i) {
                    double prod = 1.0;
                    for (int l = j + 1; l <= tau; ++l) prod *= G[(size_t)l * m + i];
                    P += q[i] * KT[(size_t)j * m + i] * prod;
                }
                const double *xj = XE + (size_t)j * d;
                for (int k = 0; k < d; ++k) y[k] += P * (-xj[k]);
            }
        }
        for (int i = 0; i < m; ++i) { /* chunk-end state */
            double A = 1.0;
            for (int l = 0; l < L; ++l) A *= G[(size_t)l * m + i];
            if (lin1) { /* + f_i = sum_j g0_j,i prod_{l=j+1..C} gs_l,i */
                for (int j = 0; j < L; ++j) {
                    double prod = 1.0;
                    for (int l = j + 1; l < L; ++l) prod *= G[(size_t)l * m + i];
                    A += G0[(size_t)j * m + i] * prod;
                }
            }
            for (int k = 0; k < d; ++k) S[(size_t)i * d + k] = A * S0[(size_t)i * d + k];
            for (int j = 0; j < L; ++j) {
                double prod = 1.0;
                for (int l = j + 1; l < L; ++l) prod *= G[(size_t)l * m + i];
                double coef = KT[(size_t)j * m + i] * prod;
                const double *xj = XE + (size_t)j * d;
                for (int k = 0; k < d; ++k) S[(size_t)i * d + k] += coef * (-xj[k]);
            }
        }
        if (J->cnorm) normalise_slots(m, d, S);
    }
}

static void *worker(void *arg)
{
    job_t *J = (job_t *)arg;
    const int m = J->m, d = J->d;
    int C = J->C > 0 ? J->C : 1;
    double *S = malloc(sizeof(double) * (size_t)m * d);
    double *S0 = malloc(sizeof(double) * (size_t)m * d);
    double *n2 = malloc(sizeof(double) * (size_t)m);
    double *w = malloc(sizeof(double) * (size_t)d);
    double *G = malloc(sizeof(double) * (size_t)C * m);
    double *KT = malloc(sizeof(double) * (size_t)C * m);
    double *XE = malloc(sizeof(double) * (size_t)C * d);
    double *GS = malloc(sizeof(double) * (size_t)C * m);
    double *G0 = malloc(sizeof(double) * (size_t)C * m);
    long long deg = 0;
    for (;;) {
        pthread_mutex_lock(&J->lock);
        int item = J->next++;
        pthread_mutex_unlock(&J->lock);
        if (item >= J->B * J->H) break;
        int b = item / J->H, h = item % J->H;
        size_t so = ((size_t)b * J->H + h) * (size_t)m * d;
        memcpy(S, J->S0 + so, sizeof(double) * (size_t)m * d);
        if (J->form == 0)
            run_exact(J, b, h, S, w, XE, &deg);
        else if (J->form == 1)
            run_chunked_tokenwise(J, b, h, S, S0, n2, G, KT, XE, GS, G0, &deg);
        else
            run_chunked_matrix(J, b, h, S, S0, n2, G, KT, XE, GS, G0, &deg);
        if (J->S_out) memcpy(J->S_out + so, S, sizeof(double) * (size_t)m * d);
    }
    pthread_mutex_lock(&J->lock);
    J->degenerate += deg;
    pthread_mutex_unlock(&J->lock);
    free(S); free(S0); free(n2); free(w); free(G); free(KT); free(XE); free(GS); free(G0);
    return NULL;
}

static long long run_lin(int form, int mode, int lin, int B, int T, int H, int m, int d, int C,
                         const double *x, const double *c, const double *q, const double *mu,
                         const double *eta, const double *S0, double *S_out, double *y,
                         int nthreads)
{
    job_t J;
    memset(&J, 0, sizeof(J));
    J.B = B; J.T = T; J.H = H; J.m = m; J.d = d; J.C = C; J.form = form; J.mode = mode;
    J.lin = lin & 3;
    J.cnorm = (lin >> 2) & 1; /* lin | 4: normalise at chunk boundaries only */
    J.x = x; J.c = c; J.q = q; J.mu = mu; J.eta = eta; J.S0 = S0; J.S_out = S_out; J.y = y;
    pthread_mutex_init(&J.lock, NULL);
    if (nthreads < 1) nthreads = 1;
    if (nthreads > B * H) nthreads = B * H;
    if (nthreads <= 1) {
        worker(&J);
    } else {
        pthread_t *th = malloc(sizeof(pthread_t) * (size_t)nthreads);
        for (int i = 0; i < nthreads; ++i) pthread_create(&th[i], NULL, worker, &J);
        for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
        free(th);
    }
    pthread_mutex_destroy(&J.lock);
    return J.degenerate;
}

static long long run(int form, int mode, int B, int T, int H, int m, int d, int C, const double *x,
                     const double *c, const double *q, const double *mu, const double *eta,
                     const double *S0, double *S_out, double *y, int nthreads)
{
    return run_lin(form, mode, 2, B, T, H, m, d, C, x, c, q, mu, eta, S0, S_out, y, nthreads);
}

/* Chunked recurrence in either linearisation of §3.4.1 (lin 2: Eq. 17,
 * recurrence_linear2; lin 1: recurrence_linear1), token by token (form 1) or through
 * the chunk closed form (form 2). lin | 4 drops the per-token normaliser and projects
 * the slots onto the unit sphere after each chunk instead (Appendix C ablation). */
long long oracle_chunked_scan_lin(int form, int mode, int lin, int B, int T, int H, int m, int d,
                                  int C, const double *x, const double *c, const double *q,
                                  const double *mu, const double *eta, const double *S0,
                                  double *S_out, double *y, int nthreads)
{
    return run_lin(form, mode, lin, B, T, H, m, d, C, x, c, q, mu, eta, S0, S_out, y, nthreads);
}

/* Whole-sequence drivers. mode 0: similarity objective (h = -x); mode 1:
 * reconstruction objective (h = phi(S) c - x, see oracle_write_input).
 * Each returns the number of zero-norm updates. */

/* Exact recurrence (chunk size 1). */
long long oracle_exact_scan_mode(int mode, int B, int T, int H, int m, int d, const double *x,
                                 const double *c, const double *q, const double *mu,
                                 const double *eta, const double *S0, double *S_out, double *y,
                                 int nthreads)
{
    return run(0, mode, B, T, H, m, d, 1, x, c, q, mu, eta, S0, S_out, y, nthreads);
}

/* Chunked recurrence of Eq. 17, chunk size C, evaluated token by token. */
long long oracle_chunked_scan_mode(int mode, int B, int T, int H, int m, int d, int C,
                                   const double *x, const double *c, const double *q,
                                   const double *mu, const double *eta, const double *S0,
                                   double *S_out, double *y, int nthreads)
{
    return run(1, mode, B, T, H, m, d, C, x, c, q, mu, eta, S0, S_out, y, nthreads);
}

/* Same definition evaluated through the chunk-level closed form (self-check). */
long long oracle_chunked_matrix_scan_mode(int mode, int B, int T, int H, int m, int d, int C,
                                          const double *x, const double *c, const double *q,
                                          const double *mu, const double *eta, const double *S0,
                                          double *S_out, double *y, int nthreads)
{
    return run(2, mode, B, T, H, m, d, C, x, c, q, mu, eta, S0, S_out, y, nthreads);
}

/* The similarity-objective drivers. */
long long oracle_exact_scan(int B, int T, int H, int m, int d, const double *x, const double *c,
                            const double *q, const double *mu, const double *eta,
                            const double *S0, double *S_out, double *y, int nthreads)
{
    return run(0, 0, B, T, H, m, d, 1, x, c, q, mu, eta, S0, S_out, y, nthreads);
}

long long oracle_chunked_scan(int B, int T, int H, int m, int d, int C, const double *x,
                              const double *c, const double *q, const double *mu,
                              const double *eta, const double *S0, double *S_out, double *y,
                              int nthreads)
{
    return run(1, 0, B, T, H, m, d, C, x, c, q, mu, eta, S0, S_out, y, nthreads);
}

long long oracle_chunked_matrix_scan(int B, int T, int H, int m, int d, int C, const double *x,
                                     const double *c, const double *q, const double *mu,
                                     const double *eta, const double *S0, double *S_out,
                                     double *y, int nthreads)
{
    return run(2, 0, B, T, H, m, d, C, x, c, q, mu, eta, S0, S_out, y, nthreads);
}

/* Read-out y = sum_i q_i s_i for every (b,h): S[B][H][m][d], q[B][H][m], y[B][H][d]
 * (Appendix D listing, y = q @ S_t; §2 eq. LA read-out). */
void oracle_readout(int B, int H, int m, int d, const double *S, const double *q, double *y)
{
    for (int bh = 0; bh < B * H; ++bh) {
        const double *Sb = S + (size_t)bh * m * d;
        const double *qb = q + (size_t)bh * m;
        double *yb = y + (size_t)bh * d;
        for (int k = 0; k < d; ++k) yb[k] = 0.0;
        for (int i = 0; i < m; ++i)
            for (int k = 0; k < d; ++k) yb[k] += qb[i] * Sb[(size_t)i * d + k];
    }
}

/* ------------------------------------------------------------------------ */
/* Backward pass: the adjoint of the forward definitions above.              */
/* ------------------------------------------------------------------------ */
/* The paper prints no backward formulas (its training differentiates the JAX
 * forward automatically, Appendix D). These are the reverse-mode derivatives of
 * the similarity-objective forward above, taken step by step in the order the
 * forward computes its intermediates, for the scalar loss
 *     L = sum_t dy_t . y_t + dS_T . S_T.
 * Every function below is pinned by central finite differences of the forward
 * drivers above (tests/test_oracle_pins.py). */

/* Adjoint of one exact slot update (§3.1.1 eq. OSR, §3.2, §3.3, Eq. 14):
 *   n2 = s.s, p = s.x, n = sqrt(n2), r = p/n2, a = eta c/n,
 *   x_perp = x - r s, w = mu s + a x_perp, s' = w/|w|.
 * gb = dL/ds' in, sb = dL/ds out; dL/dx, dL/dmu, dL/deta are added to xb, *mub,
 * *etab and dL/dc is stored in *cb. A degenerate update (n2 = 0 or w = 0) kept the
 * slot, so it passes gb through. tmp holds 3d doubles. */
static void exact_slot_bwd(int d, const double *s, const double *x, double c, double mu,
                           double eta, const double *gb, double *sb, double *xb, double *cb,
                           double *mub, double *etab, double *tmp)
{
    double *w = tmp, *xp = tmp + d, *wb = tmp + 2 * d;
    double n2 = 0.0, p = 0.0;
    for (int k = 0; k < d; ++k) { n2 += s[k] * s[k]; p += s[k] * x[k]; }
    *cb = 0.0;
    if (n2 == 0.0) { for (int k = 0; k < d; ++k) sb[k] = gb[k]; return; }
    double n = sqrt(n2), r = p / n2, a = eta * c / n, nw2 = 0.0;
    for (int k = 0; k < d; ++k) {
        xp[k] = x[k] - r * s[k];
        w[k] = mu * s[k] + a * xp[k];
        nw2 += w[k] * w[k];
    }
    if (nw2 == 0.0) { for (int k = 0; k < d; ++k) sb[k] = gb[k]; return; }
    double nw = sqrt(nw2);
    /* s' = w/|w|:  wb = (gb - s'(s'.gb)) / |w| */
    double sg = 0.0;
    for (int k = 0; k < d; ++k) sg += (w[k] / nw) * gb[k];
    for (int k = 0; k < d; ++k) wb[k] = (gb[k] - (w[k] / nw) * sg) / nw;
    /* w = mu s + a x_perp */
    double ab = 0.0, rb = 0.0;
    for (int k = 0; k < d; ++k) {
        *mub += s[k] * wb[k];
        ab += xp[k] * wb[k];
        sb[k] = mu * wb[k];
    }
    /* x_perp = x - r s, with xpb = a wb */
    for (int k = 0; k < d; ++k) {
        double xpb = a * wb[k];
        xb[k] += xpb;
        sb[k] += -r * xpb;
        rb += -s[k] * xpb;
    }
    /* r = p/n2, a = eta c/n, n = sqrt(n2) */
    double pb = rb / n2;
    double n2b = -rb * p / (n2 * n2);
    if (etab) *etab += ab * c / n;
    *cb = ab * eta / n;
    double nb = -ab * eta * c / n2;
    n2b += nb / (2.0 * n);
    /* p = s.x, n2 = s.s */
    for (int k = 0; k < d; ++k) {
        sb[k] += pb * x[k] + 2.0 * n2b * s[k];
        xb[k] += pb * s[k];
    }
}

/* Adjoint of the gates of one slot against its chunk-start state (Eq. 17, eq.
 * beta_chunk; the definitions of oracle_chunk_token_gates2 with nobeta = 0):
 *   h = -x, hh = |h|^2, hdot = h.s0, hhat = hdot/n2, khat = c/sqrt(n2),
 *   tt = khat^2 hh - n2 hhat^2 khat^2, dsq = eta^2 max(tt, 0),
 *   den = mu^2 n2 + dsq, beta = sqrt(n2)/sqrt(den),
 *   g = beta (mu + eta hhat khat), kt = -beta eta khat.
 * gateb = dL/dg and ktb = dL/dkt in; dL/dx and dL/ds0 are added to xb and s0b,
 * dL/dmu and dL/deta to *mub and *etab, dL/dc is stored in *cb. A degenerate token
 * (den = 0) had constant gates. */
static void chunk_gate_slot_bwd(int d, const double *s0, const double *x, double c, double mu,
                                double eta, double gateb, double ktb, double *xb, double *s0b,
                                double *cb, double *mub, double *etab)
{
    double n2 = 0.0, hh = 0.0, hdot = 0.0;
    for (int k = 0; k < d; ++k) {
        n2 += s0[k] * s0[k];
        hh += x[k] * x[k];
        hdot += (-x[k]) * s0[k];
    }
    double hhat = hdot / n2, khat = c / sqrt(n2);
    double tt = khat * khat * hh - n2 * hhat * hhat * khat * khat;
    double dsq = eta * eta * (tt > 0.0 ? tt : 0.0);
    double den = mu * mu * n2 + dsq;
    *cb = 0.0;
    if (den == 0.0) return;
    double beta = sqrt(n2) / sqrt(den);
    /* g = beta (mu + eta hhat khat), kt = -beta eta khat */
    double betab = gateb * (mu + eta * hhat * khat) + ktb * (-eta * khat);
    double mub_ = gateb * beta;
    double etab_ = gateb * beta * hhat * khat + ktb * (-beta * khat);
    double hhatb = gateb * beta * eta * khat;
    double khatb = gateb * beta * eta * hhat + ktb * (-beta * eta);
    /* beta = sqrt(n2) den^(-1/2) */
    double n2b = betab * beta / (2.0 * n2);
    double denb = -0.5 * betab * beta / den;
    /* den = mu^2 n2 + dsq */
    mub_ += denb * 2.0 * mu * n2;
    n2b += denb * mu * mu;
    double dsqb = denb;
    /* dsq = eta^2 max(tt, 0) */
    etab_ += dsqb * 2.0 * eta * (tt > 0.0 ? tt : 0.0);
    double ttb = tt > 0.0 ? dsqb * eta * eta : 0.0;
    /* tt = khat^2 hh - n2 hhat^2 khat^2 */
    khatb += ttb * (2.0 * khat * hh - 2.0 * n2 * hhat * hhat * khat);
    double hhb = ttb * khat * khat;
    n2b += -ttb * hhat * hhat * khat * khat;
    hhatb += -ttb * 2.0 * n2 * hhat * khat * khat;
    /* khat = c n2^(-1/2), hhat = hdot/n2 */
    *cb = khatb / sqrt(n2);
    n2b += -khatb * 0.5 * c / (n2 * sqrt(n2));
    double hdotb = hhatb / n2;
    n2b += -hhatb * hdot / (n2 * n2);
    /* hdot = -x.s0, hh = x.x, n2 = s0.s0 */
    for (int k = 0; k < d; ++k) {
        xb[k] += -hdotb * s0[k] + 2.0 * hhb * x[k];
        s0b[k] += -hdotb * x[k] + 2.0 * n2b * s0[k];
    }
    *mub += mub_;
    if (etab) *etab += etab_;
}

typedef struct {
    int B, T, H, m, d, C, form; /* form 0: exact; 1: chunked (Eq. 17), chunk C */
    const double *x, *c, *q, *mu, *eta, *S0, *dy, *dST;
    double *dx, *dc, *dq, *dmu, *deta, *dS0;
    int next;
    pthread_mutex_t lock;
} bwd_job_t;

/* One (b,h) sequence: the forward keeps every state S_t (t = -1 .. T-1), then
 * the adjoint runs backwards through the tokens. */
static void bwd_sequence(bwd_job_t *J, int b, int h, double *St, double *gb, double *s0b,
                         double *sb, double *g, double *kt, double *tmp)
{
    const int T = J->T, H = J->H, m = J->m, d = J->d, C = J->C;
    const size_t md = (size_t)m * d;
    const size_t so = ((size_t)b * H + h) * md;
    long long deg = 0;
    double *n2 = tmp + 3 * d; /* m doubles */
    memcpy(St, J->S0 + so, sizeof(double) * md);
    for (int t = 0; t < T; ++t) { /* forward, keeping the states */
        size_t tok = IDX_TOK(b, t, h, T, H);
        double eta = J->eta ? J->eta[tok] : 1.0;
        double *S = St + (size_t)(t + 1) * md;
        memcpy(S, St + (size_t)t * md, sizeof(double) * md);
        if (J->form == 0) {
            exact_token(m, d, S, J->x + tok * d, J->c + tok * m, J->q + tok * m, J->mu[tok], eta,
                        NULL, tmp, &deg);
        } else {
            const double *S0c = St + (size_t)((t / C) * C) * md; /* chunk-start state */
            for (int i = 0; i < m; ++i) {
                double a = 0.0;
                for (int k = 0; k < d; ++k) a += S0c[(size_t)i * d + k] * S0c[(size_t)i * d + k];
                n2[i] = a;
            }
            oracle_chunk_token_gates2(m, d, S0c, n2, J->x + tok * d, J->c + tok * m, J->mu[tok], eta,
                                      g, kt, NULL, &deg, NULL, NULL, 0);
            for (int i = 0; i < m; ++i)
                for (int k = 0; k < d; ++k)
                    S[(size_t)i * d + k] = g[i] * S[(size_t)i * d + k] + kt[i] * (-J->x[tok * d + k]);
        }
    }
    /* adjoint; gb = dL/dS_t */
    for (size_t e = 0; e < md; ++e) gb[e] = J->dST ? J->dST[so + e] : 0.0;
    memset(s0b, 0, sizeof(double) * md);
    for (int t = T - 1; t >= 0; --t) {
        size_t tok = IDX_TOK(b, t, h, T, H);
        const double *x = J->x + tok * d, *c = J->c + tok * m, *q = J->q + tok * m;
        const double *dy = J->dy + tok * d;
        const double mu = J->mu[tok], eta = J->eta ? J->eta[tok] : 1.0;
        const double *Sprev = St + (size_t)t * md, *Scur = St + (size_t)(t + 1) * md;
        double *xb = J->dx + tok * d, *cb = J->dc + tok * m, *qb = J->dq + tok * m;
        double mub = 0.0, etab = 0.0;
        for (int k = 0; k < d; ++k) xb[k] = 0.0;
        /* read-out y_t = sum_i q_i s_t,i (Appendix D) */
        for (int i = 0; i < m; ++i) {
            double v = 0.0;
            for (int k = 0; k < d; ++k) {
                v += dy[k] * Scur[(size_t)i * d + k];
                gb[(size_t)i * d + k] += q[i] * dy[k];
            }
            qb[i] = v;
        }
        if (J->form == 0) {
            for (int i = 0; i < m; ++i) {
                exact_slot_bwd(d, Sprev + (size_t)i * d, x, c[i], mu, eta, gb + (size_t)i * d, sb,
                               xb, cb + i, &mub, J->eta ? &etab : NULL, tmp);
                memcpy(gb + (size_t)i * d, sb, sizeof(double) * d);
            }
        } else {
            const int t0 = (t / C) * C;
            const double *S0c = St + (size_t)t0 * md;
            for (int i = 0; i < m; ++i) {
                double a = 0.0;
                for (int k = 0; k < d; ++k) a += S0c[(size_t)i * d + k] * S0c[(size_t)i * d + k];
                n2[i] = a;
            }
            oracle_chunk_token_gates2(m, d, S0c, n2, x, c, mu, eta, g, kt, NULL, &deg, NULL, NULL, 0);
            for (int i = 0; i < m; ++i) {
                /* s_t = g s_{t-1} + kt h, h = -x */
                double *gbi = gb + (size_t)i * d;
                const double *sp = Sprev + (size_t)i * d;
                double gateb = 0.0, ktb = 0.0;
                for (int k = 0; k < d; ++k) {
                    gateb += sp[k] * gbi[k];
                    ktb += (-x[k]) * gbi[k];
                    xb[k] += -kt[i] * gbi[k];
                    gbi[k] *= g[i];
                }
                chunk_gate_slot_bwd(d, S0c + (size_t)i * d, x, c[i], mu, eta, gateb, ktb, xb,
                                    s0b + (size_t)i * d, cb + i, &mub, J->eta ? &etab : NULL);
            }
            if (t == t0) { /* the chunk-start state is also the running state S_{t0-1} */
                for (size_t e = 0; e < md; ++e) { gb[e] += s0b[e]; s0b[e] = 0.0; }
            }
        }
        J->dmu[tok] = mub;
        if (J->deta) J->deta[tok] = etab;
    }
    memcpy(J->dS0 + so, gb, sizeof(double) * md);
}

static void *bwd_worker(void *arg)
{
    bwd_job_t *J = (bwd_job_t *)arg;
    const size_t md = (size_t)J->m * J->d;
    double *St = malloc(sizeof(double) * md * (size_t)(J->T + 1));
    double *gb = malloc(sizeof(double) * md), *s0b = malloc(sizeof(double) * md);
    double *sb = malloc(sizeof(double) * (size_t)J->d);
    double *g = malloc(sizeof(double) * (size_t)J->m), *kt = malloc(sizeof(double) * (size_t)J->m);
    double *tmp = malloc(sizeof(double) * (size_t)(3 * J->d + J->m));
    for (;;) {
        pthread_mutex_lock(&J->lock);
        int item = J->next++;
        pthread_mutex_unlock(&J->lock);
        if (item >= J->B * J->H) break;
        bwd_sequence(J, item / J->H, item % J->H, St, gb, s0b, sb, g, kt, tmp);
    }
    free(St); free(gb); free(s0b); free(sb); free(g); free(kt); free(tmp);
    return NULL;
}

/* Gradients of L = sum_t dy_t . y_t + dST . S_T (dST may be NULL: zero) with
 * respect to every input of the similarity-objective scan: form 0, the exact
 * recurrence; form 1, the chunked recurrence of Eq. 17 with chunk size C.
 * Outputs have the layouts of the inputs; deta may be NULL (and is not written
 * when eta is NULL, i.e. eta = 1). */
void oracle_scan_bwd(int form, int B, int T, int H, int m, int d, int C, const double *x,
                     const double *c, const double *q, const double *mu, const double *eta,
                     const double *S0, const double *dy, const double *dST, double *dx,
                     double *dc, double *dq, double *dmu, double *deta, double *dS0, int nthreads)
{
    bwd_job_t J;
    memset(&J, 0, sizeof(J));
    J.B = B; J.T = T; J.H = H; J.m = m; J.d = d; J.C = C > 0 ? C : 1; J.form = form;
    J.x = x; J.c = c; J.q = q; J.mu = mu; J.eta = eta; J.S0 = S0; J.dy = dy; J.dST = dST;
    J.dx = dx; J.dc = dc; J.dq = dq; J.dmu = dmu; J.deta = eta ? deta : NULL; J.dS0 = dS0;
    pthread_mutex_init(&J.lock, NULL);
    if (nthreads < 1) nthreads = 1;
    if (nthreads > B * H) nthreads = B * H;
    if (nthreads <= 1) {
        bwd_worker(&J);
    } else {
        pthread_t *th = malloc(sizeof(pthread_t) * (size_t)nthreads);
        for (int i = 0; i < nthreads; ++i) pthread_create(&th[i], NULL, bwd_worker, &J);
        for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
        free(th);
    }
    pthread_mutex_destroy(&J.lock);
}
