/*
 * kta_oracle.c -- plain fp64 CPU oracle for the Hybrid Linear Temporal Attention operator.
 *
 * TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the CPU-baseline leg of the
 * benchmark load this file's library. The CUDA product path never links, loads or calls it,
 * and this file includes nothing from the CUDA path.
 *
 * Source pages (cited by title and section):
 *   [K1] paper-read "Kairos: A Native World Model Stack for Physical AI" (yingwang.github.io),
 *        section 2 "Method", second pillar (hybrid linear temporal attention): the SWA, DSWA
 *        and GLA paragraphs and the four gated delta-rule equations that follow them.
 *   [K2] ai-papers.net summary of Kairos, section "3-layer hybrid temporal architecture".
 *
 * Each function evaluates its definition directly:
 *   - softmax branches: every key s < N is tested with the visibility predicate by brute force,
 *     scores are fp64 dot products, and softmax subtracts the row maximum;
 *   - GLA: the per-token recurrence, one token at a time, with an fp64 d x d state;
 *   - gated delta rule: the four recurrence lines in the order the page gives them.
 * No blocking, chunking or reordering beyond that. Inputs are the stored values (bf16 or fp32)
 * passed as float and widened to double on read; every sum is taken in double.
 *
 * Layouts (row-major): q, k, v, o are [B][N][H][d] (token-major, heads interleaved, the
 * page's (B, F*L, D) with D = H*d). Heads h0 <= h < h1 are computed; other heads of o are left
 * untouched. Gates cover only the computed heads: vector alpha [B][N][h1-h0][d]; scalar alpha
 * and beta [B][N][h1-h0]. States S0 / S_out are [B][h1-h0][d][d], stored key-major:
 * S[i][j] with i over the key dimension and j over the value dimension.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <omp.h>

#define IDX4(b, n, h, c, N, H, D) ((((int64_t)(b) * (N) + (n)) * (H) + (h)) * (D) + (c))

static int g_threads = 0;

void oracle_set_threads(int n) { g_threads = n; }

int oracle_get_threads(void) {
    return g_threads > 0 ? g_threads : omp_get_max_threads();
}

/* [K1] SWA paragraph: standard attention inside a window of L x window_size tokens, L being
 * the tokens of one frame. Reading: the window is W whole frames ending at the query's own
 * frame (the own frame is fully visible, no later frame is). */
static int swa_visible(int64_t t, int64_t s, int64_t P, int64_t W) {
    int64_t ft = t / P, fs = s / P;
    return fs <= ft && fs > ft - W;
}

/* [K1] DSWA paragraph: the same window size as SWA, but frames taken every dil-th step back
 * from the query frame: frames ft, ft-dil, ..., ft-(W-1)*dil. */
static int dswa_visible(int64_t t, int64_t s, int64_t P, int64_t W, int64_t dil) {
    int64_t ft = t / P, fs = s / P;
    if (fs > ft) return 0;
    int64_t gap = ft - fs;
    return (gap % dil) == 0 && (gap / dil) < W;
}

/* One softmax-attention output row o[b, t, h, :] over the keys that vis() admits. */
static void softmax_row(const float* q, const float* k, const float* v, double* o,
                        int64_t B, int64_t N, int64_t H, int64_t d,
                        int64_t b, int64_t h, int64_t t, int64_t P, int64_t W, int64_t dil,
                        int dilated, double scale, double* score, double* acc) {
    (void)B;
    const float* qt = q + IDX4(b, t, h, 0, N, H, d);
    double mx = -INFINITY;
    for (int64_t s = 0; s < N; ++s) {
        int vis = dilated ? dswa_visible(t, s, P, W, dil) : swa_visible(t, s, P, W);
        if (!vis) { score[s] = NAN; continue; }
        const float* ks = k + IDX4(b, s, h, 0, N, H, d);
        double dot = 0.0;
        for (int64_t c = 0; c < d; ++c) dot += (double)qt[c] * (double)ks[c];
        score[s] = scale * dot;
        if (score[s] > mx) mx = score[s];
    }
    double denom = 0.0;
    for (int64_t c = 0; c < d; ++c) acc[c] = 0.0;
    for (int64_t s = 0; s < N; ++s) {
        if (isnan(score[s])) continue;
        double p = exp(score[s] - mx);
        denom += p;
        const float* vs = v + IDX4(b, s, h, 0, N, H, d);
        for (int64_t c = 0; c < d; ++c) acc[c] += p * (double)vs[c];
    }
    double* ot = o + IDX4(b, t, h, 0, N, H, d);
    for (int64_t c = 0; c < d; ++c) ot[c] = acc[c] / denom;
}

static int softmax_branch(const float* q, const float* k, const float* v, double* o,
                          int B, int N, int H, int d, int h0, int h1,
                          int P, int W, int dil, int dilated, double scale,
                          const int64_t* rows, int64_t nrows) {
    if (B < 1 || N < 1 || H < 1 || d < 1 || P < 1 || W < 1 || dil < 1) return 1;
    if (h0 < 0 || h1 > H || h0 >= h1) return 1;
    int64_t nr = rows ? nrows : (int64_t)N;
    int64_t nh = h1 - h0;
    int64_t total = (int64_t)B * nh * nr;
    int nt = oracle_get_threads();
#pragma omp parallel num_threads(nt)
    {
        double* score = (double*)malloc(sizeof(double) * (size_t)N);
        double* acc = (double*)malloc(sizeof(double) * (size_t)d);
#pragma omp for schedule(dynamic, 4)
        for (int64_t w = 0; w < total; ++w) {
            int64_t r = w % nr;
            int64_t h = h0 + (w / nr) % nh;
            int64_t b = w / (nr * nh);
            int64_t t = rows ? rows[r] : r;
            if (t < 0 || t >= N) continue;
            softmax_row(q, k, v, o, B, N, H, d, b, h, t, P, W, dil, dilated, scale, score, acc);
        }
        free(score);
        free(acc);
    }
    return 0;
}

int oracle_swa(const float* q, const float* k, const float* v, double* o,
               int B, int N, int H, int d, int h0, int h1,
               int P, int W, double scale, const int64_t* rows, int64_t nrows) {
    return softmax_branch(q, k, v, o, B, N, H, d, h0, h1, P, W, 1, 0, scale, rows, nrows);
}

int oracle_dswa(const float* q, const float* k, const float* v, double* o,
                int B, int N, int H, int d, int h0, int h1,
                int P, int W, int dil, double scale, const int64_t* rows, int64_t nrows) {
    return softmax_branch(q, k, v, o, B, N, H, d, h0, h1, P, W, dil, 1, scale, rows, nrows);
}

/* Visibility predicates exported for the mask tests: out[i] = visible(t[i], s[i]). */
void oracle_visible(const int64_t* t, const int64_t* s, int64_t n, int P, int W, int dil,
                    int dilated, uint8_t* out) {
    for (int64_t i = 0; i < n; ++i)
        out[i] = (uint8_t)(dilated ? dswa_visible(t[i], s[i], P, W, dil)
                                   : swa_visible(t[i], s[i], P, W));
}

/* GLA with a vector forget gate, one token at a time (the form S_t = diag(alpha_t) S_{t-1}
 * + k_t^T v_t, o_t = scale * q_t S_t; row convention, S is d_k x d_v). [K1] GLA paragraph
 * gives the gated state update; the per-key-dimension gate is the configs' reading. */
int oracle_gla(const float* q, const float* k, const float* v, const float* alpha,
               const double* S0, double* o, double* S_out,
               int B, int N, int H, int d, int h0, int h1, double scale) {
    if (B < 1 || N < 0 || H < 1 || d < 1 || h0 < 0 || h1 > H || h0 >= h1) return 1;
    int64_t nh = h1 - h0;
    int nt = oracle_get_threads();
#pragma omp parallel for num_threads(nt) schedule(dynamic, 1)
    for (int64_t w = 0; w < (int64_t)B * nh; ++w) {
        int64_t b = w / nh, hg = w % nh, h = h0 + hg;
        double* S = (double*)malloc(sizeof(double) * (size_t)d * (size_t)d);
        if (S0) memcpy(S, S0 + w * d * d, sizeof(double) * (size_t)d * (size_t)d);
        else memset(S, 0, sizeof(double) * (size_t)d * (size_t)d);
        for (int64_t t = 0; t < N; ++t) {
            const float* qt = q + IDX4(b, t, h, 0, N, H, d);
            const float* kt = k + IDX4(b, t, h, 0, N, H, d);
            const float* vt = v + IDX4(b, t, h, 0, N, H, d);
            const float* at = alpha + IDX4(b, t, hg, 0, N, nh, d);
            for (int64_t i = 0; i < d; ++i)
                for (int64_t j = 0; j < d; ++j)
                    S[i * d + j] = (double)at[i] * S[i * d + j] + (double)kt[i] * (double)vt[j];
            double* ot = o + IDX4(b, t, h, 0, N, H, d);
            for (int64_t j = 0; j < d; ++j) {
                double acc = 0.0;
                for (int64_t i = 0; i < d; ++i) acc += (double)qt[i] * S[i * d + j];
                ot[j] = scale * acc;
            }
        }
        if (S_out) memcpy(S_out + w * d * d, S, sizeof(double) * (size_t)d * (size_t)d);
        free(S);
    }
    return 0;
}

/* Gated delta rule, the four lines of [K1] in the page's column convention (its state M is
 * d_v x d_k; here M[j][i] is held as S[i][j]):
 *   v_old = M_{t-1} k_t
 *   v_new = beta_t v_t + (1 - beta_t) v_old
 *   M_t   = alpha_t M_{t-1} - v_old k_t^T + v_new k_t^T
 *   o_t   = scale * M_t q_t
 * alpha_t and beta_t are scalars per token and head. erase_decayed selects the other reading of
 * the same paragraph, which says the branch is based on GatedDeltaNet: GatedDeltaNet's own update
 * decays the erase term too,
 *   M_t   = alpha_t M_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
 * i.e. alpha_t (M_{t-1} - beta_t v_old k_t^T) + beta_t v_t k_t^T. */
int oracle_delta(const float* q, const float* k, const float* v,
                 const float* alpha, const float* beta, const double* S0,
                 double* o, double* S_out,
                 int B, int N, int H, int d, int h0, int h1, double scale, int erase_decayed) {
    if (B < 1 || N < 0 || H < 1 || d < 1 || h0 < 0 || h1 > H || h0 >= h1) return 1;
    int64_t nh = h1 - h0;
    int nt = oracle_get_threads();
#pragma omp parallel for num_threads(nt) schedule(dynamic, 1)
    for (int64_t w = 0; w < (int64_t)B * nh; ++w) {
        int64_t b = w / nh, hg = w % nh, h = h0 + hg;
        double* S = (double*)malloc(sizeof(double) * (size_t)d * (size_t)d);
        double* vold = (double*)malloc(sizeof(double) * (size_t)d);
        double* vnew = (double*)malloc(sizeof(double) * (size_t)d);
        if (S0) memcpy(S, S0 + w * d * d, sizeof(double) * (size_t)d * (size_t)d);
        else memset(S, 0, sizeof(double) * (size_t)d * (size_t)d);
        for (int64_t t = 0; t < N; ++t) {
            const float* qt = q + IDX4(b, t, h, 0, N, H, d);
            const float* kt = k + IDX4(b, t, h, 0, N, H, d);
            const float* vt = v + IDX4(b, t, h, 0, N, H, d);
            double a = (double)alpha[((int64_t)b * N + t) * nh + hg];
            double be = (double)beta[((int64_t)b * N + t) * nh + hg];
            for (int64_t j = 0; j < d; ++j) {
                double acc = 0.0;
                for (int64_t i = 0; i < d; ++i) acc += S[i * d + j] * (double)kt[i];
                vold[j] = acc;
            }
            if (!erase_decayed) {
                /* the page's four lines: v_new = beta v + (1 - beta) v_old,
                   M = alpha M - v_old k^T + v_new k^T */
                for (int64_t j = 0; j < d; ++j) vnew[j] = be * (double)vt[j] + (1.0 - be) * vold[j];
                for (int64_t i = 0; i < d; ++i)
                    for (int64_t j = 0; j < d; ++j)
                        S[i * d + j] = a * S[i * d + j] - vold[j] * (double)kt[i] + vnew[j] * (double)kt[i];
            } else {
                /* decayed erase (the GatedDeltaNet form): M = alpha M (I - beta k k^T) + beta v k^T,
                   where M k = v_old is read from the undecayed state */
                for (int64_t i = 0; i < d; ++i)
                    for (int64_t j = 0; j < d; ++j)
                        S[i * d + j] = a * (S[i * d + j] - be * vold[j] * (double)kt[i])
                                       + be * (double)vt[j] * (double)kt[i];
            }
            double* ot = o + IDX4(b, t, h, 0, N, H, d);
            for (int64_t j = 0; j < d; ++j) {
                double acc = 0.0;
                for (int64_t i = 0; i < d; ++i) acc += S[i * d + j] * (double)qt[i];
                ot[j] = scale * acc;
            }
        }
        if (S_out) memcpy(S_out + w * d * d, S, sizeof(double) * (size_t)d * (size_t)d);
        free(S);
        free(vold);
        free(vnew);
    }
    return 0;
}

/* ------------------------------------------------------------------------------ backward
 * Reverse mode of the operators above: given dO, the gradients of L = sum(dO * O) with respect
 * to q, k, v and the gates, written out from the chain rule of each forward definition. Only the
 * head range [h0, h1) of the gradient arrays is written (zeroed first). */

static void zero_heads(double* x, int B, int N, int H, int d, int h0, int h1) {
    for (int64_t b = 0; b < B; ++b)
        for (int64_t t = 0; t < N; ++t)
            memset(x + IDX4(b, t, h0, 0, N, H, d), 0, sizeof(double) * (size_t)(h1 - h0) * (size_t)d);
}

/* Softmax branches: with p_ts = softmax_s(scale q_t . k_s) over the visible keys and
 * o_t = sum_s p_ts v_s: dp_ts = dO_t . v_s, ds_ts = p_ts (dp_ts - dO_t . o_t),
 * dq_t = scale sum_s ds_ts k_s, dk_s = scale sum_t ds_ts q_t, dv_s = sum_t p_ts dO_t. */
int oracle_softmax_bwd(const float* q, const float* k, const float* v, const double* dout,
                       double* dq, double* dk, double* dv,
                       int B, int N, int H, int d, int h0, int h1, int P, int W, int dil,
                       int dilated, double scale) {
    if (B < 1 || N < 0 || H < 1 || d < 1 || h0 < 0 || h1 > H || h0 >= h1 || P < 1 || W < 1 ||
        dil < 1)
        return 1;
    zero_heads(dq, B, N, H, d, h0, h1);
    zero_heads(dk, B, N, H, d, h0, h1);
    zero_heads(dv, B, N, H, d, h0, h1);
    int64_t nh = h1 - h0;
    int nt = oracle_get_threads();
#pragma omp parallel for num_threads(nt) schedule(dynamic, 1)
    for (int64_t w = 0; w < (int64_t)B * nh; ++w) {
        int64_t b = w / nh, h = h0 + w % nh;
        double* lg = (double*)malloc(sizeof(double) * (size_t)N);
        double* o = (double*)malloc(sizeof(double) * (size_t)d);
        for (int64_t t = 0; t < N; ++t) {
            const float* qt = q + IDX4(b, t, h, 0, N, H, d);
            const double* dot = dout + IDX4(b, t, h, 0, N, H, d);
            double m = -INFINITY;
            for (int64_t s = 0; s < N; ++s) {
                int vis = dilated ? dswa_visible(t, s, P, W, dil) : swa_visible(t, s, P, W);
                if (!vis) { lg[s] = -INFINITY; continue; }
                const float* ks = k + IDX4(b, s, h, 0, N, H, d);
                double acc = 0.0;
                for (int64_t i = 0; i < d; ++i) acc += (double)qt[i] * (double)ks[i];
                lg[s] = scale * acc;
                if (lg[s] > m) m = lg[s];
            }
            double den = 0.0;
            for (int64_t s = 0; s < N; ++s) {
                lg[s] = lg[s] == -INFINITY ? 0.0 : exp(lg[s] - m);
                den += lg[s];
            }
            for (int64_t j = 0; j < d; ++j) o[j] = 0.0;
            for (int64_t s = 0; s < N; ++s) {
                if (lg[s] == 0.0) continue;
                lg[s] /= den;  /* p_ts */
                const float* vs = v + IDX4(b, s, h, 0, N, H, d);
                for (int64_t j = 0; j < d; ++j) o[j] += lg[s] * (double)vs[j];
            }
            double dD = 0.0;
            for (int64_t j = 0; j < d; ++j) dD += dot[j] * o[j];
            double* dqt = dq + IDX4(b, t, h, 0, N, H, d);
            for (int64_t s = 0; s < N; ++s) {
                if (lg[s] == 0.0) continue;
                const float* ks = k + IDX4(b, s, h, 0, N, H, d);
                const float* vs = v + IDX4(b, s, h, 0, N, H, d);
                double dp = 0.0;
                for (int64_t j = 0; j < d; ++j) dp += dot[j] * (double)vs[j];
                double ds = lg[s] * (dp - dD);
                double* dks = dk + IDX4(b, s, h, 0, N, H, d);
                double* dvs = dv + IDX4(b, s, h, 0, N, H, d);
                for (int64_t i = 0; i < d; ++i) {
                    dqt[i] += scale * ds * (double)ks[i];
                    dks[i] += scale * ds * (double)qt[i];
                    dvs[i] += lg[s] * dot[i];
                }
            }
        }
        free(lg);
        free(o);
    }
    return 0;
}

/* GLA (vector gate). With G_t = dL/dS_t = scale q_t^T dO_t + diag(alpha_{t+1}) G_{t+1}:
 * dq_t = scale S_t dO_t^T, dk_t = G_t v_t^T, dv_t = k_t G_t, dalpha_t[i] = sum_j G_t[i][j]
 * S_{t-1}[i][j], and dS_0 = diag(alpha_1) G_1. States are kept from a forward pass. */
int oracle_gla_bwd(const float* q, const float* k, const float* v, const float* alpha,
                   const double* S0, const double* dout, double* dq, double* dk, double* dv,
                   double* dalpha, double* dS0, int B, int N, int H, int d, int h0, int h1,
                   double scale) {
    if (B < 1 || N < 0 || H < 1 || d < 1 || h0 < 0 || h1 > H || h0 >= h1) return 1;
    zero_heads(dq, B, N, H, d, h0, h1);
    zero_heads(dk, B, N, H, d, h0, h1);
    zero_heads(dv, B, N, H, d, h0, h1);
    int64_t nh = h1 - h0, dd = (int64_t)d * d;
    int nt = oracle_get_threads();
#pragma omp parallel for num_threads(nt) schedule(dynamic, 1)
    for (int64_t w = 0; w < (int64_t)B * nh; ++w) {
        int64_t b = w / nh, hg = w % nh, h = h0 + hg;
        double* S = (double*)malloc(sizeof(double) * (size_t)((N + 1) * dd));  /* S_0 .. S_N */
        double* G = (double*)calloc((size_t)dd, sizeof(double));
        if (S0) memcpy(S, S0 + w * dd, sizeof(double) * (size_t)dd);
        else memset(S, 0, sizeof(double) * (size_t)dd);
        for (int64_t t = 0; t < N; ++t) {
            const float* kt = k + IDX4(b, t, h, 0, N, H, d);
            const float* vt = v + IDX4(b, t, h, 0, N, H, d);
            const float* at = alpha + IDX4(b, t, hg, 0, N, nh, d);
            const double* Sp = S + t * dd;
            double* Sn = S + (t + 1) * dd;
            for (int64_t i = 0; i < d; ++i)
                for (int64_t j = 0; j < d; ++j)
                    Sn[i * d + j] = (double)at[i] * Sp[i * d + j] + (double)kt[i] * (double)vt[j];
        }
        for (int64_t t = N - 1; t >= 0; --t) {
            const float* qt = q + IDX4(b, t, h, 0, N, H, d);
            const float* kt = k + IDX4(b, t, h, 0, N, H, d);
            const float* vt = v + IDX4(b, t, h, 0, N, H, d);
            const float* at = alpha + IDX4(b, t, hg, 0, N, nh, d);
            const double* dot = dout + IDX4(b, t, h, 0, N, H, d);
            const double* St = S + (t + 1) * dd;
            const double* Sp = S + t * dd;
            for (int64_t i = 0; i < d; ++i)
                for (int64_t j = 0; j < d; ++j) G[i * d + j] += scale * (double)qt[i] * dot[j];
            double* dqt = dq + IDX4(b, t, h, 0, N, H, d);
            double* dkt = dk + IDX4(b, t, h, 0, N, H, d);
            double* dvt = dv + IDX4(b, t, h, 0, N, H, d);
            double* dat = dalpha + IDX4(b, t, hg, 0, N, nh, d);
            for (int64_t i = 0; i < d; ++i) {
                double aq = 0.0, ak = 0.0, aa = 0.0;
                for (int64_t j = 0; j < d; ++j) {
                    aq += St[i * d + j] * dot[j];
                    ak += G[i * d + j] * (double)vt[j];
                    aa += G[i * d + j] * Sp[i * d + j];
                }
                dqt[i] = scale * aq;
                dkt[i] = ak;
                dat[i] = aa;
            }
            for (int64_t j = 0; j < d; ++j) {
                double acc = 0.0;
                for (int64_t i = 0; i < d; ++i) acc += (double)kt[i] * G[i * d + j];
                dvt[j] = acc;
            }
            for (int64_t i = 0; i < d; ++i)
                for (int64_t j = 0; j < d; ++j) G[i * d + j] *= (double)at[i];
        }
        if (dS0) memcpy(dS0 + w * dd, G, sizeof(double) * (size_t)dd);
        free(S);
        free(G);
    }
    return 0;
}

/* Gated delta rule (row convention: w_t = k_t S_{t-1}, u_t = beta_t (v_t - a_t w_t) with a_t = 1
 * for the page's form and a_t = alpha_t for the decayed erase, S_t = alpha_t S_{t-1} + k_t^T u_t,
 * o_t = scale q_t S_t). With G_t = dL/dS_t = scale q_t^T dO_t + [propagated from t+1] and
 * du_t = k_t G_t:
 *   dq_t = scale S_t dO_t^T,   dv_t = beta_t du_t,   dbeta_t = du_t . (v_t - a_t w_t),
 *   dk_t = G_t u_t^T - beta_t a_t S_{t-1} du_t^T,
 *   dalpha_t = <G_t, S_{t-1}> (- beta_t du_t . w_t for the decayed erase),
 *   G_{t-1} = alpha_t G_t - beta_t a_t k_t^T du_t. */
int oracle_delta_bwd(const float* q, const float* k, const float* v, const float* alpha,
                     const float* beta, const double* S0, const double* dout, double* dq,
                     double* dk, double* dv, double* dalpha, double* dbeta, double* dS0,
                     int B, int N, int H, int d, int h0, int h1, double scale, int erase_decayed) {
    if (B < 1 || N < 0 || H < 1 || d < 1 || h0 < 0 || h1 > H || h0 >= h1) return 1;
    zero_heads(dq, B, N, H, d, h0, h1);
    zero_heads(dk, B, N, H, d, h0, h1);
    zero_heads(dv, B, N, H, d, h0, h1);
    int64_t nh = h1 - h0, dd = (int64_t)d * d;
    int nt = oracle_get_threads();
#pragma omp parallel for num_threads(nt) schedule(dynamic, 1)
    for (int64_t w = 0; w < (int64_t)B * nh; ++w) {
        int64_t b = w / nh, hg = w % nh, h = h0 + hg;
        double* S = (double*)malloc(sizeof(double) * (size_t)((N + 1) * dd));
        double* U = (double*)malloc(sizeof(double) * (size_t)(N * d + 1));
        double* Wr = (double*)malloc(sizeof(double) * (size_t)(N * d + 1));
        double* G = (double*)calloc((size_t)dd, sizeof(double));
        double* du = (double*)malloc(sizeof(double) * (size_t)d);
        if (S0) memcpy(S, S0 + w * dd, sizeof(double) * (size_t)dd);
        else memset(S, 0, sizeof(double) * (size_t)dd);
        for (int64_t t = 0; t < N; ++t) {
            const float* kt = k + IDX4(b, t, h, 0, N, H, d);
            const float* vt = v + IDX4(b, t, h, 0, N, H, d);
            double a = (double)alpha[((int64_t)b * N + t) * nh + hg];
            double be = (double)beta[((int64_t)b * N + t) * nh + hg];
            double ae = erase_decayed ? a : 1.0;
            const double* Sp = S + t * dd;
            double* Sn = S + (t + 1) * dd;
            for (int64_t j = 0; j < d; ++j) {
                double acc = 0.0;
                for (int64_t i = 0; i < d; ++i) acc += (double)kt[i] * Sp[i * d + j];
                Wr[t * d + j] = acc;
                U[t * d + j] = be * ((double)vt[j] - ae * acc);
            }
            for (int64_t i = 0; i < d; ++i)
                for (int64_t j = 0; j < d; ++j)
                    Sn[i * d + j] = a * Sp[i * d + j] + (double)kt[i] * U[t * d + j];
        }
        for (int64_t t = N - 1; t >= 0; --t) {
            const float* qt = q + IDX4(b, t, h, 0, N, H, d);
            const float* kt = k + IDX4(b, t, h, 0, N, H, d);
            const float* vt = v + IDX4(b, t, h, 0, N, H, d);
            const double* dot = dout + IDX4(b, t, h, 0, N, H, d);
            double a = (double)alpha[((int64_t)b * N + t) * nh + hg];
            double be = (double)beta[((int64_t)b * N + t) * nh + hg];
            double ae = erase_decayed ? a : 1.0;
            const double* St = S + (t + 1) * dd;
            const double* Sp = S + t * dd;
            for (int64_t i = 0; i < d; ++i)
                for (int64_t j = 0; j < d; ++j) G[i * d + j] += scale * (double)qt[i] * dot[j];
            for (int64_t j = 0; j < d; ++j) {
                double acc = 0.0;
                for (int64_t i = 0; i < d; ++i) acc += (double)kt[i] * G[i * d + j];
                du[j] = acc;
            }
            double* dqt = dq + IDX4(b, t, h, 0, N, H, d);
            double* dkt = dk + IDX4(b, t, h, 0, N, H, d);
            double* dvt = dv + IDX4(b, t, h, 0, N, H, d);
            double da = 0.0, db = 0.0;
            for (int64_t i = 0; i < d; ++i) {
                double aq = 0.0, ak = 0.0, as = 0.0;
                for (int64_t j = 0; j < d; ++j) {
                    aq += St[i * d + j] * dot[j];
                    ak += G[i * d + j] * U[t * d + j];
                    as += Sp[i * d + j] * du[j];
                    da += G[i * d + j] * Sp[i * d + j];
                }
                dqt[i] = scale * aq;
                dkt[i] = ak - be * ae * as;
            }
            for (int64_t j = 0; j < d; ++j) {
                dvt[j] = be * du[j];
                db += du[j] * ((double)vt[j] - ae * Wr[t * d + j]);
                if (erase_decayed) da -= be * du[j] * Wr[t * d + j];
            }
            dalpha[((int64_t)b * N + t) * nh + hg] = da;
            dbeta[((int64_t)b * N + t) * nh + hg] = db;
            for (int64_t i = 0; i < d; ++i)
                for (int64_t j = 0; j < d; ++j)
                    G[i * d + j] = a * G[i * d + j] - be * ae * (double)kt[i] * du[j];
        }
        if (dS0) memcpy(dS0 + w * dd, G, sizeof(double) * (size_t)dd);
        free(S);
        free(U);
        free(Wr);
        free(G);
        free(du);
    }
    return 0;
}

/* ----------------------------------------------------------------------------- projections
 * paper-read, section 2, second pillar, GLA paragraph: q_t = W_Q x_t, k_t = W_K x_t,
 * v_t = W_V x_t and beta_t = sigmoid(W_beta x_t); the forget gate alpha_t is likewise a sigmoid
 * of a projection of x_t. With every weight stacked as the rows of one matrix w [N][K], row r of
 * the result is y[r][n] = sum_k x[r][k] w[n][k] (+ bias[n] when a bias is given: the caller's
 * gate offset, not a page term); columns in [sig_c0, sig_c1) then pass through the logistic
 * sigmoid 1 / (1 + exp(-y)). rows (nrows entries) selects which rows of x to
 * compute, NULL = all M rows; y holds one output row per selected row. */
int oracle_proj(const float* x, const float* w, const float* bias, int64_t M, int64_t N, int64_t K,
                const int64_t* rows, int64_t nrows, int64_t sig_c0, int64_t sig_c1, double* y) {
  if (!x || !w || !y || M < 1 || N < 1 || K < 1) return 1;
  const int64_t R = rows ? nrows : M;
  for (int64_t i = 0; i < R; ++i)
    if (rows && (rows[i] < 0 || rows[i] >= M)) return 1;
#pragma omp parallel for schedule(static) num_threads(oracle_get_threads())
  for (int64_t i = 0; i < R; ++i) {
    const float* xr = x + (rows ? rows[i] : i) * K;
    for (int64_t n = 0; n < N; ++n) {
      const float* wr = w + n * K;
      double acc = 0.0;
      for (int64_t c = 0; c < K; ++c) acc += (double)xr[c] * (double)wr[c];
      if (bias) acc += (double)bias[n];
      if (n >= sig_c0 && n < sig_c1) acc = 1.0 / (1.0 + exp(-acc));
      y[i * N + n] = acc;
    }
  }
  return 0;
}
