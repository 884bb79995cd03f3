/*
 * CPU oracle for windowed INT8 recurrent-state decode of gated delta-rule
 * linear attention (LeapQuant, arXiv 2609.38166).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, loads or
 * calls this file; only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg do.  It shares no code, header, table or constant with the
 * CUDA path.
 *
 * It is deliberately plain and slow: one head at a time, a dense FP64 state,
 * the recurrence written as the explicit matrix product of its definition
 * (O(d^3) per token), and the state codec written step by step.  Every
 * function names the passage it follows.  Sources:
 *   [abs]  "LeapQuant: Efficient Linear Attention with Accurate Recurrent State
 *          Quantization" (mlsanity.com paper page), section "Abstract (arXiv)":
 *          per-window quantization that quantizes the state once, at the end
 *          of a window; outputs taken from the fixed low-bit state plus
 *          high-precision buffered updates; the largest outliers kept as
 *          Compensator Tokens on the update path of real tokens; smoothing of
 *          the residual before quantization; an 8-bit state.
 *   [news] bedrocknews.com article on arXiv 2609.38166v1, mechanism paragraph:
 *          outlier rows and columns kept in FP16/FP32; the comparison with
 *          naive per-token quantization; FP32 inference as the baseline.
 * The pages print no formula.  The update rules are the published Gated
 * DeltaNet and Kimi Delta Attention recurrences; the per-row INT8 grain, the
 * smoothing factor s_j = sqrt(max_i |R_ij|) and the rank-1 FP32 (v,k) form of
 * the compensators are this library's specification of the method.  Readings
 * taken where the pages are silent are marked at each step below.
 *
 * Parity pins (tests/test_oracle_pins.py) check this file against properties
 * fixed by the mathematics, not against itself: the delta-rule write and
 * orthogonal-complement identities, closed forms, a hand-derived codec
 * example, the codec round-trip bound and the error bound of the windowed
 * scheme.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { LQO_GATE_SCALAR = 0, LQO_GATE_CHANNEL = 1 };
enum { LQO_MODE_WINDOW = 0, LQO_MODE_NAIVE = 1, LQO_MODE_FP32 = 2 };
enum { LQO_SELECT_L2 = 0, LQO_SELECT_MAXABS = 1 };

typedef struct {
    int32_t d_k, d_v;          /* key / value channels: S is d_v x d_k        */
    int32_t window;            /* W: tokens between two quantizations         */
    int32_t n_comp_rows;       /* compensator rows   (ceil(n_c/2) by default) */
    int32_t n_comp_cols;       /* compensator columns (floor(n_c/2))          */
    int32_t gate;              /* LQO_GATE_SCALAR (GDN) | LQO_GATE_CHANNEL (KDA) */
    int32_t mode;              /* LQO_MODE_WINDOW | LQO_MODE_NAIVE | LQO_MODE_FP32 */
    int32_t smooth;            /* 1: per-column smoothing before quantization */
    int32_t select;            /* LQO_SELECT_L2 | LQO_SELECT_MAXABS           */
} lqo_params;

/*
 * One token of the gated delta rule, dense, in FP64.
 *   GDN  (Gated DeltaNet, named in [abs]):
 *        S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
 *   KDA  (Kimi Delta Attention, named in [abs]); reading: the per-key-channel
 *        gate multiplies the key side before the delta step,
 *        S_t = S_{t-1} diag(alpha_t) (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
 *   output o_t = S_t q_t.
 * The gate arrives as its logarithm g = log(alpha) (one value for GDN, d_k for
 * KDA).  The transition matrix A_t is formed explicitly and multiplied in, so
 * the code reads as the definition.
 */
void lqo_step(const lqo_params *p, double *S, const double *q, const double *k,
              const double *v, const double *g, double beta, double *o)
{
    const int dk = p->d_k, dv = p->d_v;
    double *A = (double *)malloc(sizeof(double) * dk * dk);
    double *Sn = (double *)malloc(sizeof(double) * dv * dk);

    /* A_t = diag(alpha) (I - beta k k^T); for GDN diag(alpha) = alpha I. */
    for (int m = 0; m < dk; ++m) {
        double alpha_m = exp(p->gate == LQO_GATE_SCALAR ? g[0] : g[m]);
        for (int j = 0; j < dk; ++j) {
            double eye = (m == j) ? 1.0 : 0.0;
            A[m * dk + j] = alpha_m * (eye - beta * k[m] * k[j]);
        }
    }
    /* S_t = S_{t-1} A_t + beta v k^T */
    for (int i = 0; i < dv; ++i) {
        for (int j = 0; j < dk; ++j) {
            double acc = 0.0;
            for (int m = 0; m < dk; ++m)
                acc += S[i * dk + m] * A[m * dk + j];
            Sn[i * dk + j] = acc + beta * v[i] * k[j];
        }
    }
    memcpy(S, Sn, sizeof(double) * dv * dk);
    /* o_t = S_t q_t */
    if (o) {
        for (int i = 0; i < dv; ++i) {
            double acc = 0.0;
            for (int j = 0; j < dk; ++j)
                acc += S[i * dk + j] * q[j];
            o[i] = acc;
        }
    }
    free(A);
    free(Sn);
}

/* Index of the largest score among those not yet taken; ties go to the lower
 * index (strict comparison while scanning upwards). */
static int argmax_free(const float *score, const unsigned char *taken, int n)
{
    int best = -1;
    for (int i = 0; i < n; ++i) {
        if (taken[i]) continue;
        if (best < 0 || score[i] > score[best]) best = i;
    }
    return best;
}

/*
 * The state codec, applied once per window, at its end ([abs]: the state is
 * quantized a single time per window), and once to the prefilled state.
 *
 * Input:  S, the dense FP64 state (d_v x d_k, row-major, d_k contiguous).
 * Output: the stored window-start state and, in place of S, its decoded value
 *         S~ = R^ + C that the next window starts from.
 *
 * All decisions are taken in FP32, the precision of the stored state:
 *  0. R = fp32(S).
 *  1. Compensator Tokens ([abs]: the largest outliers of the state stay in
 *     high precision as a few Compensator Tokens; [news]: the outliers are
 *     whole rows and columns, kept in FP16/FP32; reading: FP32).  First n_rows rows, ranked on R by
 *     L2 norm (reading; max-abs with select=1), each kept as the rank-1 pair
 *     (v = e_i, k = R[i,:]) and zeroed in R.  Then n_cols columns, ranked on
 *     the row-zeroed R, each kept as (v = R[:,j], k = e_j) and zeroed.
 *     Scores are FP32 sums in index order; ties go to the lower index.
 *  2. Smoothing ([abs]: the residual left after the compensators is smoothed
 *     before it is quantized):
 *     m_j = max_i |R_ij|, s_j = sqrt(m_j) rounded to FP32; reading: s_j = 1
 *     where m_j = 0.  Without smoothing s_j = 1.
 *  3. Per-row symmetric INT8 ([abs]: the state is held in 8 bits):
 *     R'_ij = R_ij * (1 / s_j), M_i = max_j |R'_ij|, sigma_i = M_i / 127,
 *     Q_ij = clamp(rint(R'_ij * (127 / M_i)), -127, 127) with ties to even;
 *     reading: Q_i = 0 where M_i = 0.  The scales are applied as
 *     multiplications by FP32 reciprocals (one division per column and per
 *     row); the pages fix no arithmetic for the quantizer.
 *  4. S~_ij = sigma_i Q_ij s_j + C_ij, C the sum of the compensator pairs.
 *
 * comp_idx: n_rows row indices then n_cols column indices.
 * comp_vec: n_rows k-vectors of d_k floats, then n_cols v-vectors of d_v.
 */
void lqo_encode(const lqo_params *p, int n_rows, int n_cols, int smooth, int select,
                double *S, int8_t *Q, float *sigma, float *s,
                int32_t *comp_idx, float *comp_vec)
{
    const int dk = p->d_k, dv = p->d_v;
    float *R = (float *)malloc(sizeof(float) * dv * dk);
    float *score = (float *)malloc(sizeof(float) * (dv > dk ? dv : dk));
    unsigned char *taken = (unsigned char *)calloc((size_t)(dv > dk ? dv : dk), 1);
    float *rs = (float *)malloc(sizeof(float) * dk);

    for (int e = 0; e < dv * dk; ++e) R[e] = (float)S[e];

    /* 1a. rows */
    for (int i = 0; i < dv; ++i) {
        float acc = 0.0f;
        for (int j = 0; j < dk; ++j) {
            float a = fabsf(R[i * dk + j]);
            if (select == LQO_SELECT_L2) acc = acc + a * a;
            else if (a > acc) acc = a;
        }
        score[i] = acc;
    }
    for (int c = 0; c < n_rows; ++c) {
        int i = argmax_free(score, taken, dv);
        taken[i] = 1;
        comp_idx[c] = i;
        for (int j = 0; j < dk; ++j) {
            comp_vec[c * dk + j] = R[i * dk + j];
            R[i * dk + j] = 0.0f;
        }
    }
    /* 1b. columns, ranked on the row-zeroed residual */
    memset(taken, 0, (size_t)(dv > dk ? dv : dk));
    for (int j = 0; j < dk; ++j) {
        float acc = 0.0f;
        for (int i = 0; i < dv; ++i) {
            float a = fabsf(R[i * dk + j]);
            if (select == LQO_SELECT_L2) acc = acc + a * a;
            else if (a > acc) acc = a;
        }
        score[j] = acc;
    }
    for (int c = 0; c < n_cols; ++c) {
        int j = argmax_free(score, taken, dk);
        taken[j] = 1;
        comp_idx[n_rows + c] = j;
        for (int i = 0; i < dv; ++i) {
            comp_vec[n_rows * dk + c * dv + i] = R[i * dk + j];
            R[i * dk + j] = 0.0f;
        }
    }

    /* 2. smoothing factors */
    for (int j = 0; j < dk; ++j) {
        float m = 0.0f;
        for (int i = 0; i < dv; ++i) {
            float a = fabsf(R[i * dk + j]);
            if (a > m) m = a;
        }
        s[j] = (smooth && m > 0.0f) ? sqrtf(m) : 1.0f;
    }
    /* 3. row scales and codes */
    for (int j = 0; j < dk; ++j) rs[j] = 1.0f / s[j];
    for (int i = 0; i < dv; ++i) {
        float mx = 0.0f;
        for (int j = 0; j < dk; ++j) {
            float a = fabsf(R[i * dk + j] * rs[j]);
            if (a > mx) mx = a;
        }
        sigma[i] = mx / 127.0f;
        float rho = (mx > 0.0f) ? 127.0f / mx : 0.0f;
        for (int j = 0; j < dk; ++j) {
            float code = 0.0f;
            if (mx > 0.0f) {
                code = rintf((R[i * dk + j] * rs[j]) * rho);
                if (code > 127.0f) code = 127.0f;
                if (code < -127.0f) code = -127.0f;
            }
            Q[i * dk + j] = (int8_t)code;
        }
    }
    /* 4. decoded window-start state */
    for (int i = 0; i < dv; ++i)
        for (int j = 0; j < dk; ++j)
            S[i * dk + j] = (double)sigma[i] * (double)Q[i * dk + j] * (double)s[j];
    for (int c = 0; c < n_rows; ++c) {
        int i = comp_idx[c];
        for (int j = 0; j < dk; ++j) S[i * dk + j] += (double)comp_vec[c * dk + j];
    }
    for (int c = 0; c < n_cols; ++c) {
        int j = comp_idx[n_rows + c];
        for (int i = 0; i < dv; ++i) S[i * dk + j] += (double)comp_vec[n_rows * dk + c * dv + i];
    }
    free(R);
    free(score);
    free(taken);
    free(rs);
}

/* Number of codec applications in a run of T tokens: the prefill encoding,
 * then one per window end (windowed) or one per token (naive). */
int lqo_num_encodings(const lqo_params *p, int T)
{
    if (p->mode == LQO_MODE_FP32) return 0;
    if (p->mode == LQO_MODE_NAIVE) return 1 + T;
    return 1 + T / p->window;
}

/*
 * One head through T tokens.
 *   FP32 mode:     the plain recurrence from S0 ([news]: FP32 inference is
 *                  the baseline).
 *   Windowed mode: the state is encoded from S0, then in every window the
 *                  recurrence runs densely from the decoded window-start state
 *                  and is re-encoded after tokens W, 2W, ... ([abs]).  The
 *                  buffered form a fast implementation uses reaches exactly
 *                  these outputs; this oracle never uses it.
 *   Naive mode:    the state is re-encoded after every token, with no
 *                  compensators and no smoothing ([news]: the per-token
 *                  quantization the paper compares against).
 * Arrays: q,k [T][d_k]; v [T][d_v]; g [T][1 or d_k]; beta [T]; o [T][d_v].
 * S_final (may be NULL) receives the state after the last token (decoded,
 * after any flush at T).  The *_snap arrays (each may be NULL) receive every
 * encoding in order: Q [n][d_v*d_k], sigma [n][d_v], s [n][d_k],
 * idx [n][n_rows+n_cols], vec [n][n_rows*d_k + n_cols*d_v].
 */
void lqo_run(const lqo_params *p, int T, const double *S0,
             const double *q, const double *k, const double *v, const double *g,
             const double *beta, double *o, double *S_final,
             int8_t *Q_snap, float *sigma_snap, float *s_snap,
             int32_t *idx_snap, float *vec_snap)
{
    const int dk = p->d_k, dv = p->d_v;
    const int gdim = (p->gate == LQO_GATE_SCALAR) ? 1 : dk;
    const int naive = (p->mode == LQO_MODE_NAIVE);
    const int nr = naive ? 0 : p->n_comp_rows;
    const int nc = naive ? 0 : p->n_comp_cols;
    const int sm = naive ? 0 : p->smooth;
    const int ncomp = nr + nc;
    const int nvec = nr * dk + nc * dv;

    double *S = (double *)malloc(sizeof(double) * dv * dk);
    int8_t *Q = (int8_t *)malloc((size_t)dv * dk);
    float *sigma = (float *)malloc(sizeof(float) * dv);
    float *s = (float *)malloc(sizeof(float) * dk);
    int32_t *idx = (int32_t *)malloc(sizeof(int32_t) * (ncomp > 0 ? ncomp : 1));
    float *vec = (float *)malloc(sizeof(float) * (nvec > 0 ? nvec : 1));
    int n_enc = 0;

    memcpy(S, S0, sizeof(double) * dv * dk);

#define LQO_ENCODE_AND_SNAP()                                                        \
    do {                                                                             \
        lqo_encode(p, nr, nc, sm, p->select, S, Q, sigma, s, idx, vec);              \
        if (Q_snap) memcpy(Q_snap + (size_t)n_enc * dv * dk, Q, (size_t)dv * dk);    \
        if (sigma_snap) memcpy(sigma_snap + (size_t)n_enc * dv, sigma, sizeof(float) * dv); \
        if (s_snap) memcpy(s_snap + (size_t)n_enc * dk, s, sizeof(float) * dk);      \
        if (idx_snap && ncomp) memcpy(idx_snap + (size_t)n_enc * ncomp, idx, sizeof(int32_t) * ncomp); \
        if (vec_snap && nvec) memcpy(vec_snap + (size_t)n_enc * nvec, vec, sizeof(float) * nvec); \
        ++n_enc;                                                                     \
    } while (0)

    if (p->mode != LQO_MODE_FP32) LQO_ENCODE_AND_SNAP();
    for (int t = 0; t < T; ++t) {
        lqo_step(p, S, q + (size_t)t * dk, k + (size_t)t * dk, v + (size_t)t * dv,
                 g + (size_t)t * gdim, beta[t], o + (size_t)t * dv);
        if (naive || (p->mode == LQO_MODE_WINDOW && (t + 1) % p->window == 0))
            LQO_ENCODE_AND_SNAP();
    }
#undef LQO_ENCODE_AND_SNAP
    if (S_final) memcpy(S_final, S, sizeof(double) * dv * dk);
    free(S); free(Q); free(sigma); free(s); free(idx); free(vec);
}

/*
 * lqo_run over n independent heads (each (sequence, head) pair is its own
 * recurrence), head-major arrays: S0 [n][d_v*d_k], q/k [n][T][d_k],
 * v [n][T][d_v], g [n][T][gdim], beta [n][T], o [n][T][d_v]; the optional
 * outputs are per head as in lqo_run.  OpenMP spreads heads over n_threads
 * host threads (0: the OpenMP default).
 */
void lqo_run_heads(const lqo_params *p, int n, int T, int n_threads, const double *S0,
                   const double *q, const double *k, const double *v, const double *g,
                   const double *beta, double *o, double *S_final,
                   int8_t *Q_snap, float *sigma_snap, float *s_snap,
                   int32_t *idx_snap, float *vec_snap)
{
    const int dk = p->d_k, dv = p->d_v;
    const int gdim = (p->gate == LQO_GATE_SCALAR) ? 1 : dk;
    const int naive = (p->mode == LQO_MODE_NAIVE);
    const int ncomp = naive ? 0 : p->n_comp_rows + p->n_comp_cols;
    const int nvec = naive ? 0 : p->n_comp_rows * dk + p->n_comp_cols * dv;
    const int ne = lqo_num_encodings(p, T);
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (int h = 0; h < n; ++h) {
        lqo_run(p, T, S0 + (size_t)h * dv * dk,
                q + (size_t)h * T * dk, k + (size_t)h * T * dk, v + (size_t)h * T * dv,
                g + (size_t)h * T * gdim, beta + (size_t)h * T, o + (size_t)h * T * dv,
                S_final ? S_final + (size_t)h * dv * dk : NULL,
                Q_snap ? Q_snap + (size_t)h * ne * dv * dk : NULL,
                sigma_snap ? sigma_snap + (size_t)h * ne * dv : NULL,
                s_snap ? s_snap + (size_t)h * ne * dk : NULL,
                idx_snap ? idx_snap + (size_t)h * ne * ncomp : NULL,
                vec_snap ? vec_snap + (size_t)h * ne * nvec : NULL);
    }
}

/* Host threads an OpenMP region started now would use. */
int lqo_max_threads(int n_threads)
{
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
    return omp_get_max_threads();
#else
    (void)n_threads;
    return 1;
#endif
}
