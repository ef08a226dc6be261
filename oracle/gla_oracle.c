/*
 * gla_oracle.c -- plain, slow, fp64 CPU oracle for the Simple GLA mixer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the libgla shared
 * library and its Python binding) may link, load or call this file; only the
 * test suite, the package's smoke check and the benchmark's CPU-baseline leg
 * use it.  It shares no code, header, table or constant with the CUDA path.
 *
 * What it computes (one head at a time, everything in double precision):
 *
 *   Simple Gated Linear Attention keeps one fixed-size matrix state per head
 *   and updates it once per token ("AWS serve Laplace 3B di i14 con uno stato
 *   fisso di 29,5 MB", section "GLA sostituisce i token conservati con uno
 *   stato ricorrente"; "Como i14 llevo Laplace 3B a AWS Trainium2", section
 *   "Por que atencion lineal importa": the previous context is compressed into
 *   a fixed-size state matrix).  With a scalar per-head log-decay a_t <= 0:
 *
 *       S_t = exp(a_t) * S_{t-1} + k_t^T v_t          (S is dk x dv)
 *       o_t = scale * q_t S_t                          (scale = dk^-1/2)
 *
 *   The state read by o_t already contains token t (inclusive state), and the
 *   scale is applied exactly once, to q.  The chunked form used for prefill
 *   and training ("Como i14 ...", section "Adaptaciones para AWS Trainium2",
 *   item 1: 16 chunks of 128 tokens) is an exact reorganisation of this loop,
 *   so the oracle is the loop itself, token by token.
 *
 * Layouts (all contiguous, row-major, double):
 *   q, k   [B, T, H, dk]     v, o, dO  [B, T, H, dv]     a, da  [B, T, H]
 *   s0, s_final, dsT, ds0    [B, H, dk, dv]
 *
 * Backward: the hand-derived reverse recurrence.  With G = dL/dS_t,
 *     G     += scale * q_t^T dO_t
 *     dq_t   = scale * S_t dO_t^T          dk_t = G v_t^T      dv_t = k_t G
 *     da_t   = exp(a_t) * <G, S_{t-1}>     G    = exp(a_t) * G
 * starting from G = dS_T and ending with dS_0 = G.  The states S_t are
 * recomputed forward from checkpoints every CKPT tokens, so memory stays
 * bounded at large T.  The sequential backward over chunks that the pages
 * describe ("Como i14 ...", "Adaptaciones para AWS Trainium2", item 3) is the
 * same computation grouped by chunk.
 *
 * Decode: one token per (sequence, head), state updated in place, then read.
 * Front end ("Como i14 ...", section "Diseno esencial de Laplace 3B": each
 * residual vector passes LayerNorm, then a causal depthwise Conv1d of width 4
 * with SiLU): y[t,c] = SiLU(sum_j w[c,j] * xn[t-(W-1)+j, c] + bias[c]), with
 * xn the LayerNorm output (biased variance over D, eps inside the root) and
 * positions before t = 0 taken from conv_state (zeros when absent).  Its
 * backward (gla_oracle_ln_conv_silu_bwd) is the chain rule through those
 * three stages, written out below.
 *
 * A fault switch (gla_oracle_set_fault) plants a known mistake so the tests
 * can show that each pin catches it.  It is 0 outside those tests.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define CKPT 64

/* Planted mistakes, used only by the pin tests (0 = none). */
enum {
    FAULT_NONE = 0,
    FAULT_NO_DECAY = 1,        /* S_t = S_{t-1} + k^T v (decay dropped)          */
    FAULT_EXCLUSIVE = 2,       /* o_t reads S_{t-1} instead of S_t                */
    FAULT_DOUBLE_SCALE = 3,    /* scale applied twice                             */
    FAULT_DECAY_INDEX = 4,     /* uses a_{t-1} instead of a_t                     */
    FAULT_BWD_DA_NO_EXP = 5,   /* da_t misses its exp(a_t) factor                 */
    FAULT_BWD_DK_SIGN = 6,     /* dk sign flipped                                 */
    FAULT_LN_NO_CENTER = 7,    /* LayerNorm forgets to subtract the mean          */
    FAULT_CONV_TAP_FLIP = 8,   /* conv taps applied in reverse order              */
    FAULT_BWD_SILU_SIGMOID = 9, /* front-end backward uses sigmoid(u) as SiLU'(u)  */
    FAULT_BWD_LN_NO_MEAN = 10  /* LayerNorm backward drops the mean(g) term        */
};
static int g_fault = 0;

void gla_oracle_set_fault(int f) { g_fault = f; }
int gla_oracle_get_fault(void) { return g_fault; }

int gla_oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

static double decay_at(const double* a, int t, int T, int H, int h)
{
    if (g_fault == FAULT_DECAY_INDEX) {
        if (t == 0) return 0.0;
        return a[(size_t)(t - 1) * H + h];
    }
    (void)T;
    return a[(size_t)t * H + h];
}

/* One head: token-by-token recurrence.  Pointers are pre-offset to (b, h);
 * token stride is H*d for q/k/v/o and H for a. */
static void fwd_head(const double* q, const double* k, const double* v, const double* a,
                     const double* s0, double* o, double* s_final, int T, int H, int h,
                     int dk, int dv, double scale, double* S)
{
    const double sc = (g_fault == FAULT_DOUBLE_SCALE) ? scale * scale : scale;
    if (s0) memcpy(S, s0, sizeof(double) * dk * dv);
    else memset(S, 0, sizeof(double) * dk * dv);
    for (int t = 0; t < T; ++t) {
        const double* qt = q + (size_t)t * H * dk;
        const double* kt = k + (size_t)t * H * dk;
        const double* vt = v + (size_t)t * H * dv;
        double* ot = o + (size_t)t * H * dv;
        const double g = (g_fault == FAULT_NO_DECAY) ? 1.0 : exp(decay_at(a, t, T, H, h));
        if (g_fault == FAULT_EXCLUSIVE) {
            for (int j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int i = 0; i < dk; ++i) acc += qt[i] * S[i * dv + j];
                ot[j] = sc * acc;
            }
        }
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j)
                S[i * dv + j] = g * S[i * dv + j] + kt[i] * vt[j];
        if (g_fault != FAULT_EXCLUSIVE) {
            for (int j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int i = 0; i < dk; ++i) acc += qt[i] * S[i * dv + j];
                ot[j] = sc * acc;
            }
        }
    }
    if (s_final) memcpy(s_final, S, sizeof(double) * dk * dv);
}

void gla_oracle_fwd(const double* q, const double* k, const double* v, const double* a,
                    const double* s0, double* o, double* s_final,
                    int B, int T, int H, int dk, int dv, double scale)
{
    const int units = B * H;
#pragma omp parallel
    {
        double* S = (double*)malloc(sizeof(double) * dk * dv);
#pragma omp for schedule(dynamic, 1)
        for (int u = 0; u < units; ++u) {
            const int b = u / H, h = u % H;
            const size_t tok0 = (size_t)b * T;
            fwd_head(q + (tok0 * H + h) * dk, k + (tok0 * H + h) * dk,
                     v + (tok0 * H + h) * dv, a + tok0 * H, s0 ? s0 + (size_t)u * dk * dv : NULL,
                     o + (tok0 * H + h) * dv, s_final ? s_final + (size_t)u * dk * dv : NULL,
                     T, H, h, dk, dv, scale, S);
        }
        free(S);
    }
}

/* One head of the backward.  ckpt holds S at the start of every CKPT block
 * ((nblk+1) x dk x dv), blk holds the CKPT states S_t of the block being
 * processed. */
static void bwd_head(const double* q, const double* k, const double* v, const double* a,
                     const double* s0, const double* dO, const double* dsT,
                     double* dq, double* dkk, double* dvv, double* da, double* ds0,
                     int T, int H, int h, int dk, int dv, double scale,
                     double* ckpt, double* blk, double* G)
{
    const size_t SS = (size_t)dk * dv;
    const int nblk = (T + CKPT - 1) / CKPT;
    /* forward sweep: checkpoints of S at the start of each block */
    double* S = ckpt;
    if (s0) memcpy(S, s0, sizeof(double) * SS);
    else memset(S, 0, sizeof(double) * SS);
    for (int bi = 0; bi < nblk; ++bi) {
        double* Sn = ckpt + (size_t)(bi + 1) * SS;
        memcpy(Sn, ckpt + (size_t)bi * SS, sizeof(double) * SS);
        const int t1 = (bi + 1) * CKPT < T ? (bi + 1) * CKPT : T;
        for (int t = bi * CKPT; t < t1; ++t) {
            const double g = exp(a[(size_t)t * H + h]);
            const double* kt = k + (size_t)t * H * dk;
            const double* vt = v + (size_t)t * H * dv;
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j) Sn[i * dv + j] = g * Sn[i * dv + j] + kt[i] * vt[j];
        }
    }
    /* reverse sweep */
    if (dsT) memcpy(G, dsT, sizeof(double) * SS);
    else memset(G, 0, sizeof(double) * SS);
    for (int bi = nblk - 1; bi >= 0; --bi) {
        const int t0 = bi * CKPT;
        const int t1 = (bi + 1) * CKPT < T ? (bi + 1) * CKPT : T;
        /* recompute S_t for t in [t0, t1) into blk[t - t0] */
        const double* Sp = ckpt + (size_t)bi * SS;
        for (int t = t0; t < t1; ++t) {
            double* St = blk + (size_t)(t - t0) * SS;
            const double g = exp(a[(size_t)t * H + h]);
            const double* kt = k + (size_t)t * H * dk;
            const double* vt = v + (size_t)t * H * dv;
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j) St[i * dv + j] = g * Sp[i * dv + j] + kt[i] * vt[j];
            Sp = St;
        }
        for (int t = t1 - 1; t >= t0; --t) {
            const double* St = blk + (size_t)(t - t0) * SS;
            const double* Sprev = (t == t0) ? ckpt + (size_t)bi * SS : blk + (size_t)(t - t0 - 1) * SS;
            const double* qt = q + (size_t)t * H * dk;
            const double* kt = k + (size_t)t * H * dk;
            const double* vt = v + (size_t)t * H * dv;
            const double* gt = dO + (size_t)t * H * dv;
            double* dqt = dq + (size_t)t * H * dk;
            double* dkt = dkk + (size_t)t * H * dk;
            double* dvt = dvv + (size_t)t * H * dv;
            const double g = exp(a[(size_t)t * H + h]);
            /* G += scale * q_t^T dO_t  (G is now dL/dS_t) */
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j) G[i * dv + j] += scale * qt[i] * gt[j];
            /* dq_t = scale * S_t dO_t^T */
            for (int i = 0; i < dk; ++i) {
                double acc = 0.0;
                for (int j = 0; j < dv; ++j) acc += St[i * dv + j] * gt[j];
                dqt[i] = scale * acc;
            }
            /* dk_t = G v_t^T ; dv_t = k_t G */
            for (int i = 0; i < dk; ++i) {
                double acc = 0.0;
                for (int j = 0; j < dv; ++j) acc += G[i * dv + j] * vt[j];
                dkt[i] = (g_fault == FAULT_BWD_DK_SIGN) ? -acc : acc;
            }
            for (int j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int i = 0; i < dk; ++i) acc += kt[i] * G[i * dv + j];
                dvt[j] = acc;
            }
            /* da_t = exp(a_t) <G, S_{t-1}> */
            double fr = 0.0;
            for (size_t e = 0; e < SS; ++e) fr += G[e] * Sprev[e];
            da[(size_t)t * H + h] = (g_fault == FAULT_BWD_DA_NO_EXP) ? fr : g * fr;
            /* G = exp(a_t) G  (now dL/dS_{t-1}) */
            for (size_t e = 0; e < SS; ++e) G[e] *= g;
        }
    }
    if (ds0) memcpy(ds0, G, sizeof(double) * SS);
}

void gla_oracle_bwd(const double* q, const double* k, const double* v, const double* a,
                    const double* s0, const double* dO, const double* dsT,
                    double* dq, double* dk_out, double* dv_out, double* da, double* ds0,
                    int B, int T, int H, int dk, int dv, double scale)
{
    const int units = B * H;
    const size_t SS = (size_t)dk * dv;
    const int nblk = (T + CKPT - 1) / CKPT;
#pragma omp parallel
    {
        double* ckpt = (double*)malloc(sizeof(double) * SS * (nblk + 1));
        double* blk = (double*)malloc(sizeof(double) * SS * CKPT);
        double* G = (double*)malloc(sizeof(double) * SS);
#pragma omp for schedule(dynamic, 1)
        for (int u = 0; u < units; ++u) {
            const int b = u / H, h = u % H;
            const size_t tok0 = (size_t)b * T;
            bwd_head(q + (tok0 * H + h) * dk, k + (tok0 * H + h) * dk, v + (tok0 * H + h) * dv,
                     a + tok0 * H, s0 ? s0 + (size_t)u * SS : NULL, dO + (tok0 * H + h) * dv,
                     dsT ? dsT + (size_t)u * SS : NULL, dq + (tok0 * H + h) * dk,
                     dk_out + (tok0 * H + h) * dk, dv_out + (tok0 * H + h) * dv, da + tok0 * H,
                     ds0 ? ds0 + (size_t)u * SS : NULL, T, H, h, dk, dv, scale, ckpt, blk, G);
        }
        free(ckpt);
        free(blk);
        free(G);
    }
}

/* Decode: one token for each of N sequences.  state [N_slots, H, dk, dv] is
 * updated in place; slot_idx (nullable) maps sequence n to its state slot. */
void gla_oracle_decode(double* state, const long long* slot_idx, const double* q,
                       const double* k, const double* v, const double* a, double* o,
                       int N, int H, int dk, int dv, double scale)
{
    const size_t SS = (size_t)dk * dv;
#pragma omp parallel for schedule(static)
    for (long long u = 0; u < (long long)N * H; ++u) {
        const int n = (int)(u / H), h = (int)(u % H);
        const long long slot = slot_idx ? slot_idx[n] : n;
        double* S = state + ((size_t)slot * H + h) * SS;
        const double* qt = q + (size_t)u * dk;
        const double* kt = k + (size_t)u * dk;
        const double* vt = v + (size_t)u * dv;
        const double g = (g_fault == FAULT_NO_DECAY) ? 1.0 : exp(a[u]);
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j) S[i * dv + j] = g * S[i * dv + j] + kt[i] * vt[j];
        for (int j = 0; j < dv; ++j) {
            double acc = 0.0;
            for (int i = 0; i < dk; ++i) acc += qt[i] * S[i * dv + j];
            o[(size_t)u * dv + j] = scale * acc;
        }
    }
}

/* LayerNorm (optional) -> causal depthwise conv of width W -> SiLU (optional;
 * the switches exist so the tests can pin each stage on its own).
 * x, y [B, T, D]; w [D, W] (w[c, W-1] multiplies the current token);
 * conv_state_in/out [B, W-1, D] hold the last W-1 conv inputs, oldest first. */
void gla_oracle_ln_conv_silu(const double* x, const double* ln_gamma, const double* ln_beta,
                             double ln_eps, int do_ln, const double* w, const double* bias,
                             const double* conv_state_in, double* conv_state_out, double* y,
                             int B, int T, int D, int W, int do_silu)
{
    for (int b = 0; b < B; ++b) {
        double* xn = (double*)malloc(sizeof(double) * ((size_t)T + W - 1) * D);
        /* history rows 0..W-2, then the T normalised rows */
        for (int r = 0; r < W - 1; ++r)
            for (int c = 0; c < D; ++c)
                xn[(size_t)r * D + c] =
                    conv_state_in ? conv_state_in[((size_t)b * (W - 1) + r) * D + c] : 0.0;
#pragma omp parallel for schedule(static)
        for (int t = 0; t < T; ++t) {
            const double* xr = x + ((size_t)b * T + t) * D;
            double* out = xn + ((size_t)t + W - 1) * D;
            if (!do_ln) {
                for (int c = 0; c < D; ++c) out[c] = xr[c];
                continue;
            }
            double mean = 0.0;
            for (int c = 0; c < D; ++c) mean += xr[c];
            mean /= D;
            double var = 0.0;
            for (int c = 0; c < D; ++c) var += (xr[c] - mean) * (xr[c] - mean);
            var /= D;
            const double rstd = 1.0 / sqrt(var + ln_eps);
            const double mu = (g_fault == FAULT_LN_NO_CENTER) ? 0.0 : mean;
            for (int c = 0; c < D; ++c) {
                double vln = (xr[c] - mu) * rstd;
                if (ln_gamma) vln *= ln_gamma[c];
                if (ln_beta) vln += ln_beta[c];
                out[c] = vln;
            }
        }
#pragma omp parallel for schedule(static)
        for (int t = 0; t < T; ++t) {
            for (int c = 0; c < D; ++c) {
                double acc = bias ? bias[c] : 0.0;
                for (int j = 0; j < W; ++j) {
                    const int tap = (g_fault == FAULT_CONV_TAP_FLIP) ? (W - 1 - j) : j;
                    acc += w[(size_t)c * W + tap] * xn[((size_t)t + j) * D + c];
                }
                y[((size_t)b * T + t) * D + c] = do_silu ? acc / (1.0 + exp(-acc)) : acc;
            }
        }
        if (conv_state_out)
            for (int r = 0; r < W - 1; ++r)
                for (int c = 0; c < D; ++c)
                    conv_state_out[((size_t)b * (W - 1) + r) * D + c] =
                        xn[((size_t)T + r) * D + c];
        free(xn);
    }
}

/*
 * Backward of the front end above (the per-layer LayerNorm -> causal
 * depthwise conv -> SiLU of "Como i14 ...", section "Diseno esencial de
 * Laplace 3B"), by the chain rule, for a loss whose gradient with respect to
 * y is dy.  With xn the conv inputs (history rows first), u the conv output
 * before SiLU and s = 1 / (1 + exp(-u)):
 *     du[t,c]     = dy[t,c] * s * (1 + u (1 - s))           SiLU'(u)
 *     dbias[c]    = sum_{b,t} du[t,c]
 *     dw[c,j]     = sum_{b,t} du[t,c] * xn[t-(W-1)+j, c]
 *     dxn[p,c]    = sum_j w[c,j] * du[p+(W-1)-j, c]           (du = 0 outside 0..T-1)
 *   rows p < 0 are the history: dconv_state_in[b, p+W-1, c] = dxn[p,c].
 *   LayerNorm, xhat = (x - mean) * rstd, xn = xhat * gamma + beta:
 *     dgamma[c]   = sum_{b,t} dxn * xhat      dbeta[c] = sum_{b,t} dxn
 *     g           = dxn * gamma
 *     dx          = rstd * (g - mean_c(g) - xhat * mean_c(g * xhat))
 *   (without LayerNorm, dx = dxn and dgamma = dbeta = 0).  The conv state
 *   out carries no gradient back.  All outputs are overwritten.
 */
void gla_oracle_ln_conv_silu_bwd(const double* x, const double* ln_gamma, const double* ln_beta,
                                 double ln_eps, int do_ln, const double* w, const double* bias,
                                 const double* conv_state_in, const double* dy, double* dx, double* dw,
                                 double* dbias, double* dgamma, double* dbeta, double* dconv_state_in,
                                 int B, int T, int D, int W)
{
    for (int c = 0; c < D; ++c) {
        dbias[c] = dgamma[c] = dbeta[c] = 0.0;
        for (int j = 0; j < W; ++j) dw[(size_t)c * W + j] = 0.0;
    }
    for (int b = 0; b < B; ++b) {
        const size_t rows = (size_t)T + W - 1;
        double* xn = (double*)malloc(sizeof(double) * rows * D);
        double* xh = (double*)malloc(sizeof(double) * (size_t)T * D);
        double* rs = (double*)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
        double* du = (double*)malloc(sizeof(double) * (size_t)T * D);
        double* dxn = (double*)malloc(sizeof(double) * rows * D);
        for (int r = 0; r < W - 1; ++r)
            for (int c = 0; c < D; ++c)
                xn[(size_t)r * D + c] = conv_state_in ? conv_state_in[((size_t)b * (W - 1) + r) * D + c] : 0.0;
        /* forward again: LayerNorm rows, conv, SiLU'(u) */
        for (int t = 0; t < T; ++t) {
            const double* xr = x + ((size_t)b * T + t) * D;
            double* out = xn + ((size_t)t + W - 1) * D;
            double* h = xh + (size_t)t * D;
            if (!do_ln) {
                for (int c = 0; c < D; ++c) out[c] = h[c] = xr[c];
                rs[t] = 1.0;
                continue;
            }
            double mean = 0.0, var = 0.0;
            for (int c = 0; c < D; ++c) mean += xr[c];
            mean /= D;
            for (int c = 0; c < D; ++c) var += (xr[c] - mean) * (xr[c] - mean);
            var /= D;
            rs[t] = 1.0 / sqrt(var + ln_eps);
            for (int c = 0; c < D; ++c) {
                h[c] = (xr[c] - mean) * rs[t];
                out[c] = h[c] * (ln_gamma ? ln_gamma[c] : 1.0) + (ln_beta ? ln_beta[c] : 0.0);
            }
        }
        for (int t = 0; t < T; ++t)
            for (int c = 0; c < D; ++c) {
                double u = bias ? bias[c] : 0.0;
                for (int j = 0; j < W; ++j) u += w[(size_t)c * W + j] * xn[((size_t)t + j) * D + c];
                const double sg = 1.0 / (1.0 + exp(-u));
                const double dsilu = (g_fault == FAULT_BWD_SILU_SIGMOID) ? sg : sg * (1.0 + u * (1.0 - sg));
                const double g = dy[((size_t)b * T + t) * D + c] * dsilu;
                du[(size_t)t * D + c] = g;
                dbias[c] += g;
                for (int j = 0; j < W; ++j) dw[(size_t)c * W + j] += g * xn[((size_t)t + j) * D + c];
            }
        /* dxn over all rows, history included: row r = p + W - 1 */
        for (size_t r = 0; r < rows; ++r)
            for (int c = 0; c < D; ++c) {
                double acc = 0.0;
                for (int j = 0; j < W; ++j) {
                    const long t = (long)r - j;           /* p + (W-1) - j with p = r - (W-1) */
                    if (t >= 0 && t < T) acc += w[(size_t)c * W + j] * du[(size_t)t * D + c];
                }
                dxn[r * D + c] = acc;
            }
        if (dconv_state_in)
            for (int r = 0; r < W - 1; ++r)
                for (int c = 0; c < D; ++c)
                    dconv_state_in[((size_t)b * (W - 1) + r) * D + c] = dxn[(size_t)r * D + c];
        for (int t = 0; t < T; ++t) {
            const double* d = dxn + ((size_t)t + W - 1) * D;
            const double* h = xh + (size_t)t * D;
            double* o = dx + ((size_t)b * T + t) * D;
            if (!do_ln) {
                for (int c = 0; c < D; ++c) o[c] = d[c];
                continue;
            }
            double mg = 0.0, mgh = 0.0;
            for (int c = 0; c < D; ++c) {
                const double g = d[c] * (ln_gamma ? ln_gamma[c] : 1.0);
                mg += g;
                mgh += g * h[c];
                dgamma[c] += d[c] * h[c];
                dbeta[c] += d[c];
            }
            mg /= D;
            mgh /= D;
            if (g_fault == FAULT_BWD_LN_NO_MEAN) mg = 0.0;
            for (int c = 0; c < D; ++c) {
                const double g = d[c] * (ln_gamma ? ln_gamma[c] : 1.0);
                o[c] = rs[t] * (g - mg - h[c] * mgh);
            }
        }
        free(xn);
        free(xh);
        free(rs);
        free(du);
        free(dxn);
    }
}
