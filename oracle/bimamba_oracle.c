/*
 * bimamba_oracle.c -- plain, slow, double-precision CPU oracle for the
 * bidirectional Mamba-2 mixer core.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file; only the tests, the smoke check and the CPU-baseline leg of
 * the benchmark do.  It shares no code, header, table or helper with the CUDA
 * library.
 *
 * What it computes (sources, by page title and section):
 *  - "DiffuMamba: High-Throughput Diffusion LMs with Mamba Backbone"
 *    (gist.science, Japanese technical summary, section 2 "Proposed method"):
 *    every mixer is a bidirectional Mamba-2 mixer; a forward and a reversed
 *    stream are combined by addition.  The Portuguese summary of the same
 *    paper (section 2 "Metodologia") says the same: two directions, fused.
 *  - The blog post "DiffuMamba" (metaphor-xennon), network-architecture
 *    listing: d_state = 128, d_conv = 4, expand = 2.
 *  - The Mamba-2 (SSD) recurrence, which the pages name but never print, is
 *    taken in its standard form:
 *        h_t = exp(dt_t * A) * h_{t-1} + dt_t * x_t B_t^T      (P x N per head)
 *        y_t = h_t C_t + D * x_t
 *    with A a negative scalar per head, dt per (token, head), and B, C shared
 *    by all heads of a group.
 *  - "Fixed state, long reach: constant-size caches in large-scale block
 *    diffusion" (bittide, abstract and section 1): a finished block is
 *    summarised by the forward SSM state (O(1) memory); the reverse scan is
 *    restricted to the active block; training on the block-causal objective
 *    makes cached decoding exactly equal to recomputation.
 *
 * Readings where the pages are silent (each one is listed in the design notes):
 *  - conv: depthwise, causal, tap j multiplies u[t-(K-1)+j]; zero padding
 *    before the sequence start (or the cached tail in decode).  The reversed
 *    stream uses the mirror image: tap j multiplies u[t+(K-1)-j], zero past
 *    the end.  This is exactly flip(conv(flip(u))).
 *  - the conv covers all xBC channels (x, B and C), then SiLU.
 *  - the reverse scan is the forward recurrence run from t = L-1 down to 0,
 *    i.e. flip(scan(flip(.))); its initial state is zero.
 *  - the two directions share every parameter (A, D, conv weights, dt).
 *  - the D skip term is added in each direction.
 *
 * Every function works on plain double arrays, row-major, contiguous.
 */
#include <math.h>
#include <stddef.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static double silu(double v) { return v / (1.0 + exp(-v)); }

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * Depthwise conv1d with K taps, then optional SiLU.
 *   u    : (batch, len, ch)
 *   w    : (ch, K)
 *   bias : (ch) or NULL
 *   tail : (batch, K, ch) or NULL -- the K raw tokens before t = 0, oldest
 *          first (forward direction only; ignored when reverse != 0)
 *   out  : (batch, len, ch)
 * Forward:  pre[t,c] = bias[c] + sum_j w[c,j] * u[t-(K-1)+j, c]
 *           u at negative positions = tail (if given) else 0.
 * Reverse:  pre[t,c] = bias[c] + sum_j w[c,j] * u[t+(K-1)-j, c]
 *           u at positions >= len = 0.
 */
void oracle_conv(const double *u, const double *w, const double *bias,
                 const double *tail, int batch, int len, int ch, int K,
                 int reverse, int apply_silu, double *out)
{
    for (int b = 0; b < batch; ++b) {
        for (int t = 0; t < len; ++t) {
            for (int c = 0; c < ch; ++c) {
                double acc = bias ? bias[c] : 0.0;
                for (int j = 0; j < K; ++j) {
                    long src = reverse ? (long)t + (K - 1) - j
                                       : (long)t - (K - 1) + j;
                    double v;
                    if (src >= 0 && src < len) {
                        v = u[((size_t)b * len + src) * ch + c];
                    } else if (!reverse && src < 0 && tail) {
                        /* tail holds positions -K .. -1 */
                        v = tail[((size_t)b * K + (size_t)(K + src)) * ch + c];
                    } else {
                        v = 0.0;
                    }
                    acc += w[(size_t)c * K + j] * v;
                }
                out[((size_t)b * len + t) * ch + c] = apply_silu ? silu(acc) : acc;
            }
        }
    }
}

/*
 * One direction of the selective scan, sequential in t.
 *   x    : (batch, len, H, P)
 *   Bm   : (batch, len, G, N)
 *   Cm   : (batch, len, G, N)
 *   dt   : (batch, len, H)        already positive (post-softplus)
 *   A    : (H)                    negative
 *   D    : (H)
 *   init : (batch, H, P, N) or NULL (zero state)
 *   y    : (batch, len, H, P)     written (not accumulated)
 *   fin  : (batch, H, P, N) or NULL -- state after the last processed token
 * Head h reads group h / (H / G).
 * reverse != 0 walks t = len-1 .. 0 with the same update.
 */
void oracle_scan(const double *x, const double *Bm, const double *Cm,
                 const double *dt, const double *A, const double *D,
                 const double *init, int batch, int len, int H, int P, int N,
                 int G, int reverse, double *y, double *fin)
{
    int hpg = H / G;
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int b = 0; b < batch; ++b) {
        for (int h = 0; h < H; ++h) {
            int g = h / hpg;
            double *hs = (double *)malloc(sizeof(double) * (size_t)P * N);
            if (init)
                memcpy(hs, init + ((size_t)b * H + h) * P * N,
                       sizeof(double) * (size_t)P * N);
            else
                memset(hs, 0, sizeof(double) * (size_t)P * N);
            for (int step = 0; step < len; ++step) {
                int t = reverse ? len - 1 - step : step;
                double d = dt[((size_t)b * len + t) * H + h];
                double a = exp(d * A[h]);
                const double *xt = x + (((size_t)b * len + t) * H + h) * P;
                const double *bt = Bm + (((size_t)b * len + t) * G + g) * N;
                const double *ct = Cm + (((size_t)b * len + t) * G + g) * N;
                double *yt = y + (((size_t)b * len + t) * H + h) * P;
                for (int p = 0; p < P; ++p) {
                    double *row = hs + (size_t)p * N;
                    double dx = d * xt[p];
                    double acc = 0.0;
                    for (int n = 0; n < N; ++n) {
                        row[n] = a * row[n] + dx * bt[n];
                        acc += row[n] * ct[n];
                    }
                    yt[p] = acc + D[h] * xt[p];
                }
            }
            if (fin)
                memcpy(fin + ((size_t)b * H + h) * P * N, hs,
                       sizeof(double) * (size_t)P * N);
            free(hs);
        }
    }
}

/* Split activated xBC (batch, len, ch = H*P + 2*G*N) into x, B, C. */
static void split_xbc(const double *u, int batch, int len, int H, int P,
                      int N, int G, double *x, double *Bm, double *Cm)
{
    int ch = H * P + 2 * G * N;
    for (size_t r = 0; r < (size_t)batch * len; ++r) {
        const double *src = u + r * ch;
        memcpy(x + r * H * P, src, sizeof(double) * (size_t)H * P);
        memcpy(Bm + r * G * N, src + H * P, sizeof(double) * (size_t)G * N);
        memcpy(Cm + r * G * N, src + H * P + G * N, sizeof(double) * (size_t)G * N);
    }
}

/*
 * Whole bidirectional mixer core.
 *   xbc    : (batch, len, ch) raw (pre-conv) when conv_w != NULL, otherwise
 *            already activated; ch = H*P + 2*G*N, channel order [x | B | C]
 *   conv_w : (ch, K) or NULL (no conv, no SiLU)
 *   conv_b : (ch) or NULL
 *   tail   : (batch, K, ch) or NULL -- forward conv history (decode)
 *   init   : (batch, H, P, N) or NULL -- forward initial state
 *   y      : (batch, len, H*P) = forward stream + reverse stream
 *   fin    : (batch, H, P, N) or NULL -- forward final state
 *   yf, yr : optional (batch, len, H*P) per-direction outputs (may be NULL)
 */
void oracle_bimamba(const double *xbc, const double *dt, const double *A,
                    const double *D, const double *conv_w, const double *conv_b,
                    const double *tail, const double *init, int batch, int len,
                    int H, int P, int N, int G, int K, double *y, double *fin,
                    double *yf, double *yr)
{
    int ch = H * P + 2 * G * N;
    size_t nt = (size_t)batch * len;
    double *act = (double *)malloc(sizeof(double) * nt * ch);
    double *x = (double *)malloc(sizeof(double) * nt * H * P);
    double *Bm = (double *)malloc(sizeof(double) * nt * G * N);
    double *Cm = (double *)malloc(sizeof(double) * nt * G * N);
    double *of = (double *)malloc(sizeof(double) * nt * H * P);
    double *orv = (double *)malloc(sizeof(double) * nt * H * P);

    /* forward stream */
    if (conv_w)
        oracle_conv(xbc, conv_w, conv_b, tail, batch, len, ch, K, 0, 1, act);
    else
        memcpy(act, xbc, sizeof(double) * nt * ch);
    split_xbc(act, batch, len, H, P, N, G, x, Bm, Cm);
    oracle_scan(x, Bm, Cm, dt, A, D, init, batch, len, H, P, N, G, 0, of, fin);

    /* reverse stream: mirrored conv, zero padding past the end, zero state */
    if (conv_w)
        oracle_conv(xbc, conv_w, conv_b, NULL, batch, len, ch, K, 1, 1, act);
    else
        memcpy(act, xbc, sizeof(double) * nt * ch);
    split_xbc(act, batch, len, H, P, N, G, x, Bm, Cm);
    oracle_scan(x, Bm, Cm, dt, A, D, NULL, batch, len, H, P, N, G, 1, orv, NULL);

    for (size_t i = 0; i < nt * H * P; ++i)
        y[i] = of[i] + orv[i];
    if (yf) memcpy(yf, of, sizeof(double) * nt * H * P);
    if (yr) memcpy(yr, orv, sizeof(double) * nt * H * P);
    free(act); free(x); free(Bm); free(Cm); free(of); free(orv);
}

/*
 * Cached block decode for block diffusion.  For each stream, the forward
 * stream resumes from the cached state with the cached conv tail; the reverse
 * stream covers the active block only, from a zero state, with zero padding
 * past the block end.  The result is the sum.
 *   block     : (streams, len, ch) raw xBC of the active block
 *   state     : (streams, H, P, N) forward state after the prefix
 *   tail      : (streams, K, ch) last K raw tokens of the prefix, oldest first
 *   y         : (streams, len, H*P)
 *   state_out : (streams, H, P, N) or NULL -- forward state after the block
 *   tail_out  : (streams, K, ch) or NULL   -- last K raw tokens of
 *               prefix + block, oldest first
 * This is oracle_bimamba with tail and init on the forward stream, so it
 * reuses that definition directly.
 */
void oracle_block_decode(const double *block, const double *dt, const double *A,
                         const double *D, const double *conv_w,
                         const double *conv_b, const double *state,
                         const double *tail, int streams, int len, int H, int P,
                         int N, int G, int K, double *y, double *state_out,
                         double *tail_out)
{
    oracle_bimamba(block, dt, A, D, conv_w, conv_b, tail, state, streams, len,
                   H, P, N, G, K, y, state_out, NULL, NULL);
    if (tail_out) {
        int ch = H * P + 2 * G * N;
        for (int s = 0; s < streams; ++s) {
            for (int k = 0; k < K; ++k) {
                /* position len - K + k of the concatenation tail | block */
                long pos = (long)len - K + k;
                const double *src;
                if (pos >= 0)
                    src = block + ((size_t)s * len + pos) * ch;
                else
                    src = tail + ((size_t)s * K + (size_t)(K + pos)) * ch;
                memcpy(tail_out + ((size_t)s * K + k) * ch, src,
                       sizeof(double) * ch);
            }
        }
    }
}

/*
 * Untied directions.  The blog post "DiffuMamba" (metaphor-xennon),
 * network-architecture listing, builds the bidirectional mixer from two
 * separate Mamba modules: one reads the sequence as it is, the other reads
 * it reversed and its output is reversed back; the two outputs are
 * concatenated and a Linear layer maps 2d back to d.  The technical
 * summaries (section 2) combine the two streams by addition instead.  This
 * function gives each stream its own parameters and offers both fusions:
 *   *_f, *_r : forward / reverse stream inputs and parameters (xbc, dt, A,
 *              D, conv taps, conv bias), shaped as in oracle_bimamba
 *   init     : (batch, H, P, N) or NULL -- forward initial state
 *   concat   : 0 -> y (batch, len, H*P) = forward + reverse
 *              1 -> y (batch, len, 2*H*P), per token [forward | reverse]
 *              (the Linear after the concatenation is not part of the scan)
 *   fin      : (batch, H, P, N) or NULL -- forward final state
 * Each stream is exactly the corresponding stream of oracle_bimamba run
 * with that stream's parameters.
 */
void oracle_bimamba_untied(const double *xbc_f, const double *xbc_r,
                           const double *dt_f, const double *dt_r,
                           const double *A_f, const double *A_r,
                           const double *D_f, const double *D_r,
                           const double *conv_w_f, const double *conv_w_r,
                           const double *conv_b_f, const double *conv_b_r,
                           const double *init, int batch, int len, int H,
                           int P, int N, int G, int K, int concat, double *y,
                           double *fin)
{
    int ch = H * P + 2 * G * N;
    size_t nt = (size_t)batch * len;
    size_t hp = (size_t)H * P;
    double *act = (double *)malloc(sizeof(double) * nt * ch);
    double *x = (double *)malloc(sizeof(double) * nt * hp);
    double *Bm = (double *)malloc(sizeof(double) * nt * G * N);
    double *Cm = (double *)malloc(sizeof(double) * nt * G * N);
    double *of = (double *)malloc(sizeof(double) * nt * hp);
    double *orv = (double *)malloc(sizeof(double) * nt * hp);

    /* forward stream, forward parameters */
    if (conv_w_f)
        oracle_conv(xbc_f, conv_w_f, conv_b_f, NULL, batch, len, ch, K, 0, 1, act);
    else
        memcpy(act, xbc_f, sizeof(double) * nt * ch);
    split_xbc(act, batch, len, H, P, N, G, x, Bm, Cm);
    oracle_scan(x, Bm, Cm, dt_f, A_f, D_f, init, batch, len, H, P, N, G, 0, of, fin);

    /* reverse stream, reverse parameters: mirrored conv, zero state */
    if (conv_w_r)
        oracle_conv(xbc_r, conv_w_r, conv_b_r, NULL, batch, len, ch, K, 1, 1, act);
    else
        memcpy(act, xbc_r, sizeof(double) * nt * ch);
    split_xbc(act, batch, len, H, P, N, G, x, Bm, Cm);
    oracle_scan(x, Bm, Cm, dt_r, A_r, D_r, NULL, batch, len, H, P, N, G, 1, orv, NULL);

    for (size_t r = 0; r < nt; ++r) {
        if (concat) {
            memcpy(y + r * 2 * hp, of + r * hp, sizeof(double) * hp);
            memcpy(y + r * 2 * hp + hp, orv + r * hp, sizeof(double) * hp);
        } else {
            for (size_t i = 0; i < hp; ++i) y[r * hp + i] = of[r * hp + i] + orv[r * hp + i];
        }
    }
    free(act); free(x); free(Bm); free(Cm); free(of); free(orv);
}

/*
 * Backward of one direction of the selective scan (no conv): the adjoint of
 * the recurrence above, for the training objective the cached-decode page's
 * block-causal training implies.  Given dy = dL/dy (same shape as y), it ADDS
 * dL/d(input) into the gradient buffers (any of which may be NULL), so that
 * calling it once per direction accumulates the bidirectional gradient.
 * With g_s = dL/dh_s carried backward along the walk:
 *   g_s      = dy_s C_s^T + a_{s+1} g_{s+1}
 *   dC_s    += h_s^T dy_s            dD   += dy_s . x_s
 *   dx_s    += D dy_s + dt_s g_s B_s dB_s += dt_s g_s^T x_s
 *   ddt_s   += <g_s, x_s B_s^T> + A a_s <g_s, h_{s-1}>
 *   dA      += dt_s a_s <g_s, h_{s-1}>
 *   dinit   += a_0 g_0    (the state entering the walk)
 * Shapes as in oracle_scan; dA, dD : (H); dinit : (batch, H, P, N).
 * Sequential (the group-shared B, C and the per-head A, D gradients are sums
 * over heads, batch and time).
 */
void oracle_scan_backward(const double *x, const double *Bm, const double *Cm,
                          const double *dt, const double *A, const double *D,
                          const double *init, const double *dy, int batch,
                          int len, int H, int P, int N, int G, int reverse,
                          double *dx, double *dB, double *dC, double *ddt,
                          double *dA, double *dD, double *dinit)
{
    int hpg = H / G;
    size_t pn = (size_t)P * N;
    double *hs = (double *)malloc(sizeof(double) * pn * (size_t)(len + 1));
    double *g = (double *)malloc(sizeof(double) * pn);
    for (int b = 0; b < batch; ++b) {
        for (int h = 0; h < H; ++h) {
            int grp = h / hpg;
            /* forward pass, keeping every state: hs[0] = entering state,
               hs[s + 1] = state after walk step s */
            if (init)
                memcpy(hs, init + ((size_t)b * H + h) * pn, sizeof(double) * pn);
            else
                memset(hs, 0, sizeof(double) * pn);
            for (int s = 0; s < len; ++s) {
                int t = reverse ? len - 1 - s : s;
                double d = dt[((size_t)b * len + t) * H + h];
                double a = exp(d * A[h]);
                const double *xt = x + (((size_t)b * len + t) * H + h) * P;
                const double *bt = Bm + (((size_t)b * len + t) * G + grp) * N;
                const double *prev = hs + (size_t)s * pn;
                double *cur = hs + (size_t)(s + 1) * pn;
                for (int p = 0; p < P; ++p)
                    for (int n = 0; n < N; ++n)
                        cur[(size_t)p * N + n] = a * prev[(size_t)p * N + n] + d * xt[p] * bt[n];
            }
            /* backward along the walk */
            memset(g, 0, sizeof(double) * pn);
            for (int s = len - 1; s >= 0; --s) {
                int t = reverse ? len - 1 - s : s;
                size_t ti = (size_t)b * len + t;
                double d = dt[ti * H + h];
                double a = exp(d * A[h]);
                const double *xt = x + (ti * H + h) * P;
                const double *bt = Bm + (ti * G + grp) * N;
                const double *ct = Cm + (ti * G + grp) * N;
                const double *dyt = dy + (ti * H + h) * P;
                const double *cur = hs + (size_t)(s + 1) * pn;
                const double *prev = hs + (size_t)s * pn;
                double da = 0.0, dd_in = 0.0, dDh = 0.0;
                for (int p = 0; p < P; ++p) {
                    double gx = 0.0;
                    for (int n = 0; n < N; ++n) {
                        double *gp = g + (size_t)p * N + n;
                        *gp += dyt[p] * ct[n];
                        if (dC) dC[(ti * G + grp) * N + n] += cur[(size_t)p * N + n] * dyt[p];
                        if (dB) dB[(ti * G + grp) * N + n] += d * (*gp) * xt[p];
                        gx += (*gp) * bt[n];
                        da += (*gp) * prev[(size_t)p * N + n];
                        dd_in += (*gp) * xt[p] * bt[n];
                    }
                    if (dx) dx[(ti * H + h) * P + p] += D[h] * dyt[p] + d * gx;
                    dDh += dyt[p] * xt[p];
                }
                if (dD) dD[h] += dDh;
                if (ddt) ddt[ti * H + h] += dd_in + A[h] * a * da;
                if (dA) dA[h] += d * a * da;
                for (size_t i = 0; i < pn; ++i) g[i] *= a;
            }
            if (dinit)
                for (size_t i = 0; i < pn; ++i) dinit[((size_t)b * H + h) * pn + i] += g[i];
        }
    }
    free(hs);
    free(g);
}

/*
 * Backward of oracle_conv (with SiLU) without a tail: given dout = dL/dout,
 * ADDS dL/du, dL/dw and dL/dbias (any may be NULL).  With pre the conv's
 * pre-activation, silu'(v) = s(v) (1 + v (1 - s(v))), s the logistic sigmoid:
 *   dpre[t,c]    = dout[t,c] silu'(pre[t,c])
 *   du[src,c]   += w[c,j] dpre[t,c]   for each tap j (src as in the forward)
 *   dw[c,j]     += dpre[t,c] u[src,c]
 *   dbias[c]    += dpre[t,c]
 */
void oracle_conv_backward(const double *u, const double *w, const double *bias,
                          const double *dout, int batch, int len, int ch, int K,
                          int reverse, double *du, double *dw, double *dbias)
{
    for (int b = 0; b < batch; ++b) {
        for (int t = 0; t < len; ++t) {
            for (int c = 0; c < ch; ++c) {
                double pre = bias ? bias[c] : 0.0;
                for (int j = 0; j < K; ++j) {
                    long src = reverse ? (long)t + (K - 1) - j : (long)t - (K - 1) + j;
                    if (src >= 0 && src < len)
                        pre += w[(size_t)c * K + j] * u[((size_t)b * len + src) * ch + c];
                }
                double sg = 1.0 / (1.0 + exp(-pre));
                double dpre = dout[((size_t)b * len + t) * ch + c] * sg * (1.0 + pre * (1.0 - sg));
                if (dbias) dbias[c] += dpre;
                for (int j = 0; j < K; ++j) {
                    long src = reverse ? (long)t + (K - 1) - j : (long)t - (K - 1) + j;
                    if (src < 0 || src >= len) continue;
                    if (du) du[((size_t)b * len + src) * ch + c] += w[(size_t)c * K + j] * dpre;
                    if (dw) dw[(size_t)c * K + j] += dpre * u[((size_t)b * len + src) * ch + c];
                }
            }
        }
    }
}
