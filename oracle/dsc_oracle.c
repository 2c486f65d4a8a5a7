/*
 * CPU oracle for the causal dynamic short convolution.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or call
 * this file; only the tests, the smoke check and the benchmark's CPU-baseline leg
 * use it.  It shares no code, header, table or helper with the CUDA library.
 *
 * Plain, single-threaded C in double precision, written from the defining
 * formulas of "Convolucoes Curtas Dinamicas Melhoram Transformers"
 * (gist.science/pt/paper/2606.03825), section "Metodologia > Convolucoes Curtas
 * Dinamicas":
 *   - Mecanismo:       y_t = sum_{k=0}^{W-1} w(t)_k (.) x_{t-k}
 *   - Parametrizacao:  w(t) from a learned linear map; (1) low-rank factorisation
 *                      of rank R, w(t) = z_t U; (2) head-wise tying, one filter
 *                      shared by G consecutive channels
 *   - Posicionamento:  residual, X = X + dynamicShortConv(X)
 * and the static depthwise causal convolution that the method generalises
 * (same page, "Declaracao do Problema").
 *
 * Readings taken where the page is silent:
 *   - positions before the start of a sequence count as zero, per sequence b;
 *   - tap k = 0 multiplies the current token x_t;
 *   - channel c belongs to filter group g(c) = floor(c / G);
 *   - U column j = g*W + k, so reshape(z U, [B,T,D/G,W]) is the explicit w;
 *   - no normalisation, bias or scaling is applied to w;
 *   - the residual is always added.
 *
 * Layouts (row-major, all contiguous):
 *   x, y, dy, dx : [B, T, D]
 *   w, dw        : [B, T, D/G, W]        (explicit dynamic filters)
 *   z, dz        : [B, T, R]
 *   U, dU        : [R, (D/G)*W]
 *   ws, dws      : [D, W]                (static filters)
 *
 * The backward functions follow from the forward by the chain rule; y is linear
 * in x and in w, so
 *   dx[b,s,c]   = dy[b,s,c] + sum_{k<W, s+k<T} w[b,s+k,g(c),k] dy[b,s+k,c]
 *   dw[b,t,g,k] = sum_{c: g(c)=g, t-k>=0} dy[b,t,c] x[b,t-k,c]
 *   dz[b,t,r]   = sum_j dw[b,t,j] U[r,j]
 *   dU[r,j]     = sum_{b,t} z[b,t,r] dw[b,t,j]
 * The backward is written in scatter form: one token's filter row at a time,
 * each product added into the dx row it belongs to.
 */
#include <stdlib.h>
#include <string.h>

/* y = x + dynconv(x; w), explicit filters. */
void oracle_fwd(const double *x, const double *w, double *y,
                int B, int T, int D, int G, int W)
{
    const int NG = D / G;
    for (int b = 0; b < B; ++b)
        for (int t = 0; t < T; ++t)
            for (int c = 0; c < D; ++c) {
                const int g = c / G;
                const double *wt = w + (((size_t)b * T + t) * NG + g) * W;
                double acc = x[((size_t)b * T + t) * D + c];
                for (int k = 0; k < W; ++k) {
                    if (t - k < 0) break;
                    acc += wt[k] * x[((size_t)b * T + (t - k)) * D + c];
                }
                y[((size_t)b * T + t) * D + c] = acc;
            }
}

/* w[b,t,:] = z[b,t,:] U  (plain triple loop; column j = g*W + k). */
void oracle_lowrank_weights(const double *z, const double *U, double *w,
                            int B, int T, int D, int G, int W, int R)
{
    const int N = (D / G) * W;
    for (size_t bt = 0; bt < (size_t)B * T; ++bt)
        for (int j = 0; j < N; ++j) {
            double s = 0.0;
            for (int r = 0; r < R; ++r)
                s += z[bt * R + r] * U[(size_t)r * N + j];
            w[bt * N + j] = s;
        }
}

/* y = x + dynconv(x; w = z U), the filter row of token t formed from z_t. */
int oracle_fwd_lowrank(const double *x, const double *z, const double *U, double *y,
                       int B, int T, int D, int G, int W, int R)
{
    const int N = (D / G) * W;
    double *wt = (double *)malloc(sizeof(double) * (size_t)N);
    if (!wt) return 1;
    for (int b = 0; b < B; ++b)
        for (int t = 0; t < T; ++t) {
            const size_t bt = (size_t)b * T + t;
            for (int j = 0; j < N; ++j) {
                double s = 0.0;
                for (int r = 0; r < R; ++r)
                    s += z[bt * R + r] * U[(size_t)r * N + j];
                wt[j] = s;
            }
            for (int c = 0; c < D; ++c) {
                const int g = c / G;
                double acc = x[bt * D + c];
                for (int k = 0; k < W; ++k) {
                    if (t - k < 0) break;
                    acc += wt[g * W + k] * x[(bt - k) * D + c];
                }
                y[bt * D + c] = acc;
            }
        }
    free(wt);
    return 0;
}

/* Backward of oracle_fwd: dx [B,T,D] and dw [B,T,D/G,W]. */
void oracle_bwd(const double *x, const double *w, const double *dy,
                double *dx, double *dw, int B, int T, int D, int G, int W)
{
    const int NG = D / G;
    const size_t nx = (size_t)B * T * D;
    memcpy(dx, dy, sizeof(double) * nx);               /* residual path */
    memset(dw, 0, sizeof(double) * (size_t)B * T * NG * W);
    for (int b = 0; b < B; ++b)
        for (int t = 0; t < T; ++t) {
            const size_t bt = (size_t)b * T + t;
            for (int c = 0; c < D; ++c) {
                const int g = c / G;
                const double gy = dy[bt * D + c];
                for (int k = 0; k < W; ++k) {
                    if (t - k < 0) break;
                    /* y_t[c] += w_t[g,k] x_{t-k}[c] */
                    dx[(bt - k) * D + c] += w[(bt * NG + g) * W + k] * gy;
                    dw[(bt * NG + g) * W + k] += gy * x[(bt - k) * D + c];
                }
            }
        }
}

/* Backward of oracle_fwd_lowrank: dx [B,T,D], dz [B,T,R], dU [R,(D/G)*W]. */
int oracle_bwd_lowrank(const double *x, const double *z, const double *U, const double *dy,
                       double *dx, double *dz, double *dU,
                       int B, int T, int D, int G, int W, int R)
{
    const int N = (D / G) * W;
    double *wt = (double *)malloc(sizeof(double) * (size_t)N);
    double *dwt = (double *)malloc(sizeof(double) * (size_t)N);
    if (!wt || !dwt) { free(wt); free(dwt); return 1; }
    memcpy(dx, dy, sizeof(double) * (size_t)B * T * D);  /* residual path */
    memset(dU, 0, sizeof(double) * (size_t)R * N);
    for (int b = 0; b < B; ++b)
        for (int t = 0; t < T; ++t) {
            const size_t bt = (size_t)b * T + t;
            for (int j = 0; j < N; ++j) {
                double s = 0.0;
                for (int r = 0; r < R; ++r)
                    s += z[bt * R + r] * U[(size_t)r * N + j];
                wt[j] = s;
                dwt[j] = 0.0;
            }
            for (int c = 0; c < D; ++c) {
                const int g = c / G;
                const double gy = dy[bt * D + c];
                for (int k = 0; k < W; ++k) {
                    if (t - k < 0) break;
                    dx[(bt - k) * D + c] += wt[g * W + k] * gy;
                    dwt[g * W + k] += gy * x[(bt - k) * D + c];
                }
            }
            /* w_t = z_t U  =>  dz_t = dw_t U^T,  dU += z_t^T dw_t */
            for (int r = 0; r < R; ++r) {
                double s = 0.0;
                for (int j = 0; j < N; ++j)
                    s += dwt[j] * U[(size_t)r * N + j];
                dz[bt * R + r] = s;
                const double zr = z[bt * R + r];
                for (int j = 0; j < N; ++j)
                    dU[(size_t)r * N + j] += zr * dwt[j];
            }
        }
    free(wt);
    free(dwt);
    return 0;
}

/* Static depthwise causal convolution: y = x + conv(x; ws), ws [D,W] fixed over t. */
void oracle_static_fwd(const double *x, const double *ws, double *y,
                       int B, int T, int D, int W)
{
    for (int b = 0; b < B; ++b)
        for (int t = 0; t < T; ++t)
            for (int c = 0; c < D; ++c) {
                double acc = x[((size_t)b * T + t) * D + c];
                for (int k = 0; k < W; ++k) {
                    if (t - k < 0) break;
                    acc += ws[(size_t)c * W + k] * x[((size_t)b * T + (t - k)) * D + c];
                }
                y[((size_t)b * T + t) * D + c] = acc;
            }
}

/* Backward of oracle_static_fwd: dx [B,T,D], dws [D,W] summed over all b, t. */
void oracle_static_bwd(const double *x, const double *ws, const double *dy,
                       double *dx, double *dws, int B, int T, int D, int W)
{
    memcpy(dx, dy, sizeof(double) * (size_t)B * T * D);
    memset(dws, 0, sizeof(double) * (size_t)D * W);
    for (int b = 0; b < B; ++b)
        for (int t = 0; t < T; ++t)
            for (int c = 0; c < D; ++c) {
                const size_t bt = (size_t)b * T + t;
                const double gy = dy[bt * D + c];
                for (int k = 0; k < W; ++k) {
                    if (t - k < 0) break;
                    dx[(bt - k) * D + c] += ws[(size_t)c * W + k] * gy;
                    dws[(size_t)c * W + k] += gy * x[(bt - k) * D + c];
                }
            }
}

/*
 * One decode step: token t of each of B sequences, with the W-1 tokens before it
 * taken from a rolling window instead of from the sequence itself (the page notes
 * that inference still needs engineering: "Significancia e Alegacoes").  The same
 * formula as above at a single position:
 *   y_t[c] = x_t[c] + w_t[g(c),0] x_t[c] + sum_{k=1}^{W-1} w_t[g(c),k] x_{t-k}[c]
 * Layouts (row-major):
 *   x_t, y_t   : [B, D]
 *   state      : [B, W-1, D], row i holds x_{t-(W-1)+i} (oldest first; zeros before
 *                the start of a sequence), so x_{t-k} is row W-1-k
 *   state_out  : [B, W-1, D], the window after the step: rows shifted by one, x_t last
 */
static void decode_one(const double *x_t, const double *wt, const double *state,
                       double *y_t, double *state_out, int D, int G, int W)
{
    for (int c = 0; c < D; ++c) {
        const int g = c / G;
        double acc = x_t[c];
        acc += wt[g * W + 0] * x_t[c];
        for (int k = 1; k < W; ++k)
            acc += wt[g * W + k] * state[(size_t)(W - 1 - k) * D + c];
        y_t[c] = acc;
    }
    for (int i = 0; i + 1 < W - 1; ++i)
        for (int c = 0; c < D; ++c)
            state_out[(size_t)i * D + c] = state[(size_t)(i + 1) * D + c];
    if (W > 1)
        for (int c = 0; c < D; ++c)
            state_out[(size_t)(W - 2) * D + c] = x_t[c];
}

/* Decode step with explicit filters w_t [B, D/G, W]. */
void oracle_decode(const double *x_t, const double *w_t, const double *state,
                   double *y_t, double *state_out, int B, int D, int G, int W)
{
    const int NG = D / G;
    for (int b = 0; b < B; ++b)
        decode_one(x_t + (size_t)b * D, w_t + (size_t)b * NG * W,
                   state + (size_t)b * (W - 1) * D, y_t + (size_t)b * D,
                   state_out + (size_t)b * (W - 1) * D, D, G, W);
}

/* Decode step with low-rank filters w_t = z_t U; z_t [B, R], U [R, (D/G)*W]. */
int oracle_decode_lowrank(const double *x_t, const double *z_t, const double *U,
                          const double *state, double *y_t, double *state_out,
                          int B, int D, int G, int W, int R)
{
    const int N = (D / G) * W;
    double *wt = (double *)malloc(sizeof(double) * (size_t)N);
    if (!wt) return 1;
    for (int b = 0; b < B; ++b) {
        for (int j = 0; j < N; ++j) {
            double s = 0.0;
            for (int r = 0; r < R; ++r)
                s += z_t[(size_t)b * R + r] * U[(size_t)r * N + j];
            wt[j] = s;
        }
        decode_one(x_t + (size_t)b * D, wt, state + (size_t)b * (W - 1) * D,
                   y_t + (size_t)b * D, state_out + (size_t)b * (W - 1) * D, D, G, W);
    }
    free(wt);
    return 0;
}

/* Rotary position embedding of the first n_rot channels of y, in place.
 *
 * "Metodologia > Convolucoes Curtas Dinamicas > Posicionamento": the convolution is
 * applied to the Q, K and V projections before RoPE, so the op's output on the Q and K
 * channels is rotated next.  Reading: RoPE in its original form, pairs of adjacent
 * channels (2i, 2i+1) of each head of dh channels rotated by the angle of pair i at
 * the token's position t in its sequence, whose cosine and sine are given:
 *   y'[2i]   = y[2i] cos - y[2i+1] sin
 *   y'[2i+1] = y[2i] sin + y[2i+1] cos
 * Channels n_rot..D-1 (V) are not rotated.  transpose != 0 applies the inverse
 * rotation (angle -theta), which is the transpose the backward needs.
 *   y  : [B, T, D]
 *   cs : [T, dh/2, 2]   (cos, sin) per position and pair
 * Requires dh even and n_rot a multiple of dh, n_rot <= D. */
void oracle_rope(double *y, const double *cs, int B, int T, int D, int dh, int n_rot, int transpose)
{
    const int np = dh / 2;
    for (int b = 0; b < B; ++b)
        for (int t = 0; t < T; ++t) {
            double *row = y + ((size_t)b * T + t) * D;
            for (int c0 = 0; c0 < n_rot; c0 += dh)
                for (int i = 0; i < np; ++i) {
                    const double co = cs[((size_t)t * np + i) * 2 + 0];
                    const double si = transpose ? -cs[((size_t)t * np + i) * 2 + 1]
                                                : cs[((size_t)t * np + i) * 2 + 1];
                    const double a = row[c0 + 2 * i], e = row[c0 + 2 * i + 1];
                    row[c0 + 2 * i] = a * co - e * si;
                    row[c0 + 2 * i + 1] = a * si + e * co;
                }
        }
}
