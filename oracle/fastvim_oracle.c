/*
 * fastvim_oracle.c -- fp64 CPU oracle of the FastVim SSM layer ("pooled selective scan").
 *
 * TEST INFRASTRUCTURE, NOT PRODUCT CODE: only the test suite, the package smoke check and the
 * benchmark's CPU-baseline / reference leg may call it.  Plain nested loops, no blocking, no
 * fusion, no reordering beyond what the method's definition states, so that each step can be
 * checked against the method description by eye.  Layouts and citations: fastvim_oracle.h.
 *
 * Readings of points the pages leave open (each is a choice, stated once):
 *   - POOL_W averages over the w index and leaves T = h tokens, matching the summary page's
 *     "(B,h,w,D) -> (B,h,1,D)"; POOL_H averages over h and leaves T = w.
 *   - Bbar x = Delta * B * x (Euler form of the input term) unless zoh_exact is set; Abar is
 *     always the exact exp(Delta A).
 *   - The backward scan runs t = T-1 .. 0 from a zero state and writes its output at the same
 *     t; the directions are summed without averaging before the single gate.
 *   - D has one row per direction; the skip adds (sum over directions of D) * x.
 *   - Masked pooling divides by the full pooled-over length S (w for POOL_W, h for POOL_H),
 *     not by the number of kept tokens; an empty row pools to zero and is still scanned.
 */
#include "fastvim_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static int pooled_len(int h, int w, int axis) { return axis == FVO_POOL_W ? h : w; }
static int pooled_over(int h, int w, int axis) { return axis == FVO_POOL_W ? w : h; }

static int popcount2(unsigned f) { return (int)((f & 1u) != 0) + (int)((f & 2u) != 0); }

/* softplus(v) = log(1 + e^v), written in the overflow-free form max(v,0) + log1p(e^{-|v|}). */
static double softplus(double v) { return (v > 0 ? v : 0.0) + log1p(exp(-fabs(v))); }

/* SiLU(v) = v * sigmoid(v). */
static double silu(double v) { return v / (1.0 + exp(-v)); }

/* Mean pooling (summary page, "方法详解" item 2; glossary "Mean Pooling"): for POOL_W,
 * xbar[b][i] = (1/w) sum_j x[b][i][j]; for POOL_H, xbar[b][j] = (1/h) sum_i x[b][i][j]. */
int fvo_pool(const float* x, int B, int h, int w, int E, int pool_axis, double pool_scale,
             double* xbar)
{
    if (B < 0 || h <= 0 || w <= 0 || E <= 0 || (pool_axis != FVO_POOL_W && pool_axis != FVO_POOL_H))
        return FVO_BAD_SHAPE;
    const int T = pooled_len(h, w, pool_axis), S = pooled_over(h, w, pool_axis);
    for (int b = 0; b < B; ++b)
        for (int t = 0; t < T; ++t)
            for (int e = 0; e < E; ++e) {
                double acc = 0.0;
                for (int s = 0; s < S; ++s) {
                    const int i = (pool_axis == FVO_POOL_W) ? t : s;
                    const int j = (pool_axis == FVO_POOL_W) ? s : t;
                    acc += (double)x[(((size_t)b * h + i) * w + j) * E + e];
                }
                xbar[((size_t)b * T + t) * E + e] = pool_scale * acc / (double)S;
            }
    return FVO_OK;
}

/* Row of each kept token (summary page, "方法详解" item 6: FastMaskVim transposes by the
 * kept-token index).  A grid id g = r*w + c lies in row r = g / w (POOL_W) or, after the
 * index-map transpose, in column c = g % w (POOL_H).  Ids must lie in [0, h*w) and be unique
 * within a sample.  row_off/row_tok list each row's kept tokens in ascending k. */
int fvo_mask_rows(const int32_t* keep_idx, int B, int K, int h, int w, int pool_axis,
                  int32_t* row_of, int32_t* row_off, int32_t* row_tok)
{
    if (B < 0 || K < 0 || h <= 0 || w <= 0 || (pool_axis != FVO_POOL_W && pool_axis != FVO_POOL_H))
        return FVO_BAD_SHAPE;
    const int T = pooled_len(h, w, pool_axis);
    const long G = (long)h * w;
    int status = FVO_OK;
    unsigned char* seen = (unsigned char*)calloc((size_t)G, 1);
    if (!seen) return FVO_NO_MEMORY;
    for (int b = 0; b < B; ++b) {
        memset(seen, 0, (size_t)G);
        for (int k = 0; k < K; ++k) {
            const int32_t g = keep_idx[(size_t)b * K + k];
            int32_t r = -1;
            if (g < 0 || g >= G || seen[g]) {
                status = FVO_BAD_INDEX;
            } else {
                seen[g] = 1;
                r = (pool_axis == FVO_POOL_W) ? g / w : g % w;
            }
            row_of[(size_t)b * K + k] = r;
        }
        int32_t* off = row_off + (size_t)b * (T + 1);
        for (int t = 0; t <= T; ++t) off[t] = 0;
        for (int k = 0; k < K; ++k) {
            const int32_t r = row_of[(size_t)b * K + k];
            if (r >= 0) off[r + 1] += 1;
        }
        for (int t = 0; t < T; ++t) off[t + 1] += off[t];
        int pos = 0;
        for (int t = 0; t < T; ++t)
            for (int k = 0; k < K; ++k)
                if (row_of[(size_t)b * K + k] == t) row_tok[(size_t)b * K + pos++] = k;
        for (; pos < K; ++pos) row_tok[(size_t)b * K + pos] = -1;
    }
    free(seen);
    return status;
}

/* Masked mean pooling (summary page, "方法详解" item 6: normalise by the fixed width):
 * xbar[b][t] = pool_scale * (sum over kept tokens k of row t of x[b][k]) / S. */
int fvo_pool_masked(const float* x, const int32_t* row_off, const int32_t* row_tok, int B,
                    int K, int T, int S, int E, double pool_scale, double* xbar)
{
    if (B < 0 || K < 0 || T <= 0 || S <= 0 || E <= 0) return FVO_BAD_SHAPE;
    for (int b = 0; b < B; ++b)
        for (int t = 0; t < T; ++t)
            for (int e = 0; e < E; ++e) {
                double acc = 0.0;
                for (int p = row_off[(size_t)b * (T + 1) + t]; p < row_off[(size_t)b * (T + 1) + t + 1]; ++p) {
                    const int k = row_tok[(size_t)b * K + p];
                    acc += (double)x[((size_t)b * K + k) * E + e];
                }
                xbar[((size_t)b * T + t) * E + e] = pool_scale * acc / (double)S;
            }
    return FVO_OK;
}

/* Input-dependent projections (summary page, "方法详解" item 3; glossary "Selective Scan"):
 * u = W_x xbar gives dt_low (R values), B (N) and C (N) per pooled token and direction;
 * Delta[e] = softplus(sum_r W_dt[e][r] dt_low[r] + b_dt[e]). */
int fvo_proj(const double* xbar, int B, int T, int E, int nd, int R, int N, const float* W_x,
             const float* W_dt, const float* b_dt, double* u, double* delta)
{
    if (B < 0 || T <= 0 || E <= 0 || nd < 1 || nd > 2 || R <= 0 || N <= 0) return FVO_BAD_SHAPE;
    const int J = R + 2 * N;
    const size_t M = (size_t)B * T;
    for (int k = 0; k < nd; ++k)
        for (size_t m = 0; m < M; ++m) {
            double* um = u + ((size_t)k * M + m) * J;
            for (int j = 0; j < J; ++j) {
                double acc = 0.0;
                for (int e = 0; e < E; ++e)
                    acc += (double)W_x[((size_t)k * J + j) * E + e] * xbar[m * E + e];
                um[j] = acc;
            }
            for (int e = 0; e < E; ++e) {
                double acc = (double)b_dt[(size_t)k * E + e];
                for (int r = 0; r < R; ++r)
                    acc += (double)W_dt[((size_t)k * E + e) * R + r] * um[r];
                delta[((size_t)k * M + m) * E + e] = softplus(acc);
            }
        }
    return FVO_OK;
}

/* ZOH discretisation and the selective scans (summary page, "方法详解" items 3-4; glossary
 * "State Space Model").  For direction slot k, channel e and state n, with A = -exp(A_log):
 *   Abar_t = exp(Delta_t A),  Bbar_t x_t = Delta_t B_t x_t  (zoh_exact: (Abar_t - 1)/A B_t x_t)
 *   forward : h_t = Abar_t h_{t-1} + Bbar_t x_t,  t = 0..T-1,  h_{-1} = 0
 *   backward: h_t = Abar_t h_{t+1} + Bbar_t x_t,  t = T-1..0,  h_T  = 0
 *   ys[t] += C_t . h_t  (summed over both directions). */
int fvo_scan(const double* xbar, const double* delta, const double* u, const float* A_log,
             int B, int T, int E, int nd, int R, int N, unsigned dir_flags, int zoh_exact,
             double* ys)
{
    if (B < 0 || T <= 0 || E <= 0 || R <= 0 || N <= 0 || (dir_flags & ~3u) != 0 ||
        popcount2(dir_flags) != nd)
        return FVO_BAD_SHAPE;
    const int J = R + 2 * N;
    const size_t M = (size_t)B * T;
    for (size_t m = 0; m < M * E; ++m) ys[m] = 0.0;
    int k = 0;
    for (unsigned dir = FVO_FWD; dir <= FVO_BWD; dir <<= 1) {
        if (!(dir_flags & dir)) continue;
        for (int b = 0; b < B; ++b)
            for (int e = 0; e < E; ++e)
                for (int n = 0; n < N; ++n) {
                    const double A = -exp((double)A_log[((size_t)k * E + e) * N + n]);
                    double hs = 0.0;
                    for (int step = 0; step < T; ++step) {
                        const int t = (dir == FVO_FWD) ? step : T - 1 - step;
                        const size_t m = (size_t)b * T + t;
                        const double dt = delta[((size_t)k * M + m) * E + e];
                        const double* um = u + ((size_t)k * M + m) * J;
                        const double Bn = um[R + n], Cn = um[R + N + n];
                        const double Abar = exp(dt * A);
                        const double Bbar = zoh_exact ? (Abar - 1.0) / A * Bn : dt * Bn;
                        hs = Abar * hs + Bbar * xbar[m * E + e];
                        ys[m * E + e] += Cn * hs;
                    }
                }
        ++k;
    }
    return FVO_OK;
}

/* The states the scans above pass through (the same recurrences, stored instead of read out):
 * hin[k][b][s][e][n] = the state of direction slot k entering its s-th step in scan order
 * (time t = s forward, t = T-1-s backward), so hin[.][.][0] = 0.  For the gradient, which
 * restarts the recurrence from stored states. */
int fvo_scan_states(const double* xbar, const double* delta, const double* u, const float* A_log,
                    int B, int T, int E, int nd, int R, int N, unsigned dir_flags, int zoh_exact,
                    double* hin)
{
    if (B < 0 || T <= 0 || E <= 0 || R <= 0 || N <= 0 || (dir_flags & ~3u) != 0 ||
        popcount2(dir_flags) != nd)
        return FVO_BAD_SHAPE;
    const int J = R + 2 * N;
    const size_t rows = (size_t)B * T;
    int slot = 0;
    for (unsigned d = FVO_FWD; d <= FVO_BWD; d <<= 1) {
        if ((dir_flags & d) == 0) continue;
        for (int b = 0; b < B; ++b)
            for (int e = 0; e < E; ++e)
                for (int n = 0; n < N; ++n) {
                    const double a_n = -exp((double)A_log[((size_t)slot * E + e) * N + n]);
                    double h = 0.0;
                    for (int s = 0; s < T; ++s) {
                        hin[((((size_t)slot * B + b) * T + s) * E + e) * N + n] = h;
                        const int t = d == FVO_FWD ? s : T - 1 - s;
                        const size_t row = (size_t)b * T + t;
                        const double dlt = delta[((size_t)slot * rows + row) * E + e];
                        const double bn = u[((size_t)slot * rows + row) * J + R + n];
                        const double ab = exp(dlt * a_n);
                        const double q = zoh_exact ? (ab - 1.0) / a_n * bn : dlt * bn;
                        h = ab * h + q * xbar[row * E + e];
                    }
                }
        ++slot;
    }
    return FVO_OK;
}

/* Post-SSM LayerNorm over the E channels of one token (gptget.net summary of 2502.00594,
 * "方法详解" item 5: the repeated output goes through the skip connection and a LayerNorm;
 * pith.science verdict, referee report: the post-SSM LayerNorm is the one VMamba adds before
 * the gate).  Standard layer normalisation with the biased variance:
 *   LN(s)_e = gamma_e (s_e - mu) / sqrt(var + eps) + beta_e,
 *   mu = (1/E) sum_e s_e,  var = (1/E) sum_e (s_e - mu)^2. */
static void layernorm_row(double* s, int E, const float* gamma, const float* beta, double eps)
{
    double mu = 0.0;
    for (int e = 0; e < E; ++e) mu += s[e];
    mu /= (double)E;
    double var = 0.0;
    for (int e = 0; e < E; ++e) {
        const double d = s[e] - mu;
        var += d * d;
    }
    var /= (double)E;
    const double inv = 1.0 / sqrt(var + eps);
    for (int e = 0; e < E; ++e) s[e] = (double)gamma[e] * ((s[e] - mu) * inv) + (double)beta[e];
}

static int ln_args_ok(const float* ln_gamma, const float* ln_beta, double ln_eps)
{
    if ((ln_gamma == NULL) != (ln_beta == NULL)) return 0;
    return ln_gamma == NULL || (ln_eps >= 0.0 && isfinite(ln_eps));
}

/* One output token: s = ys row + (sum_k D[k]) x (the repeat and the skip), optionally
 * LayerNorm(s), then y = SiLU(z) * s.  tmp: E doubles of scratch. */
static void gate_token(const float* x, const float* z, const double* ysr, const float* D, int E, int nd,
                       const float* ln_gamma, const float* ln_beta, double ln_eps, double* tmp, double* y)
{
    for (int e = 0; e < E; ++e) {
        double Dsum = 0.0;
        for (int k = 0; k < nd; ++k) Dsum += (double)D[(size_t)k * E + e];
        tmp[e] = ysr[e] + Dsum * (double)x[e];
    }
    if (ln_gamma) layernorm_row(tmp, E, ln_gamma, ln_beta, ln_eps);
    for (int e = 0; e < E; ++e) y[e] = silu((double)z[e]) * tmp[e];
}

/* Repeat, skip and gate (pith.science verdict, "key_machinery": the repeat restores the token
 * count before the D x skip; ijyty.com Vision Mamba article, section 2.1: gate(z, y_fwd + y_bwd)):
 *   y[b][i][j] = SiLU(z[b][i][j]) * N(ys[b][t(i,j)] + (sum_k D[k]) * x[b][i][j]),
 * N = the post-SSM LayerNorm when ln_gamma is given, else the identity. */
int fvo_gate_dense(const float* x, const float* z, const double* ys, const float* D, int B,
                   int h, int w, int E, int nd, int pool_axis, const float* ln_gamma,
                   const float* ln_beta, double ln_eps, double* y)
{
    if (B < 0 || h <= 0 || w <= 0 || E <= 0 || nd < 1 || nd > 2) return FVO_BAD_SHAPE;
    if (!ln_args_ok(ln_gamma, ln_beta, ln_eps)) return FVO_BAD_SHAPE;
    const int T = pooled_len(h, w, pool_axis);
    double* tmp = (double*)malloc(sizeof(double) * (size_t)E);
    if (!tmp) return FVO_NO_MEMORY;
    for (int b = 0; b < B; ++b)
        for (int i = 0; i < h; ++i)
            for (int j = 0; j < w; ++j) {
                const int t = (pool_axis == FVO_POOL_W) ? i : j;
                const size_t g = (((size_t)b * h + i) * w + j) * E;
                gate_token(x + g, z + g, ys + ((size_t)b * T + t) * E, D, E, nd, ln_gamma, ln_beta, ln_eps,
                           tmp, y + g);
            }
    free(tmp);
    return FVO_OK;
}

/* Masked form: each kept token takes the pooled output of its row (repeat only to kept
 * indices).  A token whose index was rejected (row_of < 0) gets 0. */
int fvo_gate_masked(const float* x, const float* z, const double* ys, const float* D,
                    const int32_t* row_of, int B, int K, int T, int E, int nd, const float* ln_gamma,
                    const float* ln_beta, double ln_eps, double* y)
{
    if (B < 0 || K < 0 || T <= 0 || E <= 0 || nd < 1 || nd > 2) return FVO_BAD_SHAPE;
    if (!ln_args_ok(ln_gamma, ln_beta, ln_eps)) return FVO_BAD_SHAPE;
    double* tmp = (double*)malloc(sizeof(double) * (size_t)E);
    if (!tmp) return FVO_NO_MEMORY;
    for (int b = 0; b < B; ++b)
        for (int k = 0; k < K; ++k) {
            const int32_t t = row_of[(size_t)b * K + k];
            const size_t g = ((size_t)b * K + k) * E;
            if (t < 0) {
                for (int e = 0; e < E; ++e) y[g + e] = 0.0;
                continue;
            }
            gate_token(x + g, z + g, ys + ((size_t)b * T + t) * E, D, E, nd, ln_gamma, ln_beta, ln_eps, tmp,
                       y + g);
        }
    free(tmp);
    return FVO_OK;
}

/* ---- The block's Conv1D in front of the layer -------------------------------------------------
 * gptget.net summary of 2502.00594, "方法详解" item 2: the tokens go through Norm, the expansion
 * layer and a Conv1D, and the layer pools the Conv1D's output; ijyty.com Vision Mamba article,
 * section 2.1 code: the forward and the backward SSM each take the output of their own Conv1D
 * of the expanded tokens, the backward one run over the reversed sequence.
 * Readings taken (the pages give no more):
 *   - depthwise (one filter of dc taps and a bias per channel and direction), zero padding;
 *   - the block's token sequence runs line by line along the pooled-over axis: position
 *     p = t * S + s holds token (i, j) = (t, s) under POOL_W and (s, t) under POOL_H (the
 *     transposed grid of an alternate block, flattened row by row), L = h * w positions;
 *   - forward slot:  xc[p] = act(b + sum_{q<dc} w[q] x[p - (dc-1) + q])  (x = 0 before p = 0)
 *     backward slot: xc[p] = act(b + sum_{q<dc} w[q] x[p + (dc-1) - q])  (x = 0 past L - 1),
 *     i.e. the same causal filter run over the reversed sequence and reversed back;
 *   - act is the identity, or SiLU when conv_silu is set (Mamba-family blocks follow the
 *     Conv1D with SiLU; the pages do not say).
 * Layouts: conv_w [nd][E][dc], conv_b [nd][E]; xc [nd][B][h][w][E] (the grid layout of x). */
static void seq_token(int p, int h, int w, int pool_axis, int* i, int* j)
{
    const int S = pooled_over(h, w, pool_axis);
    const int t = p / S, s = p % S;
    *i = (pool_axis == FVO_POOL_W) ? t : s;
    *j = (pool_axis == FVO_POOL_W) ? s : t;
}

int fvo_conv(const float* x, int B, int h, int w, int E, int pool_axis, unsigned dir_flags, int dc,
             const float* conv_w, const float* conv_b, int conv_silu, double* xc)
{
    if (B < 0 || h <= 0 || w <= 0 || E <= 0 || dc < 1 || (dir_flags & ~3u) != 0 || dir_flags == 0 ||
        (pool_axis != FVO_POOL_W && pool_axis != FVO_POOL_H))
        return FVO_BAD_SHAPE;
    const int L = h * w;
    const size_t img = (size_t)L * E;
    int k = 0;
    for (unsigned dir = FVO_FWD; dir <= FVO_BWD; dir <<= 1) {
        if (!(dir_flags & dir)) continue;
        for (int b = 0; b < B; ++b)
            for (int p = 0; p < L; ++p) {
                int i, j;
                seq_token(p, h, w, pool_axis, &i, &j);
                for (int e = 0; e < E; ++e) {
                    double acc = (double)conv_b[(size_t)k * E + e];
                    for (int q = 0; q < dc; ++q) {
                        const int pp = (dir == FVO_FWD) ? p - (dc - 1) + q : p + (dc - 1) - q;
                        if (pp < 0 || pp >= L) continue;
                        int ii, jj;
                        seq_token(pp, h, w, pool_axis, &ii, &jj);
                        acc += (double)conv_w[((size_t)k * E + e) * dc + q] *
                               (double)x[(size_t)b * img + ((size_t)ii * w + jj) * E + e];
                    }
                    xc[((size_t)k * B + b) * img + ((size_t)i * w + j) * E + e] = conv_silu ? silu(acc) : acc;
                }
            }
        ++k;
    }
    return FVO_OK;
}

/* Mean pooling (as fvo_pool) of a grid held in fp64: the convolved tokens. */
int fvo_pool_d(const double* x, int B, int h, int w, int E, int pool_axis, double pool_scale, double* xbar)
{
    if (B < 0 || h <= 0 || w <= 0 || E <= 0 || (pool_axis != FVO_POOL_W && pool_axis != FVO_POOL_H))
        return FVO_BAD_SHAPE;
    const int T = pooled_len(h, w, pool_axis), S = pooled_over(h, w, pool_axis);
    for (int b = 0; b < B; ++b)
        for (int t = 0; t < T; ++t)
            for (int e = 0; e < E; ++e) {
                double acc = 0.0;
                for (int s = 0; s < S; ++s) {
                    const int i = (pool_axis == FVO_POOL_W) ? t : s;
                    const int j = (pool_axis == FVO_POOL_W) ? s : t;
                    acc += x[(((size_t)b * h + i) * w + j) * E + e];
                }
                xbar[((size_t)b * T + t) * E + e] = pool_scale * acc / (double)S;
            }
    return FVO_OK;
}

/* Repeat + skip (+ LayerNorm) + gate when every direction has its own convolved input:
 *   y[b][i][j] = SiLU(z[b][i][j]) * N(ys[b][t(i,j)] + sum_k D[k] * xc[k][b][i][j]). */
int fvo_gate_dense_conv(const double* xc, const float* z, const double* ys, const float* D, int B, int h,
                        int w, int E, int nd, int pool_axis, const float* ln_gamma, const float* ln_beta,
                        double ln_eps, double* y)
{
    if (B < 0 || h <= 0 || w <= 0 || E <= 0 || nd < 1 || nd > 2) return FVO_BAD_SHAPE;
    if (!ln_args_ok(ln_gamma, ln_beta, ln_eps)) return FVO_BAD_SHAPE;
    const int T = pooled_len(h, w, pool_axis);
    const size_t all = (size_t)B * h * w * E;
    double* tmp = (double*)malloc(sizeof(double) * (size_t)E);
    if (!tmp) return FVO_NO_MEMORY;
    for (int b = 0; b < B; ++b)
        for (int i = 0; i < h; ++i)
            for (int j = 0; j < w; ++j) {
                const int t = (pool_axis == FVO_POOL_W) ? i : j;
                const size_t g = (((size_t)b * h + i) * w + j) * E;
                for (int e = 0; e < E; ++e) {
                    double v = ys[((size_t)b * T + t) * E + e];
                    for (int k = 0; k < nd; ++k) v += (double)D[(size_t)k * E + e] * xc[(size_t)k * all + g + e];
                    tmp[e] = v;
                }
                if (ln_gamma) layernorm_row(tmp, E, ln_gamma, ln_beta, ln_eps);
                for (int e = 0; e < E; ++e) y[g + e] = silu((double)z[g + e]) * tmp[e];
            }
    free(tmp);
    return FVO_OK;
}

/* One image of the layer with the Conv1D in front: each direction slot k convolves x with its
 * own filter, pools its own convolved tokens, projects and scans them with its own parameters;
 * the scan outputs are summed and the skip adds each direction's D times its own convolved
 * input.  Scratch: xc [nd][h][w][E], xbar [T][E], u [T][J], delta [T][E], ys and ysk [T][E]. */
static int forward_one_conv(const float* x, const float* z, const float* A_log, const float* D,
                            const float* W_x, const float* W_dt, const float* b_dt, int h, int w, int E,
                            int N, int R, int pool_axis, unsigned dir_flags, double pool_scale, int zoh_exact,
                            int dc, const float* conv_w, const float* conv_b, int conv_silu,
                            const float* ln_gamma, const float* ln_beta, double ln_eps, double* y,
                            double* xc, double* xbar, double* u, double* delta, double* ys, double* ysk)
{
    const int nd = popcount2(dir_flags);
    const int T = pooled_len(h, w, pool_axis);
    const int J = R + 2 * N;
    const size_t img = (size_t)h * w * E;
    int st = fvo_conv(x, 1, h, w, E, pool_axis, dir_flags, dc, conv_w, conv_b, conv_silu, xc);
    if (st) return st;
    for (size_t m = 0; m < (size_t)T * E; ++m) ys[m] = 0.0;
    int k = 0;
    for (unsigned dir = FVO_FWD; dir <= FVO_BWD; dir <<= 1) {
        if (!(dir_flags & dir)) continue;
        if ((st = fvo_pool_d(xc + (size_t)k * img, 1, h, w, E, pool_axis, pool_scale, xbar))) return st;
        if ((st = fvo_proj(xbar, 1, T, E, 1, R, N, W_x + (size_t)k * J * E, W_dt + (size_t)k * E * R,
                           b_dt + (size_t)k * E, u, delta)))
            return st;
        if ((st = fvo_scan(xbar, delta, u, A_log + (size_t)k * E * N, 1, T, E, 1, R, N, dir, zoh_exact, ysk)))
            return st;
        for (size_t m = 0; m < (size_t)T * E; ++m) ys[m] += ysk[m];
        ++k;
    }
    return fvo_gate_dense_conv(xc, z, ys, D, 1, h, w, E, nd, pool_axis, ln_gamma, ln_beta, ln_eps, y);
}

int fvo_forward_conv(const float* x, const float* z, const float* A_log, const float* D,
                     const float* W_x, const float* W_dt, const float* b_dt, int B, int h, int w, int E,
                     int N, int R, int pool_axis, unsigned dir_flags, double pool_scale, int zoh_exact, int dc,
                     const float* conv_w, const float* conv_b, int conv_silu, const float* ln_gamma,
                     const float* ln_beta, double ln_eps, int nthreads, double* y)
{
    const int nd = popcount2(dir_flags);
    if (B < 0 || h <= 0 || w <= 0 || E <= 0 || N <= 0 || R <= 0 || nd < 1 || dc < 1 ||
        (dir_flags & ~3u) != 0 || (pool_axis != FVO_POOL_W && pool_axis != FVO_POOL_H) || !conv_w ||
        !conv_b || !ln_args_ok(ln_gamma, ln_beta, ln_eps))
        return FVO_BAD_SHAPE;
    const int T = pooled_len(h, w, pool_axis);
    const int J = R + 2 * N;
    const size_t img = (size_t)h * w * E;
    int status = FVO_OK;
    if (nthreads < 1) nthreads = 1;
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads) if (nthreads > 1)
#endif
    for (int b = 0; b < B; ++b) {
        double* xc = (double*)malloc(sizeof(double) * (size_t)nd * img);
        double* xbar = (double*)malloc(sizeof(double) * (size_t)T * E);
        double* u = (double*)malloc(sizeof(double) * (size_t)T * J);
        double* delta = (double*)malloc(sizeof(double) * (size_t)T * E);
        double* ys = (double*)malloc(sizeof(double) * (size_t)T * E);
        double* ysk = (double*)malloc(sizeof(double) * (size_t)T * E);
        int st = FVO_NO_MEMORY;
        if (xc && xbar && u && delta && ys && ysk)
            st = forward_one_conv(x + (size_t)b * img, z + (size_t)b * img, A_log, D, W_x, W_dt, b_dt, h, w, E, N,
                                  R, pool_axis, dir_flags, pool_scale, zoh_exact, dc, conv_w, conv_b, conv_silu,
                                  ln_gamma, ln_beta, ln_eps, y + (size_t)b * img, xc, xbar, u, delta, ys, ysk);
        free(xc); free(xbar); free(u); free(delta); free(ys); free(ysk);
        if (st != FVO_OK) {
#ifdef _OPENMP
#pragma omp critical
#endif
            {
                if (status == FVO_OK) status = st;
            }
        }
    }
    return status;
}

/* One image through the whole chain; scratch is owned by the caller. */
static int forward_one(const float* x, const float* z, const float* A_log, const float* D,
                       const float* W_x, const float* W_dt, const float* b_dt,
                       const int32_t* keep_idx, int h, int w, int E, int N, int R, int K,
                       int pool_axis, unsigned dir_flags, double pool_scale, int zoh_exact,
                       const float* ln_gamma, const float* ln_beta, double ln_eps,
                       double* y, double* xbar, double* u, double* delta, double* ys,
                       int32_t* row_of, int32_t* row_off, int32_t* row_tok)
{
    const int nd = popcount2(dir_flags);
    const int T = pooled_len(h, w, pool_axis), S = pooled_over(h, w, pool_axis);
    int st, idx_status = FVO_OK;
    if (keep_idx) {
        idx_status = fvo_mask_rows(keep_idx, 1, K, h, w, pool_axis, row_of, row_off, row_tok);
        if (idx_status != FVO_OK && idx_status != FVO_BAD_INDEX) return idx_status;
        st = fvo_pool_masked(x, row_off, row_tok, 1, K, T, S, E, pool_scale, xbar);
    } else {
        st = fvo_pool(x, 1, h, w, E, pool_axis, pool_scale, xbar);
    }
    if (st) return st;
    if ((st = fvo_proj(xbar, 1, T, E, nd, R, N, W_x, W_dt, b_dt, u, delta))) return st;
    if ((st = fvo_scan(xbar, delta, u, A_log, 1, T, E, nd, R, N, dir_flags, zoh_exact, ys))) return st;
    if (keep_idx)
        st = fvo_gate_masked(x, z, ys, D, row_of, 1, K, T, E, nd, ln_gamma, ln_beta, ln_eps, y);
    else
        st = fvo_gate_dense(x, z, ys, D, 1, h, w, E, nd, pool_axis, ln_gamma, ln_beta, ln_eps, y);
    return st ? st : idx_status;
}

int fvo_forward(const float* x, const float* z, const float* A_log, const float* D,
                const float* W_x, const float* W_dt, const float* b_dt,
                const int32_t* keep_idx, int B, int h, int w, int E, int N, int R, int K,
                int pool_axis, unsigned dir_flags, double pool_scale, int zoh_exact,
                const float* ln_gamma, const float* ln_beta, double ln_eps, int nthreads, double* y)
{
    const int nd = popcount2(dir_flags);
    if (B < 0 || h <= 0 || w <= 0 || E <= 0 || N <= 0 || R <= 0 || nd < 1 ||
        (dir_flags & ~3u) != 0 || (pool_axis != FVO_POOL_W && pool_axis != FVO_POOL_H) ||
        (keep_idx && (K < 0 || K > h * w)) || !ln_args_ok(ln_gamma, ln_beta, ln_eps))
        return FVO_BAD_SHAPE;
    const int T = pooled_len(h, w, pool_axis);
    const int J = R + 2 * N;
    const size_t tok = keep_idx ? (size_t)K : (size_t)h * w;
    int status = FVO_OK;
    if (nthreads < 1) nthreads = 1;
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads) if (nthreads > 1)
#endif
    for (int b = 0; b < B; ++b) {
        double* xbar = (double*)malloc(sizeof(double) * (size_t)T * E);
        double* u = (double*)malloc(sizeof(double) * (size_t)nd * T * J);
        double* delta = (double*)malloc(sizeof(double) * (size_t)nd * T * E);
        double* ys = (double*)malloc(sizeof(double) * (size_t)T * E);
        int32_t* row_of = (int32_t*)malloc(sizeof(int32_t) * (size_t)(K > 0 ? K : 1));
        int32_t* row_off = (int32_t*)malloc(sizeof(int32_t) * (size_t)(T + 1));
        int32_t* row_tok = (int32_t*)malloc(sizeof(int32_t) * (size_t)(K > 0 ? K : 1));
        int st = FVO_NO_MEMORY;
        if (xbar && u && delta && ys && row_of && row_off && row_tok)
            st = forward_one(x + (size_t)b * tok * E, z + (size_t)b * tok * E, A_log, D, W_x,
                             W_dt, b_dt, keep_idx ? keep_idx + (size_t)b * K : NULL, h, w, E, N,
                             R, K, pool_axis, dir_flags, pool_scale, zoh_exact, ln_gamma, ln_beta,
                             ln_eps, y + (size_t)b * tok * E, xbar, u, delta, ys, row_of, row_off, row_tok);
        free(xbar); free(u); free(delta); free(ys); free(row_of); free(row_off); free(row_tok);
        if (st != FVO_OK) {
#ifdef _OPENMP
#pragma omp critical
#endif
            {
                if (status == FVO_OK || status == FVO_BAD_INDEX) status = st;
            }
        }
    }
    return status;
}
