/*
 * fastvim_oracle.h -- fp64 CPU oracle of the FastVim SSM layer ("pooled selective scan").
 *
 * TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only the test suite, the package's smoke check and
 * the benchmark's CPU-baseline / reference leg may load or call this library.  It shares no
 * code, header, table or helper with the CUDA library; the two only ever meet through the
 * seeded synthetic inputs that both are handed.
 *
 * What it computes follows the method description of FastVim (Kapse et al., arXiv 2502.00594):
 *   - gptget.net summary of 2502.00594, section "方法详解" (method details), items 1-6:
 *     reshape to (B,h,w,D), mean-pool along one grid axis to (B,h,1,D), input-dependent
 *     B, C and Delta = softplus(Parameter + s_Delta(x)), ZOH discretisation, forward and
 *     backward selective scan of the pooled sequence, repeat along the pooled axis, skip;
 *   - same page, glossary "State Space Model": h_t = A h_{t-1} + B x_t, y_t = C h_t + D x_t;
 *   - pith.science verdict on 2502.00594, field "key_machinery": the repeat restores the token
 *     count before the D x_t skip connection (so the skip uses full-resolution x);
 *   - ijyty.com Vision Mamba article, section 2.1 code: the block gates the sum of the forward
 *     and backward SSM outputs with z;
 *   - optional post-SSM LayerNorm after the skip and before the gate (summary page, "方法详解"
 *     item 5; verdict page, referee report on the VMamba post-SSM LayerNorm).
 *
 * All arithmetic is fp64; inputs are fp32 arrays as the GPU library sees them.
 * Layouts (row-major, last index fastest):
 *   dense  x, z        [B][h][w][E]          masked x, z      [B][K][E]
 *   keep_idx           [B][K] int32, grid id r*w + c
 *   A_log              [nd][E][N]            D                [nd][E]
 *   W_x                [nd][R+2N][E]  (rows: dt_low | B | C)
 *   W_dt               [nd][E][R]            b_dt             [nd][E]
 *   xbar               [B][T][E]             u                [nd][B][T][R+2N]
 *   delta              [nd][B][T][E]         ys               [B][T][E]
 * Parameter slot k (0..nd-1) belongs to the k-th enabled direction in the order FWD, BWD.
 */
#ifndef FASTVIM_ORACLE_H
#define FASTVIM_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { FVO_OK = 0, FVO_BAD_SHAPE = 2, FVO_BAD_INDEX = 4, FVO_NO_MEMORY = 8 };
enum { FVO_POOL_W = 0, FVO_POOL_H = 1 };
enum { FVO_FWD = 1, FVO_BWD = 2 };

/* Mean pooling of a dense grid along one axis (pooled length T, pooled-over length S). */
int fvo_pool(const float* x, int B, int h, int w, int E, int pool_axis, double pool_scale,
             double* xbar);

/* Row bucketing of kept-token indices: row_of[B][K] (pooled token of each kept token),
 * row_off[B][T+1] and row_tok[B][K] (kept-token ordinals grouped by row, ascending k). */
int fvo_mask_rows(const int32_t* keep_idx, int B, int K, int h, int w, int pool_axis,
                  int32_t* row_of, int32_t* row_off, int32_t* row_tok);

/* Masked pooling: xbar[b][t] = pool_scale * (sum of kept tokens in row t) / S. */
int fvo_pool_masked(const float* x, const int32_t* row_off, const int32_t* row_tok, int B,
                    int K, int T, int S, int E, double pool_scale, double* xbar);

/* x_proj and dt_proj + softplus on the pooled tokens. */
int fvo_proj(const double* xbar, int B, int T, int E, int nd, int R, int N, const float* W_x,
             const float* W_dt, const float* b_dt, double* u, double* delta);

/* ZOH discretisation + forward/backward selective scans, directions summed. zoh_exact = 0:
 * Bbar x = Delta B x; zoh_exact = 1: Bbar = (exp(Delta A) - 1) / A * B. */
int fvo_scan(const double* xbar, const double* delta, const double* u, const float* A_log,
             int B, int T, int E, int nd, int R, int N, unsigned dir_flags, int zoh_exact,
             double* ys);

/* The scans' states: hin [nd][B][T][E][N], hin[k][b][s] = the state of direction slot k entering
 * its s-th step in scan order (zero at s = 0). */
int fvo_scan_states(const double* xbar, const double* delta, const double* u, const float* A_log,
                    int B, int T, int E, int nd, int R, int N, unsigned dir_flags, int zoh_exact,
                    double* hin);

/* Repeat + D x skip (+ the post-SSM LayerNorm over E when ln_gamma, ln_beta [E] are given,
 * both or neither, ln_eps >= 0) + SiLU(z) gate on the dense grid. */
int fvo_gate_dense(const float* x, const float* z, const double* ys, const float* D, int B,
                   int h, int w, int E, int nd, int pool_axis, const float* ln_gamma,
                   const float* ln_beta, double ln_eps, double* y);

/* Same on the kept tokens, each taking the pooled output of its row. */
int fvo_gate_masked(const float* x, const float* z, const double* ys, const float* D,
                    const int32_t* row_of, int B, int K, int T, int E, int nd, const float* ln_gamma,
                    const float* ln_beta, double ln_eps, double* y);

/* The whole layer, one image at a time (OpenMP over images when nthreads > 1).
 * keep_idx == NULL: dense x, z, y [B][h][w][E]; otherwise masked [B][K][E]. */
int fvo_forward(const float* x, const float* z, const float* A_log, const float* D,
                const float* W_x, const float* W_dt, const float* b_dt,
                const int32_t* keep_idx, int B, int h, int w, int E, int N, int R, int K,
                int pool_axis, unsigned dir_flags, double pool_scale, int zoh_exact,
                const float* ln_gamma, const float* ln_beta, double ln_eps, int nthreads, double* y);

/* The block's Conv1D in front of the layer (depthwise, dc taps, zero padding), one filter per
 * direction slot: conv_w [nd][E][dc], conv_b [nd][E]; the sequence runs line by line along the
 * pooled-over axis (position t*S + s); the forward slot's filter is causal, the backward slot's
 * runs over the reversed sequence; SiLU after it when conv_silu.  xc [nd][B][h][w][E]. */
int fvo_conv(const float* x, int B, int h, int w, int E, int pool_axis, unsigned dir_flags, int dc,
             const float* conv_w, const float* conv_b, int conv_silu, double* xc);

/* Mean pooling of an fp64 grid [B][h][w][E] (the convolved tokens of one direction). */
int fvo_pool_d(const double* x, int B, int h, int w, int E, int pool_axis, double pool_scale, double* xbar);

/* Repeat + skip (+ LayerNorm) + gate with a convolved input per direction:
 * y = SiLU(z) * N(ys[t] + sum_k D[k] * xc[k]), xc [nd][B][h][w][E]. */
int fvo_gate_dense_conv(const double* xc, const float* z, const double* ys, const float* D, int B, int h,
                        int w, int E, int nd, int pool_axis, const float* ln_gamma, const float* ln_beta,
                        double ln_eps, double* y);

/* The whole dense layer with the Conv1D in front: x is the Conv1D's input; each direction
 * pools, projects and scans its own convolved tokens, and the skip adds each direction's D
 * times its own convolved input (OpenMP over images when nthreads > 1). */
int fvo_forward_conv(const float* x, const float* z, const float* A_log, const float* D,
                     const float* W_x, const float* W_dt, const float* b_dt, int B, int h, int w, int E,
                     int N, int R, int pool_axis, unsigned dir_flags, double pool_scale, int zoh_exact, int dc,
                     const float* conv_w, const float* conv_b, int conv_silu, const float* ln_gamma,
                     const float* ln_beta, double ln_eps, int nthreads, double* y);

/* The gradient of the layer (fastvim_oracle_grad.c): given dy = dL/dy (layout of y), writes
 * dx, dz (layouts of x, z) and the parameter gradients summed over the batch, dA_log [nd][E][N],
 * dD [nd][E], dW_x [nd][R+2N][E], dW_dt [nd][E][R], db_dt [nd][E]; with the post-SSM LayerNorm
 * (ln_gamma, ln_beta [E], both or neither) also dln_gamma, dln_beta [E].
 * Tokens whose id is rejected (masked) get dx = dz = 0 and the call returns FVO_BAD_INDEX. */
int fvo_backward(const float* x, const float* z, const float* A_log, const float* D, const float* W_x,
                 const float* W_dt, const float* b_dt, const int32_t* keep_idx, int B, int h, int w, int E,
                 int N, int R, int K, int pool_axis, unsigned dir_flags, double pool_scale, int zoh_exact,
                 const float* ln_gamma, const float* ln_beta, double ln_eps, const float* dy, int nthreads,
                 double* dx, double* dz, double* dA_log, double* dD, double* dW_x, double* dW_dt, double* db_dt,
                 double* dln_gamma, double* dln_beta);

#ifdef __cplusplus
}
#endif
#endif
