/*
 * fastvim_ssm.h -- C ABI of the B200 (sm_100a) FastVim SSM layer, the "pooled selective scan".
 *
 * The layer (FastVim, Kapse et al., arXiv 2502.00594; gptget.net summary of the paper, section
 * "方法详解" (method details), items 1-6, and glossary "State Space Model"):
 *
 *   1. grid index map   x[B][h][w][E] is the post-Conv1D activation of an h x w token grid
 *                       (channels last).  No copy, transpose or flip is made: the pooled axis
 *                       is the pool_axis flag, the scan direction is a loop order.
 *   2. mean pooling     POOL_W: xbar[b][t] = pool_scale/w * sum_j x[b][t][j], T = h tokens
 *                       ("(B,h,w,D) -> (B,h,1,D)");  POOL_H: mean over i, T = w tokens.
 *   3. projections      per direction k: [dt_low | B | C] = W_x[k] xbar  (R, N, N values),
 *                       Delta[e] = softplus(W_dt[k][e] . dt_low + b_dt[k][e]).
 *   4. ZOH              A = -exp(A_log[k]);  Abar = exp(Delta A);  Bbar x = Delta B xbar
 *                       (FV_FLAG_ZOH_EXACT: Bbar = (Abar - 1) / A * B).
 *   5. scans            forward  h_t = Abar_t h_{t-1} + Bbar_t x_t, t = 0 .. T-1;
 *                       backward the same for t = T-1 .. 0; both from a zero state;
 *                       ys[t] = sum over enabled directions of C_t . h_t.
 *   6. repeat+skip+gate y[b][i][j] = SiLU(z[b][i][j]) * (ys[b][t(i,j)] + (sum_k D[k]) * x[b][i][j])
 *                       (pith.science verdict on 2502.00594, "key_machinery": the repeat comes
 *                       before the D x skip; ijyty.com Vision Mamba article, section 2.1: the
 *                       gate is applied to the sum of the two directions).
 *   masked (FastMaskVim; "方法详解" item 6): x, z, y are [B][K][E] kept tokens with grid ids
 *                       keep_idx[B][K] = r*w + c.  A kept token pools into row r (POOL_W) or
 *                       column c (POOL_H); each pooled token is the sum of its kept tokens
 *                       divided by the FIXED full length (w for POOL_W, h for POOL_H); an
 *                       empty row pools to 0 and is still scanned; each kept token takes the
 *                       output of its row.  Ids must be in [0, h*w) and unique per sample.
 *
 * Conventions for every entry point:
 *   - All tensors are fp32 (keep_idx int32), row-major, and live in DEVICE memory unless an
 *     entry point says otherwise.  Every pointer must be 16-byte aligned.
 *   - Parameters are stacked per enabled direction on a leading nd axis (nd = number of bits
 *     set in dir_flags), slot 0 = FWD when enabled, then BWD:
 *       A_log [nd][E][N], D [nd][E], W_x [nd][R+2N][E] (rows dt_low | B | C),
 *       W_dt [nd][E][R], b_dt [nd][E].
 *   - Ownership: the caller allocates and frees every buffer, including the workspace.  The
 *     library never allocates device memory, never frees, and (except fastvim_ssm_forward_host
 *     and fastvim_get_device_status) never synchronises.  Work is queued on the caller's
 *     stream (a cudaStream_t passed as void*, NULL = the legacy default stream).
 *   - Errors: argument errors are detected on the host and returned before anything is
 *     queued.  Launch failures return FV_ERR_CUDA (fastvim_last_error() has the CUDA
 *     message).  Errors found on the device (a bad keep index) never trap: the kernels skip
 *     the bad token, record FV_ERR_INDEX in the workspace, and fastvim_get_device_status()
 *     reports it; the output of a call that recorded a device error is unspecified.
 *   - Limits: E % 4 == 0, 1 <= N <= 16, 1 <= R, R + 2N <= 96, T <= 4096, h*w <= 2^20 for the
 *     masked layer, and the per-image scan tile must fit in shared memory (checked; returns
 *     FV_ERR_UNSUPPORTED otherwise).
 */
#ifndef FASTVIM_SSM_H
#define FASTVIM_SSM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define FASTVIM_SSM_ABI_VERSION 6

#if defined(__GNUC__)
#define FV_API __attribute__((visibility("default")))
#else
#define FV_API
#endif

typedef enum {
    FV_OK = 0,
    FV_ERR_NULL = 1,        /* a required pointer is NULL                                  */
    FV_ERR_SHAPE = 2,       /* a size or flag is out of range                              */
    FV_ERR_ALIGN = 3,       /* a pointer is not 16-byte aligned                            */
    FV_ERR_INDEX = 4,       /* (device) a keep index is out of range or repeated           */
    FV_ERR_WORKSPACE = 5,   /* workspace missing, too small or not 256-byte aligned        */
    FV_ERR_CUDA = 6,        /* a CUDA call failed; see fastvim_last_error()                */
    FV_ERR_TIMEOUT = 7,     /* (device) a bounded wait gave up                             */
    FV_ERR_UNSUPPORTED = 8, /* valid layer, but beyond this build's limits                 */
    FV_ERR_ALIAS = 9        /* y overlaps x or z                                           */
} fv_status;

enum { FV_POOL_W = 0, /* mean over w, T = h tokens (column pooling) */
       FV_POOL_H = 1  /* mean over h, T = w tokens (row pooling)    */ };
enum { FV_DIR_FWD = 1u, FV_DIR_BWD = 2u };
enum {
    FV_FLAG_ZOH_EXACT = 1u,   /* Bbar = (exp(Delta A) - 1) / A * B instead of Delta B            */
    FV_FLAG_PATH_STAGED = 2u, /* force the staged kernels (pool, proj, scan, epilogue launches)  */
    FV_FLAG_PATH_FUSED = 4u,  /* force the single persistent launch (dense layers only;
                                 FV_ERR_UNSUPPORTED when the layer does not fit it)             */
    FV_FLAG_TRACE = 8u,       /* fused launch: record one entry per task in the workspace
                                 (fv_ws_layout.trace); costs a little time, for profiling      */
    FV_FLAG_LAYERNORM = 16u,  /* post-SSM LayerNorm before the gate (ln_gamma, ln_beta, ln_eps) */
    FV_FLAG_CONV_SILU = 32u,  /* SiLU after the block's Conv1D (needs d_conv > 0)               */
    FV_FLAG_KEEP_STATES = 64u /* training: the scans also store their 16 states every 8 steps
                                 (fv_ws_layout.ckpt, B nd 2 ceil(T/16) E 64 bytes more
                                 workspace) so that the gradient call reads them instead of
                                 running the recurrences a first time; y is unchanged          */
};
/* Without a PATH flag a dense layer without FV_FLAG_LAYERNORM whose images hold >= 16 MiB of x
 * runs the fused launch, every other layer the staged kernels; both compute the same layer.  The fused launch gates image b
 * L rounds after it pools it, L chosen from the layer's shape; the environment variable
 * FASTVIM_FUSED_LAG (an integer 3..64, read by every call that takes the fused launch) replaces
 * that choice.  It is a test hook: the tests run the schedule at its smallest safe lag (3) and at
 * large ones; results do not depend on it.  No other environment variable is read. */

typedef struct {
    int B, h, w, E, N, R;    /* batch, grid height/width, channels, d_state, dt_rank        */
    int pool_axis;           /* FV_POOL_W or FV_POOL_H                                       */
    unsigned dir_flags;      /* FV_DIR_FWD | FV_DIR_BWD, at least one                        */
    int K;                   /* kept tokens per sample (masked layer); 0 = dense grid        */
    float pool_scale;        /* factor on the pooled mean; 0 is read as 1 (plain mean)       */
    unsigned flags;          /* FV_FLAG_*                                                    */
    const float* x;          /* dense [B][h][w][E] | masked [B][K][E]                        */
    const float* z;          /* same shape as x                                              */
    const float* A_log;      /* [nd][E][N]                                                   */
    const float* D;          /* [nd][E]                                                      */
    const float* W_x;        /* [nd][R+2N][E]                                                */
    const float* W_dt;       /* [nd][E][R]                                                   */
    const float* b_dt;       /* [nd][E]                                                      */
    const int32_t* keep_idx; /* NULL (dense) or [B][K] grid ids r*w + c                      */
    float* y;                /* same shape as x; must not overlap x or z                     */
    /* Post-SSM LayerNorm, with FV_FLAG_LAYERNORM (summary page, "方法详解" item 5: after the
     * repeat and the skip; verdict page: VMamba's post-SSM LayerNorm), over the E channels of
     * each token, before the gate:
     *   y = SiLU(z) * (ln_gamma * (s - mean(s)) / sqrt(var(s) + ln_eps) + ln_beta),
     *   s = ys[t] + (sum_k D[k]) * x,  var the biased variance over E.
     * With the flag: ln_gamma and ln_beta [E] are required (FV_ERR_NULL), ln_eps must be > 0 and
     * finite (FV_ERR_SHAPE), E <= 4096 (FV_ERR_UNSUPPORTED).  Without it both must be NULL
     * (FV_ERR_SHAPE) and ln_eps is ignored. */
    const float* ln_gamma;   /* NULL or [E]                                                  */
    const float* ln_beta;    /* NULL or [E]                                                  */
    float ln_eps;            /* LayerNorm epsilon (e.g. 1e-5)                                */
    /* The block's Conv1D in front of the layer, with d_conv > 0 (dense layers).  The summary
     * page ("方法详解" item 2) pools the output of the block's Conv1D; the Vim article's code
     * (section 2.1) gives each direction its own Conv1D of the expanded tokens, the backward one
     * run over the reversed sequence.  With d_conv > 0, x is the Conv1D's INPUT (the x half of
     * the expansion layer's output) and, per channel, for direction slot k
     *   forward slot:  xc_k[p] = act(conv_b[k] + sum_{q<d_conv} conv_w[k][q] x[p - (d_conv-1) + q])
     *   backward slot: xc_k[p] = act(conv_b[k] + sum_{q<d_conv} conv_w[k][q] x[p + (d_conv-1) - q])
     * with x = 0 outside the sequence and act = SiLU under FV_FLAG_CONV_SILU, else the identity.
     * The sequence is the block's token order p = t * S + s: the pooled lines t in order and the
     * tokens s along each line (row-major for POOL_W, column-major for POOL_H), so a line's first
     * tokens see the end of the line before.  Each direction then pools, projects and scans its
     * own xc_k, and the skip is sum_k D[k] * xc_k.  xc is never written to memory.
     * d_conv: 0 (no Conv1D: x is its output) or 1..4 (> 4: FV_ERR_UNSUPPORTED); conv_w
     * [nd][E][d_conv] and conv_b [nd][E] are required with d_conv > 0 (FV_ERR_NULL) and must be
     * NULL without (FV_ERR_SHAPE), as must FV_FLAG_CONV_SILU; masked layers, the single
     * persistent launch (FV_FLAG_PATH_FUSED) and the gradient return FV_ERR_UNSUPPORTED with it. */
    int d_conv;              /* taps of the depthwise Conv1D, 0 = none                        */
    const float* conv_w;     /* NULL or [nd][E][d_conv]                                      */
    const float* conv_b;     /* NULL or [nd][E]                                              */
} fv_ssm_args;

/* Byte offsets of the intermediates inside a workspace (for inspection and tests). */
typedef struct {
    size_t total_bytes;  /* what fastvim_ssm_workspace_size returns                          */
    size_t status;       /* uint32 device status word (+ one uint32 of scratch)              */
    size_t xbar;         /* fp32 [B][nx][T][E] pooled tokens; nx = nd with the Conv1D (each
                            direction pools its own convolved tokens), else 1              */
    size_t u;            /* fp32 projections dt_low | B | C: [B][nd] blocks of [T][R+2N], each
                            block starting every ceil(T (R+2N) / 32) * 32 floats            */
    size_t ys;           /* fp32 [B][T][E] scan output summed over directions                */
    size_t row_of;       /* int32 [B][K] pooled row of each kept token (masked), else 0      */
    size_t row_off;      /* int32 [B][T+1] CSR row offsets (masked), else 0                  */
    size_t row_tok;      /* int32 [B][K] kept-token ordinals grouped by row, ascending       */
    size_t delta;        /* fp32 [nd][B][T][E] step sizes Delta = softplus(dt_proj) of the
                            staged kernels; 0 on the fused launch (they stay on chip)       */
    size_t ctrl;         /* uint32 control block of the fused launch (dense layers), else 0  */
    size_t trace;        /* FV_FLAG_TRACE on the fused launch: uint64 [trace_records][4]:
                            w0 = kind << 60 | image << 32 | index (kind 0 pool, 1 scan, 2 gate, 3 x_proj),
                            w1 = SM id << 32 | CTA id, w2 = start (ns, %globaltimer),
                            w3 = wait_ns << 40 | total_ns (from start to the task's end)        */
    size_t trace_records;  /* number of trace entries (tasks of the call), else 0               */
    size_t ckpt;         /* FV_FLAG_KEEP_STATES: fp32 [B][nd][2 ceil(T/16)][E][16], zero past N;
                            slot 2i+h = the 16 states entering the h-th 8-step half of the
                            i-th 16-step chunk [16c, 16c+16) of the time axis in the scan's
                            order (forward: before step 16i+8h; the backward scan starts
                            with the last, possibly shorter, chunk); a chunk of <= 8 steps
                            has no slot 2i+1; else 0                                        */
    size_t scan_dt;      /* reserved, 0                                                      */
    int T, S, nd;        /* pooled length, pooled-over length, number of directions          */
} fv_ws_layout;

/* Human-readable name of a status code (static string, never NULL). */
FV_API const char* fastvim_status_string(fv_status s);

/* Message of the last CUDA failure seen by this thread ("" if none). */
FV_API const char* fastvim_last_error(void);

/* ABI version (FASTVIM_SSM_ABI_VERSION). */
FV_API int fastvim_abi_version(void);

/* Host-side argument check of a forward call, without touching the GPU or dereferencing any
 * tensor pointer.  Returns FV_OK or the first error found. */
FV_API fv_status fastvim_ssm_validate(const fv_ssm_args* args);

/* Workspace bytes a forward call needs (0 when the arguments are invalid). */
FV_API size_t fastvim_ssm_workspace_size(const fv_ssm_args* args);

/* Where each intermediate sits inside the workspace. */
FV_API fv_status fastvim_ssm_workspace_layout(const fv_ssm_args* args, fv_ws_layout* out);

/* Number of kernel launches one fastvim_ssm_forward call queues (memsets excluded; 0 when the
 * arguments are invalid or B == 0). */
FV_API int fastvim_ssm_launch_count(const fv_ssm_args* args);

/* Name of the i-th kernel launch of a forward call ("" when out of range); static string. */
FV_API const char* fastvim_ssm_launch_name(const fv_ssm_args* args, int i);

/* The layer: queue pool -> projections -> scans -> repeat/skip/gate on `stream`.
 * ws: device workspace of at least fastvim_ssm_workspace_size(args) bytes, 256-byte aligned,
 * no initial contents required, not shared with a concurrently running call.  Every launch of
 * the call goes to `stream`, in order. */
FV_API fv_status fastvim_ssm_forward(const fv_ssm_args* args, void* ws, size_t ws_bytes, void* stream);

/* fastvim_ssm_forward with timing marks: `events` holds n_events >= 2 * launch_count CUDA
 * events (cudaEvent_t, created by the caller); events[2i] and events[2i+1] are recorded just
 * before and just after the i-th kernel launch, on the stream that launch runs on, so their
 * elapsed time is the device duration of launch i.  Same results as fastvim_ssm_forward. */
FV_API fv_status fastvim_ssm_forward_events(const fv_ssm_args* args, void* ws, size_t ws_bytes,
                                            void* stream, void* const* events, int n_events);

/* End-to-end variant for host-resident data.  `host` names pinned HOST buffers for x, z,
 * the parameters, keep_idx and y; `dev` names DEVICE buffers of the same shapes (its sizes
 * and flags must equal host's).  Copies the inputs host -> device, runs the layer, copies y
 * device -> host and waits for the stream, so y is ready in host memory on return.  The batch
 * runs as chunks of whole images (about 64 MB of x each, at most 16 chunks) in a pipeline: the
 * upload of one chunk, the layer on the previous one (on `stream`) and the download of the one
 * before overlap, on two streams the call creates and destroys.  The device status word of ws
 * reports the first device error of any chunk.  Each chunk reuses the workspace from its start,
 * so with FV_FLAG_KEEP_STATES it holds the last chunk's scan states only (this entry point has no
 * gradient counterpart). */
FV_API fv_status fastvim_ssm_forward_host(const fv_ssm_args* host, const fv_ssm_args* dev, void* ws,
                                   size_t ws_bytes, void* stream);

/* fastvim_ssm_forward for callers that cannot allocate device memory.  There is no counterpart
 * in the paper; this is an interface convenience.  Some callers only ever receive device
 * buffers for their inputs and outputs from a host framework that owns all device memory and
 * offers them no allocator, or must not call cudaMalloc/cudaFree because those calls can stall
 * the whole device.  This entry point needs no workspace argument: its scratch is a fixed
 * 16 MiB array in device memory, part of this library's device code, held until the process
 * exits.
 *   - Limit: fastvim_ssm_workspace_size(args) must be <= 16 MiB (e.g. the 224 px FastVim-T
 *     layer at batch 128 needs about 6 MiB); larger layers return FV_ERR_UNSUPPORTED with a
 *     message in fastvim_last_error() and queue nothing; split the batch or use
 *     fastvim_ssm_forward.
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 *   - The first call on a device looks up that device's scratch address (with the device
 *     current).  CUDA loads the library's device code lazily, so this first call is also
 *     where the 16 MiB are committed on that device: it can fail with FV_ERR_CUDA when the
 *     device is out of memory.  Make that first call before any stream capture begins.
 *   - All calls on a device share the one scratch array: calls that may overlap on the GPU
 *     (different streams, no ordering between them) race and give wrong results; on the
 *     single-launch path one call's reset of the shared control block can also leave the
 *     other call's blocks waiting until their bounded wait (1 s) runs out, and that timeout
 *     is not reported (see below).  Calls queued on one stream are ordered and safe.  Each
 *     call resets what must start at zero; the contents left by a previous call need no
 *     clearing.
 *   - The device status word lives in the shared scratch and is not readable through this
 *     entry point; use fastvim_ssm_forward with a workspace where FV_ERR_INDEX or
 *     FV_ERR_TIMEOUT must be seen.  Likewise a gradient call needs the forward's workspace,
 *     which this entry point does not expose: FV_FLAG_KEEP_STATES only costs scratch here.
 * Inputs, outputs and the returned status are as for fastvim_ssm_forward. */
FV_API fv_status fastvim_ssm_forward_noalloc(const fv_ssm_args* args, void* stream);

/* Self-test of the bounded wait that the fused launch uses between its tasks: queues one CTA
 * that waits on a counter nothing increments, for limit_us microseconds (1 .. 10^7), after which
 * it records FV_ERR_TIMEOUT in the status word of `ws` (>= 1 KB, 256-byte aligned) and exits.
 * fastvim_get_device_status(ws, stream) then returns FV_ERR_TIMEOUT; the context stays usable. */
FV_API fv_status fastvim_selftest_bounded_wait(void* ws, size_t ws_bytes, unsigned limit_us, void* stream);

/* Self-test of the device math the layer uses instead of CUDA's full-precision functions, for
 * checking against a reference on the host: out[i] = f(in[i]) for i < n, with f chosen by `fn`:
 *   0  softplus(v) = log(1 + e^v)   (SFU exp2 and reciprocal, an odd series of atanh)
 *   1  SiLU(v) = v / (1 + e^-v)      (SFU exp2 and reciprocal; the gate)
 *   2  2^v                           (SFU exp2, inputs below -126 flush to 0; the ZOH exponential)
 * in, out: DEVICE float arrays of n elements (16-byte aligned, not overlapping); queued on
 * `stream`.  Returns FV_ERR_SHAPE for an unknown fn or n < 0, FV_ERR_NULL for a NULL array. */
FV_API fv_status fastvim_selftest_math(int fn, const float* in, float* out, int n, void* stream);

/* Waits for `stream`, then reads the device status word of a workspace used by the last
 * forward call: FV_OK, FV_ERR_INDEX or FV_ERR_TIMEOUT (or FV_ERR_CUDA if the read fails). */
FV_API fv_status fastvim_get_device_status(const void* ws, void* stream);

/* ---- Gradient (training) ---------------------------------------------------------------------
 * FastVim is trained end to end (summary page, "实验结果": faster pre-training and fine-tuning);
 * the pages give no backward rule, so this is the exact derivative of the layer above, by the
 * chain rule in reverse step order: for an upstream gradient dy = dL/dy of a scalar loss L it
 * returns dx = dL/dx, dz = dL/dz and the parameter gradients summed over the batch.  Dense and
 * masked layers, both pool axes, one or two directions, pool_scale, FV_FLAG_ZOH_EXACT and the
 * post-SSM LayerNorm (FV_FLAG_LAYERNORM: also dln_gamma, dln_beta).  Masked tokens whose id the
 * forward rejected (FV_ERR_INDEX) get dx = dz = 0. */
typedef struct {
    const float* dy;  /* dL/dy, the shape of y (dense [B][h][w][E] | masked [B][K][E])         */
    float* dx;        /* dL/dx, the shape of x (written)                                      */
    float* dz;        /* dL/dz, the shape of z (written)                                      */
    float* dA_log;    /* [nd][E][N]      } parameter gradients, summed over the batch;          */
    float* dD;        /* [nd][E]         } written (not accumulated into): the call zeroes     */
    float* dW_x;      /* [nd][R+2N][E]   } them.  The sums run in fp32 over per-block partial  */
    float* dW_dt;     /* [nd][E][R]      } sums added in a fixed order (no atomics), so two    */
    float* db_dt;     /* [nd][E]         } calls on one GPU give the same bits.                */
    float* dln_gamma; /* [E] with FV_FLAG_LAYERNORM (written, like the above), else NULL          */
    float* dln_beta;  /* [E] with FV_FLAG_LAYERNORM, else NULL                                    */
} fv_ssm_grads;

/* Byte offsets of the gradient's intermediates inside its workspace. */
typedef struct {
    size_t total_bytes;  /* what fastvim_ssm_backward_workspace_size returns                 */
    size_t dys;          /* float [B][T][E]   dL/dys: ds summed over each pooled row's tokens  */
    size_t dxbar;        /* float [B][T][E]   dL/dxbar                                         */
    size_t du;           /* float, the layout of the forward's u: d dt_low | dB | dC           */
    size_t dxs;          /* float [B][nd][T][E]  the scans' share of dL/dxbar per direction     */
    size_t ckpt;         /* float [B][nd][2 ceil(T/16)][E][16]  scan state entering every 8 steps;
                            0 with FV_FLAG_KEEP_STATES (the forward's are read)               */
    size_t status;       /* uint32 device status word (FV_ERR_TIMEOUT from a bounded wait), read
                            by fastvim_get_device_status(ws, stream); the call clears it       */
    size_t delta;        /* float [nd][B][T][E] step sizes Delta, computed by the gradient call
                            when the forward workspace holds none (fv_ws_layout.delta == 0),
                            else 0 (the forward's are read)                                   */
    size_t partials;     /* float scratch from here to the end: per-block partial sums of du and
                            of the parameter gradients, added in a fixed order                 */
} fv_bwd_ws_layout;

/* Workspace bytes a gradient call needs (0 when the arguments are invalid). */
FV_API size_t fastvim_ssm_backward_workspace_size(const fv_ssm_args* args);
FV_API fv_status fastvim_ssm_backward_workspace_layout(const fv_ssm_args* args, fv_bwd_ws_layout* out);

/* Kernel launches of one gradient call (0 when invalid or B == 0) and the name of the i-th. */
FV_API int fastvim_ssm_backward_launch_count(const fv_ssm_args* args);
FV_API const char* fastvim_ssm_backward_launch_name(const fv_ssm_args* args, int i);

/* Queue the gradient on `stream`.
 * args: the forward call's arguments (the same tensors; y is not read and may be NULL).
 * fwd_ws: the workspace of a fastvim_ssm_forward (or _events) call with these args that is
 *   complete or queued earlier on `stream`: the gradient reads its pooled tokens, projections,
 *   scan outputs, (masked) row lists and, with FV_FLAG_KEEP_STATES, the scan states.  fwd_ws_bytes >= fastvim_ssm_workspace_size(args).
 * ws: the gradient's own workspace, >= fastvim_ssm_backward_workspace_size(args) bytes, 256-byte
 *   aligned, no initial contents; fwd_ws and ws must not overlap.
 * grads: device arrays, 16-byte aligned; dx and dz must not overlap each other, x, z or dy.
 * Errors: as fastvim_ssm_forward for args; FV_ERR_NULL for a missing grads array (dy, dx, dz may
 * be NULL when B == 0; dln_gamma, dln_beta are required with FV_FLAG_LAYERNORM); FV_ERR_SHAPE
 * for dln_gamma or dln_beta without the flag; FV_ERR_ALIGN, FV_ERR_ALIAS as above;
 * FV_ERR_WORKSPACE for a missing, short or misaligned fwd_ws or ws. */
FV_API fv_status fastvim_ssm_backward(const fv_ssm_args* args, const fv_ssm_grads* grads, const void* fwd_ws,
                                      size_t fwd_ws_bytes, void* ws, size_t ws_bytes, void* stream);

/* fastvim_ssm_backward with timing marks, as fastvim_ssm_forward_events:
 * n_events >= 2 * fastvim_ssm_backward_launch_count(args). */
FV_API fv_status fastvim_ssm_backward_events(const fv_ssm_args* args, const fv_ssm_grads* grads,
                                             const void* fwd_ws, size_t fwd_ws_bytes, void* ws, size_t ws_bytes,
                                             void* stream, void* const* events, int n_events);

#ifdef __cplusplus
}
#endif
#endif /* FASTVIM_SSM_H */
