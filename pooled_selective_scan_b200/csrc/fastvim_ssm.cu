// fastvim_ssm.cu -- C ABI of the FastVim SSM layer: validation, workspace planning, launches.
// The layer's definition, the argument layouts and the error contract are in fastvim_ssm.h.
#include "fastvim_ssm.h"

#include <stdio.h>
#include <string.h>

#include <stdlib.h>

#include <mutex>
#include <vector>
#include <algorithm>

#include "fv_common.cuh"
#include "fv_fused.cuh"
#include "fv_dt_tc.cuh"
#include "fv_kernels.cuh"
#include "fv_backward.cuh"

namespace {

thread_local char g_last_error[512] = "";

void note_cuda(cudaError_t e, const char* where) {
    snprintf(g_last_error, sizeof g_last_error, "%s: %s (%d)", where, cudaGetErrorString(e), (int)e);
}

int popc2(unsigned f) { return (int)((f & 1u) != 0) + (int)((f & 2u) != 0); }
bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }
size_t round256(size_t v) { return (v + 255) & ~(size_t)255; }

constexpr int kMaxT = 4096;
constexpr long long kMaxMaskGrid = 1ll << 20;
constexpr int kMaxLnE = 4096;  // channels of a LayerNorm row (shared-memory rows of the LN epilogue)

size_t bucket_smem_bytes(const fv::Shape& sh) {
    const long long G = (long long)sh.h * sh.w;
    return (size_t)(((G + 31) >> 5) + 2ll * sh.T) * sizeof(unsigned);
}

// Sizes and flags only; no pointer is dereferenced.
fv_status make_shape(const fv_ssm_args* a, fv::Shape* sh) {
    if (!a) return FV_ERR_NULL;
    if (a->B < 0 || a->h < 1 || a->w < 1 || a->E < 4 || a->N < 1 || a->R < 1) return FV_ERR_SHAPE;
    if (a->pool_axis != FV_POOL_W && a->pool_axis != FV_POOL_H) return FV_ERR_SHAPE;
    if (a->dir_flags == 0 || (a->dir_flags & ~3u) != 0) return FV_ERR_SHAPE;
    if ((a->flags & ~(unsigned)(FV_FLAG_ZOH_EXACT | FV_FLAG_PATH_STAGED | FV_FLAG_PATH_FUSED | FV_FLAG_TRACE |
                                FV_FLAG_LAYERNORM | FV_FLAG_CONV_SILU | FV_FLAG_KEEP_STATES)) != 0)
        return FV_ERR_SHAPE;
    if (a->d_conv < 0) return FV_ERR_SHAPE;
    if (a->d_conv == 0 && (a->flags & FV_FLAG_CONV_SILU)) return FV_ERR_SHAPE;  // SiLU of no Conv1D
    if ((a->flags & FV_FLAG_PATH_STAGED) && (a->flags & FV_FLAG_PATH_FUSED)) return FV_ERR_SHAPE;
    if (a->E % 4 != 0) return FV_ERR_SHAPE;
    if (a->K < 0 || (long long)a->K > (long long)a->h * a->w) return FV_ERR_SHAPE;
    if (!(a->pool_scale == a->pool_scale) || a->pool_scale > 3.0e38f || a->pool_scale < -3.0e38f)
        return FV_ERR_SHAPE;
    if (a->N > fv::kMaxN || a->R + 2 * a->N > fv::kMaxJ) return FV_ERR_UNSUPPORTED;
    const long long tok = a->K > 0 ? (long long)a->K : (long long)a->h * a->w;
    if ((long long)a->B * tok * a->E >= (1ll << 40)) return FV_ERR_UNSUPPORTED;
    sh->B = a->B; sh->h = a->h; sh->w = a->w; sh->E = a->E; sh->N = a->N; sh->R = a->R;
    sh->pool_axis = a->pool_axis;
    sh->T = a->pool_axis == FV_POOL_W ? a->h : a->w;
    sh->S = a->pool_axis == FV_POOL_W ? a->w : a->h;
    sh->nd = popc2(a->dir_flags);
    sh->J = a->R + 2 * a->N;
    sh->NJ = sh->nd * sh->J;
    sh->K = a->K;
    sh->dir_flags = a->dir_flags;
    sh->zoh_exact = (a->flags & FV_FLAG_ZOH_EXACT) ? 1 : 0;
    sh->path_flags = a->flags & (FV_FLAG_PATH_STAGED | FV_FLAG_PATH_FUSED);
    sh->trace = (a->flags & FV_FLAG_TRACE) ? 1 : 0;
    sh->pool_scale = a->pool_scale == 0.f ? 1.f : a->pool_scale;
    sh->SL = a->E / 4;
    sh->ln = (a->flags & FV_FLAG_LAYERNORM) ? 1 : 0;
    sh->ln_eps = sh->ln ? a->ln_eps : 0.f;
    if (sh->ln && !(a->ln_eps > 0.f && a->ln_eps <= 3.0e38f)) return FV_ERR_SHAPE;
    if (sh->ln && a->E > kMaxLnE) return FV_ERR_UNSUPPORTED;
    sh->dc = a->d_conv;
    sh->conv_silu = (a->flags & FV_FLAG_CONV_SILU) ? 1 : 0;
    sh->nx = a->d_conv > 0 ? sh->nd : 1;
    sh->keep = (a->flags & FV_FLAG_KEEP_STATES) ? 1 : 0;
    if (a->d_conv > fv::kMaxConv) return FV_ERR_UNSUPPORTED;
    if (a->d_conv > 0 && a->K > 0) return FV_ERR_UNSUPPORTED;  // the Conv1D is for dense grids
    if (sh->T > kMaxT) return FV_ERR_UNSUPPORTED;
    if (a->K > 0 && (long long)a->h * a->w > kMaxMaskGrid) return FV_ERR_UNSUPPORTED;
    if ((long long)sh->B * sh->T >= (1ll << 31)) return FV_ERR_UNSUPPORTED;
    return FV_OK;
}

fv_status check_pointers(const fv_ssm_args* a, const fv::Shape& sh) {
    if (!a->A_log || !a->D || !a->W_x || !a->W_dt || !a->b_dt) return FV_ERR_NULL;
    if (sh.B > 0 && (!a->x || !a->z || !a->y)) return FV_ERR_NULL;
    if (sh.K > 0 && sh.B > 0 && !a->keep_idx) return FV_ERR_NULL;
    if (sh.K == 0 && a->keep_idx) return FV_ERR_SHAPE;  // a keep list needs K
    if (sh.ln && (!a->ln_gamma || !a->ln_beta)) return FV_ERR_NULL;
    if (!sh.ln && (a->ln_gamma || a->ln_beta)) return FV_ERR_SHAPE;  // LayerNorm weights need the flag
    if (sh.dc > 0 && (!a->conv_w || !a->conv_b)) return FV_ERR_NULL;
    if (sh.dc == 0 && (a->conv_w || a->conv_b)) return FV_ERR_SHAPE;  // Conv1D weights need d_conv
    const void* ps[] = {a->x, a->z, a->y, a->A_log, a->D, a->W_x, a->W_dt, a->b_dt, a->keep_idx, a->ln_gamma,
                        a->ln_beta, a->conv_w, a->conv_b};
    for (const void* p : ps)
        if (p && !aligned16(p)) return FV_ERR_ALIGN;
    if (sh.B > 0) {
        const size_t tok = sh.K > 0 ? (size_t)sh.K : (size_t)sh.h * sh.w;
        const size_t bytes = (size_t)sh.B * tok * sh.E * sizeof(float);
        const uintptr_t y0 = (uintptr_t)a->y, y1 = y0 + bytes;
        const uintptr_t x0 = (uintptr_t)a->x, z0 = (uintptr_t)a->z;
        if ((x0 < y1 && y0 < x0 + bytes) || (z0 < y1 && y0 < z0 + bytes)) return FV_ERR_ALIAS;
    }
    return FV_OK;
}

enum class Path { Staged, Fused, Invalid };
int device_sm_count();
Path choose_path(const fv::Shape& sh);
fv::FusedPlan plan_fused(const fv::Shape& sh);

fv_status plan_layout(const fv::Shape& sh, fv_ws_layout* L) {
    memset(L, 0, sizeof *L);
    size_t off = 0;
    // word 0: the call's device status; word 1: scratch of fastvim_ssm_forward_host
    L->status = off; off = round256(off + 2 * sizeof(unsigned));
    L->xbar = off; off = round256(off + (size_t)sh.B * sh.nx * sh.T * sh.E * sizeof(float));
    L->u = off; off = round256(off + (size_t)sh.nd * sh.B * fv::u_block_stride(sh.T, sh.J) * sizeof(float));
    L->ys = off; off = round256(off + (size_t)sh.B * sh.T * sh.E * sizeof(float));
    if (choose_path(sh) != Path::Fused && fv::staged_delta_kernel(sh)) {  // step sizes of the staged dt_proj kernel
        L->delta = off; off = round256(off + (size_t)sh.nd * sh.B * sh.T * sh.E * sizeof(float));
    }
    if (sh.keep) {  // the scan states every 8 steps, for the gradient
        L->ckpt = off; off = round256(off + (size_t)sh.B * sh.nd * fv::ckpt_count(sh.T) * sh.E * 16 * sizeof(float));
    }
    if (sh.K > 0) {
        L->row_of = off; off = round256(off + (size_t)sh.B * sh.K * sizeof(int32_t));
        L->row_off = off; off = round256(off + (size_t)sh.B * (sh.T + 1) * sizeof(int32_t));
        L->row_tok = off; off = round256(off + (size_t)sh.B * sh.K * sizeof(int32_t));
    } else {
        // dense layers: the control block of the fused launch
        L->ctrl = off; off = round256(off + (size_t)(fv::kCtrlHeaderWords + fv::kCtrlCounters * (size_t)sh.B) * sizeof(unsigned));
        if (sh.trace && choose_path(sh) == Path::Fused) {
            const fv::FusedPlan pl = plan_fused(sh);
            L->trace = off;
            L->trace_records = pl.total;
            off = round256(off + (size_t)pl.total * 4 * sizeof(unsigned long long));
        }
    }
    L->total_bytes = off;
    L->T = sh.T; L->S = sh.S; L->nd = sh.nd;
    return FV_OK;
}

// The library is built for sm_100a only: 227 KB of opt-in shared memory per CTA.
constexpr size_t kMaxSmemOptin = 227 * 1024;
// Latency of one image's pool -> x_proj -> scan chain inside the fused launch: the scan task runs
// the T steps of its recurrences in sequence (traces on B200: 55 us at T = 128, 36 us at T = 64),
// the projection and the last pooling tasks add about 40 us.
double chain_latency_us(const fv::Shape& sh) { return 40.0 + 0.5 * sh.T; }

fv_status check_limits(const fv::Shape& sh) {
    if (fv::seq_smem_floats(sh) * sizeof(float) > kMaxSmemOptin) return FV_ERR_UNSUPPORTED;
    if (fv::fused_proj_smem_floats(sh) * sizeof(float) > kMaxSmemOptin) return FV_ERR_UNSUPPORTED;
    if (sh.K > 0 && bucket_smem_bytes(sh) > kMaxSmemOptin) return FV_ERR_UNSUPPORTED;
    return FV_OK;
}


// Grid lines per P/E task: the fewest that give each task at least 384 KB of x.  Every task costs
// a ticket (a contended atomic, ~1 us under full HBM load), so fewer, larger streaming tasks pay:
// B200, 2048 px layer, 2.17 -> 2.13 ms going from one 196 KB line to two per task.
int fused_lines_per_task(const fv::Shape& sh) {
    const size_t line = (size_t)sh.S * sh.E * sizeof(float);
    int lp = 1;
    while (lp < fv::kMaxLP && lp < sh.T && (size_t)lp * line < ((size_t)384 << 10)) ++lp;
    return lp;
}

bool fused_possible(const fv::Shape& sh) {
    if (sh.K > 0 || sh.B < 1 || sh.dc > 0) return false;
    // a token row of x (and of z) must fit half a ring stage; a thread holds at most 2 float4 slots
    if ((size_t)sh.E * sizeof(float) > (size_t)fv::kStageBytes / 2) return false;
    if (sh.SL > fv::kMaxSlots * fv::kFusedThreads) return false;
    if (fv::fused_smem_floats(sh, fused_lines_per_task(sh)) * sizeof(float) > kMaxSmemOptin) return false;
    // tickets are 32-bit: every task of the call must be numbered
    const long long per_image = 2ll * sh.T + (sh.T + fv::kQT - 1) / fv::kQT +
                                (sh.E + fv::fused_ech(sh.nd) - 1) / fv::fused_ech(sh.nd);
    if ((long long)sh.B * per_image >= (1ll << 31)) return false;
    return true;
}

// Which implementation runs: the fused single launch for dense layers with large images (>= 16 MiB
// of x per image: there the overlap of projections and scans with streaming pays; measured on B200,
// 2.19 vs 2.35 ms at 2048 px, while at 1024 px the staged kernels win, 1.41 vs 1.83 ms) without
// the post-SSM LayerNorm, the staged kernels otherwise; flags can force either.
Path choose_path(const fv::Shape& sh) {
    const bool ok = fused_possible(sh);
    if (sh.path_flags & FV_FLAG_PATH_STAGED) return Path::Staged;
    if (sh.path_flags & FV_FLAG_PATH_FUSED) return ok ? Path::Fused : Path::Invalid;
    // with the post-SSM LayerNorm the staged epilogue (tokens in registers) is the faster one
    // (2048 px: 2.20 ms staged vs 2.41 ms fused on B200)
    if (sh.ln) return Path::Staged;
    const size_t img = (size_t)sh.h * sh.w * sh.E * sizeof(float);
    return (ok && img >= ((size_t)16 << 20)) ? Path::Fused : Path::Staged;
}

fv::FusedPlan plan_fused(const fv::Shape& sh) {
    fv::FusedPlan pl;
    pl.LP = fused_lines_per_task(sh);
    pl.nP = (sh.T + pl.LP - 1) / pl.LP;
    pl.nQ = (sh.T + fv::kQT - 1) / fv::kQT;
    pl.ECH = fv::fused_ech(sh.nd);
    pl.nS = (sh.E + pl.ECH - 1) / pl.ECH;
    pl.ctP = fv::kStageBytes / (sh.E * (int)sizeof(float));
    pl.ctE = fv::kStageBytes / 2 / (sh.E * (int)sizeof(float));
    // Lag: enough rounds to cover one image's pool -> proj -> scan chain (chain_latency_us) at the
    // rate one round streams, plus one (B200, 2048 px: L = 7 measured 2.14-2.16 ms, L = 9
    // 2.22-2.23; holding the first gates back further, so that the start's pooling-only rounds
    // cover the first chain, measured no better); it streams (x twice, z and y once: 16 E bytes per grid token at
    // ~6.5 TB/s).  (Keeping x in L2 across that window does not happen: traffic of this size
    // evicts first-touch lines whatever their L2 eviction priority.)
    const double round_us = (double)sh.h * sh.w * sh.E * 16.0 / 6.5e6;
    long long lag = (long long)(chain_latency_us(sh) / (round_us > 0.01 ? round_us : 0.01)) + 1;
    // FASTVIM_FUSED_LAG replaces the choice (a test hook, declared in the header: the tests run
    // the schedule at its smallest safe lag and at large ones)
    if (const char* env = getenv("FASTVIM_FUSED_LAG")) {
        const long long v = atoll(env);
        if (v >= 3 && v <= 64) lag = v;
    }
    // Image b's scans come in round b+2, its gates in round b+L: L >= 3 keeps every consumer after
    // its producers in ticket order (the deadlock-freedom argument of the fused kernel).
    pl.L = (int)(lag < 3 ? 3 : (lag > 64 ? 64 : lag));
    pl.B = sh.B;
    // rounds r = 0 .. B+L-1; [R1, R2) hold Q, P, E and S alike
    const int rounds = sh.B + pl.L;
    pl.R1 = pl.L > 1 ? pl.L : 1;
    pl.R2 = sh.B > pl.R1 ? sh.B : pl.R1;
    unsigned c = 0;
    for (int r = 0; r < pl.R1; ++r) c += fv::fused_round_size(pl, r);
    pl.c1 = c;
    pl.c2 = c + (unsigned)(pl.R2 - pl.R1) * fv::fused_round_size(pl, pl.R1);
    c = pl.c2;
    for (int r = pl.R2; r < rounds; ++r) c += fv::fused_round_size(pl, r);
    pl.total = c;
    pl.smem_bytes = fv::fused_smem_floats(sh, pl.LP) * sizeof(float);
    pl.wait_limit_ns = fv::kWaitLimitNs;
    return pl;
}

// Kernels that take more than 48 KB of dynamic shared memory need an opt-in per device.
template <typename Kern>
cudaError_t ensure_smem(Kern kernel, size_t bytes) {
    if (bytes <= 48 * 1024) return cudaSuccess;
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

#define FV_LAUNCH_CHECK(where)                         \
    do {                                               \
        cudaError_t e_ = cudaGetLastError();           \
        if (e_ != cudaSuccess) {                       \
            note_cuda(e_, where);                      \
            return FV_ERR_CUDA;                        \
        }                                              \
    } while (0)

// Records events[2i] just before and events[2i+1] just after the i-th kernel launch, on the
// stream of that launch, when an event list is given.
struct EventMarks {
    void* const* ev;
    int n, next;
    cudaError_t before(cudaStream_t st) {
        if (!ev || next >= n) return cudaSuccess;
        return cudaEventRecord((cudaEvent_t)ev[2 * next], st);
    }
    cudaError_t after(cudaStream_t st) {
        if (!ev || next >= n) return cudaSuccess;
        return cudaEventRecord((cudaEvent_t)ev[2 * next++ + 1], st);
    }
};

#define FV_MARK_CALL(marks, st, call)                          \
    do {                                                       \
        cudaError_t e_ = (marks).before(st);                   \
        if (e_ != cudaSuccess) {                               \
            note_cuda(e_, "event record");                     \
            return FV_ERR_CUDA;                                \
        }                                                      \
        fv_status s_ = (call);                                 \
        if (s_ != FV_OK) return s_;                            \
        if ((e_ = (marks).after(st)) != cudaSuccess) {         \
            note_cuda(e_, "event record");                     \
            return FV_ERR_CUDA;                                \
        }                                                      \
    } while (0)

// The post-SSM LayerNorm epilogue keeps each lane's share of a token in registers up to 1536
// channels (without the Conv1D, whose skip needs each token's sequence neighbours).
bool ln_uses_reg_kernel(const fv::Shape& sh) { return sh.dc == 0 && fv::ln_reg_nsl(sh.SL) > 0; }

// Launches of a staged call: pool (masked: bucket, pool), x_proj, scans, epilogue.
int launch_count_of(const fv::Shape& sh) {
    if (sh.B == 0) return 0;
    const Path path = choose_path(sh);
    if (path == Path::Invalid) return 0;
    if (path == Path::Fused) return 1;
    return (sh.K > 0 ? 5 : 4) + (fv::staged_delta_kernel(sh) ? 1 : 0);
}

const char* launch_name_of(const fv::Shape& sh, int i) {
    static const char* dense[] = {"pool_dense_kernel", "proj_gemm_kernel", "dt_proj_kernel", "scan_seq_kernel",
                                  "epilogue_dense_kernel"};
    static const char* conv[] = {"pool_conv_kernel", "proj_gemm_kernel", "dt_proj_kernel", "scan_seq_kernel",
                                 "epilogue_conv_kernel"};
    static const char* masked[] = {"mask_bucket_kernel", "mask_pool_kernel", "proj_gemm_kernel", "dt_proj_kernel",
                                   "scan_seq_kernel", "mask_epilogue_kernel"};
    const int n = launch_count_of(sh);
    if (i < 0 || i >= n) return "";
    if (choose_path(sh) == Path::Fused) return "fused_layer_kernel";
    if (sh.ln && i == n - 1) return ln_uses_reg_kernel(sh) ? "ln_epilogue_reg_kernel" : "ln_epilogue_kernel";
    const int first_scan = sh.K > 0 ? 3 : 2;  // without the dt_proj kernel the later launches move up one
    const int j = (!fv::staged_delta_kernel(sh) && i >= first_scan) ? i + 1 : i;
    return sh.K > 0 ? masked[j] : (sh.dc > 0 ? conv[j] : dense[j]);
}

template <int ND, bool Z>
fv_status launch_fused_t(const fv::Shape& sh, const fv::FusedPlan& pl, const fv::FusedPtrs& ptrs, cudaStream_t st) {
    auto kern = fv::fused_layer_kernel<ND, Z>;
    cudaError_t e = ensure_smem(kern, pl.smem_bytes);
    if (e != cudaSuccess) { note_cuda(e, "fused smem attribute"); return FV_ERR_CUDA; }
    int dev = 0, sms = 0, per_sm = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess ||
        (e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, fv::kFusedThreads, pl.smem_bytes)) != cudaSuccess) {
        note_cuda(e, "fused occupancy query");
        return FV_ERR_CUDA;
    }
    if (per_sm < 1) return FV_ERR_UNSUPPORTED;
    long long grid = (long long)sms * per_sm;
    if (grid > (long long)pl.total) grid = pl.total;
    kern<<<(unsigned)grid, fv::kFusedThreads, pl.smem_bytes, st>>>(sh, pl, ptrs);
    FV_LAUNCH_CHECK("fused_layer_kernel");
    return FV_OK;
}

fv::FusedPtrs fused_ptrs(const fv_ssm_args* a, const fv_ws_layout& L, char* ws) {
    fv::FusedPtrs p;
    p.x = a->x; p.z = a->z; p.A_log = a->A_log; p.D = a->D; p.W_x = a->W_x; p.W_dt = a->W_dt; p.b_dt = a->b_dt;
    p.y = a->y;
    p.ln_gamma = a->ln_gamma;
    p.ln_beta = a->ln_beta;
    p.xbar = (float*)(ws + L.xbar);
    p.u = (float*)(ws + L.u);
    p.ys = (float*)(ws + L.ys);
    p.status = (unsigned*)(ws + L.status);
    p.ctrl = L.ctrl ? (unsigned*)(ws + L.ctrl) : nullptr;
    p.trace = L.trace_records ? (unsigned long long*)(ws + L.trace) : nullptr;
    p.ckpt = L.ckpt ? (float*)(ws + L.ckpt) : nullptr;
    return p;
}

fv_status launch_fused(const fv::Shape& sh, const fv_ssm_args* a, const fv_ws_layout& L, char* ws, cudaStream_t st) {
    const fv::FusedPlan pl = plan_fused(sh);
    const fv::FusedPtrs p = fused_ptrs(a, L, ws);
    if (sh.nd == 2) return sh.zoh_exact ? launch_fused_t<2, true>(sh, pl, p, st) : launch_fused_t<2, false>(sh, pl, p, st);
    return sh.zoh_exact ? launch_fused_t<1, true>(sh, pl, p, st) : launch_fused_t<1, false>(sh, pl, p, st);
}

// Staged: every (image, 128-channel tile, direction) recurrence, one thread each.  With both
// directions the two add into ys, which is zeroed first.
fv_status launch_scan_seq(const fv::Shape& sh, const fv_ssm_args* a, const fv_ws_layout& L, char* ws, cudaStream_t st) {
    float* ys = (float*)(ws + L.ys);
    cudaError_t e;
    if (sh.nd == 2 && (e = cudaMemsetAsync(ys, 0, (size_t)sh.B * sh.T * sh.E * sizeof(float), st)) != cudaSuccess) {
        note_cuda(e, "scan output reset");
        return FV_ERR_CUDA;
    }
    const size_t smem = fv::seq_smem_floats(sh) * sizeof(float);
    const bool din = fv::staged_delta_kernel(sh);
    auto kern = sh.zoh_exact ? (din ? fv::scan_seq_kernel<true, true> : fv::scan_seq_kernel<true, false>)
                             : (din ? fv::scan_seq_kernel<false, true> : fv::scan_seq_kernel<false, false>);
    if ((e = ensure_smem(kern, smem)) != cudaSuccess) { note_cuda(e, "scan smem attribute"); return FV_ERR_CUDA; }
    const long long tiles = (sh.E + fv::kSeqThreads - 1) / fv::kSeqThreads;
    const long long grid = (long long)sh.B * tiles * sh.nd;
    if (grid >= (1ll << 31)) return FV_ERR_UNSUPPORTED;
    kern<<<(unsigned)grid, fv::kSeqThreads, smem, st>>>(sh, (const float*)(ws + L.u), (const float*)(ws + L.xbar),
                                                         a->A_log, a->W_dt, a->b_dt,
                                                         din ? (const float*)(ws + L.delta) : nullptr, ys,
                                                         L.ckpt ? (float*)(ws + L.ckpt) : nullptr);
    FV_LAUNCH_CHECK("scan_seq_kernel");
    return FV_OK;
}

// Staged pooling (masked: bucketing of the kept ids, then pooling).
fv_status staged_front(const fv::Shape& sh, const fv_ssm_args* a, const fv_ws_layout& L, char* ws, unsigned* status,
                       cudaStream_t st, EventMarks& marks) {
    const int M = sh.B * sh.T;
    float* xbar = (float*)(ws + L.xbar);
    if (sh.K == 0) {
        FV_MARK_CALL(marks, st, ([&]() -> fv_status {
            // a whole number of token groups of SL threads each (no idle threads)
            const int threads = sh.SL <= fv::kThreads ? (fv::kThreads / sh.SL) * sh.SL : fv::kThreads;
            if (sh.dc > 0) {
                fv::pool_conv_kernel<<<M, threads, 0, st>>>(sh, a->x, a->conv_w, a->conv_b, xbar);
                FV_LAUNCH_CHECK("pool_conv_kernel");
            } else {
                fv::pool_dense_kernel<<<M, threads, 0, st>>>(sh, a->x, xbar);
                FV_LAUNCH_CHECK("pool_dense_kernel");
            }
            return FV_OK;
        })());
        return FV_OK;
    }
    const size_t bsm = bucket_smem_bytes(sh);
    cudaError_t e = ensure_smem(fv::mask_bucket_kernel, bsm);
    if (e != cudaSuccess) { note_cuda(e, "bucket smem attribute"); return FV_ERR_CUDA; }
    FV_MARK_CALL(marks, st, ([&]() -> fv_status {
        fv::mask_bucket_kernel<<<sh.B, fv::kThreads, bsm, st>>>(sh, a->keep_idx, (int32_t*)(ws + L.row_of),
                                                                (int32_t*)(ws + L.row_off),
                                                                (int32_t*)(ws + L.row_tok), status);
        FV_LAUNCH_CHECK("mask_bucket_kernel");
        return FV_OK;
    })());
    FV_MARK_CALL(marks, st, ([&]() -> fv_status {
        const int threads = sh.SL <= fv::kThreads ? fv::kThreads
                                                  : std::min(fv::kMaskPoolMaxThreads, (sh.SL + 31) / 32 * 32);
        fv::mask_pool_kernel<<<M, threads, 0, st>>>(sh, a->x, (const int32_t*)(ws + L.row_off),
                                                         (const int32_t*)(ws + L.row_tok), xbar);
        FV_LAUNCH_CHECK("mask_pool_kernel");
        return FV_OK;
    })());
    return FV_OK;
}

// Staged x_proj: one GEMM over all pooled tokens of the chunk.
fv_status launch_proj_gemm(const fv::Shape& sh, const fv_ssm_args* a, const fv_ws_layout& L, char* ws, cudaStream_t st) {
    cudaError_t e = ensure_smem(fv::proj_gemm_kernel, fv::kPgSmemBytes);
    if (e != cudaSuccess) { note_cuda(e, "proj smem attribute"); return FV_ERR_CUDA; }
    const long long M = (long long)sh.B * sh.T;
    const int nz = sh.NJ / sh.nx;  // outputs per pooled-token set
    const dim3 grid((unsigned)((M + fv::kPgM - 1) / fv::kPgM), (unsigned)((nz + fv::kPgN - 1) / fv::kPgN),
                    (unsigned)sh.nx);
    if (M >= (1ll << 31) / 2) return FV_ERR_UNSUPPORTED;
    fv::proj_gemm_kernel<<<grid, fv::kPgThreads, fv::kPgSmemBytes, st>>>(sh, (const float*)(ws + L.xbar), a->W_x,
                                                                        (float*)(ws + L.u));
    FV_LAUNCH_CHECK("proj_gemm_kernel");
    return FV_OK;
}

// dt_proj + softplus: Delta for every pooled token of the batch and direction, on the tensor
// cores (fv_dt_tc.cuh), one CTA per 128 tokens x 128 channels of a direction.
fv_status launch_dt_proj_to(const fv::Shape& sh, const float* u, const float* W_dt, const float* b_dt, float* delta,
                            unsigned* status, cudaStream_t st) {
    const long long M = (long long)sh.B * sh.T;
    if (M >= (1ll << 31) / 2) return FV_ERR_UNSUPPORTED;
    cudaError_t e = ensure_smem(fv::dt_proj_kernel, fv::kDtSmemBytes);
    if (e != cudaSuccess) { note_cuda(e, "dt_proj smem attribute"); return FV_ERR_CUDA; }
    const dim3 grid((unsigned)((M + fv::kDtM - 1) / fv::kDtM), (unsigned)((sh.E + fv::kDtN - 1) / fv::kDtN),
                    (unsigned)sh.nd);
    fv::dt_proj_kernel<<<grid, fv::kDtThreads, fv::kDtSmemBytes, st>>>(sh, u, W_dt, b_dt, delta, status);
    FV_LAUNCH_CHECK("dt_proj_kernel");
    return FV_OK;
}
fv_status launch_dt_proj(const fv::Shape& sh, const fv_ssm_args* a, const fv_ws_layout& L, char* ws, cudaStream_t st) {
    return launch_dt_proj_to(sh, (const float*)(ws + L.u), a->W_dt, a->b_dt, (float*)(ws + L.delta),
                             (unsigned*)(ws + L.status), st);
}
// Staged x_proj, dt_proj + softplus as its own GEMM from dt_rank 32 (else inside the scans), then
// ZOH + scans.
fv_status staged_middle(const fv::Shape& sh, const fv_ssm_args* a, const fv_ws_layout& L, char* ws, cudaStream_t st,
                        EventMarks& marks) {
    FV_MARK_CALL(marks, st, launch_proj_gemm(sh, a, L, ws, st));
    if (fv::staged_delta_kernel(sh)) FV_MARK_CALL(marks, st, launch_dt_proj(sh, a, L, ws, st));
    FV_MARK_CALL(marks, st, launch_scan_seq(sh, a, L, ws, st));
    return FV_OK;
}

// Staged repeat + skip (+ LayerNorm) + gate.
fv_status staged_back(const fv::Shape& sh, const fv_ssm_args* a, const fv_ws_layout& L, char* ws, cudaStream_t st,
                      EventMarks& marks) {
    const float* ys = (const float*)(ws + L.ys);
    if (sh.ln && ln_uses_reg_kernel(sh)) {
        const size_t smem = (size_t)3 * sh.SL * sizeof(float4);
        const int nsl = fv::ln_reg_nsl(sh.SL);
        // the widest rows (12 slots per lane) take two warps per token at 6 slots each
        auto kern = nsl == 1 ? fv::ln_epilogue_reg_kernel<1, 1> : nsl == 2 ? fv::ln_epilogue_reg_kernel<2, 1>
                  : nsl == 3 ? fv::ln_epilogue_reg_kernel<3, 1> : nsl == 4 ? fv::ln_epilogue_reg_kernel<4, 1>
                  : nsl == 6 ? fv::ln_epilogue_reg_kernel<6, 1> : nsl == 8 ? fv::ln_epilogue_reg_kernel<8, 1>
                  : fv::ln_epilogue_reg_kernel<6, 2>;
        cudaError_t e = ensure_smem(kern, smem);
        if (e != cudaSuccess) { note_cuda(e, "LayerNorm epilogue smem attribute"); return FV_ERR_CUDA; }
        int per_sm = 0;
        if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, fv::kLnRegWarps * 32, smem)) !=
            cudaSuccess) {
            note_cuda(e, "LayerNorm epilogue occupancy");
            return FV_ERR_CUDA;
        }
        const long long ntok = (long long)sh.B * (sh.K > 0 ? (long long)sh.K : (long long)sh.h * sh.w);
        // persistent over tokens: four waves of resident blocks, a warp per token at a time
        long long grid = (long long)std::max(per_sm, 1) * device_sm_count() * 4;
        const long long need = (ntok + fv::kLnRegWarps - 1) / fv::kLnRegWarps;
        if (grid > need) grid = need;
        FV_MARK_CALL(marks, st, ([&]() -> fv_status {
            kern<<<(unsigned)grid, fv::kLnRegWarps * 32, smem, st>>>(sh, a->x, a->z, ys, a->D, a->ln_gamma, a->ln_beta,
                                                                     sh.K > 0 ? (const int32_t*)(ws + L.row_of)
                                                                              : nullptr,
                                                                     a->y);
            FV_LAUNCH_CHECK("ln_epilogue_reg_kernel");
            return FV_OK;
        })());
    } else if (sh.ln) {
        const size_t smem = fv::ln_epilogue_smem_bytes(sh);
        auto kern = sh.dc > 0 ? fv::ln_epilogue_kernel<true> : fv::ln_epilogue_kernel<false>;
        cudaError_t e = ensure_smem(kern, smem);
        if (e != cudaSuccess) { note_cuda(e, "LayerNorm epilogue smem attribute"); return FV_ERR_CUDA; }
        const long long ntok = (long long)sh.B * (sh.K > 0 ? (long long)sh.K : (long long)sh.h * sh.w);
        const long long per = (long long)fv::kLnWarps * fv::kLnTokensPerWarp;
        const long long grid = (ntok + per - 1) / per;
        if (grid >= (1ll << 31)) return FV_ERR_UNSUPPORTED;
        FV_MARK_CALL(marks, st, ([&]() -> fv_status {
            kern<<<(unsigned)grid, fv::kLnWarps * 32, smem, st>>>(
                sh, a->x, a->z, ys, a->D, a->ln_gamma, a->ln_beta,
                sh.K > 0 ? (const int32_t*)(ws + L.row_of) : nullptr, a->conv_w, a->conv_b, a->y);
            FV_LAUNCH_CHECK("ln_epilogue_kernel");
            return FV_OK;
        })());
    } else if (sh.K == 0 && sh.dc > 0) {
        FV_MARK_CALL(marks, st, ([&]() -> fv_status {
            const int threads = sh.SL <= fv::kThreads ? (fv::kThreads / sh.SL) * sh.SL : fv::kThreads;
            fv::epilogue_conv_kernel<<<sh.B * sh.T, threads, 0, st>>>(sh, a->x, a->z, ys, a->D, a->conv_w, a->conv_b,
                                                                       a->y);
            FV_LAUNCH_CHECK("epilogue_conv_kernel");
            return FV_OK;
        })());
    } else if (sh.K == 0) {
        FV_MARK_CALL(marks, st, ([&]() -> fv_status {
            fv::epilogue_dense_kernel<<<sh.B * sh.T, fv::kThreads, 0, st>>>(sh, a->x, a->z, ys, a->D, a->y);
            FV_LAUNCH_CHECK("epilogue_dense_kernel");
            return FV_OK;
        })());
    } else {
        const int nkb = (sh.K + fv::kMaskEpiTokens - 1) / fv::kMaskEpiTokens;
        const size_t msm = (size_t)sh.SL * sizeof(float4);
        cudaError_t e = ensure_smem(fv::mask_epilogue_kernel, msm);
        if (e != cudaSuccess) { note_cuda(e, "masked epilogue smem attribute"); return FV_ERR_CUDA; }
        FV_MARK_CALL(marks, st, ([&]() -> fv_status {
            fv::mask_epilogue_kernel<<<sh.B * nkb, fv::kThreads, msm, st>>>(sh, a->x, a->z, ys, a->D,
                                                                           (const int32_t*)(ws + L.row_of), a->y);
            FV_LAUNCH_CHECK("mask_epilogue_kernel");
            return FV_OK;
        })());
    }
    return FV_OK;
}

fv_status forward_impl(const fv_ssm_args* a, void* ws_v, size_t ws_bytes, cudaStream_t st,
                       void* const* events = nullptr, int n_events = 0) {
    fv::Shape sh;
    fv_status s = make_shape(a, &sh);
    if (s != FV_OK) return s;
    if ((s = check_pointers(a, sh)) != FV_OK) return s;
    fv_ws_layout L;
    plan_layout(sh, &L);
    if (!ws_v || ws_bytes < L.total_bytes || ((uintptr_t)ws_v & 255u) != 0) return FV_ERR_WORKSPACE;
    if ((s = check_limits(sh)) != FV_OK) return s;
    if (events && n_events < 2 * launch_count_of(sh)) return FV_ERR_SHAPE;
    EventMarks marks{events, launch_count_of(sh), 0};
    char* ws = (char*)ws_v;
    unsigned* status = (unsigned*)(ws + L.status);
    cudaError_t e = cudaMemsetAsync(status, 0, sizeof(unsigned), st);
    if (e != cudaSuccess) { note_cuda(e, "status reset"); return FV_ERR_CUDA; }
    if (sh.B == 0) return FV_OK;
    const Path path = choose_path(sh);
    if (path == Path::Invalid) return FV_ERR_UNSUPPORTED;
    if (path == Path::Fused) {
        // control block (ticket, abort flag, per-image counters) starts at zero
        e = cudaMemsetAsync(ws + L.ctrl, 0, (fv::kCtrlHeaderWords + fv::kCtrlCounters * (size_t)sh.B) * sizeof(unsigned), st);
        if (e != cudaSuccess) { note_cuda(e, "control reset"); return FV_ERR_CUDA; }
        FV_MARK_CALL(marks, st, launch_fused(sh, a, L, ws, st));
        return FV_OK;
    }

    if ((s = staged_front(sh, a, L, ws, status, st, marks)) != FV_OK) return s;
    if ((s = staged_middle(sh, a, L, ws, st, marks)) != FV_OK) return s;
    return staged_back(sh, a, L, ws, st, marks);
}

}  // namespace

extern "C" {

const char* fastvim_status_string(fv_status s) {
    switch (s) {
        case FV_OK: return "FV_OK";
        case FV_ERR_NULL: return "FV_ERR_NULL: a required pointer is NULL";
        case FV_ERR_SHAPE: return "FV_ERR_SHAPE: a size or flag is out of range";
        case FV_ERR_ALIGN: return "FV_ERR_ALIGN: a pointer is not 16-byte aligned";
        case FV_ERR_INDEX: return "FV_ERR_INDEX: a keep index is out of range or repeated";
        case FV_ERR_WORKSPACE: return "FV_ERR_WORKSPACE: workspace missing, too small or misaligned";
        case FV_ERR_CUDA: return "FV_ERR_CUDA: a CUDA call failed";
        case FV_ERR_TIMEOUT: return "FV_ERR_TIMEOUT: a bounded device wait gave up";
        case FV_ERR_UNSUPPORTED: return "FV_ERR_UNSUPPORTED: beyond this build's limits";
        case FV_ERR_ALIAS: return "FV_ERR_ALIAS: y overlaps x or z";
    }
    return "unknown fv_status";
}

const char* fastvim_last_error(void) { return g_last_error; }

int fastvim_abi_version(void) { return FASTVIM_SSM_ABI_VERSION; }

fv_status fastvim_ssm_validate(const fv_ssm_args* args) {
    fv::Shape sh;
    fv_status s = make_shape(args, &sh);
    if (s != FV_OK) return s;
    return check_pointers(args, sh);
}

size_t fastvim_ssm_workspace_size(const fv_ssm_args* args) {
    fv::Shape sh;
    if (make_shape(args, &sh) != FV_OK) return 0;
    fv_ws_layout L;
    plan_layout(sh, &L);
    return L.total_bytes;
}

fv_status fastvim_ssm_workspace_layout(const fv_ssm_args* args, fv_ws_layout* out) {
    if (!out) return FV_ERR_NULL;
    fv::Shape sh;
    fv_status s = make_shape(args, &sh);
    if (s != FV_OK) return s;
    return plan_layout(sh, out);
}

int fastvim_ssm_launch_count(const fv_ssm_args* args) {
    fv::Shape sh;
    if (make_shape(args, &sh) != FV_OK) return 0;
    return launch_count_of(sh);
}

const char* fastvim_ssm_launch_name(const fv_ssm_args* args, int i) {
    fv::Shape sh;
    if (make_shape(args, &sh) != FV_OK) return "";
    return launch_name_of(sh, i);
}

fv_status fastvim_ssm_forward(const fv_ssm_args* args, void* ws, size_t ws_bytes, void* stream) {
    return forward_impl(args, ws, ws_bytes, (cudaStream_t)stream);
}

fv_status fastvim_ssm_forward_events(const fv_ssm_args* args, void* ws, size_t ws_bytes, void* stream,
                                     void* const* events, int n_events) {
    if (!events) return FV_ERR_NULL;
    return forward_impl(args, ws, ws_bytes, (cudaStream_t)stream, events, n_events);
}

namespace {
// x bytes per chunk of images in fastvim_ssm_forward_host, and the most chunks it makes.
constexpr size_t kHostChunkBytes = (size_t)64 << 20;
constexpr int kHostMaxChunks = 16;

// Streams and events of one fastvim_ssm_forward_host call, released on every exit path.
struct HostPipe {
    cudaStream_t up = nullptr, down = nullptr;
    std::vector<cudaEvent_t> ev;
    ~HostPipe() {
        if (up) cudaStreamSynchronize(up);
        if (down) cudaStreamSynchronize(down);
        for (cudaEvent_t e : ev)
            if (e) cudaEventDestroy(e);
        if (up) cudaStreamDestroy(up);
        if (down) cudaStreamDestroy(down);
    }
    cudaEvent_t make() {
        cudaEvent_t e = nullptr;
        if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) e = nullptr;
        ev.push_back(e);
        return e;
    }
};
}  // namespace

fv_status fastvim_ssm_forward_host(const fv_ssm_args* host, const fv_ssm_args* dev, void* ws,
                                   size_t ws_bytes, void* stream) {
    if (!host || !dev) return FV_ERR_NULL;
    fv::Shape sh, shd;
    fv_status s = make_shape(host, &sh);
    if (s != FV_OK) return s;
    if ((s = make_shape(dev, &shd)) != FV_OK) return s;
    if (host->B != dev->B || host->h != dev->h || host->w != dev->w || host->E != dev->E ||
        host->N != dev->N || host->R != dev->R || host->K != dev->K || host->pool_axis != dev->pool_axis ||
        host->dir_flags != dev->dir_flags || host->flags != dev->flags || host->pool_scale != dev->pool_scale ||
        host->d_conv != dev->d_conv ||
        ((host->flags & FV_FLAG_LAYERNORM) && host->ln_eps != dev->ln_eps))
        return FV_ERR_SHAPE;
    if ((s = check_pointers(host, sh)) != FV_OK) return s;
    if ((s = check_pointers(dev, shd)) != FV_OK) return s;
    {
        fv_ws_layout L;
        plan_layout(sh, &L);
        if (!ws || ws_bytes < L.total_bytes || ((uintptr_t)ws & 255u) != 0) return FV_ERR_WORKSPACE;
        if ((s = check_limits(sh)) != FV_OK) return s;
    }
    cudaStream_t st = (cudaStream_t)stream;
    const size_t tok = sh.K > 0 ? (size_t)sh.K : (size_t)sh.h * sh.w;
    const size_t img = tok * sh.E * sizeof(float);  // bytes of one image's x, z or y
    const size_t nd = (size_t)sh.nd;

    // The images are independent, so the batch runs as chunks of images in a three-stage
    // pipeline: chunk c's x and z go up on one stream while chunk c-1 is computed on the caller's
    // stream and chunk c-2's y comes down on a third (the two copy directions run concurrently).
    int chunks = 1;
    if (sh.B > 1) {
        const size_t want = ((size_t)sh.B * img + kHostChunkBytes - 1) / kHostChunkBytes;
        chunks = (int)std::min<size_t>(std::min<size_t>(want, (size_t)kHostMaxChunks), (size_t)sh.B);
        if (chunks < 1) chunks = 1;
    }
    const int per = sh.B > 0 ? (sh.B + chunks - 1) / chunks : 0;
    chunks = per > 0 ? (sh.B + per - 1) / per : 1;

    HostPipe pp;
    auto cuda_fail = [&](cudaError_t e, const char* where) { note_cuda(e, where); return FV_ERR_CUDA; };
    cudaError_t e = cudaStreamCreateWithFlags(&pp.up, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&pp.down, cudaStreamNonBlocking);
    if (e != cudaSuccess) return cuda_fail(e, "host pipeline streams");
    cudaEvent_t start = pp.make(), down_done = pp.make();
    std::vector<cudaEvent_t> up_done(chunks), computed(chunks);
    for (int c = 0; c < chunks; ++c) { up_done[c] = pp.make(); computed[c] = pp.make(); }
    for (cudaEvent_t v : pp.ev)
        if (!v) return cuda_fail(cudaErrorMemoryAllocation, "host pipeline events");

    // the copies start after the work the caller queued before this call
    if ((e = cudaEventRecord(start, st)) != cudaSuccess) return cuda_fail(e, "event record");
    if ((e = cudaStreamWaitEvent(pp.up, start, 0)) != cudaSuccess) return cuda_fail(e, "stream wait");
    struct Copy { void* dst; const void* src; size_t bytes; } params[] = {
        {(void*)dev->A_log, host->A_log, nd * sh.E * sh.N * sizeof(float)},
        {(void*)dev->D, host->D, nd * sh.E * sizeof(float)},
        {(void*)dev->W_x, host->W_x, nd * sh.J * sh.E * sizeof(float)},
        {(void*)dev->W_dt, host->W_dt, nd * sh.E * sh.R * sizeof(float)},
        {(void*)dev->b_dt, host->b_dt, nd * sh.E * sizeof(float)},
        {(void*)dev->keep_idx, host->keep_idx, sh.K > 0 ? (size_t)sh.B * sh.K * sizeof(int32_t) : 0},
        {(void*)dev->ln_gamma, host->ln_gamma, sh.ln ? (size_t)sh.E * sizeof(float) : 0},
        {(void*)dev->ln_beta, host->ln_beta, sh.ln ? (size_t)sh.E * sizeof(float) : 0},
        {(void*)dev->conv_w, host->conv_w, nd * sh.E * (size_t)sh.dc * sizeof(float)},
        {(void*)dev->conv_b, host->conv_b, sh.dc > 0 ? nd * sh.E * sizeof(float) : 0},
    };
    for (const Copy& c : params) {
        if (c.bytes == 0 || !c.dst) continue;
        if ((e = cudaMemcpyAsync(c.dst, c.src, c.bytes, cudaMemcpyHostToDevice, pp.up)) != cudaSuccess)
            return cuda_fail(e, "host->device copy");
    }
    unsigned* status = (unsigned*)ws;  // word 0 of the layout; word 1 keeps the first error
    if (chunks > 1 && (e = cudaMemsetAsync(status + 1, 0, sizeof(unsigned), st)) != cudaSuccess)
        return cuda_fail(e, "status reset");
    for (int c = 0; c < chunks; ++c) {
        const int b0 = c * per, nb = std::max(0, std::min(per, sh.B - b0));
        const size_t off = (size_t)b0 * tok * sh.E;  // float offset of the chunk's first image
        const size_t bytes = (size_t)nb * img;
        if (bytes > 0) {
            if ((e = cudaMemcpyAsync((void*)(dev->x + off), host->x + off, bytes, cudaMemcpyHostToDevice, pp.up)) != cudaSuccess ||
                (e = cudaMemcpyAsync((void*)(dev->z + off), host->z + off, bytes, cudaMemcpyHostToDevice, pp.up)) != cudaSuccess)
                return cuda_fail(e, "host->device copy");
        }
        if ((e = cudaEventRecord(up_done[c], pp.up)) != cudaSuccess) return cuda_fail(e, "event record");
        if ((e = cudaStreamWaitEvent(st, up_done[c], 0)) != cudaSuccess) return cuda_fail(e, "stream wait");
        fv_ssm_args a = *dev;
        a.B = nb;
        if (bytes > 0) { a.x = dev->x + off; a.z = dev->z + off; a.y = dev->y + off; }
        if (sh.K > 0 && nb > 0) a.keep_idx = dev->keep_idx + (size_t)b0 * sh.K;
        if ((s = forward_impl(&a, ws, ws_bytes, st)) != FV_OK) return s;
        if (chunks > 1) {
            fv::status_fold_kernel<<<1, 32, 0, st>>>(status + 1, status);
            FV_LAUNCH_CHECK("status_fold_kernel");
        }
        if ((e = cudaEventRecord(computed[c], st)) != cudaSuccess) return cuda_fail(e, "event record");
        if ((e = cudaStreamWaitEvent(pp.down, computed[c], 0)) != cudaSuccess) return cuda_fail(e, "stream wait");
        if (bytes > 0 &&
            (e = cudaMemcpyAsync(host->y + off, dev->y + off, bytes, cudaMemcpyDeviceToHost, pp.down)) != cudaSuccess)
            return cuda_fail(e, "device->host copy");
    }
    if (chunks > 1) {  // the call's status word reports the first error of any chunk
        fv::status_fold_kernel<<<1, 32, 0, st>>>(status, status + 1);
        FV_LAUNCH_CHECK("status_fold_kernel");
    }
    if ((e = cudaEventRecord(down_done, pp.down)) != cudaSuccess) return cuda_fail(e, "event record");
    if ((e = cudaStreamWaitEvent(st, down_done, 0)) != cudaSuccess) return cuda_fail(e, "stream wait");
    if ((e = cudaStreamSynchronize(st)) != cudaSuccess) return cuda_fail(e, "stream synchronize");
    return FV_OK;
}

fv_status fastvim_selftest_bounded_wait(void* ws, size_t ws_bytes, unsigned limit_us, void* stream) {
    if (!ws) return FV_ERR_NULL;
    if (ws_bytes < 1024 || ((uintptr_t)ws & 255u) != 0) return FV_ERR_WORKSPACE;
    if (limit_us == 0 || limit_us > 10u * 1000u * 1000u) return FV_ERR_SHAPE;
    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t e = cudaMemsetAsync(ws, 0, 1024, st);
    if (e != cudaSuccess) { note_cuda(e, "selftest reset"); return FV_ERR_CUDA; }
    unsigned* status = (unsigned*)ws;
    unsigned* ctrl = (unsigned*)((char*)ws + 256);
    fv::bounded_wait_selftest_kernel<<<1, 32, 0, st>>>(status, ctrl, (unsigned long long)limit_us * 1000ull);
    FV_LAUNCH_CHECK("bounded_wait_selftest_kernel");
    return FV_OK;
}

fv_status fastvim_selftest_math(int fn, const float* in, float* out, int n, void* stream) {
    if (fn < 0 || fn > 2 || n < 0) return FV_ERR_SHAPE;
    if (n == 0) return FV_OK;
    if (!in || !out) return FV_ERR_NULL;
    if (((uintptr_t)in & 15u) || ((uintptr_t)out & 15u)) return FV_ERR_ALIGN;
    if ((const char*)out < (const char*)(in + n) && (const char*)in < (const char*)(out + n)) return FV_ERR_ALIAS;
    fv::math_selftest_kernel<<<(n + 255) / 256, 256, 0, (cudaStream_t)stream>>>(fn, in, out, n);
    FV_LAUNCH_CHECK("math_selftest_kernel");
    return FV_OK;
}

fv_status fastvim_get_device_status(const void* ws, void* stream) {
    if (!ws) return FV_ERR_NULL;
    cudaStream_t st = (cudaStream_t)stream;
    unsigned v = 0;
    cudaError_t e = cudaMemcpyAsync(&v, ws, sizeof v, cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) { note_cuda(e, "status read"); return FV_ERR_CUDA; }
    return (fv_status)v;
}

}  // extern "C"

// ------------------------------------------------------------------------------------------------
// Allocation-free entry point: the forward call with its workspace in a fixed static device
// array instead of caller-provided memory.
// ------------------------------------------------------------------------------------------------
namespace {

// 16 MiB of device memory on every GPU where this library's device code is loaded (CUDA loads it
// lazily, at the first symbol lookup or launch on that device), held until the process exits.
constexpr size_t kStaticScratchBytes = (size_t)16 << 20;
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

constexpr int kMaxScratchDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxScratchDevices] = {};

// Device address of g_static_scratch on the current device.  Host code only sees a host-side
// stand-in under that name, so the real address is asked from the runtime, once per device,
// with that device current.
fv_status static_scratch_address(void** out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) { note_cuda(e, "cudaGetDevice"); return FV_ERR_CUDA; }
    if (dev < 0 || dev >= kMaxScratchDevices) return FV_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_static_scratch);
        if (e != cudaSuccess || !p) {
            note_cuda(e, "cudaGetSymbolAddress(static scratch)");
            return FV_ERR_CUDA;
        }
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return FV_OK;
}

}  // namespace

extern "C" fv_status fastvim_ssm_forward_noalloc(const fv_ssm_args* args, void* stream) {
    fv::Shape sh;
    fv_status s = make_shape(args, &sh);
    if (s != FV_OK) return s;
    if ((s = check_pointers(args, sh)) != FV_OK) return s;
    fv_ws_layout L;
    plan_layout(sh, &L);
    if (L.total_bytes > kStaticScratchBytes) {
        snprintf(g_last_error, sizeof g_last_error,
                 "fastvim_ssm_forward_noalloc: this layer needs %zu bytes of scratch, above the %zu-byte "
                 "static scratch; split the batch or use fastvim_ssm_forward with a workspace",
                 L.total_bytes, kStaticScratchBytes);
        return FV_ERR_UNSUPPORTED;
    }
    void* scratch = nullptr;
    if ((s = static_scratch_address(&scratch)) != FV_OK) return s;
    // Every region of the workspace is written before it is read within one call, and each call
    // resets the status word itself, so the contents left by an earlier call need no clearing.
    return forward_impl(args, scratch, kStaticScratchBytes, (cudaStream_t)stream);
}

// ------------------------------------------------------------------------------------------------
// Gradient of the layer.
// ------------------------------------------------------------------------------------------------
namespace {

struct BwdLayout {
    size_t status, dys, dxbar, du, dxs, ckpt, delta;
    // per-block partial sums, added in a fixed order by bwd_reduce_kernel
    size_t partials, part_du, part_dA, part_wdt, part_bdt, part_wx, part_gate;
    size_t total;
};

// Caps that size the partial-sum scratch independently of the GPU: blocks of the persistent gate
// gradient, and K splits of the dW_x GEMM.
constexpr int kMaxGateBlocks = 2048;
constexpr int kMaxWxSplits = 64;

// Whether the forward call's workspace holds the step sizes Delta (staged path, dt_rank >= 32);
// otherwise the gradient computes them into its own workspace first.
bool fwd_has_delta(const fv::Shape& sh) {
    fv_ws_layout FL;
    plan_layout(sh, &FL);
    return FL.delta != 0;
}

BwdLayout plan_bwd(const fv::Shape& sh) {
    BwdLayout L{};
    size_t off = 0;
    const size_t bte = (size_t)sh.B * sh.T * sh.E * sizeof(float);
    L.status = off; off = round256(off + 2 * sizeof(unsigned));
    L.dys = off; off = round256(off + bte);
    L.dxbar = off; off = round256(off + bte);
    L.du = off; off = round256(off + (size_t)sh.nd * sh.B * fv::u_block_stride(sh.T, sh.J) * sizeof(float));
    L.dxs = off; off = round256(off + (size_t)sh.nd * bte);
    if (!sh.keep) {  // else the forward kept the scan states in its workspace
        L.ckpt = off;
        off = round256(off + (size_t)sh.B * sh.nd * fv::bs_nckpt(sh.T) * sh.E * 16 * sizeof(float));
    }
    if (!fwd_has_delta(sh)) {
        L.delta = off;
        off = round256(off + (size_t)sh.nd * sh.B * sh.T * sh.E * sizeof(float));
    }
    const size_t f = sizeof(float), ne = (size_t)sh.nd * sh.B * sh.E;
    L.partials = off;
    L.part_du = off;
    off = round256(off + (size_t)((sh.E + fv::kBsCh - 1) / fv::kBsCh) * sh.nd * sh.B * fv::u_block_stride(sh.T, sh.J) * f);
    L.part_dA = off; off = round256(off + ne * sh.N * f);
    L.part_wdt = off; off = round256(off + ne * sh.R * f);
    L.part_bdt = off; off = round256(off + ne * f);
    L.part_wx = off; off = round256(off + (size_t)kMaxWxSplits * sh.nd * sh.J * sh.E * f);
    L.part_gate = off; off = round256(off + (size_t)kMaxGateBlocks * (sh.ln ? 3 : 1) * sh.E * f);
    L.total = off;
    return L;
}

// Launch order of a gradient call: gate (through the LayerNorm with FV_FLAG_LAYERNORM), dt_proj
// (when the forward workspace holds no step sizes), scans (with dt_proj's gradient), dW_x, dxbar,
// pooling.
// The LayerNorm gate gradient keeps each token in registers across groups of up to 8 warps
// (E <= 2048); wider rows take the shared-memory-row kernel.
bool bwd_ln_uses_reg(const fv::Shape& sh) { return fv::bwd_lnr_wpt(sh.SL) <= 8; }
int bwd_launch_count_of(const fv::Shape& sh) { return sh.B == 0 ? 0 : (fwd_has_delta(sh) ? 7 : 8); }
const char* bwd_launch_name_of(const fv::Shape& sh, int i) {
    static const char* dense[] = {"bwd_gate_dense_kernel", "dt_proj_kernel", "bwd_scan_kernel", "bwd_reduce_kernel:du",
                                  "bwd_dwx_kernel", "bwd_dxbar_kernel", "bwd_pool_dense_kernel",
                                  "bwd_reduce_kernel:params"};
    static const char* masked[] = {"bwd_gate_masked_kernel", "dt_proj_kernel", "bwd_scan_kernel", "bwd_reduce_kernel:du",
                                   "bwd_dwx_kernel", "bwd_dxbar_kernel", "bwd_pool_masked_kernel",
                                   "bwd_reduce_kernel:params"};
    const int n = bwd_launch_count_of(sh);
    if (i < 0 || i >= n) return "";
    if (i == 0 && sh.ln) return bwd_ln_uses_reg(sh) ? "bwd_ln_gate_reg_kernel" : "bwd_ln_gate_kernel";
    const int j = (n == 7 && i >= 1) ? i + 1 : i;
    return sh.K > 0 ? masked[j] : dense[j];
}

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
    const uintptr_t a0 = (uintptr_t)a, b0 = (uintptr_t)b;
    return a && b && a0 < b0 + nb && b0 < a0 + na;
}

fv_status check_grads(const fv_ssm_args* a, const fv::Shape& sh, const fv_ssm_grads* g) {
    if (!g) return FV_ERR_NULL;
    if (!g->dA_log || !g->dD || !g->dW_x || !g->dW_dt || !g->db_dt) return FV_ERR_NULL;
    if (sh.B > 0 && (!g->dy || !g->dx || !g->dz)) return FV_ERR_NULL;
    if (sh.ln && (!g->dln_gamma || !g->dln_beta)) return FV_ERR_NULL;
    if (!sh.ln && (g->dln_gamma || g->dln_beta)) return FV_ERR_SHAPE;  // LayerNorm gradients need the flag
    const void* ps[] = {g->dy, g->dx, g->dz, g->dA_log, g->dD, g->dW_x, g->dW_dt, g->db_dt, g->dln_gamma, g->dln_beta};
    for (const void* p : ps)
        if (p && !aligned16(p)) return FV_ERR_ALIGN;
    if (sh.B > 0) {
        const size_t tok = sh.K > 0 ? (size_t)sh.K : (size_t)sh.h * sh.w;
        const size_t n = (size_t)sh.B * tok * sh.E * sizeof(float);
        if (overlaps(g->dx, n, g->dz, n) || overlaps(g->dx, n, g->dy, n) || overlaps(g->dz, n, g->dy, n) ||
            overlaps(g->dx, n, a->x, n) || overlaps(g->dx, n, a->z, n) || overlaps(g->dz, n, a->x, n) ||
            overlaps(g->dz, n, a->z, n))
            return FV_ERR_ALIAS;
    }
    return FV_OK;
}

// Tokens in flight per thread of the dense gate gradient.  B200, 2048 px layer: 2 tokens (64
// registers, 30 warps per SM) stream at 0.945 of the copy rate, 4 tokens (99 registers, 18 warps)
// at 0.79.
constexpr int kBwdGateTokens = 2;

int device_sm_count() {
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        sms <= 0)
        return 148;
    return sms;
}

// Tokens per split of dW_x (a multiple of the kernel's 16-token k-step) for about `splits` splits of
// M; the splits that result are ceil(M / chunk).
int bwd_kchunk(int M, int splits) {
    const int kchunk = (M + splits - 1) / splits;
    return (kchunk + fv::kGwK - 1) / fv::kGwK * fv::kGwK;
}

// dW_x partials: one instantiation per row count ceil(J / 16) (J <= kMaxJ = 96)
fv_status launch_bwd_dwx(const fv::Shape& sh, const float* du, const float* xbar, float* part, int splits,
                         int kchunk, cudaStream_t st) {
    const dim3 grid((sh.E + fv::kGwE - 1) / fv::kGwE, sh.nd * splits);
    const bool vec = (sh.J & 3) == 0;
#define FV_DWX(RT)                                                                                      \
    case RT:                                                                                            \
        if (vec) fv::bwd_dwx_kernel<RT, true><<<grid, fv::kThreads, 0, st>>>(sh, du, xbar, part, splits, kchunk); \
        else fv::bwd_dwx_kernel<RT, false><<<grid, fv::kThreads, 0, st>>>(sh, du, xbar, part, splits, kchunk); \
        break;
    switch ((sh.J + 15) / 16) {
        FV_DWX(1)
        FV_DWX(2)
        FV_DWX(3)
        FV_DWX(4)
        FV_DWX(5)
        FV_DWX(6)
        default: return FV_ERR_UNSUPPORTED;
    }
#undef FV_DWX
    FV_LAUNCH_CHECK("bwd_dwx_kernel");
    return FV_OK;
}

// Splits of a reduction over the M = B T pooled tokens: about 4 blocks per SM in all.
int bwd_splits(int M, int tiles, int sms) {
    int s = (4 * sms + tiles - 1) / tiles;
    const int most = (M + 255) / 256;  // at least 256 tokens per split
    if (s > most) s = most;
    return s < 1 ? 1 : s;
}

fv_status backward_impl(const fv_ssm_args* args, const fv_ssm_grads* g, const void* fwd_v, size_t fwd_bytes,
                        void* ws_v, size_t ws_bytes, cudaStream_t st, void* const* events = nullptr, int n_events = 0) {
    fv::Shape sh;
    fv_status s = make_shape(args, &sh);
    if (s != FV_OK) return s;
    // y is not read: a NULL y stands for "no output", checked as dx (which must not overlap x, z)
    fv_ssm_args ac = *args;
    if (!ac.y && g) ac.y = g->dx;
    const fv_ssm_args* a = &ac;
    if ((s = check_pointers(a, sh)) != FV_OK) return s;
    if ((s = check_grads(a, sh, g)) != FV_OK) return s;
    if (sh.dc > 0) return FV_ERR_UNSUPPORTED;  // the gradient through the Conv1D is not built
    fv_ws_layout FL;
    plan_layout(sh, &FL);
    const BwdLayout L = plan_bwd(sh);
    if (!fwd_v || fwd_bytes < FL.total_bytes || ((uintptr_t)fwd_v & 255u)) return FV_ERR_WORKSPACE;
    if (!ws_v || ws_bytes < L.total || ((uintptr_t)ws_v & 255u)) return FV_ERR_WORKSPACE;
    if (overlaps(fwd_v, FL.total_bytes, ws_v, L.total)) return FV_ERR_WORKSPACE;
    const size_t scan_smem = fv::bs_smem_floats(sh.R) * sizeof(float);
    if (scan_smem > kMaxSmemOptin) return FV_ERR_UNSUPPORTED;
    if (events && n_events < 2 * bwd_launch_count_of(sh)) return FV_ERR_SHAPE;
    EventMarks marks{events, bwd_launch_count_of(sh), 0};

    // parameter gradients: written by the final fixed-order reduction; an empty batch sums to zero
    const size_t nA = (size_t)sh.nd * sh.E * sh.N, nE = (size_t)sh.nd * sh.E, nWx = (size_t)sh.nd * sh.J * sh.E,
                 nWdt = (size_t)sh.nd * sh.E * sh.R;
    cudaError_t e = cudaSuccess;
    if (sh.B == 0 && ((e = cudaMemsetAsync(g->dA_log, 0, nA * sizeof(float), st)) != cudaSuccess ||
        (e = cudaMemsetAsync(g->dD, 0, nE * sizeof(float), st)) != cudaSuccess ||
        (e = cudaMemsetAsync(g->dW_x, 0, nWx * sizeof(float), st)) != cudaSuccess ||
        (e = cudaMemsetAsync(g->dW_dt, 0, nWdt * sizeof(float), st)) != cudaSuccess ||
        (e = cudaMemsetAsync(g->db_dt, 0, nE * sizeof(float), st)) != cudaSuccess ||
        (sh.ln && (e = cudaMemsetAsync(g->dln_gamma, 0, (size_t)sh.E * sizeof(float), st)) != cudaSuccess) ||
        (sh.ln && (e = cudaMemsetAsync(g->dln_beta, 0, (size_t)sh.E * sizeof(float), st)) != cudaSuccess))) {
        note_cuda(e, "gradient reset");
        return FV_ERR_CUDA;
    }
    if (sh.B == 0) return FV_OK;
    const char* fw = (const char*)fwd_v;
    char* ws = (char*)ws_v;
    const float* xbar = (const float*)(fw + FL.xbar);
    const float* u = (const float*)(fw + FL.u);
    const float* ys = (const float*)(fw + FL.ys);
    float* dys = (float*)(ws + L.dys);
    float* dxbar = (float*)(ws + L.dxbar);
    float* du = (float*)(ws + L.du);
    float* dxs = (float*)(ws + L.dxs);
    // the scan states every 8 steps: kept by the forward (FV_FLAG_KEEP_STATES), else pass 1 of
    // bwd_scan_kernel writes them here
    float* ckpt = sh.keep ? (float*)(fw + FL.ckpt) : (float*)(ws + L.ckpt);
    // the step sizes: the forward's (staged, dt_rank >= 32), else computed below into ws
    const float* delta = L.delta ? (const float*)(ws + L.delta) : (const float*)(fw + FL.delta);
    float* part_du = (float*)(ws + L.part_du);
    float* part_dA = (float*)(ws + L.part_dA);
    float* part_wdt = (float*)(ws + L.part_wdt);
    float* part_bdt = (float*)(ws + L.part_bdt);
    float* part_gate = (float*)(ws + L.part_gate);
    // the status word starts clear
    if ((e = cudaMemsetAsync(ws + L.status, 0, 2 * sizeof(unsigned), st)) != cudaSuccess) {
        note_cuda(e, "status reset");
        return FV_ERR_CUDA;
    }
    const int sms = device_sm_count();
    const int M = sh.B * sh.T;
    // one pass of bwd_reduce_kernel over `n` segments
    auto reduce = [&](const fv::RedSegs& segs, int n, const char* where) -> fv_status {
        long long most = 1;
        for (int i = 0; i < n; ++i) most = std::max(most, segs.seg[i].L);
        const long long want = (most + 31) / 32;  // 32 outputs per block at a time
        const dim3 grid((unsigned)std::min<long long>(want, 8ll * sms), (unsigned)n);
        fv::bwd_reduce_kernel<<<grid, fv::kRedWarps * 32, 0, st>>>(segs);
        FV_LAUNCH_CHECK(where);
        return FV_OK;
    };

    // 1. gate, skip and repeat
    // the gate kernels are persistent over pooled rows: one wave of resident blocks
    auto resident = [&](auto kern, int threads, size_t smem = 0) {
        int per_sm = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, smem) != cudaSuccess || per_sm < 1)
            per_sm = 1;
        return std::min(std::min(M, per_sm * sms), kMaxGateBlocks);
    };
    int gate_blocks = 0;  // rows of part_gate the gate kernel fills
    if (sh.ln && bwd_ln_uses_reg(sh)) {
        const int threads = 32 * fv::bwd_lnr_wpt(sh.SL) * fv::bwd_lnr_groups(sh.SL);
        const size_t smem = fv::bwd_lnr_smem_bytes(sh.SL);
        const int32_t* row_off = sh.K > 0 ? (const int32_t*)(fw + FL.row_off) : nullptr;
        const int32_t* row_tok = sh.K > 0 ? (const int32_t*)(fw + FL.row_tok) : nullptr;
        const bool one = fv::bwd_lnr_nsl(sh.SL) == 1;
        auto kern = sh.K > 0 ? (one ? fv::bwd_ln_gate_reg_kernel<1, true> : fv::bwd_ln_gate_reg_kernel<2, true>)
                             : (one ? fv::bwd_ln_gate_reg_kernel<1, false> : fv::bwd_ln_gate_reg_kernel<2, false>);
        if ((e = ensure_smem(kern, smem)) != cudaSuccess) {
            note_cuda(e, "LayerNorm gradient smem attribute");
            return FV_ERR_CUDA;
        }
        const int grid = gate_blocks = resident(kern, threads, smem);
        FV_MARK_CALL(marks, st, ([&]() -> fv_status {
            kern<<<grid, threads, smem, st>>>(sh, a->x, a->z, g->dy, ys, a->D, a->ln_gamma, a->ln_beta, row_off, row_tok,
                                              g->dx, g->dz, dys, part_gate);
            FV_LAUNCH_CHECK("bwd_ln_gate_reg_kernel");
            return FV_OK;
        })());
    } else if (sh.ln) {
        const int warps = fv::bwd_ln_warps(sh.SL);
        const size_t smem = fv::bwd_ln_smem_bytes(sh.SL, warps);
        const int32_t* row_off = sh.K > 0 ? (const int32_t*)(fw + FL.row_off) : nullptr;
        const int32_t* row_tok = sh.K > 0 ? (const int32_t*)(fw + FL.row_tok) : nullptr;
        FV_MARK_CALL(marks, st, ([&]() -> fv_status {
            if (sh.K > 0) {
                if ((e = ensure_smem(fv::bwd_ln_gate_kernel<true>, smem)) != cudaSuccess) {
                    note_cuda(e, "LayerNorm gradient smem attribute");
                    return FV_ERR_CUDA;
                }
                const int grid = gate_blocks = resident(fv::bwd_ln_gate_kernel<true>, 32 * warps, smem);
                fv::bwd_ln_gate_kernel<true><<<grid, 32 * warps, smem, st>>>(sh, a->x, a->z, g->dy, ys, a->D,
                                                                             a->ln_gamma, a->ln_beta, row_off, row_tok,
                                                                             g->dx, g->dz, dys, part_gate);
            } else {
                if ((e = ensure_smem(fv::bwd_ln_gate_kernel<false>, smem)) != cudaSuccess) {
                    note_cuda(e, "LayerNorm gradient smem attribute");
                    return FV_ERR_CUDA;
                }
                const int grid = gate_blocks = resident(fv::bwd_ln_gate_kernel<false>, 32 * warps, smem);
                fv::bwd_ln_gate_kernel<false><<<grid, 32 * warps, smem, st>>>(sh, a->x, a->z, g->dy, ys, a->D,
                                                                              a->ln_gamma, a->ln_beta, row_off,
                                                                              row_tok, g->dx, g->dz, dys, part_gate);
            }
            FV_LAUNCH_CHECK("bwd_ln_gate_kernel");
            return FV_OK;
        })());
    } else if (sh.K == 0) {
        const int threads = fv::bwd_groups(sh.SL) * fv::bwd_slot_width(sh.SL);
        auto kern = fv::bwd_gate_dense_kernel<kBwdGateTokens>;
        const int grid = gate_blocks = resident(kern, threads);
        FV_MARK_CALL(marks, st, ([&]() -> fv_status {
            kern<<<grid, threads, 0, st>>>(sh, a->x, a->z, g->dy, ys, a->D, g->dx, g->dz, dys, part_gate);
            FV_LAUNCH_CHECK("bwd_gate_dense_kernel");
            return FV_OK;
        })());
    } else {
        const int32_t* row_off = (const int32_t*)(fw + FL.row_off);
        const int32_t* row_tok = (const int32_t*)(fw + FL.row_tok);
        const int threads = fv::bwd_mgroups(sh.SL) * fv::bwd_mslot_width(sh.SL);
        const int grid = gate_blocks = resident(fv::bwd_gate_masked_kernel, threads);
        FV_MARK_CALL(marks, st, ([&]() -> fv_status {
            fv::bwd_gate_masked_kernel<<<grid, threads, 0, st>>>(sh, a->x, a->z, g->dy, ys, a->D, row_off, row_tok,
                                                                       g->dx, g->dz, dys, part_gate);
            FV_LAUNCH_CHECK("bwd_gate_masked_kernel");
            return FV_OK;
        })());
    }
    // 2. the step sizes (when the forward kept none), then the adjoint of the scans
    if (L.delta)
        FV_MARK_CALL(marks, st, launch_dt_proj_to(sh, u, a->W_dt, a->b_dt, (float*)(ws + L.delta),
                                                  (unsigned*)(ws + L.status), st));
    FV_MARK_CALL(marks, st, ([&]() -> fv_status {
        const dim3 grid(sh.B, sh.nd, (sh.E + fv::kBsCh - 1) / fv::kBsCh);
        if (sh.zoh_exact) {
            if ((e = ensure_smem(fv::bwd_scan_kernel<true>, scan_smem)) != cudaSuccess) {
                note_cuda(e, "scan gradient smem attribute");
                return FV_ERR_CUDA;
            }
            fv::bwd_scan_kernel<true><<<grid, fv::kBsThreads, scan_smem, st>>>(sh, u, xbar, dys, a->A_log, a->W_dt, delta,
                                                                              ckpt, dxs, part_du, part_dA, part_wdt,
                                                                              part_bdt);
        } else {
            if ((e = ensure_smem(fv::bwd_scan_kernel<false>, scan_smem)) != cudaSuccess) {
                note_cuda(e, "scan gradient smem attribute");
                return FV_ERR_CUDA;
            }
            fv::bwd_scan_kernel<false><<<grid, fv::kBsThreads, scan_smem, st>>>(sh, u, xbar, dys, a->A_log, a->W_dt,
                                                                               delta, ckpt, dxs, part_du, part_dA,
                                                                               part_wdt, part_bdt);
        }
        FV_LAUNCH_CHECK("bwd_scan_kernel");
        return FV_OK;
    })());
    // du = the sum of the 64-channel tiles' shares, in tile order
    {
        const int tiles = (sh.E + fv::kBsCh - 1) / fv::kBsCh;
        const long long ub = (long long)fv::u_block_stride(sh.T, sh.J), L_du = (long long)sh.nd * sh.B * ub;
        fv::RedSegs segs{};
        segs.seg[0] = fv::RedSeg{part_du, du, L_du, L_du, 0, ub, (long long)sh.T * sh.J, tiles, 1};
        FV_MARK_CALL(marks, st, reduce(segs, 1, "bwd_reduce_kernel (du)"));
    }
    // 3. x_proj: dW_x = du^T xbar (split-K partials), dxbar = the scans' share + sum_k du[k] W_x[k]
    const int wx_tiles = ((sh.E + fv::kGwE - 1) / fv::kGwE) * sh.nd;
    const int wx_chunk = bwd_kchunk(M, std::min(bwd_splits(M, wx_tiles, sms), kMaxWxSplits));
    const int wx_splits = (M + wx_chunk - 1) / wx_chunk;
    FV_MARK_CALL(marks, st, launch_bwd_dwx(sh, du, xbar, (float*)(ws + L.part_wx), wx_splits, wx_chunk, st));
    FV_MARK_CALL(marks, st, ([&]() -> fv_status {
        const dim3 grid((M + fv::kGxM - 1) / fv::kGxM, (sh.E + fv::kGxE - 1) / fv::kGxE);
        fv::bwd_dxbar_kernel<<<grid, fv::kThreads, 0, st>>>(sh, du, a->W_x, dxs, dxbar);
        FV_LAUNCH_CHECK("bwd_dxbar_kernel");
        return FV_OK;
    })());
    // 4. pooling
    if (sh.K == 0) {
        const int threads = fv::bwd_groups(sh.SL) * fv::bwd_slot_width(sh.SL);
        FV_MARK_CALL(marks, st, ([&]() -> fv_status {
            fv::bwd_pool_dense_kernel<<<M, threads, 0, st>>>(sh, dxbar, g->dx);
            FV_LAUNCH_CHECK("bwd_pool_dense_kernel");
            return FV_OK;
        })());
    } else {
        const int32_t* row_of = (const int32_t*)(fw + FL.row_of);
        const long long ntok = (long long)sh.B * sh.K;
        if (ntok >= (1ll << 31)) return FV_ERR_UNSUPPORTED;
        FV_MARK_CALL(marks, st, ([&]() -> fv_status {
            fv::bwd_pool_masked_kernel<<<(unsigned)ntok, 128, 0, st>>>(sh, row_of, dxbar, g->dx, g->dz);
            FV_LAUNCH_CHECK("bwd_pool_masked_kernel");
            return FV_OK;
        })());
    }
    // 5. the batch sums of the parameter gradients, each added in a fixed order (images, K splits,
    // gate blocks), so that every run gives the same bits
    {
        const long long E = sh.E, nd = sh.nd, ne = nd * E;
        fv::RedSegs segs{};
        int n = 0;
        segs.seg[n++] = fv::RedSeg{part_dA, g->dA_log, ne * sh.N, ne * sh.N, 0, 0, 0, sh.B, 1};
        segs.seg[n++] = fv::RedSeg{part_wdt, g->dW_dt, ne * sh.R, ne * sh.R, 0, 0, 0, sh.B, 1};
        segs.seg[n++] = fv::RedSeg{part_bdt, g->db_dt, ne, ne, 0, 0, 0, sh.B, 1};
        segs.seg[n++] = fv::RedSeg{(const float*)(ws + L.part_wx), g->dW_x, (long long)nWx, (long long)nWx, 0, 0, 0,
                                   wx_splits, 1};
        if (sh.ln) {  // part_gate rows: dgamma | dbeta | dD per gate block
            segs.seg[n++] = fv::RedSeg{part_gate, g->dln_gamma, E, 3 * E, 0, 0, 0, gate_blocks, 1};
            segs.seg[n++] = fv::RedSeg{part_gate + E, g->dln_beta, E, 3 * E, 0, 0, 0, gate_blocks, 1};
            segs.seg[n++] = fv::RedSeg{part_gate + 2 * E, g->dD, E, 3 * E, E, 0, 0, gate_blocks, (int)nd};
        } else {  // dD is the same sum for every direction
            segs.seg[n++] = fv::RedSeg{part_gate, g->dD, E, E, E, 0, 0, gate_blocks, (int)nd};
        }
        FV_MARK_CALL(marks, st, reduce(segs, n, "bwd_reduce_kernel (params)"));
    }
    return FV_OK;
}

}  // namespace

extern "C" {

size_t fastvim_ssm_backward_workspace_size(const fv_ssm_args* args) {
    fv::Shape sh;
    if (make_shape(args, &sh) != FV_OK) return 0;
    return plan_bwd(sh).total;
}

fv_status fastvim_ssm_backward_workspace_layout(const fv_ssm_args* args, fv_bwd_ws_layout* out) {
    if (!out) return FV_ERR_NULL;
    fv::Shape sh;
    fv_status s = make_shape(args, &sh);
    if (s != FV_OK) return s;
    const BwdLayout L = plan_bwd(sh);
    out->total_bytes = L.total;
    out->dys = L.dys; out->dxbar = L.dxbar; out->du = L.du; out->dxs = L.dxs; out->ckpt = L.ckpt;
    out->status = L.status; out->delta = L.delta; out->partials = L.partials;
    return FV_OK;
}

int fastvim_ssm_backward_launch_count(const fv_ssm_args* args) {
    fv::Shape sh;
    if (make_shape(args, &sh) != FV_OK) return 0;
    return bwd_launch_count_of(sh);
}

const char* fastvim_ssm_backward_launch_name(const fv_ssm_args* args, int i) {
    fv::Shape sh;
    if (make_shape(args, &sh) != FV_OK) return "";
    return bwd_launch_name_of(sh, i);
}

fv_status fastvim_ssm_backward(const fv_ssm_args* args, const fv_ssm_grads* grads, const void* fwd_ws,
                               size_t fwd_ws_bytes, void* ws, size_t ws_bytes, void* stream) {
    return backward_impl(args, grads, fwd_ws, fwd_ws_bytes, ws, ws_bytes, (cudaStream_t)stream);
}

fv_status fastvim_ssm_backward_events(const fv_ssm_args* args, const fv_ssm_grads* grads, const void* fwd_ws,
                                      size_t fwd_ws_bytes, void* ws, size_t ws_bytes, void* stream,
                                      void* const* events, int n_events) {
    if (!events) return FV_ERR_NULL;
    return backward_impl(args, grads, fwd_ws, fwd_ws_bytes, ws, ws_bytes, (cudaStream_t)stream, events, n_events);
}

}  // extern "C"
