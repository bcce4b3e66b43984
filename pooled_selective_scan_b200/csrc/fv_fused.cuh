// fv_fused.cuh -- the dense FastVim SSM layer as ONE persistent, image-pipelined launch (sm_100a),
// and the projection task body that the staged launches reuse.
//
// The layer's pooled tokens depend on ALL of an image's x, and every output token depends on the
// whole image's scan, so x must be read once for pooling and once more for the D x skip.  One
// persistent launch (two 256-thread CTAs per SM) streams the images through four task kinds,
//
//   P(b, g)  pool LP grid lines of image b into pooled tokens     (TMA bulk-copy ring over x)
//   Q(b, q)  x_proj of 16 pooled tokens of image b                (fp32 GEMM, cp.async pipeline)
//   S(b, c)  dt_proj + softplus, ZOH and the forward/backward scans of a channel tile of image b
//   E(b, g)  repeat + D x skip + SiLU(z) gate for LP grid lines  (TMA ring over x and z; y stored)
//
// taken from a global ticket counter in the order  [Q_{r-1}][P_r][E_{r-L}][S_{r-2}]  for r = 0, 1,
// ..., so that every CTA keeps streaming while other CTAs project and scan: the x_proj GEMMs, the
// scans and all the waits between them overlap the HBM traffic of other images.  Each image's
// projections come one round after its pools and its scans one round after that, and its gates
// L >= 3 rounds after its pools, so that consumers rarely wait.  (Keeping x in the 126 MB L2
// between pool and gate does not work at these traffic volumes: first-touch lines are evicted
// whatever their eviction priority, so x is simply streamed twice.)
//
// Dependencies are per-image counters (pool, proj, scan) released by producer CTAs and acquired by
// consumer CTAs.  A CTA only ever waits for tasks with smaller tickets, which were handed to CTAs
// that are already running, so the schedule cannot deadlock whatever the number of resident CTAs.
// Every wait is bounded (1 s): on expiry the CTA records FV_ERR_TIMEOUT in the status word, raises
// the abort flag (which makes every other CTA stop taking work), lets its own copies in flight
// land, and exits.
//
// The scan of one (direction, channel) is split into 8 time chunks held by 8 lanes.  Pass 1 runs
// each chunk from a zero state, giving the chunk's affine map h -> P h + H (P = product of the
// Abar, taken as one exp2 of the summed step sizes); a 3-step shuffle scan over the 8 lanes
// composes the maps in scan order; pass 2 reruns each chunk from its true incoming state and
// emits C_t . h_t.  All 16 states of a lane stay in registers; the sequential depth is ~2 T/8 + 3
// instead of T.
#pragma once

#include "fv_common.cuh"

namespace fv {

constexpr int kFusedThreads = 256;       // two persistent CTAs per SM
constexpr int kScanChunks = 8;           // time chunks (lanes) per (direction, channel)
constexpr int kScanStates = 16;          // states per lane (N <= 16, unused ones are zero)
constexpr int kBCStride = 2 * kScanStates + 4;  // floats per token row of B|C in shared memory
constexpr int kMaxLP = 4;                // grid lines per P/E task at most
constexpr int kRingStages = 4;           // TMA bulk-copy ring of the streaming tasks
constexpr int kStageBytes = 24 * 1024;   // per stage: P tasks x only; E tasks x and z halves
constexpr int kMaxSlots = 2;             // float4 slots per thread in P tasks: E <= 2048
constexpr int kQT = 16;                  // pooled tokens per projection task
constexpr int kQK = 32;                  // channels per projection K-step
constexpr int kQPad = kQK + 4;           // padded row of a projection tile (16-byte aligned)
// cp.async pipeline depth of the projection K-loop for TN = 3, 4, 6 outputs per thread
__host__ __device__ constexpr int q_stages(int TN) { return TN <= 3 ? 5 : (TN == 4 ? 4 : 3); }
__host__ __device__ constexpr int q_tn(int NJ) { return NJ <= 96 ? 3 : (NJ <= 128 ? 4 : 6); }
constexpr unsigned long long kWaitLimitNs = 1000000000ull;

// Control block at the start of the fused workspace region (zeroed before every call):
//   [0] ticket counter  [1] abort flag  [64 ..] pool_cnt[B], proj_cnt[B], scan_cnt[B]
constexpr int kCtrlHeaderWords = 64;
constexpr int kCtrlCounters = 3;  // counters per image

enum FusedTask { kTaskNone = -1, kTaskPool = 0, kTaskScan = 1, kTaskGate = 2, kTaskProj = 3 };

struct FusedPlan {
    int LP;      // grid lines per P and E task
    int nP;      // P tasks (and E tasks) per image
    int nQ;      // Q tasks per image
    int nS;      // S tasks per image
    int ECH;     // channels per S task
    int CL;      // time steps per scan chunk: ceil(T / 8)
    int L;       // E of image r - L is issued in round r
    int B;
    int ctP;     // tokens per ring chunk in P tasks
    int ctE;     // tokens per ring chunk in E tasks
    unsigned total;       // number of tickets
    unsigned c1, c2;      // first tickets of rounds R1 and R2
    int R1, R2;           // rounds [R1, R2) all have the same composition
    size_t smem_bytes;    // dynamic shared memory per CTA
    unsigned long long wait_limit_ns;
};

struct FusedPtrs {
    const float* x;
    const float* z;
    const float* A_log;
    const float* D;
    const float* W_x;
    const float* W_dt;
    const float* b_dt;
    float* y;
    float* xbar;   // [B][T][E]
    float* u;      // [nd][B] blocks of [T][J] (see u_offset)
    float* ys;     // [B][T][E]
    float* bcs;    // [nd][B][8 CL][kBCStride]: B | C rows in the scan's chunk-interleaved order
    float* dts;    // [nd][B][Tr]: dt_low rows [T][R], block padded to Tr = ceil(T R / 32) * 32
    unsigned* status;
    unsigned* ctrl;
    unsigned long long* trace;  // NULL, or 4 words per ticket
};

// Per-CTA state of the TMA ring, kept across tasks.
struct Ring {
    unsigned long long* full;  // [kRingStages] mbarriers
    char* buf;                 // [kRingStages][kStageBytes]
    unsigned count;            // chunks issued (and consumed) by this CTA so far
};

__host__ __device__ __forceinline__ int fused_ech(int nd) { return kFusedThreads / (kScanChunks * nd); }
// Per-(direction, image) block strides of the scan-ready copies, in floats.
__host__ __device__ __forceinline__ size_t fused_bcs_stride(int T) {
    return (size_t)kScanChunks * ((T + kScanChunks - 1) / kScanChunks) * kBCStride;
}
__host__ __device__ __forceinline__ size_t fused_dts_stride(int T, int R) { return (((size_t)T * R + 31) / 32) * 32; }
__host__ __device__ __forceinline__ int fused_xstride(int nd) { return fused_ech(nd) + 4; }

// Dynamic shared memory (floats) per task kind; the fused launch takes the maximum.
__host__ __device__ __forceinline__ size_t fused_proj_smem_floats(const Shape& sh) {
    const int tn = q_tn(sh.NJ);
    return (size_t)q_stages(tn) * ((size_t)kQT * kQPad + (size_t)32 * tn * kQPad);
}
__host__ __device__ __forceinline__ size_t fused_scan_smem_floats(const Shape& sh) {
    const int CL = (sh.T + kScanChunks - 1) / kScanChunks;
    const size_t rows = (size_t)kScanChunks * CL;
    const int XS = fused_xstride(sh.nd);
    return (size_t)sh.nd * rows * kBCStride + (size_t)(sh.nd + 1) * rows * XS +
           (size_t)sh.nd * fused_dts_stride(sh.T, sh.R) + (size_t)sh.nd * fused_ech(sh.nd) * (sh.R + 1) +
           (size_t)sh.T;
}
__host__ __device__ __forceinline__ size_t fused_smem_floats(const Shape& sh, int LP) {
    const size_t ring = (size_t)kRingStages * kStageBytes / 4;
    const size_t pool = ring + (size_t)kFusedThreads * 4;
    const size_t gate = ring + (size_t)(LP + 1) * sh.E;
    const size_t proj = fused_proj_smem_floats(sh);
    const size_t scan = fused_scan_smem_floats(sh);
    size_t m = pool > gate ? pool : gate;
    m = m > proj ? m : proj;
    return m > scan ? m : scan;
}

// Ticket -> (task kind, image, index within the image).  Round r holds, in this order,
//   Q of image r-1 (if 0 <= r-1 < B), P of image r (if r < B), E of image r-L (if 0 <= r-L < B),
//   S of image r-2 (if 0 <= r-2 < B),
// for r = 0 .. B+L-1.  Rounds [R1, R2) all have the same composition; the few rounds outside are
// walked one by one.
__host__ __device__ __forceinline__ void fused_round_parts(const FusedPlan& pl, int r, bool& q, bool& pp, bool& ee,
                                                           bool& ss) {
    q = (r >= 1 && r - 1 < pl.B);
    pp = r < pl.B;
    ee = (r >= pl.L && r - pl.L < pl.B);
    ss = (r >= 2 && r - 2 < pl.B);
}
__host__ __device__ __forceinline__ unsigned fused_round_size(const FusedPlan& pl, int r) {
    bool q, pp, ee, ss;
    fused_round_parts(pl, r, q, pp, ee, ss);
    return (q ? pl.nQ : 0) + (pp ? pl.nP : 0) + (ee ? pl.nP : 0) + (ss ? pl.nS : 0);
}
__device__ __forceinline__ void fused_decode(const FusedPlan& pl, unsigned tk, int& kind, int& b, int& idx) {
    unsigned base = 0;
    int r = 0;
    if (tk >= pl.c1) {
        const unsigned mid = fused_round_size(pl, pl.R1);
        if (tk < pl.c2 && mid) {
            const unsigned q = (tk - pl.c1) / mid;
            r = pl.R1 + (int)q;
            base = pl.c1 + q * mid;
        } else {
            r = pl.R2;
            base = pl.c2;
        }
    }
    for (;;) {
        const unsigned sz = fused_round_size(pl, r);
        if (tk < base + sz) break;
        base += sz;
        ++r;
    }
    unsigned off = tk - base;
    bool q, pp, ee, ss;
    fused_round_parts(pl, r, q, pp, ee, ss);
    if (q) {
        if (off < (unsigned)pl.nQ) { kind = kTaskProj; b = r - 1; idx = (int)off; return; }
        off -= pl.nQ;
    }
    if (pp) {
        if (off < (unsigned)pl.nP) { kind = kTaskPool; b = r; idx = (int)off; return; }
        off -= pl.nP;
    }
    if (ee) {
        if (off < (unsigned)pl.nP) { kind = kTaskGate; b = r - pl.L; idx = (int)off; return; }
        off -= pl.nP;
    }
    kind = kTaskScan;
    b = r - 2;
    idx = (int)off;
}

// Thread 0 waits (bounded) until *cnt >= target; the verdict is broadcast to the CTA.
__device__ __forceinline__ bool cta_wait(const unsigned* cnt, unsigned target, unsigned* status,
                                         unsigned* abort_flag, unsigned long long limit_ns, int* s_flag) {
    if (threadIdx.x == 0) {
        int ok = 1;
        if (ld_acquire_gpu(cnt) < target) {
            const unsigned long long t0 = globaltimer_ns();
            while (ld_acquire_gpu(cnt) < target) {
                if (ld_acquire_gpu(abort_flag)) { ok = 0; break; }
                if (globaltimer_ns() - t0 > limit_ns) {
                    set_status(status, kStatusTimeout);
                    atomicExch(abort_flag, 1u);
                    ok = 0;
                    break;
                }
                __nanosleep(128);
            }
        }
        *s_flag = ok;
    }
    __syncthreads();
    return *s_flag != 0;
}

// All of this CTA's global writes so far become visible before the counter moves (no counter:
// the task runs in a staged launch, where the launch boundary orders it).
__device__ __forceinline__ void cta_signal(unsigned* cnt) {
    __syncthreads();
    if (threadIdx.x == 0 && cnt) {
        __threadfence();
        red_release_gpu_add(cnt, 1u);
    }
}

// Thread 0 waits (bounded) for a ring stage to fill; the verdict is broadcast to the CTA.  On a
// timeout the status word and the abort flag are set.
__device__ __forceinline__ bool ring_wait(unsigned long long* bar, unsigned parity, const FusedPtrs& p,
                                          unsigned long long limit_ns, int* s_flag) {
    if (threadIdx.x == 0) {
        int ok = 1;
        if (!mbar_try_wait(bar, parity)) {
            const unsigned long long t0 = globaltimer_ns();
            while (!mbar_try_wait(bar, parity)) {
                if (globaltimer_ns() - t0 > limit_ns) {
                    set_status(p.status, kStatusTimeout);
                    atomicExch(p.ctrl + 1, 1u);
                    ok = 0;
                    break;
                }
            }
        }
        *s_flag = ok;
    }
    __syncthreads();
    return *s_flag != 0;
}

// Before a CTA gives up in the middle of a streaming task: let the copies it still has in flight
// land (bounded), so that none writes into shared memory after the CTA is gone.
__device__ __forceinline__ void ring_drain(Ring& rg, unsigned first, unsigned last, unsigned long long limit_ns) {
    if (threadIdx.x == 0) {
        for (unsigned g = first; g < last; ++g) {
            unsigned long long* bar = rg.full + (g % kRingStages);
            const unsigned parity = (g / kRingStages) & 1u;
            const unsigned long long t0 = globaltimer_ns();
            while (!mbar_try_wait(bar, parity))
                if (globaltimer_ns() - t0 > limit_ns) break;
        }
    }
    __syncthreads();
}

__device__ __forceinline__ float4 f4_mul(const float4& v, float s) {
    return make_float4(v.x * s, v.y * s, v.z * s, v.w * s);
}

// Issue ring chunk q of a streaming task: tokens [i*ct, i*ct + n) of grid line l, from x (and z
// for gate tasks) into stage `st`.  POOL_W lines are contiguous (one copy per tensor); POOL_H
// lines take one copy per token.
__device__ __forceinline__ void ring_issue(const Shape& sh, const FusedPtrs& p, int b, int t0, int q, int nch, int ct,
                                           bool with_z, unsigned long long* bar, char* stage, uint64_t pol) {
    const int l = q / nch, i = q - l * nch;
    const int tok0 = i * ct;
    const int n = min(ct, sh.S - tok0);
    const unsigned tok_bytes = (unsigned)sh.E * 4u;
    const size_t base = dense_base(sh, b, t0 + l);
    const size_t stride = dense_stride(sh);
    mbar_arrive_expect_tx(bar, (with_z ? 2u : 1u) * (unsigned)n * tok_bytes);
    char* zdst = stage + kStageBytes / 2;
    if (sh.pool_axis == 0) {
        const size_t off = base + (size_t)tok0 * stride;
        bulk_g2s(stage, p.x + off, (unsigned)n * tok_bytes, bar, pol);
        if (with_z) bulk_g2s(zdst, p.z + off, (unsigned)n * tok_bytes, bar, pol);
    } else {
        for (int j = 0; j < n; ++j) {
            const size_t off = base + (size_t)(tok0 + j) * stride;
            bulk_g2s(stage + (size_t)j * tok_bytes, p.x + off, tok_bytes, bar, pol);
            if (with_z) bulk_g2s(zdst + (size_t)j * tok_bytes, p.z + off, tok_bytes, bar, pol);
        }
    }
}

// Thread -> (float4 slot(s), token group) of a token row of E channels (pooling).
struct SlotMap {
    int G;        // token groups
    int g;        // this thread's group (g < G for active threads)
    int slot[kMaxSlots];
    int nslot;    // valid slots of this thread
};
__device__ __forceinline__ SlotMap slot_map(int SL) {
    SlotMap m;
    if (SL <= kFusedThreads) {
        m.G = kFusedThreads / SL;
        m.g = threadIdx.x / SL;
        m.slot[0] = threadIdx.x % SL;
        m.slot[1] = 0;
        m.nslot = m.g < m.G ? 1 : 0;
    } else {
        m.G = 1;
        m.g = 0;
        m.slot[0] = threadIdx.x;
        m.slot[1] = threadIdx.x + kFusedThreads;
        m.nslot = threadIdx.x + kFusedThreads < SL ? 2 : 1;
    }
    return m;
}

// ---- P: pool grid lines [t0, t0+LP) of image b ------------------------------------------------
__device__ __forceinline__ bool fused_pool(const Shape& sh, const FusedPlan& pl, const FusedPtrs& p, int b, int g,
                                           float* smem, Ring& rg, uint64_t pol_keep, int* s_flag) {
    const int E = sh.E, SL = sh.SL;
    float4* part = reinterpret_cast<float4*>(smem + kRingStages * kStageBytes / 4);  // [256] float4
    const int t0 = g * pl.LP;
    const int nl = min(sh.T, t0 + pl.LP) - t0;
    const float scale = sh.pool_scale / (float)sh.S;
    const size_t m0 = (size_t)b * sh.T + t0;
    const int ct = pl.ctP;
    const int nch = (sh.S + ct - 1) / ct;
    const int nq = nl * nch;
    const SlotMap sm = slot_map(SL);
    const unsigned g0 = rg.count;
    if (threadIdx.x == 0) {
        fence_proxy_async_smem();
        for (int q = 0; q < min(kRingStages, nq); ++q) {
            const unsigned gg = g0 + q;
            ring_issue(sh, p, b, t0, q, nch, ct, false, rg.full + gg % kRingStages,
                       rg.buf + (size_t)(gg % kRingStages) * kStageBytes, pol_keep);
        }
    }
    float4 acc[kMaxSlots];
    for (int q = 0; q < nq; ++q) {
        const unsigned gg = g0 + q;
        const int st = gg % kRingStages;
        if (!ring_wait(rg.full + st, (gg / kRingStages) & 1u, p, pl.wait_limit_ns, s_flag)) {
            ring_drain(rg, gg + 1, g0 + min(nq, q + kRingStages), pl.wait_limit_ns);
            return false;
        }
        const int i = q % nch;
        if (i == 0) {
#pragma unroll
            for (int k = 0; k < kMaxSlots; ++k) acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        const int n = min(ct, sh.S - i * ct);
        const float4* chunk = reinterpret_cast<const float4*>(rg.buf + (size_t)st * kStageBytes);
#pragma unroll
        for (int k = 0; k < kMaxSlots; ++k)
            if (k < sm.nslot)
                for (int j = sm.g; j < n; j += sm.G) f4_add(acc[k], chunk[(size_t)j * SL + sm.slot[k]]);
        if (i == nch - 1) {
            float4* out = reinterpret_cast<float4*>(p.xbar + (m0 + q / nch) * E);
            if (SL <= kFusedThreads) {
                part[threadIdx.x] = acc[0];
                __syncthreads();
                if (threadIdx.x < SL) {
                    float4 sum = part[threadIdx.x];
                    for (int qq = 1; qq < sm.G; ++qq) f4_add(sum, part[qq * SL + threadIdx.x]);
                    out[threadIdx.x] = f4_mul(sum, scale);
                }
            } else {
#pragma unroll
                for (int k = 0; k < kMaxSlots; ++k)
                    if (k < sm.nslot) out[sm.slot[k]] = f4_mul(acc[k], scale);
            }
        }
        __syncthreads();  // everyone is done with stage st
        if (threadIdx.x == 0 && q + kRingStages < nq)
            ring_issue(sh, p, b, t0, q + kRingStages, nch, ct, false, rg.full + st, rg.buf + (size_t)st * kStageBytes,
                       pol_keep);
    }
    rg.count = g0 + nq;
    cta_signal(p.ctrl ? p.ctrl + kCtrlHeaderWords + b : nullptr);
    return true;
}

// ---- Q: x_proj of pooled tokens [q*16, q*16+16) of image b ------------------------------------
// u = W_x . xbar as a register-blocked fp32 GEMM (2 tokens x TN outputs per thread: TN = 3, 4 or
// 6 for nd(R+2N) <= 96, 128 or 192 outputs; weight rows past nd(R+2N) are zero-filled), 32-channel
// K-steps in a 5-, 4- or 3-stage cp.async pipeline.  Besides u, the task writes the scan-ready copies: B | C
// of each token into its chunk-interleaved row, dt_low into a dense [T][R] block.
template <int TN, int kQStages>
__device__ __forceinline__ void fused_proj_t(const Shape& sh, const FusedPlan& pl, const FusedPtrs& p, int b, int q,
                                             float* smem) {
    const int T = sh.T, E = sh.E, J = sh.J, NJ = sh.NJ, R = sh.R, N = sh.N;
    constexpr int WROWS = 32 * TN;
    constexpr int TM = kQT / 8;
    const int tq0 = q * kQT;
    const int mt = min(kQT, T - tq0);
    const size_t m0 = (size_t)b * T + tq0;
    float* xs = smem;                                // [kQStages][kQT][kQPad]
    float* ws = xs + kQStages * kQT * kQPad;         // [kQStages][WROWS][kQPad]
    const int tg = threadIdx.x & 7, cg = threadIdx.x >> 3;   // tokens tg + 8 i, outputs cg + 32 j
    const int nk = (E + kQK - 1) / kQK;
    auto load = [&](int kk) {
        const int e0 = kk * kQK;
        const int st = kk % kQStages;
        float* xb = xs + st * kQT * kQPad;
        float* wb = ws + st * WROWS * kQPad;
        for (int v = threadIdx.x; v < kQT * (kQK / 4); v += kFusedThreads) {
            const int r = v >> 3, c4 = (v & 7) * 4;
            const bool ok = r < mt && e0 + c4 < E;
            cp_async16(xb + r * kQPad + c4, ok ? (const void*)(p.xbar + (m0 + r) * E + e0 + c4) : (const void*)p.xbar,
                       ok ? 16u : 0u);
        }
        for (int v = threadIdx.x; v < WROWS * (kQK / 4); v += kFusedThreads) {
            const int r = v >> 3, c4 = (v & 7) * 4;
            const bool ok = r < NJ && e0 + c4 < E;
            cp_async16(wb + r * kQPad + c4, ok ? (const void*)(p.W_x + (size_t)r * E + e0 + c4) : (const void*)p.W_x,
                       ok ? 16u : 0u);
        }
    };
    float acc[TM][TN];
#pragma unroll
    for (int i = 0; i < TM; ++i)
#pragma unroll
        for (int j = 0; j < TN; ++j) acc[i][j] = 0.f;
#pragma unroll
    for (int kk = 0; kk < kQStages - 1; ++kk) {
        if (kk < nk) load(kk);
        cp_async_commit();
    }
    for (int kk = 0; kk < nk; ++kk) {
        cp_async_wait<kQStages - 2>();
        __syncthreads();  // K-step kk has landed for every thread; step kk-1's buffer is free
        if (kk + kQStages - 1 < nk) load(kk + kQStages - 1);
        cp_async_commit();
        const int st = kk % kQStages;
        const float* xb = xs + st * kQT * kQPad;
        const float* wb = ws + st * WROWS * kQPad;
#pragma unroll 2
        for (int c = 0; c < kQK; c += 4) {
            float4 xv[TM], wv[TN];
#pragma unroll
            for (int i = 0; i < TM; ++i) xv[i] = *reinterpret_cast<const float4*>(xb + (tg + 8 * i) * kQPad + c);
#pragma unroll
            for (int j = 0; j < TN; ++j) wv[j] = *reinterpret_cast<const float4*>(wb + (cg + 32 * j) * kQPad + c);
#pragma unroll
            for (int i = 0; i < TM; ++i)
#pragma unroll
                for (int j = 0; j < TN; ++j)
                    acc[i][j] = fmaf(wv[j].w, xv[i].w,
                                     fmaf(wv[j].z, xv[i].z, fmaf(wv[j].y, xv[i].y, fmaf(wv[j].x, xv[i].x, acc[i][j]))));
        }
    }
    cp_async_wait<0>();
    const int CL = pl.CL;
    const size_t bstride = fused_bcs_stride(T), dstride = fused_dts_stride(T, R);
#pragma unroll
    for (int j = 0; j < TN; ++j) {
        const int jj = cg + 32 * j;
        if (jj < NJ) {
            const int k = jj / J, jc = jj - k * J;
            float* bcb = p.bcs + ((size_t)k * sh.B + b) * bstride;
            float* dtb = p.dts + ((size_t)k * sh.B + b) * dstride;
#pragma unroll
            for (int i = 0; i < TM; ++i) {
                const int r = tg + 8 * i;
                if (r < mt) {
                    const int t = tq0 + r;
                    const float v = acc[i][j];
                    p.u[u_offset(sh, k, b, t) + jc] = v;
                    if (!p.bcs) continue;  // staged launches scan from u alone
                    if (jc < R) {
                        dtb[(size_t)t * R + jc] = v;
                    } else {
                        const int nb = jc - R;
                        float* row = bcb + (size_t)((t % CL) * kScanChunks + t / CL) * kBCStride;
                        row[nb < N ? nb : kScanStates + (nb - N)] = v;
                        if (nb == 0)  // unused state slots of this token read as zero
                            for (int n = N; n < kScanStates; ++n) {
                                row[n] = 0.f;
                                row[kScanStates + n] = 0.f;
                            }
                    }
                }
            }
        }
    }
    cta_signal(p.ctrl ? p.ctrl + kCtrlHeaderWords + sh.B + b : nullptr);
}

__device__ __forceinline__ void fused_proj(const Shape& sh, const FusedPlan& pl, const FusedPtrs& p, int b, int q,
                                           float* smem) {
    switch (q_tn(sh.NJ)) {
        case 3: fused_proj_t<3, q_stages(3)>(sh, pl, p, b, q, smem); break;
        case 4: fused_proj_t<4, q_stages(4)>(sh, pl, p, b, q, smem); break;
        default: fused_proj_t<6, q_stages(6)>(sh, pl, p, b, q, smem); break;
    }
}

// ---- S: dt_proj + softplus, ZOH and scans of channels [e0, e0 + ECH) of image b -----------------
// Shared rows are stored in chunk-interleaved time order p(t) = (t % CL) * 8 + t / CL, so that at
// any step the 8 chunk lanes read 8 consecutive rows (bank-conflict free with the paddings).
template <int ND, bool ZOH_EXACT>
__device__ __forceinline__ void fused_scan(const Shape& sh, const FusedPlan& pl, const FusedPtrs& p, int b, int tile,
                                           float* smem) {
    constexpr int ECH = kFusedThreads / (kScanChunks * ND);
    constexpr int XS = ECH + 4;
    constexpr int NS = kScanStates;
    const int T = sh.T, E = sh.E, N = sh.N, R = sh.R;
    const int CL = pl.CL;
    const int rows = kScanChunks * CL;
    const int e0 = tile * ECH;
    float* bc = smem;                          // [ND][rows][kBCStride]: B_0..B_15 | C_0..C_15
    float* dx = bc + ND * rows * kBCStride;    // [ND][rows][XS]: Delta, then y of that direction
    float* xsm = dx + ND * rows * XS;          // [rows][XS]: pooled tokens
    const int DTS = (int)fused_dts_stride(T, R);
    float* dtl = xsm + rows * XS;              // [ND][DTS]: dt_low rows [T][R]
    float* wdt = dtl + ND * DTS;               // [ND][ECH][R+1]: dt_proj rows (+ bias)
    int* post = reinterpret_cast<int*>(wdt + ND * ECH * (R + 1));  // [T]: p(t)
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    constexpr int kWarps = kFusedThreads / 32;
    // Stage the tile's inputs with 16-byte asynchronous copies (all in flight together): the
    // scan-ready B | C rows and dt_low rows written by the projection tasks, the pooled tokens of
    // the tile's channels; and the tile's dt_proj rows and biases.
    {
        const int nbc = rows * kBCStride / 4, ndt = DTS / 4;
        for (int k = 0; k < ND; ++k) {
            const float* sb = p.bcs + ((size_t)k * sh.B + b) * fused_bcs_stride(T);
            const float* sd = p.dts + ((size_t)k * sh.B + b) * DTS;
            for (int v = threadIdx.x; v < nbc; v += kFusedThreads) cp_async16(bc + k * rows * kBCStride + 4 * v, sb + 4 * v, 16u);
            for (int v = threadIdx.x; v < ndt; v += kFusedThreads) cp_async16(dtl + k * DTS + 4 * v, sd + 4 * v, 16u);
        }
        for (int t = threadIdx.x; t < T; t += kFusedThreads) post[t] = (t % CL) * kScanChunks + t / CL;
        __syncthreads();
        for (int v = threadIdx.x; v < T * (ECH / 4); v += kFusedThreads) {
            const int t = v / (ECH / 4), c4 = (v % (ECH / 4)) * 4;
            const bool ok = e0 + c4 < E;
            cp_async16(xsm + post[t] * XS + c4, ok ? (const void*)(p.xbar + ((size_t)b * T + t) * E + e0 + c4)
                                                   : (const void*)p.xbar, ok ? 16u : 0u);
        }
        cp_async_commit();
        for (int i = threadIdx.x; i < ND * ECH * (R + 1); i += kFusedThreads) {
            const int k = i / (ECH * (R + 1));
            const int rem = i - k * ECH * (R + 1);
            const int c = rem / (R + 1), r = rem - c * (R + 1);
            const int e = e0 + c;
            float v = 0.f;
            if (e < E) v = r < R ? __ldg(p.W_dt + ((size_t)k * E + e) * R + r) : __ldg(p.b_dt + (size_t)k * E + e);
            wdt[i] = v;
        }
        cp_async_wait<0>();
        __syncthreads();
    }
    // Delta = softplus(W_dt . dt_low + b_dt) for this tile: lane -> channel, warps -> tokens
    {
        constexpr int kTPerWarpPass = 32 / ECH > 0 ? 32 / ECH : 1;
        const int c = lane % ECH;
        const int tsub = lane / ECH;
        const bool live = e0 + c < E;
        for (int k = 0; k < ND; ++k) {
            const float* wr = wdt + (k * ECH + c) * (R + 1);
            for (int t = warp * kTPerWarpPass + tsub; t < T; t += kWarps * kTPerWarpPass) {
                const float* dl = dtl + k * DTS + t * R;
                float a = wr[R];
#pragma unroll 4
                for (int r = 0; r < R; ++r) a = fmaf(wr[r], dl[r], a);
                dx[(k * rows + post[t]) * XS + c] = live ? softplus_fast(a) : 0.f;
            }
        }
    }
    __syncthreads();

    const int chunk = lane & 7;
    constexpr int kWarpsPerDir = ECH / 4;
    const int kd = warp / kWarpsPerDir;
    const int ch = (warp - kd * kWarpsPerDir) * 4 + (lane >> 3);
    const int e = e0 + ch;
    const bool active = e < E;
    const bool fwd = (ND == 2) ? (kd == 0) : ((sh.dir_flags & 1u) != 0);
    constexpr float kLog2e = 1.4426950408889634f;
    float A2[NS], h[NS];
    float An[NS], Ainv[NS];  // used by the exact-ZOH input term only
#pragma unroll
    for (int n = 0; n < NS; ++n) {
        const float A = (active && n < N) ? -expf(__ldg(p.A_log + ((size_t)kd * E + e) * N + n)) : 0.f;
        A2[n] = A * kLog2e;
        An[n] = A;
        Ainv[n] = A != 0.f ? 1.f / A : 0.f;
        h[n] = 0.f;
    }
    const int c_lo = chunk * CL;
    const int c_hi = min(T, c_lo + CL);
    const int len = c_hi > c_lo ? c_hi - c_lo : 0;
    const float* bck = bc + kd * rows * kBCStride;
    float* dxk = dx + kd * rows * XS;

    // pass 1: this chunk from a zero state
    float sdt = 0.f;
    for (int s = 0; s < len; ++s) {
        const int t = fwd ? c_lo + s : c_hi - 1 - s;
        const int pos = (t - c_lo) * kScanChunks + chunk;
        const float dt = dxk[pos * XS + ch];
        const float xv = xsm[pos * XS + ch];
        const float dtx = dt * xv;
        sdt += dt;
        const float4* Bq = reinterpret_cast<const float4*>(bck + pos * kBCStride);
#pragma unroll
        for (int q = 0; q < NS / 4; ++q) {
            const float4 bv = Bq[q];
            const float bb[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int n = 4 * q + i;
                const float dA = ex2_approx(dt * A2[n]);
                const float bx = ZOH_EXACT ? expm1f(dt * An[n]) * Ainv[n] * bb[i] * xv : dtx * bb[i];
                h[n] = fmaf(dA, h[n], bx);
            }
        }
    }
    // compose the chunk maps h -> P h + H along the scan order (lanes 0..7 forward, 7..0 backward;
    // the direction is uniform within a warp)
    if (fwd) {
#pragma unroll
        for (int n = 0; n < NS; ++n) {
            float P = ex2_approx(A2[n] * sdt), H = h[n];
#pragma unroll
            for (int d = 1; d < kScanChunks; d <<= 1) {
                const float Pp = __shfl_up_sync(0xffffffffu, P, d, kScanChunks);
                const float Hp = __shfl_up_sync(0xffffffffu, H, d, kScanChunks);
                if (chunk >= d) {
                    H = fmaf(P, Hp, H);
                    P = P * Pp;
                }
            }
            const float Hin = __shfl_up_sync(0xffffffffu, H, 1, kScanChunks);
            h[n] = chunk == 0 ? 0.f : Hin;
        }
    } else {
#pragma unroll
        for (int n = 0; n < NS; ++n) {
            float P = ex2_approx(A2[n] * sdt), H = h[n];
#pragma unroll
            for (int d = 1; d < kScanChunks; d <<= 1) {
                const float Pp = __shfl_down_sync(0xffffffffu, P, d, kScanChunks);
                const float Hp = __shfl_down_sync(0xffffffffu, H, d, kScanChunks);
                if (chunk + d < kScanChunks) {
                    H = fmaf(P, Hp, H);
                    P = P * Pp;
                }
            }
            const float Hin = __shfl_down_sync(0xffffffffu, H, 1, kScanChunks);
            h[n] = chunk == kScanChunks - 1 ? 0.f : Hin;
        }
    }
    // pass 2: rerun the chunk from its incoming state and emit C_t . h_t
    for (int s = 0; s < len; ++s) {
        const int t = fwd ? c_lo + s : c_hi - 1 - s;
        const int pos = (t - c_lo) * kScanChunks + chunk;
        const float dt = dxk[pos * XS + ch];
        const float xv = xsm[pos * XS + ch];
        const float dtx = dt * xv;
        const float4* Bq = reinterpret_cast<const float4*>(bck + pos * kBCStride);
        const float4* Cq = Bq + NS / 4;
        float y = 0.f;
#pragma unroll
        for (int q = 0; q < NS / 4; ++q) {
            const float4 bv = Bq[q], cv = Cq[q];
            const float bb[4] = {bv.x, bv.y, bv.z, bv.w};
            const float cc[4] = {cv.x, cv.y, cv.z, cv.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int n = 4 * q + i;
                const float dA = ex2_approx(dt * A2[n]);
                const float bx = ZOH_EXACT ? expm1f(dt * An[n]) * Ainv[n] * bb[i] * xv : dtx * bb[i];
                h[n] = fmaf(dA, h[n], bx);
                y = fmaf(cc[i], h[n], y);
            }
        }
        dxk[pos * XS + ch] = y;  // the slot held this step's Delta, read above by this lane only
    }
    __syncthreads();
    for (int t = warp; t < T; t += kWarps) {
        const int pos = post[t];
        for (int c = lane; c < ECH; c += 32) {
            const int ee = e0 + c;
            float sum = dx[pos * XS + c];
            if (ND == 2) sum += dx[(rows + pos) * XS + c];
            if (ee < E) p.ys[((size_t)b * T + t) * E + ee] = sum;
        }
    }
    cta_signal(p.ctrl ? p.ctrl + kCtrlHeaderWords + 2 * sh.B + b : nullptr);
}

// ---- E: repeat + skip + gate for grid lines [t0, t0+LP) of image b -------------------------------
// x and z stream through the ring (x mostly hits L2); every thread takes consecutive float4s of a
// chunk (all 256 threads busy for any E), and y is stored straight from registers (evict-first).
__device__ __forceinline__ bool fused_gate(const Shape& sh, const FusedPlan& pl, const FusedPtrs& p, int b, int g,
                                           float* smem, Ring& rg, uint64_t pol_stream, int* s_flag) {
    const int SL = sh.SL, E = sh.E;
    const int t0 = g * pl.LP;
    const int nl = min(sh.T, t0 + pl.LP) - t0;
    const int ct = pl.ctE;
    const int nch = (sh.S + ct - 1) / ct;
    const int nq = nl * nch;
    const size_t stride4 = dense_stride(sh) >> 2;
    float* dsum = smem + kRingStages * kStageBytes / 4;   // [E]  sum_k D_k
    float* ysl = dsum + E;                                // [LP][E] scan output of the lines
    const unsigned g0 = rg.count;
    if (threadIdx.x == 0) {
        fence_proxy_async_smem();
        for (int q = 0; q < min(kRingStages, nq); ++q) {
            const unsigned gg = g0 + q;
            ring_issue(sh, p, b, t0, q, nch, ct, true, rg.full + gg % kRingStages,
                       rg.buf + (size_t)(gg % kRingStages) * kStageBytes, pol_stream);
        }
    }
    for (int e = threadIdx.x; e < E; e += kFusedThreads) {
        float d = __ldg(p.D + e);
        if (sh.nd == 2) d += __ldg(p.D + E + e);
        dsum[e] = d;
    }
    for (int i = threadIdx.x; i < nl * E; i += kFusedThreads) {
        const int l = i / E, e = i - l * E;
        ysl[i] = __ldcg(p.ys + ((size_t)b * sh.T + t0 + l) * E + e);
    }
    const float inv_sl = 1.f / (float)SL;
    for (int q = 0; q < nq; ++q) {
        const unsigned gg = g0 + q;
        const int st = gg % kRingStages;
        const int l = q / nch, i = q - l * nch;
        if (!ring_wait(rg.full + st, (gg / kRingStages) & 1u, p, pl.wait_limit_ns, s_flag)) {
            ring_drain(rg, gg + 1, g0 + min(nq, q + kRingStages), pl.wait_limit_ns);
            return false;
        }
        const int tok0 = i * ct;
        const int n = min(ct, sh.S - tok0);
        const float4* xc = reinterpret_cast<const float4*>(rg.buf + (size_t)st * kStageBytes);
        const float4* zc = reinterpret_cast<const float4*>(rg.buf + (size_t)st * kStageBytes + kStageBytes / 2);
        const float4* ys4 = reinterpret_cast<const float4*>(ysl + (size_t)l * E);
        const float4* d4 = reinterpret_cast<const float4*>(dsum);
        float4* y4 = reinterpret_cast<float4*>(p.y + dense_base(sh, b, t0 + l));
        for (int f = threadIdx.x; f < n * SL; f += kFusedThreads) {
            const int j = (int)(((float)f + 0.5f) * inv_sl);  // f / SL (exact for f < 2^16)
            const int slot = f - j * SL;
            const float4 xv = xc[f], zv = zc[f], yv = ys4[slot], dv = d4[slot];
            const float4 o = make_float4(silu_fast(zv.x) * fmaf(dv.x, xv.x, yv.x),
                                         silu_fast(zv.y) * fmaf(dv.y, xv.y, yv.y),
                                         silu_fast(zv.z) * fmaf(dv.z, xv.z, yv.z),
                                         silu_fast(zv.w) * fmaf(dv.w, xv.w, yv.w));
            st_hint(y4 + (size_t)(tok0 + j) * stride4 + slot, o, pol_stream);
        }
        __syncthreads();  // everyone is done with stage st
        if (threadIdx.x == 0 && q + kRingStages < nq)
            ring_issue(sh, p, b, t0, q + kRingStages, nch, ct, true, rg.full + st, rg.buf + (size_t)st * kStageBytes,
                       pol_stream);
    }
    rg.count = g0 + nq;
    return true;
}

// ---- the persistent kernel ----------------------------------------------------------------------
template <int ND, bool ZOH_EXACT>
__global__ void __launch_bounds__(kFusedThreads, 2)
fused_layer_kernel(Shape sh, FusedPlan pl, FusedPtrs p) {
    extern __shared__ __align__(128) float smem_f[];
    __shared__ __align__(8) unsigned long long s_full[kRingStages];
    __shared__ int s_task[3];
    __shared__ int s_flag;
    __shared__ unsigned s_ticket;
    __shared__ unsigned long long s_t0, s_t1;
    const uint64_t pol_keep = l2_policy_evict_first();  // x is re-read by the gate tasks from HBM
    const uint64_t pol_stream = l2_policy_evict_first();
    unsigned* abort_flag = p.ctrl + 1;
    unsigned* cnt_pool = p.ctrl + kCtrlHeaderWords;
    unsigned* cnt_proj = cnt_pool + sh.B;
    unsigned* cnt_scan = cnt_proj + sh.B;
    Ring rg;
    rg.full = s_full;
    rg.buf = reinterpret_cast<char*>(smem_f);
    rg.count = 0;
    if (threadIdx.x == 0) {
        for (int i = 0; i < kRingStages; ++i) mbar_init(&s_full[i], 1);
        fence_mbar_init();
    }
    for (;;) {
        __syncthreads();
        if (threadIdx.x == 0) {
            int kind = kTaskNone, b = 0, idx = 0;
            const unsigned tk = atomicAdd(p.ctrl, 1u);
            if (tk < pl.total && ld_acquire_gpu(abort_flag) == 0u) fused_decode(pl, tk, kind, b, idx);
            s_task[0] = kind;
            s_task[1] = b;
            s_task[2] = idx;
            s_ticket = tk;
            if (p.trace) s_t0 = globaltimer_ns();
        }
        __syncthreads();
        const int kind = s_task[0], b = s_task[1], idx = s_task[2];
        if (kind == kTaskNone) return;
        if (kind == kTaskPool) {
            if (p.trace && threadIdx.x == 0) s_t1 = globaltimer_ns();
            if (!fused_pool(sh, pl, p, b, idx, smem_f, rg, pol_keep, &s_flag)) return;
        } else if (kind == kTaskProj) {
            if (!cta_wait(cnt_pool + b, (unsigned)pl.nP, p.status, abort_flag, pl.wait_limit_ns, &s_flag)) return;
            if (p.trace && threadIdx.x == 0) s_t1 = globaltimer_ns();
            fused_proj(sh, pl, p, b, idx, smem_f);
        } else if (kind == kTaskScan) {
            if (!cta_wait(cnt_proj + b, (unsigned)pl.nQ, p.status, abort_flag, pl.wait_limit_ns, &s_flag)) return;
            if (p.trace && threadIdx.x == 0) s_t1 = globaltimer_ns();
            fused_scan<ND, ZOH_EXACT>(sh, pl, p, b, idx, smem_f);
        } else {
            if (!cta_wait(cnt_scan + b, (unsigned)pl.nS, p.status, abort_flag, pl.wait_limit_ns, &s_flag)) return;
            if (p.trace && threadIdx.x == 0) s_t1 = globaltimer_ns();
            if (!fused_gate(sh, pl, p, b, idx, smem_f, rg, pol_stream, &s_flag)) return;
        }
        if (p.trace) {
            __syncthreads();
            if (threadIdx.x == 0) {
                unsigned smid;
                asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
                unsigned long long* rec = p.trace + 4ull * s_ticket;
                rec[0] = ((unsigned long long)kind << 60) | ((unsigned long long)b << 32) | (unsigned)idx;
                rec[1] = ((unsigned long long)smid << 32) | blockIdx.x;
                rec[2] = s_t0;
                rec[3] = ((s_t1 - s_t0) << 40) | ((globaltimer_ns() - s_t0) & ((1ull << 40) - 1));
            }
        }
    }
}

// Staged launch of the projection task body: one CTA per task, ordered by the launch boundaries
// instead of counters.
__global__ void __launch_bounds__(kFusedThreads, 2) proj_tasks_kernel(Shape sh, FusedPlan pl, FusedPtrs p) {
    extern __shared__ __align__(128) float smem_f[];
    fused_proj(sh, pl, p, blockIdx.x / pl.nQ, blockIdx.x % pl.nQ, smem_f);
}

// A single CTA that waits, with the layer's bounded wait, on a counter that nothing increments:
// exercises the timeout path (status FV_ERR_TIMEOUT, clean exit) without the layer.
__global__ void bounded_wait_selftest_kernel(unsigned* status, unsigned* ctrl, unsigned long long limit_ns) {
    __shared__ int s_flag;
    const bool ok = cta_wait(ctrl + kCtrlHeaderWords, 1u, status, ctrl + 1, limit_ns, &s_flag);
    if (threadIdx.x == 0 && ok) set_status(status, 1u);  // unreachable unless the counter moved
}

}  // namespace fv
