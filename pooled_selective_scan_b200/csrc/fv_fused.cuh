// fv_fused.cuh -- the dense FastVim SSM layer as ONE persistent, image-pipelined launch (sm_100a).
//
// The layer's pooled tokens depend on ALL of an image's x, and every output token depends on the
// whole image's scan, so x must be read once for pooling and once more for the D x skip.  One
// persistent launch (two 256-thread CTAs per SM) streams the images through four task kinds,
//
//   P(b, g)  pool LP grid lines of image b into pooled tokens     (TMA bulk-copy ring over x)
//   Q(b, q)  x_proj of 16 pooled tokens of image b                (fp32 GEMM, cp.async pipeline)
//   S(b, c)  dt_proj + softplus, ZOH and the forward/backward scans of 128 channels of image b
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
// An S task runs one recurrence per thread over the whole pooled sequence (fv_scan.cuh): 256
// threads = 128 channels x 2 directions.  The image's P tasks zero its scan output, so both
// directions add into it.
#pragma once

#include "fv_common.cuh"
#include "fv_scan.cuh"

namespace fv {

constexpr int kFusedThreads = 256;       // two persistent CTAs per SM
constexpr int kMaxLP = 4;                // grid lines per P/E task at most
constexpr int kRingStages = 4;           // TMA bulk-copy ring of the streaming tasks
constexpr int kStageBytes = 24 * 1024;   // per stage: P tasks x only; E tasks x and z halves
constexpr int kMaxSlots = 2;             // float4 slots per thread in P tasks: E <= 2048
constexpr int kLnCache = 3;              // LayerNorm: float4 slots of s a lane keeps in registers
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
    int ECH;     // channels per S task (and direction)
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
    const float* ln_gamma;  // [E] (FV_FLAG_LAYERNORM) or NULL
    const float* ln_beta;
    float* xbar;   // [B][T][E]
    float* u;      // [B][nd] blocks of [T][J] (see u_offset)
    float* ys;     // [B][T][E]
    unsigned* status;
    unsigned* ctrl;
    unsigned long long* trace;  // NULL, or 4 words per ticket
    float* ckpt;                // NULL, or the kept scan states (FV_FLAG_KEEP_STATES)
};

// Per-CTA state of the TMA ring, kept across tasks.
struct Ring {
    unsigned long long* full;  // [kRingStages] mbarriers
    char* buf;                 // [kRingStages][kStageBytes]
    unsigned count;            // chunks issued (and consumed) by this CTA so far
};

// Channels per S task: 256 threads cover 128 channels x 2 directions, or 256 channels x 1.
__host__ __device__ __forceinline__ int fused_ech(int nd) { return kFusedThreads / nd; }

// Dynamic shared memory (floats) per task kind; the fused launch takes the maximum.
__host__ __device__ __forceinline__ size_t fused_proj_smem_floats(const Shape& sh) {
    const int tn = q_tn(sh.NJ);
    return (size_t)q_stages(tn) * ((size_t)kQT * kQPad + (size_t)32 * tn * kQPad);
}
__host__ __device__ __forceinline__ size_t fused_scan_smem_floats(const Shape& sh) {
    return seq_smem_floats(kFusedThreads, sh.nd, sh.R);
}
__host__ __device__ __forceinline__ size_t fused_smem_floats(const Shape& sh, int LP) {
    const size_t ring = (size_t)kRingStages * kStageBytes / 4;
    const size_t pool = ring + (size_t)kFusedThreads * 4;
    const size_t gate = ring + (size_t)(LP + 1 + (sh.ln ? 2 : 0)) * sh.E;
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
            // the image's scan output starts at zero: both directions add into it
            float4* yz = reinterpret_cast<float4*>(p.ys + (m0 + q / nch) * E);
            const bool zero_ys = sh.nd == 2;
            if (SL <= kFusedThreads) {
                part[threadIdx.x] = acc[0];
                __syncthreads();
                if (threadIdx.x < SL) {
                    float4 sum = part[threadIdx.x];
                    for (int qq = 1; qq < sm.G; ++qq) f4_add(sum, part[qq * SL + threadIdx.x]);
                    out[threadIdx.x] = f4_mul(sum, scale);
                    if (zero_ys) yz[threadIdx.x] = make_float4(0.f, 0.f, 0.f, 0.f);
                }
            } else {
#pragma unroll
                for (int k = 0; k < kMaxSlots; ++k)
                    if (k < sm.nslot) {
                        out[sm.slot[k]] = f4_mul(acc[k], scale);
                        if (zero_ys) yz[sm.slot[k]] = make_float4(0.f, 0.f, 0.f, 0.f);
                    }
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
// K-steps in a 5-, 4- or 3-stage cp.async pipeline.  The result goes to u (image-major blocks).
template <int TN, int kQStages>
__device__ __forceinline__ void fused_proj_t(const Shape& sh, const FusedPlan& pl, const FusedPtrs& p, int b, int q,
                                             float* smem) {
    const int T = sh.T, E = sh.E, J = sh.J, NJ = sh.NJ;
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
#pragma unroll
    for (int j = 0; j < TN; ++j) {
        const int jj = cg + 32 * j;
        if (jj < NJ) {
            const int k = jj / J, jc = jj - k * J;
#pragma unroll
            for (int i = 0; i < TM; ++i) {
                const int r = tg + 8 * i;
                if (r < mt) p.u[u_offset(sh, k, b, tq0 + r) + jc] = acc[i][j];
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

// ---- S: dt_proj + softplus, ZOH and both scans of channels [e0, e0 + ECH) of image b -------------
// 256 threads = ECH channels x ND directions, one recurrence each (fv_scan.cuh).  ys of image b
// was zeroed by the image's P tasks when both directions add into it.
template <int ND, bool ZOH_EXACT>
__device__ __forceinline__ void fused_scan(const Shape& sh, const FusedPlan& pl, const FusedPtrs& p, int b, int tile,
                                           float* smem) {
    const int e0 = tile * pl.ECH;
    seq_scan<kFusedThreads, ND, ZOH_EXACT>(sh, p.u, p.xbar, p.A_log, p.W_dt, p.b_dt, nullptr, p.ys + (size_t)b * sh.T * sh.E + e0,
                                           sh.E, b, e0, 0, smem, p.ckpt);
    cta_signal(p.ctrl ? p.ctrl + kCtrlHeaderWords + 2 * sh.B + b : nullptr);
}

// ---- E: repeat + skip + gate for grid lines [t0, t0+LP) of image b -------------------------------
// x and z stream through the ring (x mostly hits L2); every thread takes consecutive float4s of a
// chunk (all 256 threads busy for any E), and y is stored straight from registers (evict-first).
__device__ __forceinline__ bool fused_gate(const Shape& sh, const FusedPlan& pl, const FusedPtrs& p, int b, int g,
                                           float* smem, Ring& rg, uint64_t pol_stream, const unsigned* scan_done,
                                           unsigned* abort_flag, int* s_flag, unsigned long long* t_ready) {
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
    // x and z are on their way; now the image's scans must be done before its ys is read
    if (!cta_wait(scan_done, (unsigned)pl.nS, p.status, abort_flag, pl.wait_limit_ns, s_flag)) {
        ring_drain(rg, g0, g0 + min(kRingStages, nq), pl.wait_limit_ns);
        return false;
    }
    if (t_ready && threadIdx.x == 0) *t_ready = globaltimer_ns();  // trace: when the scans were seen done
    for (int i = threadIdx.x; i < nl * E; i += kFusedThreads) {
        const int l = i / E, e = i - l * E;
        ysl[i] = __ldcg(p.ys + ((size_t)b * sh.T + t0 + l) * E + e);
    }
    float* gam = ysl + (size_t)pl.LP * E;  // [E], [E]: LayerNorm gamma, beta
    float* bet = gam + E;
    if (sh.ln)
        for (int e = threadIdx.x; e < E; e += kFusedThreads) {
            gam[e] = __ldg(p.ln_gamma + e);
            bet[e] = __ldg(p.ln_beta + e);
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
        if (sh.ln) {
            // post-SSM LayerNorm: one warp per token of the stage; s = ys + (sum D) x is kept in
            // registers for the first kLnCache slots of each lane and recomputed from the stage
            // beyond; mean and variance from one warp reduction of sums about the shift K = s[0]
            const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
            const float4* g4 = reinterpret_cast<const float4*>(gam);
            const float4* b4 = reinterpret_cast<const float4*>(bet);
            const float invE = 1.f / (float)E;
            for (int j = warp; j < n; j += kFusedThreads / 32) {
                const float4* xr = xc + (size_t)j * SL;
                const float4* zr = zc + (size_t)j * SL;
                const float K = fmaf(dsum[0], xr[0].x, ysl[(size_t)l * E]);
                float4 sc[kLnCache];
                float m1 = 0.f, m2 = 0.f;
#pragma unroll
                for (int u = 0; u < kLnCache; ++u) {
                    const int slot = lane + 32 * u;
                    if (slot < SL) {
                        sc[u] = f4_fma(d4[slot], xr[slot], ys4[slot]);
                        ln_accum(sc[u], K, m1, m2);
                    }
                }
                for (int slot = lane + 32 * kLnCache; slot < SL; slot += 32)
                    ln_accum(f4_fma(d4[slot], xr[slot], ys4[slot]), K, m1, m2);
                float mean, rstd;
                ln_stats(m1, m2, K, invE, sh.ln_eps, mean, rstd);
                float4* yrow = y4 + (size_t)(tok0 + j) * stride4;
#pragma unroll
                for (int u = 0; u < kLnCache; ++u) {
                    const int slot = lane + 32 * u;
                    if (slot < SL) st_hint(yrow + slot, ln_gate4(sc[u], zr[slot], g4[slot], b4[slot], mean, rstd), pol_stream);
                }
                for (int slot = lane + 32 * kLnCache; slot < SL; slot += 32)
                    st_hint(yrow + slot, ln_gate4(f4_fma(d4[slot], xr[slot], ys4[slot]), zr[slot], g4[slot], b4[slot],
                                                  mean, rstd), pol_stream);
            }
        } else
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
    // (Claiming the next ticket while a task runs would hide the atomic's latency, but a pooling
    // ticket held behind a 60 us scan task stalls that image's whole chain: measured 3.5 ms.)
    for (;;) {
        __syncthreads();
        if (threadIdx.x == 0) {
            int kind = kTaskNone, b = 0, idx = 0;
            const unsigned tk = atomicAdd(p.ctrl, 1u);
            if (tk < pl.total && ld_relaxed_gpu(abort_flag) == 0u) fused_decode(pl, tk, kind, b, idx);
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
            // the gate waits for its scans inside, after its loads have started
            if (!fused_gate(sh, pl, p, b, idx, smem_f, rg, pol_stream, cnt_scan + b, abort_flag, &s_flag,
                            p.trace ? &s_t1 : nullptr))
                return;
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


// A single CTA that waits, with the layer's bounded wait, on a counter that nothing increments:
// exercises the timeout path (status FV_ERR_TIMEOUT, clean exit) without the layer.
__global__ void bounded_wait_selftest_kernel(unsigned* status, unsigned* ctrl, unsigned long long limit_ns) {
    __shared__ int s_flag;
    const bool ok = cta_wait(ctrl + kCtrlHeaderWords, 1u, status, ctrl + 1, limit_ns, &s_flag);
    if (threadIdx.x == 0 && ok) set_status(status, 1u);  // unreachable unless the counter moved
}

}  // namespace fv
