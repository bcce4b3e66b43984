// fv_scan.cuh -- dt_proj + softplus, ZOH discretisation and the selective scans of the FastVim SSM
// layer over the pooled sequence (sm_100a, fp32), shared by the staged scan kernel and the scan
// tasks of the fused launch.
//
// FastVim (gptget.net summary of arXiv 2502.00594, section "方法详解" items 3-4): per direction k,
// Delta = softplus(W_dt[k] dt_low + b_dt[k]), Abar = exp(Delta A), Bbar x = Delta B x (Euler; the
// exact-ZOH flag uses (Abar - 1) / A B x), h_t = Abar_t h_{t-1} + Bbar_t x_t from a zero state, the
// backward direction over t = T-1 .. 0, and ys = the sum over directions of C_t . h_t.
//
// 10^4 - 10^5 independent (image, channel, direction) recurrences of T = 14 .. 128 steps: each
// thread runs one recurrence sequentially over the whole pooled sequence, one exp2 per state and
// step, its 16 states in registers.  The per-step inputs that all channels of an image and
// direction share (B, C and dt_low: the projection row u[t] = [dt_low | B | C]) and the thread
// block's pooled tokens stream through shared memory in chunks of 16 steps, double-buffered with
// cp.async.  A backward chunk is staged in reverse, so slot i is always the i-th step taken and
// every shared-memory offset in the loops is a constant.  The step sizes Delta come either from a
// buffer written beforehand (the staged path: dt_proj + softplus as their own GEMM kernel, staged
// per chunk like the pooled tokens) or are computed per chunk up front by each thread (the fused
// launch: dt_low staged transposed, the thread's W_dt row in shared memory); either way the
// sequential loop holds only the state update.  With both directions enabled each direction adds
// its output into ys, which the caller zeroes beforehand: two float additions into +0 give the
// same sum in either order.
#pragma once

#include "fv_common.cuh"

namespace fv {

constexpr int kSeqThreads = 128;   // channels per CTA of the staged scan kernel (64 measured slower: the
                                   // per-image B, C, dt_low staging and W_dt loads double)
constexpr int kSeqChunk = 16;      // steps per staged chunk
constexpr int kSeqStates = 16;     // states per thread (N <= 16; unused ones stay zero)

__host__ __device__ __forceinline__ int seq_r4(int R) { return (R + 3) & ~3; }
// Row stride (floats) of the per-thread W_dt rows: a multiple of 4 whose quarter is odd, so the
// 8 lanes of a 128-bit shared load hit 8 distinct bank quads.
__host__ __device__ __forceinline__ int seq_wstride(int R) {
    const int r4 = seq_r4(R);
    return ((r4 / 4) & 1) ? r4 + 8 : r4 + 4;
}
// Shared memory (floats) of a scan over NT threads covering NDC directions.
__host__ __device__ __forceinline__ size_t seq_smem_floats(int NT, int NDC, int R) {
    const int r4 = seq_r4(R);
    return (size_t)NT * seq_wstride(R)                          // W_dt rows [NT][WS]
           + 2 * (size_t)NDC * kSeqChunk * 2 * kSeqStates       // B | C rows [2][NDC][16][32]
           + 2 * (size_t)NDC * r4 * kSeqChunk                   // dt_low, transposed [2][NDC][R4][16]
           + 2 * (size_t)kSeqChunk * NT;                        // pooled tokens [2][NDC][16][NT/NDC]
}
// Shared memory (floats) of a scan reading Delta from a buffer: B | C rows, Delta and pooled-token
// chunks, double-buffered.
__host__ __device__ __forceinline__ size_t seq_smem_floats_dt(int NT, int NDC) {
    return 2 * (size_t)NDC * kSeqChunk * 2 * kSeqStates + 2 * 2 * (size_t)kSeqChunk * NT;
}
// The staged path computes Delta in its own tensor-core GEMM kernel when dt_rank R >= 32; with
// shorter dt_proj dot products the scan computes them per chunk itself, which measured faster (the
// extra launch and the Delta round trip cost more than the R multiply-adds per step save).
__host__ __device__ __forceinline__ bool staged_delta_kernel(const Shape& sh) { return sh.R >= 32; }
__host__ __device__ __forceinline__ size_t seq_smem_floats(const Shape& sh) {
    return staged_delta_kernel(sh) ? seq_smem_floats_dt(kSeqThreads, 1) : seq_smem_floats(kSeqThreads, 1, sh.R);
}

// One step of the recurrence of a thread's 16 states: h = Abar h + Bbar x with Abar = 2^(dt A log2 e)
// and Bbar x = dt B x (Euler) or (Abar - 1) / A B x (exact ZOH); returns y = C . h.  bcrow: the
// step's B (16 floats) then C (16 floats).
template <bool ZOH_EXACT>
__device__ __forceinline__ float seq_step(float dt, float xv, const float* __restrict__ bcrow,
                                          const float (&A2)[kSeqStates], const float (&An)[kSeqStates],
                                          const float (&Ainv)[kSeqStates], float (&h)[kSeqStates]) {
    constexpr int NS = kSeqStates;
    const float dtx = dt * xv;
    const float4* Bq = reinterpret_cast<const float4*>(bcrow);
    const float4* Cq = Bq + NS / 4;
    float yp4[4] = {0.f, 0.f, 0.f, 0.f};  // four partial sums: short dependency chains
#pragma unroll
    for (int q = 0; q < NS / 4; ++q) {
        const float4 bv = Bq[q], cv = Cq[q];
        const float bb[4] = {bv.x, bv.y, bv.z, bv.w};
        const float cc[4] = {cv.x, cv.y, cv.z, cv.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int n = 4 * q + j;
            const float dA = ex2_approx(dt * A2[n]);
            const float bx = ZOH_EXACT ? expm1f(dt * An[n]) * Ainv[n] * bb[j] * xv : dtx * bb[j];
            h[n] = fmaf(dA, h[n], bx);
            yp4[j] = fmaf(cc[j], h[n], yp4[j]);
        }
    }
    return (yp4[0] + yp4[1]) + (yp4[2] + yp4[3]);
}

// Store a thread's 16 states at `ck` (the chunk loops skip it when the states are not kept or the
// channel is past E).
__device__ __forceinline__ void keep_state(float* ck, const float (&h)[kSeqStates]) {
    static_assert(kSeqStates == 16 && kSeqChunk == 2 * kCkptSteps, "checkpoint layout");
    float4* d = reinterpret_cast<float4*>(ck);
#pragma unroll
    for (int q = 0; q < 4; ++q) d[q] = make_float4(h[4 * q], h[4 * q + 1], h[4 * q + 2], h[4 * q + 3]);
}

// dt_proj + softplus and the recurrence over one staged chunk of `len` steps (LEN = 16 for a full
// chunk, 0 for a shorter one).  Slot i holds the i-th step taken; y of slot i goes to yp + i * ystep.
template <int LEN, int XSTRIDE, bool ZOH_EXACT>
__device__ __forceinline__ void seq_chunk(const float* __restrict__ bc, const float* __restrict__ dtT,
                                          const float* __restrict__ xs, const float* __restrict__ wrow, int R4,
                                          float bias, int len, const float (&A2)[kSeqStates],
                                          const float (&An)[kSeqStates], const float (&Ainv)[kSeqStates],
                                          float (&h)[kSeqStates], float* yp, ptrdiff_t ystep, bool live, bool add,
                                          float* ck, size_t ck_stride) {
    const int n_steps = LEN ? LEN : len;
    float dl[kSeqChunk];
#pragma unroll
    for (int i = 0; i < kSeqChunk; ++i) dl[i] = bias;
    for (int r4 = 0; r4 < R4; r4 += 4) {
        const float4 w = *reinterpret_cast<const float4*>(wrow + r4);
        const float wq[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float4* d4 = reinterpret_cast<const float4*>(dtT + (r4 + q) * kSeqChunk);
#pragma unroll
            for (int i4 = 0; i4 < kSeqChunk / 4; ++i4) {
                const float4 d = d4[i4];
                dl[4 * i4 + 0] = fmaf(wq[q], d.x, dl[4 * i4 + 0]);
                dl[4 * i4 + 1] = fmaf(wq[q], d.y, dl[4 * i4 + 1]);
                dl[4 * i4 + 2] = fmaf(wq[q], d.z, dl[4 * i4 + 2]);
                dl[4 * i4 + 3] = fmaf(wq[q], d.w, dl[4 * i4 + 3]);
            }
        }
    }
#pragma unroll
    for (int i = 0; i < kSeqChunk; ++i) {
        if (LEN || i < n_steps) {
            if (i % kCkptSteps == 0 && ck) keep_state(ck + (i / kCkptSteps) * ck_stride, h);
            const float y = seq_step<ZOH_EXACT>(softplus_fast(dl[i]), xs[i * XSTRIDE], bc + i * 2 * kSeqStates, A2,
                                                An, Ainv, h);
            if (live) {
                if (add) atomicAdd(yp, y);
                else *yp = y;
            }
            yp += ystep;
        }
    }
}

// The recurrence over one staged chunk with Delta read from shared memory (dts[i * XSTRIDE]: the
// i-th step taken).
template <int LEN, int XSTRIDE, bool ZOH_EXACT>
__device__ __forceinline__ void seq_chunk_dt(const float* __restrict__ bc, const float* __restrict__ dts,
                                             const float* __restrict__ xs, int len, const float (&A2)[kSeqStates],
                                             const float (&An)[kSeqStates], const float (&Ainv)[kSeqStates],
                                             float (&h)[kSeqStates], float* yp, ptrdiff_t ystep, bool live, bool add,
                                             float* ck, size_t ck_stride) {
    const int n_steps = LEN ? LEN : len;
#pragma unroll
    for (int i = 0; i < kSeqChunk; ++i) {
        if (LEN || i < n_steps) {
            if (i % kCkptSteps == 0 && ck) keep_state(ck + (i / kCkptSteps) * ck_stride, h);
            const float y = seq_step<ZOH_EXACT>(dts[i * XSTRIDE], xs[i * XSTRIDE], bc + i * 2 * kSeqStates, A2, An,
                                                Ainv, h);
            if (live) {
                if (add) atomicAdd(yp, y);
                else *yp = y;
            }
            yp += ystep;
        }
    }
}

// The scans of image b, channels [e0, e0 + NT / NDC), parameter slots k0 .. k0 + NDC - 1, by
// threads 0 .. NT-1 of the CTA: thread (slot kk, channel c) = (threadIdx.x / (NT/NDC),
// threadIdx.x % (NT/NDC)).  u: projections (u_offset layout), xbar: pooled tokens (xbar_offset:
// with the Conv1D each direction reads its own).  DT_IN: Delta is read from `delta`
// (delta_offset layout, softplus applied) and W_dt, b_dt are not used; otherwise dt_proj and the
// softplus run here per chunk.  The output of step t, channel e0 + c goes to ys0[t * ys_stride + c]
// ([T][E] rows: ys0 = ys + b T E + e0), zeroed by the caller when both directions add into it.
// smem: seq_smem_floats_dt(NT, NDC) floats with DT_IN, else seq_smem_floats(NT, NDC, R).
// ckpt: NULL, or the kept states (ckpt_offset layout; FV_FLAG_KEEP_STATES), written before every
// 8th step.
template <int NT, int NDC, bool ZOH_EXACT, bool DT_IN = false>
__device__ __forceinline__ void seq_scan(const Shape& sh, const float* __restrict__ u, const float* __restrict__ xbar,
                                         const float* __restrict__ A_log, const float* __restrict__ W_dt,
                                         const float* __restrict__ b_dt, const float* __restrict__ delta,
                                         float* __restrict__ ys0, int ys_stride, int b, int e0, int k0, float* smem,
                                         float* __restrict__ ckpt) {
    constexpr int NS = kSeqStates;
    constexpr int ECH = NT / NDC;             // channels per direction
    const int T = sh.T, E = sh.E, N = sh.N, R = sh.R, J = sh.J;
    const int R4 = DT_IN ? 0 : seq_r4(R), WS = DT_IN ? 0 : seq_wstride(R);
    const int kk = threadIdx.x / ECH, c = threadIdx.x - kk * ECH;
    const int k = k0 + kk;
    const int e = e0 + c;
    const bool live = e < E;
    float* sw = smem;                                            // [NT][WS] (not with DT_IN)
    float* sbc = sw + NT * WS;                                   // [2][NDC][16][32]
    float* sdt = sbc + 2 * NDC * kSeqChunk * 2 * kSeqStates;     // [2][NDC][R4][16], DT_IN: [2][NDC][16][ECH]
    float* sxs = sdt + (DT_IN ? 2 * kSeqChunk * NT : 2 * NDC * R4 * kSeqChunk);  // [2][NDC][16][ECH]
    auto dir_fwd = [&](int kd) { return sh.nd == 2 ? kd == 0 : (sh.dir_flags & 1u) != 0; };
    const bool fwd = dir_fwd(k);

    if (!DT_IN) {
        // W_dt rows of the block's (direction, channel) pairs: coalesced reads, padding columns zero
        for (int i = threadIdx.x; i < NT * R4; i += NT) {
            const int row = i / max(R4, 1), r = i - row * R4;
            const int kd = k0 + row / ECH, ee = e0 + row % ECH;
            sw[row * WS + r] = (ee < E && r < R) ? __ldg(W_dt + ((size_t)kd * E + ee) * R + r) : 0.f;
        }
    }
    constexpr float kLog2e = 1.4426950408889634f;
    float A2[NS], An[NS], Ainv[NS], h[NS];
#pragma unroll
    for (int n = 0; n < NS; ++n) {
        const float A = (live && n < N) ? -expf(__ldg(A_log + ((size_t)k * E + e) * N + n)) : 0.f;
        A2[n] = A * kLog2e;
        An[n] = A;
        Ainv[n] = A != 0.f ? 1.f / A : 0.f;
        h[n] = 0.f;
    }
    const float bias = (live && !DT_IN) ? __ldg(b_dt + (size_t)k * E + e) : 0.f;
    const bool add = sh.nd == 2;

    const int nchunks = (T + kSeqChunk - 1) / kSeqChunk;
    // [16][ECH] rows of a per-channel tensor (pooled tokens, Delta) for chunk slots of kd
    auto stage_rows = [&](float* dst, int t0, int len, bool f, auto src_of) {
        for (int v = threadIdx.x; v < kSeqChunk * (ECH / 4); v += NT) {
            const int slot = v / (ECH / 4), c4 = (v - slot * (ECH / 4)) * 4;
            const int t = t0 + (f ? slot : len - 1 - slot);
            const bool ok = slot < len && e0 + c4 < E;
            const float* src = ok ? src_of(t) + e0 + c4 : nullptr;
            cp_async16(dst + slot * ECH + c4, ok ? (const void*)src : (const void*)xbar, ok ? 16u : 0u);
        }
    };
    // stage iteration `it` into buffer buf for every slot; slot i of a chunk <- step t0 + i
    // (forward) or t0 + len - 1 - i (backward)
    auto stage = [&](int it, int buf) {
        for (int kd = 0; kd < NDC; ++kd) {
            const bool f = dir_fwd(k0 + kd);
            const int ci = f ? it : nchunks - 1 - it;
            const int t0 = ci * kSeqChunk, len = min(kSeqChunk, T - t0);
            const float* ub = u + u_offset(sh, k0 + kd, b, 0);
            float* bcb = sbc + (buf * NDC + kd) * kSeqChunk * 2 * kSeqStates;
            for (int i = threadIdx.x; i < kSeqChunk * 2 * kSeqStates; i += NT) {
                const int slot = i >> 5, j = i & 31, n = j & 15;
                const int t = t0 + (f ? slot : len - 1 - slot);
                const bool ok = slot < len && n < N;
                cp_async4z(bcb + i, ok ? ub + (size_t)t * J + R + (j < kSeqStates ? n : N + n) : ub, ok);
            }
            if (DT_IN) {
                stage_rows(sdt + (buf * NDC + kd) * kSeqChunk * ECH, t0, len, f,
                           [&](int t) { return delta + delta_offset(sh, k0 + kd, b, t); });
            } else {
                float* dtb = sdt + (buf * NDC + kd) * R4 * kSeqChunk;
                for (int i = threadIdx.x; i < R4 * kSeqChunk; i += NT) {
                    const int r = i >> 4, slot = i & 15;
                    const int t = t0 + (f ? slot : len - 1 - slot);
                    const bool ok = slot < len && r < R;
                    cp_async4z(dtb + i, ok ? ub + (size_t)t * J + r : ub, ok);
                }
            }
            stage_rows(sxs + (buf * NDC + kd) * kSeqChunk * ECH, t0, len, f,
                       [&](int t) { return xbar + xbar_offset(sh, b, sh.nx > 1 ? k0 + kd : 0, t); });
        }
        cp_async_commit();
    };

    stage(0, 0);
    for (int it = 0; it < nchunks; ++it) {
        if (it + 1 < nchunks) {
            stage(it + 1, (it + 1) & 1);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        const int buf = it & 1;
        const int ci = fwd ? it : nchunks - 1 - it;
        const int t0 = ci * kSeqChunk, len = min(kSeqChunk, T - t0);
        const int tfirst = fwd ? t0 : t0 + len - 1;
        float* yp = ys0 + (size_t)tfirst * ys_stride + c;
        const ptrdiff_t ystep = fwd ? (ptrdiff_t)ys_stride : -(ptrdiff_t)ys_stride;
        const float* bcb = sbc + (buf * NDC + kk) * kSeqChunk * 2 * kSeqStates;
        const float* xb = sxs + (buf * NDC + kk) * kSeqChunk * ECH + c;
        // the chunk's two kept states (before its steps 0 and 8), or none
        float* ck = (ckpt && live) ? ckpt + ckpt_offset(sh, b, k, 2 * it, e) : nullptr;
        const size_t cks = (size_t)E * 16;
        if (DT_IN) {
            const float* db = sdt + (buf * NDC + kk) * kSeqChunk * ECH + c;
            if (len == kSeqChunk)
                seq_chunk_dt<kSeqChunk, ECH, ZOH_EXACT>(bcb, db, xb, len, A2, An, Ainv, h, yp, ystep, live, add, ck,
                                                        cks);
            else
                seq_chunk_dt<0, ECH, ZOH_EXACT>(bcb, db, xb, len, A2, An, Ainv, h, yp, ystep, live, add, ck, cks);
        } else {
            const float* dtb = sdt + (buf * NDC + kk) * R4 * kSeqChunk;
            const float* wrow = sw + threadIdx.x * WS;
            if (len == kSeqChunk)
                seq_chunk<kSeqChunk, ECH, ZOH_EXACT>(bcb, dtb, xb, wrow, R4, bias, len, A2, An, Ainv, h, yp, ystep,
                                                     live, add, ck, cks);
            else
                seq_chunk<0, ECH, ZOH_EXACT>(bcb, dtb, xb, wrow, R4, bias, len, A2, An, Ainv, h, yp, ystep, live,
                                             add, ck, cks);
        }
        __syncthreads();  // the buffer is refilled by the next iteration's stage()
    }
}

}  // namespace fv
