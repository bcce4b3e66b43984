// fv_kernels.cuh -- the staged kernels of the FastVim SSM layer (sm_100a, fp32).
//
// Step map (FastVim, arXiv 2502.00594; gptget.net summary of the paper, section "方法详解"):
//   pool_dense_kernel / mask_bucket_kernel + mask_pool_kernel   item 2 (and item 6, masked)
//   proj_gemm_kernel (x_proj over every pooled token)            item 3
//   scan_seq_kernel (dt_proj + softplus, ZOH, both scans)       items 3-4
//   epilogue_dense_kernel / mask_epilogue_kernel                item 5 (repeat, skip, gate)
// Pooling and the epilogues are HBM streaming; the scans are MUFU/issue bound.
#pragma once

#include "fv_common.cuh"
#include "fv_scan.cuh"

namespace fv {

// ------------------------------------------------------------------------------------------
// Pooling
// ------------------------------------------------------------------------------------------

// Sum of tokens s0, s0+G, s0+2G, ... < S of one float4 column; four loads in flight.
__device__ __forceinline__ float4 sum_line(const float4* __restrict__ p, size_t st4, int s0, int G,
                                           int S) {
    float4 a0 = make_float4(0.f, 0.f, 0.f, 0.f), a1 = a0, a2 = a0, a3 = a0;
    int s = s0;
    for (; s + 7 * G < S; s += 8 * G) {  // eight tokens in flight
        float4 v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) v[u] = ld_stream(p + (size_t)(s + u * G) * st4);
        f4_add(a0, v[0]); f4_add(a1, v[1]); f4_add(a2, v[2]); f4_add(a3, v[3]);
        f4_add(a0, v[4]); f4_add(a1, v[5]); f4_add(a2, v[6]); f4_add(a3, v[7]);
    }
    if (s + 3 * G < S) {  // then four, for short lines
        float4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) v[u] = ld_stream(p + (size_t)(s + u * G) * st4);
        f4_add(a0, v[0]); f4_add(a1, v[1]); f4_add(a2, v[2]); f4_add(a3, v[3]);
        s += 4 * G;
    }
    for (; s < S; s += G) f4_add(a0, ld_stream(p + (size_t)s * st4));
    f4_add(a0, a1); f4_add(a2, a3); f4_add(a0, a2);
    return a0;
}

__device__ __forceinline__ float4 f4_scale(float4 v, float s) {
    return make_float4(v.x * s, v.y * s, v.z * s, v.w * s);
}

// Keeps the first device error of a sequence of calls: *dst = *dst ? *dst : *src.
__global__ void status_fold_kernel(unsigned* dst, const unsigned* src) {
    if (threadIdx.x == 0 && *dst == 0u) *dst = *src;
}

// One CTA per pooled token (b, t): mean of the S grid tokens of line t, 128-bit loads, no copy
// or transpose of the grid (the pooled axis only changes the base/stride of the index map).
__global__ void __launch_bounds__(kThreads)
pool_dense_kernel(Shape sh, const float* __restrict__ x, float* __restrict__ xbar) {
    __shared__ float4 part[kThreads];
    const int bt = blockIdx.x;
    const int b = bt / sh.T, t = bt - b * sh.T;
    const float4* base = reinterpret_cast<const float4*>(x + dense_base(sh, b, t));
    const size_t st4 = dense_stride(sh) >> 2;
    const float scale = sh.pool_scale / (float)sh.S;
    float4* out = reinterpret_cast<float4*>(xbar + (size_t)bt * sh.E);
    const int SL = sh.SL;
    if (SL <= kThreads) {
        const int G = kThreads / SL;  // launched with G * SL threads
        const int slot = threadIdx.x % SL, g = threadIdx.x / SL;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        if (g < G) acc = sum_line(base + slot, st4, g, G, sh.S);
        part[threadIdx.x] = acc;
        __syncthreads();
        if (threadIdx.x < SL) {
            float4 s = part[threadIdx.x];
            for (int q = 1; q < G; ++q) f4_add(s, part[q * SL + threadIdx.x]);
            out[threadIdx.x] = f4_scale(s, scale);
        }
    } else {
        for (int slot = threadIdx.x; slot < SL; slot += kThreads)
            out[slot] = f4_scale(sum_line(base + slot, st4, 0, 1, sh.S), scale);
    }
}

// Per-sample row bucketing of kept-token ids (one CTA per sample).  Validates every id (in
// range, not repeated), writes row_of[k] (-1 for a rejected id), the CSR offsets row_off[0..T]
// and row_tok (the sample's kept-token ordinals grouped by row, ascending k inside a row; the
// tail past the valid count is -1).  The stable scatter runs in one warp, 32 ids at a time,
// ranking equal rows with __match_any_sync, so the result does not depend on timing.
__global__ void __launch_bounds__(kThreads)
mask_bucket_kernel(Shape sh, const int32_t* __restrict__ keep_idx, int32_t* row_of, int32_t* row_off,
                   int32_t* row_tok, unsigned* status) {
    extern __shared__ unsigned smem_u[];
    const int G = sh.h * sh.w;
    const int nwords = (G + 31) >> 5;
    const int T = sh.T, K = sh.K;
    unsigned* bitmap = smem_u;
    int* cnt = reinterpret_cast<int*>(bitmap + nwords);  // [T]
    int* cursor = cnt + T;                               // [T]
    const int b = blockIdx.x;
    int32_t* rof = row_of + (size_t)b * K;
    for (int i = threadIdx.x; i < nwords; i += kThreads) bitmap[i] = 0u;
    for (int i = threadIdx.x; i < T; i += kThreads) cnt[i] = 0;
    __syncthreads();
    bool bad = false;
    for (int k = threadIdx.x; k < K; k += kThreads) {
        const int g = keep_idx[(size_t)b * K + k];
        int r = -1;
        if (g >= 0 && g < G) {
            const unsigned bit = 1u << (g & 31);
            const unsigned old = atomicOr(&bitmap[g >> 5], bit);
            if (!(old & bit)) r = (sh.pool_axis == 0) ? g / sh.w : g % sh.w;
        }
        if (r < 0) bad = true;
        else atomicAdd(&cnt[r], 1);
        rof[k] = r;
    }
    if (bad) set_status(status, kStatusIndex);
    __syncthreads();
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        int32_t* off = row_off + (size_t)b * (T + 1);
        int carry = 0;
        for (int base = 0; base < T; base += 32) {
            const int r = base + lane;
            const int v = (r < T) ? cnt[r] : 0;
            int incl = v;
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const int n = __shfl_up_sync(0xffffffffu, incl, d);
                if (lane >= d) incl += n;
            }
            if (r < T) {
                cursor[r] = carry + incl - v;
                off[r] = carry + incl - v;
            }
            carry += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) off[T] = carry;
        __syncwarp();
        int32_t* tok = row_tok + (size_t)b * K;
        const unsigned lt = (1u << lane) - 1u;
        for (int k0 = 0; k0 < K; k0 += 32) {
            const int k = k0 + lane;
            const int r = (k < K) ? rof[k] : -1;
            const unsigned peers = __match_any_sync(0xffffffffu, r);
            const int rank = __popc(peers & lt);
            const int pos = (r >= 0) ? cursor[r] + rank : 0;
            __syncwarp();
            if (r >= 0) {
                tok[pos] = k;
                if (lane == 31 - __clz(peers)) cursor[r] = pos + 1;
            }
            __syncwarp();
        }
        for (int p = carry + lane; p < K; p += 32) tok[p] = -1;
    }
}

// One CTA per pooled row (b, t) of a masked sample: sum of the row's kept tokens divided by the
// fixed full length S (an empty row pools to 0).  Up to 256 float4 slots per token: groups of SL
// threads split the row's tokens; wider rows: one thread per slot (launched with SL threads
// rounded up to whole warps, up to 1024), so no thread takes two slots while others take one.
constexpr int kMaskPoolMaxThreads = 1024;
__global__ void __launch_bounds__(kMaskPoolMaxThreads, 2)
mask_pool_kernel(Shape sh, const float* __restrict__ x, const int32_t* __restrict__ row_off,
                 const int32_t* __restrict__ row_tok, float* __restrict__ xbar) {
    __shared__ float4 part[kThreads];
    const int bt = blockIdx.x;
    const int b = bt / sh.T, t = bt - b * sh.T;
    const int32_t* off = row_off + (size_t)b * (sh.T + 1);
    const int p0 = off[t], p1 = off[t + 1];
    const int32_t* tok = row_tok + (size_t)b * sh.K;
    const float4* xb = reinterpret_cast<const float4*>(x + (size_t)b * sh.K * sh.E);
    const float scale = sh.pool_scale / (float)sh.S;
    float4* out = reinterpret_cast<float4*>(xbar + (size_t)bt * sh.E);
    const int SL = sh.SL;
    if (SL <= kThreads) {
        const int G = kThreads / SL;
        const int slot = threadIdx.x % SL, g = threadIdx.x / SL;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        if (g < G)
            for (int p = p0 + g; p < p1; p += G) f4_add(acc, ld_stream(xb + (size_t)tok[p] * SL + slot));
        part[threadIdx.x] = acc;
        __syncthreads();
        if (threadIdx.x < SL) {
            float4 s = part[threadIdx.x];
            for (int q = 1; q < G; ++q) f4_add(s, part[q * SL + threadIdx.x]);
            out[threadIdx.x] = f4_scale(s, scale);
        }
    } else {
        for (int slot = threadIdx.x; slot < SL; slot += blockDim.x) {
            float4 a0 = make_float4(0.f, 0.f, 0.f, 0.f);
            int p = p0;
            for (; p + 3 < p1; p += 4) {  // four kept tokens in flight, added in kept order
                const float4 v0 = ld_stream(xb + (size_t)tok[p] * SL + slot);
                const float4 v1 = ld_stream(xb + (size_t)tok[p + 1] * SL + slot);
                const float4 v2 = ld_stream(xb + (size_t)tok[p + 2] * SL + slot);
                const float4 v3 = ld_stream(xb + (size_t)tok[p + 3] * SL + slot);
                f4_add(a0, v0); f4_add(a0, v1); f4_add(a0, v2); f4_add(a0, v3);
            }
            for (; p < p1; ++p) f4_add(a0, ld_stream(xb + (size_t)tok[p] * SL + slot));
            out[slot] = f4_scale(a0, scale);
        }
    }
}

// ------------------------------------------------------------------------------------------
// Repeat + skip + gate: y = SiLU(z) * (ys[row] + (sum_k D_k) x), streamed with 128-bit accesses.
// ------------------------------------------------------------------------------------------
// SiLU(z) * (ys + (sum D) x) for four channels; SiLU with the SFU exp2 and reciprocal (silu_fast).
__device__ __forceinline__ float4 gate4(const float4& xv, const float4& zv, const float4& ysv, const float4& dv) {
    return make_float4(silu_fast(zv.x) * fmaf(dv.x, xv.x, ysv.x), silu_fast(zv.y) * fmaf(dv.y, xv.y, ysv.y),
                       silu_fast(zv.z) * fmaf(dv.z, xv.z, ysv.z), silu_fast(zv.w) * fmaf(dv.w, xv.w, ysv.w));
}

__device__ __forceinline__ float4 dsum4(const float* __restrict__ D, int nd, int SL, int slot) {
    const float4* D4 = reinterpret_cast<const float4*>(D);
    float4 dv = D4[slot];
    if (nd == 2) f4_add(dv, D4[SL + slot]);
    return dv;
}

__device__ __forceinline__ void gate_line(const float4* __restrict__ x4, const float4* __restrict__ z4,
                                          float4* __restrict__ y4, size_t st4, int s0, int G, int S,
                                          const float4& ysv, const float4& dv) {
    int s = s0;
    for (; s + G < S; s += 2 * G) {
        const size_t o0 = (size_t)s * st4, o1 = (size_t)(s + G) * st4;
        const float4 x0 = ld_stream(x4 + o0), z0 = ld_stream(z4 + o0);
        const float4 x1 = ld_stream(x4 + o1), z1 = ld_stream(z4 + o1);
        st_stream(y4 + o0, gate4(x0, z0, ysv, dv));
        st_stream(y4 + o1, gate4(x1, z1, ysv, dv));
    }
    if (s < S) {
        const size_t o0 = (size_t)s * st4;
        st_stream(y4 + o0, gate4(ld_stream(x4 + o0), ld_stream(z4 + o0), ysv, dv));
    }
}

// One CTA per pooled token (b, t): writes the S grid tokens of line t.
__global__ void __launch_bounds__(kThreads)
epilogue_dense_kernel(Shape sh, const float* __restrict__ x, const float* __restrict__ z,
                      const float* __restrict__ ys, const float* __restrict__ D, float* __restrict__ y) {
    const int bt = blockIdx.x;
    const int b = bt / sh.T, t = bt - b * sh.T;
    const size_t off4 = dense_base(sh, b, t) >> 2;
    const size_t st4 = dense_stride(sh) >> 2;
    const float4* x4 = reinterpret_cast<const float4*>(x) + off4;
    const float4* z4 = reinterpret_cast<const float4*>(z) + off4;
    float4* y4 = reinterpret_cast<float4*>(y) + off4;
    const float4* ys4 = reinterpret_cast<const float4*>(ys + (size_t)bt * sh.E);
    const int SL = sh.SL;
    if (SL <= kThreads) {
        const int G = kThreads / SL;
        const int slot = threadIdx.x % SL, g = threadIdx.x / SL;
        if (g < G) gate_line(x4 + slot, z4 + slot, y4 + slot, st4, g, G, sh.S, ys4[slot], dsum4(D, sh.nd, SL, slot));
    } else {
        for (int slot = threadIdx.x; slot < SL; slot += kThreads)
            gate_line(x4 + slot, z4 + slot, y4 + slot, st4, 0, 1, sh.S, ys4[slot], dsum4(D, sh.nd, SL, slot));
    }
}

constexpr int kMaskEpiTokens = 16;  // kept tokens per masked-epilogue CTA

// One CTA per (sample b, block of kMaskEpiTokens kept tokens); a rejected token gets 0.
__global__ void __launch_bounds__(kThreads)
mask_epilogue_kernel(Shape sh, const float* __restrict__ x, const float* __restrict__ z,
                     const float* __restrict__ ys, const float* __restrict__ D,
                     const int32_t* __restrict__ row_of, float* __restrict__ y) {
    extern __shared__ float4 mdsum[];      // [SL] sum_k D_k
    __shared__ int rows[kMaskEpiTokens];   // pooled row of each of the CTA's kept tokens
    const int nkb = (sh.K + kMaskEpiTokens - 1) / kMaskEpiTokens;
    const int b = blockIdx.x / nkb;
    const int k0 = (blockIdx.x - b * nkb) * kMaskEpiTokens;
    const int SL = sh.SL;
    for (int slot = threadIdx.x; slot < SL; slot += kThreads) mdsum[slot] = dsum4(D, sh.nd, SL, slot);
    if (threadIdx.x < kMaskEpiTokens) {
        const int k = k0 + threadIdx.x;
        rows[threadIdx.x] = k < sh.K ? row_of[(size_t)b * sh.K + k] : -1;
    }
    __syncthreads();
    const int n = min(kMaskEpiTokens, sh.K - k0) * SL;  // float4 elements of the CTA's tokens
    const float inv_sl = 1.f / (float)SL;
    const size_t obase = ((size_t)b * sh.K + k0) * SL;  // the tokens are contiguous rows
    const float4* x4 = reinterpret_cast<const float4*>(x) + obase;
    const float4* z4 = reinterpret_cast<const float4*>(z) + obase;
    const float4* ys4 = reinterpret_cast<const float4*>(ys) + (size_t)b * sh.T * SL;
    float4* y4 = reinterpret_cast<float4*>(y) + obase;
    const float4 zero = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int f0 = threadIdx.x; f0 < n; f0 += 2 * kThreads) {  // two elements per thread in flight
        float4 xv[2], zv[2], yv[2];
        int slot[2], r[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int f = f0 + u * kThreads;
            r[u] = -1;
            if (f < n) {
                const int kk = (int)(((float)f + 0.5f) * inv_sl);  // f / SL (exact for f < 2^16)
                slot[u] = f - kk * SL;
                r[u] = rows[kk];
                if (r[u] >= 0) {
                    xv[u] = ld_stream(x4 + f);
                    zv[u] = ld_stream(z4 + f);
                    yv[u] = __ldcg(ys4 + (size_t)r[u] * SL + slot[u]);
                }
            }
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int f = f0 + u * kThreads;
            if (f < n) st_stream(y4 + f, r[u] >= 0 ? gate4(xv[u], zv[u], yv[u], mdsum[slot[u]]) : zero);
        }
    }
}

// ---- The block's Conv1D in front of the layer (dense layers, staged kernels) ---------------------
// Summary page, "方法详解" item 2 (the layer pools the output of the block's Conv1D) and the Vim
// article's section 2.1 code (one Conv1D per direction, the backward one over the reversed
// sequence).  Depthwise, d_conv <= 4 taps, zero padding, along the block's sequence p = t S + s.
// Nothing convolved is stored: the pooling and the epilogue recompute it from x as they stream it,
// each thread sliding a window of 7 tokens (p - 3 .. p + 3) of one float4 slot along a run of
// consecutive sequence positions, so every token row is loaded once per run (plus 6 halo rows).
struct ConvSlot {
    float4 w[2][kMaxConv];  // taps of direction slots 0, 1, right-aligned in a 4-wide window (zero-padded)
    float4 b[2];            // biases
};

// Filters of float4 slot `slot` (channels 4 slot .. 4 slot + 3).  conv_w [nd][E][dc], conv_b [nd][E].
__device__ __forceinline__ ConvSlot conv_slot(const Shape& sh, const float* __restrict__ conv_w,
                                              const float* __restrict__ conv_b, int slot) {
    ConvSlot c;
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        c.b[k] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int q = 0; q < kMaxConv; ++q) c.w[k][q] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (k < sh.nd) {
            c.b[k] = __ldg(reinterpret_cast<const float4*>(conv_b + (size_t)k * sh.E) + slot);
            const float* wk = conv_w + ((size_t)k * sh.E + 4 * slot) * sh.dc;
#pragma unroll
            for (int qq = 0; qq < kMaxConv; ++qq) {  // window tap qq holds filter tap qq - (4 - dc)
                const int q = qq - (kMaxConv - sh.dc);
                if (q >= 0)
                    c.w[k][qq] = make_float4(__ldg(wk + q), __ldg(wk + sh.dc + q), __ldg(wk + 2 * sh.dc + q),
                                             __ldg(wk + 3 * sh.dc + q));
            }
        }
    }
    return c;
}

__device__ __forceinline__ float4 f4_silu(const float4& v) {
    return make_float4(silu_fast(v.x), silu_fast(v.y), silu_fast(v.z), silu_fast(v.w));
}

// The convolved value of direction slot k at the window's centre: a forward slot reads the window
// tokens p - 3 .. p (taps in order), a backward slot p + 3 .. p (the same filter on the reversed
// sequence).
__device__ __forceinline__ float4 conv_at(const Shape& sh, const ConvSlot& c, int k, bool fwd, const float4 (&win)[7]) {
    float4 a = c.b[k];
#pragma unroll
    for (int q = 0; q < kMaxConv; ++q) a = f4_fma(c.w[k][q], fwd ? win[q] : win[6 - q], a);
    return sh.conv_silu ? f4_silu(a) : a;
}

// Sequence cursor of image b: position (t, s), t = line, s = token along it.
struct SeqPos {
    int t, s;
};
__device__ __forceinline__ void seq_step(const Shape& sh, SeqPos& p) {
    if (++p.s == sh.S) { p.s = 0; ++p.t; }
}
__device__ __forceinline__ SeqPos seq_back(const Shape& sh, SeqPos p, int n) {
    p.s -= n;
    while (p.s < 0) { p.s += sh.S; --p.t; }
    return p;
}
// Slot `slot` of the token at position p of image b (zero outside the sequence).
__device__ __forceinline__ float4 seq_load(const Shape& sh, const float4* __restrict__ x4, int b, const SeqPos& p,
                                           int slot) {
    if (p.t < 0 || p.t >= sh.T) return make_float4(0.f, 0.f, 0.f, 0.f);
    return ld_stream(x4 + ((dense_base(sh, b, p.t) + (size_t)p.s * dense_stride(sh)) >> 2) + slot);
}

// Runs `emit(s, xc0, xc1, zv)` for the tokens s in [s0, s1) of line t of image b, xc0 and xc1
// the convolved values of direction slots 0 and 1 (xc1 unused with one direction), zv the token's
// z (with WITH_Z).  Loads run one batch of kU tokens ahead of the arithmetic, so 2 kU tokens are
// in flight (kU = 4 for the pooling, 2 for the epilogue, whose registers also hold z); tokens inside line t are addressed from the line's base, the halo beyond it through
// the sequence cursor.
template <bool WITH_Z, int kU, class Emit>
__device__ __forceinline__ void conv_line_run(const Shape& sh, const float* __restrict__ x, const float* __restrict__ z,
                                              const ConvSlot& c, int b, int t, int s0, int s1, int slot, Emit&& emit) {
    const float4* x4 = reinterpret_cast<const float4*>(x);
    const size_t line4 = (dense_base(sh, b, t) >> 2) + slot;
    const size_t st4 = dense_stride(sh) >> 2;
    const int S = sh.S;
    const bool fwd0 = (sh.dir_flags & 1u) != 0;  // slot 0 is the forward direction when it is enabled
    auto load_x = [&](int s) -> float4 {
        if (s >= 0 && s < S) return ld_stream(x4 + line4 + (size_t)s * st4);
        SeqPos p{t, s};
        while (p.s < 0) { p.s += S; --p.t; }
        while (p.s >= S) { p.s -= S; ++p.t; }
        return seq_load(sh, x4, b, p, slot);
    };
    auto load_z = [&](int s) -> float4 {
        return (WITH_Z && s < s1) ? ld_stream(reinterpret_cast<const float4*>(z) + line4 + (size_t)s * st4)
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
    };
    float4 win[7];
#pragma unroll
    for (int i = 0; i < 6; ++i) win[i + 1] = load_x(s0 - 3 + i);  // positions s0 - 3 .. s0 + 2
    float4 nx[kU], nz[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
        nx[u] = load_x(s0 + 3 + u);
        nz[u] = load_z(s0 + u);
    }
    for (int s = s0; s < s1; s += kU) {
        float4 cx[kU], cz[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            cx[u] = nx[u];
            cz[u] = nz[u];
        }
        if (s + kU < s1) {
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                nx[u] = load_x(s + kU + 3 + u);
                nz[u] = load_z(s + kU + u);
            }
        }
#pragma unroll
        for (int u = 0; u < kU; ++u) {
#pragma unroll
            for (int i = 0; i < 6; ++i) win[i] = win[i + 1];
            win[6] = cx[u];
            if (s + u < s1) {
                const float4 a = conv_at(sh, c, 0, fwd0, win);
                const float4 bb = sh.nd == 2 ? conv_at(sh, c, 1, false, win) : a;
                emit(s + u, a, bb, cz[u]);
            }
        }
    }
}

// Thread layout of the conv kernels: G groups of SL threads (one float4 slot each) per CTA, group
// g taking a contiguous run of the line's tokens; above 256 slots one group loops over the slots.
__device__ __forceinline__ void conv_groups(const Shape& sh, int& G, int& g, int& slot0, int& slot_step) {
    if (sh.SL <= kThreads) {
        G = kThreads / sh.SL;
        g = threadIdx.x / sh.SL;
        slot0 = threadIdx.x - g * sh.SL;
        slot_step = sh.SL;  // one slot
    } else {
        G = 1;
        g = 0;
        slot0 = threadIdx.x;
        slot_step = kThreads;
    }
}

// One CTA per pooled token (b, t): each direction slot pools its own convolved tokens of line t,
// xbar[b][k][t] = pool_scale / S * sum_s xc_k(t, s).
__global__ void __launch_bounds__(kThreads, 2)
pool_conv_kernel(Shape sh, const float* __restrict__ x, const float* __restrict__ conv_w,
                 const float* __restrict__ conv_b, float* __restrict__ xbar) {
    __shared__ float4 part[2][kThreads];
    const int bt = blockIdx.x;
    const int b = bt / sh.T, t = bt - b * sh.T;
    const float scale = sh.pool_scale / (float)sh.S;
    int G, g, slot0, sstep;
    conv_groups(sh, G, g, slot0, sstep);
    const int run = (sh.S + G - 1) / G;
    const int s0 = g * run, s1 = min(sh.S, s0 + run);
    for (int slot = slot0; slot < sh.SL; slot += sstep) {
        float4 acc0 = make_float4(0.f, 0.f, 0.f, 0.f), acc1 = acc0;
        if (g < G && s0 < s1) {
            const ConvSlot c = conv_slot(sh, conv_w, conv_b, slot);
            conv_line_run<false, 4>(sh, x, nullptr, c, b, t, s0, s1, slot,
                                 [&](int, const float4& a, const float4& bb, const float4&) {
                                     f4_add(acc0, a);
                                     f4_add(acc1, bb);
                                 });
        }
        if (G == 1) {
            reinterpret_cast<float4*>(xbar + xbar_offset(sh, b, 0, t))[slot] = f4_scale(acc0, scale);
            if (sh.nd == 2) reinterpret_cast<float4*>(xbar + xbar_offset(sh, b, 1, t))[slot] = f4_scale(acc1, scale);
        } else {
            part[0][threadIdx.x] = acc0;
            part[1][threadIdx.x] = acc1;
            __syncthreads();
            if (threadIdx.x < sh.SL) {
                for (int k = 0; k < sh.nd; ++k) {
                    float4 v = part[k][threadIdx.x];
                    for (int q = 1; q < G; ++q) f4_add(v, part[k][q * sh.SL + threadIdx.x]);
                    reinterpret_cast<float4*>(xbar + xbar_offset(sh, b, k, t))[threadIdx.x] = f4_scale(v, scale);
                }
            }
        }
    }
}

// One CTA per pooled token (b, t): y = SiLU(z) * (ys[b][t] + sum_k D[k] * xc_k) for the tokens of
// line t, the convolved values recomputed from x.
__global__ void __launch_bounds__(kThreads, 2)
epilogue_conv_kernel(Shape sh, const float* __restrict__ x, const float* __restrict__ z,
                     const float* __restrict__ ys, const float* __restrict__ D, const float* __restrict__ conv_w,
                     const float* __restrict__ conv_b, float* __restrict__ y) {
    const int bt = blockIdx.x;
    const int b = bt / sh.T, t = bt - b * sh.T;
    const size_t base4 = dense_base(sh, b, t) >> 2;
    const size_t st4 = dense_stride(sh) >> 2;
    float4* y4 = reinterpret_cast<float4*>(y) + base4;
    int G, g, slot0, sstep;
    conv_groups(sh, G, g, slot0, sstep);
    if (g >= G) return;
    const int run = (sh.S + G - 1) / G;
    const int s0 = g * run, s1 = min(sh.S, s0 + run);
    if (s0 >= s1) return;
    for (int slot = slot0; slot < sh.SL; slot += sstep) {
        const ConvSlot c = conv_slot(sh, conv_w, conv_b, slot);
        const float4 ysv = __ldcg(reinterpret_cast<const float4*>(ys + ((size_t)b * sh.T + t) * sh.E) + slot);
        const float4 d0 = __ldg(reinterpret_cast<const float4*>(D) + slot);
        const float4 d1 = sh.nd == 2 ? __ldg(reinterpret_cast<const float4*>(D + sh.E) + slot)
                                     : make_float4(0.f, 0.f, 0.f, 0.f);
        conv_line_run<true, 2>(sh, x, z, c, b, t, s0, s1, slot, [&](int s, const float4& a, const float4& bb,
                                                                 const float4& zv) {
            const size_t o = (size_t)s * st4 + slot;
            const float4 sv = f4_fma(d1, bb, f4_fma(d0, a, ysv));
            st_stream(y4 + o, make_float4(silu_fast(zv.x) * sv.x, silu_fast(zv.y) * sv.y, silu_fast(zv.z) * sv.z,
                                          silu_fast(zv.w) * sv.w));
        });
    }
}

// The skip term sum_k D[k] * xc_k of one float4 slot of one token (i, j) of image b, loading the
// token's sequence neighbours directly (the LayerNorm epilogue, which walks tokens, not runs).
__device__ __forceinline__ float4 conv_skip_at(const Shape& sh, const float* __restrict__ x,
                                               const float* __restrict__ conv_w, const float* __restrict__ conv_b,
                                               const float* __restrict__ D, int b, int i, int j, int slot) {
    const ConvSlot c = conv_slot(sh, conv_w, conv_b, slot);
    const SeqPos p = sh.pool_axis == 0 ? SeqPos{i, j} : SeqPos{j, i};
    SeqPos q = seq_back(sh, p, 3);
    float4 win[7];
#pragma unroll
    for (int u = 0; u < 7; ++u) {
        win[u] = seq_load(sh, reinterpret_cast<const float4*>(x), b, q, slot);
        seq_step(sh, q);
    }
    const bool fwd0 = (sh.dir_flags & 1u) != 0;
    float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
    s = f4_fma(__ldg(reinterpret_cast<const float4*>(D) + slot), conv_at(sh, c, 0, fwd0, win), s);
    if (sh.nd == 2) s = f4_fma(__ldg(reinterpret_cast<const float4*>(D + sh.E) + slot), conv_at(sh, c, 1, false, win), s);
    return s;
}

// ---- Staged epilogue with the post-SSM LayerNorm (dense and masked) ------------------------------
// s = ys[t] + (sum_k D[k]) x;  y = SiLU(z) * (gamma * (s - mean) * rsqrt(var + eps) + beta), mean and
// (biased) variance over the E channels of the token (summary page, "方法详解" item 5: repeat,
// skip, LayerNorm; VMamba's post-SSM LayerNorm sits before the gate).  One warp per token: x and z
// are streamed once (loads batched kLnBatch slots per lane) into shared-memory rows; the mean and
// variance come from one warp reduction of sums about a shift K (the token's first s value), which
// keeps var = E[(s-K)^2] - E[s-K]^2 free of cancellation when |mean| >> std.
constexpr int kLnWarps = 4;
constexpr int kLnTokensPerWarp = 4;
constexpr int kLnBatch = 4;

__host__ __forceinline__ size_t ln_epilogue_smem_bytes(const Shape& sh) {
    return (size_t)(3 + 2 * kLnWarps) * sh.SL * sizeof(float4);  // sum D, gamma, beta; per warp s and z rows
}

template <bool CONV>
__global__ void __launch_bounds__(kLnWarps * 32)
ln_epilogue_kernel(Shape sh, const float* __restrict__ x, const float* __restrict__ z,
                   const float* __restrict__ ys, const float* __restrict__ D, const float* __restrict__ gamma,
                   const float* __restrict__ beta, const int32_t* __restrict__ row_of,
                   const float* __restrict__ conv_w, const float* __restrict__ conv_b, float* __restrict__ y) {
    extern __shared__ float4 lsm[];
    const int SL = sh.SL;
    float4* dsum = lsm;
    float4* g4 = dsum + SL;
    float4* b4 = g4 + SL;
    for (int slot = threadIdx.x; slot < SL; slot += kLnWarps * 32) {
        dsum[slot] = dsum4(D, sh.nd, SL, slot);
        g4[slot] = __ldg(reinterpret_cast<const float4*>(gamma) + slot);
        b4[slot] = __ldg(reinterpret_cast<const float4*>(beta) + slot);
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float4* srow = b4 + SL + (size_t)warp * 2 * SL;
    float4* zrow = srow + SL;
    const long long per_img = sh.K > 0 ? (long long)sh.K : (long long)sh.h * sh.w;
    const long long ntok = (long long)sh.B * per_img;
    const long long tok0 = ((long long)blockIdx.x * kLnWarps + warp) * kLnTokensPerWarp;
    const float invE = 1.f / (float)sh.E;
    const float4* x4 = reinterpret_cast<const float4*>(x);
    const float4* z4 = reinterpret_cast<const float4*>(z);
    float4* y4 = reinterpret_cast<float4*>(y);
    for (int q = 0; q < kLnTokensPerWarp; ++q) {
        const long long tok = tok0 + q;
        if (tok >= ntok) break;
        const int b = (int)(tok / per_img);
        const long long r = tok - (long long)b * per_img;
        int t;
        if (sh.K > 0) {
            t = row_of[tok];  // < 0: a rejected id, output 0
        } else {
            const int i = (int)(r / sh.w), j = (int)(r - (long long)i * sh.w);
            t = sh.pool_axis == 0 ? i : j;
        }
        const size_t o = (size_t)tok * SL;
        if (t < 0) {
            for (int slot = lane; slot < SL; slot += 32) st_stream(y4 + o + slot, make_float4(0.f, 0.f, 0.f, 0.f));
            continue;
        }
        const float4* ys4 = reinterpret_cast<const float4*>(ys + ((size_t)b * sh.T + t) * sh.E);
        // shift: the token's first s value (the same value in every lane; with the Conv1D the
        // first scan output, any value near the data will do)
        const float K = CONV ? __ldcg(ys + ((size_t)b * sh.T + t) * sh.E)
                                  : fmaf(dsum[0].x, __ldcg(x + o * 4), __ldcg(ys + ((size_t)b * sh.T + t) * sh.E));
        float m1 = 0.f, m2 = 0.f;
        for (int base = lane; base < SL; base += 32 * kLnBatch) {
            float4 xv[kLnBatch], zv[kLnBatch], yv[kLnBatch];
#pragma unroll
            for (int u = 0; u < kLnBatch; ++u) {
                const int slot = base + 32 * u;
                if (slot < SL) {
                    if (!CONV) xv[u] = ld_stream(x4 + o + slot);
                    zv[u] = ld_stream(z4 + o + slot);
                    yv[u] = __ldcg(ys4 + slot);
                }
            }
            if (CONV) {  // the skip from each direction's convolved tokens, loaded by sequence position
                const int i = (int)(r / sh.w), j = (int)(r - (long long)i * sh.w);
#pragma unroll
                for (int u = 0; u < kLnBatch; ++u) {
                    const int slot = base + 32 * u;
                    if (slot < SL) xv[u] = conv_skip_at(sh, x, conv_w, conv_b, D, b, i, j, slot);
                }
            }
#pragma unroll
            for (int u = 0; u < kLnBatch; ++u) {
                const int slot = base + 32 * u;
                if (slot < SL) {
                    const float4 sv = CONV ? make_float4(yv[u].x + xv[u].x, yv[u].y + xv[u].y, yv[u].z + xv[u].z,
                                                              yv[u].w + xv[u].w)
                                                : f4_fma(dsum[slot], xv[u], yv[u]);
                    srow[slot] = sv;
                    zrow[slot] = zv[u];
                    ln_accum(sv, K, m1, m2);
                }
            }
        }
        float mean, rstd;
        ln_stats(m1, m2, K, invE, sh.ln_eps, mean, rstd);
        for (int slot = lane; slot < SL; slot += 32)
            st_stream(y4 + o + slot, ln_gate4(srow[slot], zrow[slot], g4[slot], b4[slot], mean, rstd));
    }
}

// The same epilogue for rows of up to 1536 channels (without the Conv1D), with each lane's share of
// the token's s = ys[t] + (sum D) x held in registers (NSL float4 slots per lane) instead of
// shared-memory rows: eight warps per CTA and no per-warp shared memory, so occupancy is set by
// registers alone.  Per token: x, ys and z are loaded at once, s and its shifted moments formed,
// the warp reduction gives the mean and 1/sqrt(var + eps), and y is stored.
constexpr int kLnRegWarps = 8;
__host__ __device__ __forceinline__ int ln_reg_nsl(int SL) {
    const int need = (SL + 31) / 32;
    return need <= 4 ? need : (need <= 6 ? 6 : (need <= 8 ? 8 : (need <= 12 ? 12 : 0)));
}

// WPT warps per token (WPT = 2 for the widest rows: half the registers per thread, so two CTAs
// per SM instead of one); the group's moments meet behind a named barrier, in warp order.
template <int NSL, int WPT>
__global__ void __launch_bounds__(kLnRegWarps * 32)
ln_epilogue_reg_kernel(Shape sh, const float* __restrict__ x, const float* __restrict__ z,
                       const float* __restrict__ ys, const float* __restrict__ D, const float* __restrict__ gamma,
                       const float* __restrict__ beta, const int32_t* __restrict__ row_of, float* __restrict__ y) {
    constexpr int G = 32 * WPT, NG = kLnRegWarps / WPT;  // threads per token, tokens per block
    extern __shared__ float4 lrs[];
    __shared__ float red[kLnRegWarps][2];
    const int SL = sh.SL;
    float4* dsum = lrs;
    float4* g4 = dsum + SL;
    float4* b4 = g4 + SL;
    for (int slot = threadIdx.x; slot < SL; slot += kLnRegWarps * 32) {
        dsum[slot] = dsum4(D, sh.nd, SL, slot);
        g4[slot] = __ldg(reinterpret_cast<const float4*>(gamma) + slot);
        b4[slot] = __ldg(reinterpret_cast<const float4*>(beta) + slot);
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int grp = warp / WPT, wig = warp - grp * WPT, gt = wig * 32 + lane;
    const long long per_img = sh.K > 0 ? (long long)sh.K : (long long)sh.h * sh.w;
    const long long ntok = (long long)sh.B * per_img;
    const float invE = 1.f / (float)sh.E;
    // this thread's slots are gt + G u: one base pointer per tensor, constant offsets per slot
    const int nsl = (SL - gt + G - 1) / G;  // slots of this thread
    const float4* dl = dsum + gt;
    const float4* gl = g4 + gt;
    const float4* bl = b4 + gt;
    for (long long tok = (long long)blockIdx.x * NG + grp; tok < ntok; tok += (long long)gridDim.x * NG) {
        const int b = (int)(tok / per_img);
        const long long r = tok - (long long)b * per_img;
        int t;
        if (sh.K > 0) {
            t = row_of[tok];  // < 0: a rejected id, output 0
        } else {
            const int i = (int)(r / sh.w), j = (int)(r - (long long)i * sh.w);
            t = sh.pool_axis == 0 ? i : j;
        }
        const size_t o = (size_t)tok * SL + gt;
        float4* yl = reinterpret_cast<float4*>(y) + o;
        if (t < 0) {
#pragma unroll
            for (int u = 0; u < NSL; ++u)
                if (u < nsl) st_stream(yl + G * u, make_float4(0.f, 0.f, 0.f, 0.f));
            continue;
        }
        const float4* xl = reinterpret_cast<const float4*>(x) + o;
        const float* ysr = ys + ((size_t)b * sh.T + t) * sh.E;
        const float4* yl4 = reinterpret_cast<const float4*>(ysr) + gt;
        const float4* zl = reinterpret_cast<const float4*>(z) + o;
        float4 sv[NSL], zv[NSL];
#pragma unroll
        for (int u = 0; u < NSL; ++u) {  // x, ys and z at once: one memory round trip per token
            sv[u] = u < nsl ? f4_fma(dl[G * u], ld_stream(xl + G * u), __ldcg(yl4 + G * u))
                            : make_float4(0.f, 0.f, 0.f, 0.f);
            zv[u] = u < nsl ? ld_stream(zl + G * u) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        // wide rows (6+ slots per lane): the group's next token into L2 meanwhile (measured on B200:
        // 0.82 -> 0.92 of the copy rate at E = 1,536, 0.92 -> 0.93 at E = 768, but 0.935 -> 0.92 at
        // E = 384)
        const long long tn = tok + (long long)gridDim.x * NG;
        if (NSL >= 6 && tn < ntok) {
            const size_t on = (size_t)tn * SL + gt;
#pragma unroll
            for (int u = 0; u < NSL; ++u)
                if (u < nsl) {
                    prefetch_l2(reinterpret_cast<const float4*>(x) + on + G * u);
                    prefetch_l2(reinterpret_cast<const float4*>(z) + on + G * u);
                }
        }
        // shift: the token's first s value (lane 0 of the group's first warp holds it)
        const float K = WPT == 1 ? __shfl_sync(0xffffffffu, sv[0].x, 0)
                                 : fmaf(dsum[0].x, __ldcg(x + (size_t)tok * sh.E), __ldcg(ysr));
        float m1 = 0.f, m2 = 0.f;
#pragma unroll
        for (int u = 0; u < NSL; ++u)
            if (u < nsl) ln_accum(sv[u], K, m1, m2);
        float mean, rstd;
        if (WPT == 1) {
            ln_stats(m1, m2, K, invE, sh.ln_eps, mean, rstd);
        } else {
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                m1 += __shfl_xor_sync(0xffffffffu, m1, off);
                m2 += __shfl_xor_sync(0xffffffffu, m2, off);
            }
            if (lane == 0) {
                red[warp][0] = m1;
                red[warp][1] = m2;
            }
            asm volatile("bar.sync %0, %1;" : : "r"(1 + grp), "r"(G) : "memory");
            m1 = red[grp * WPT][0];
            m2 = red[grp * WPT][1];
#pragma unroll
            for (int w = 1; w < WPT; ++w) {
                m1 += red[grp * WPT + w][0];
                m2 += red[grp * WPT + w][1];
            }
            // the slots are read again only after the group's next barrier
            asm volatile("bar.sync %0, %1;" : : "r"(1 + grp), "r"(G) : "memory");
            const float d = m1 * invE;
            mean = K + d;
            rstd = rsqrtf(fmaxf(m2 * invE - d * d, 0.f) + sh.ln_eps);
        }
#pragma unroll
        for (int u = 0; u < NSL; ++u)
            if (u < nsl) st_stream(yl + G * u, ln_gate4(sv[u], zv[u], gl[G * u], bl[G * u], mean, rstd));
    }
}

// ---- Staged x_proj: one fp32 GEMM over every pooled token of the batch ---------------------------
// u[b][k][t][j] = sum_e W_x[k][j][e] * xbar[b][t][e]: C[m][n] = sum_e A[m][e] B[n][e] with M = B T
// pooled tokens, N = nd (R + 2N) outputs, K = E; both operands E-contiguous.  With the Conv1D each
// direction has its own pooled tokens: blockIdx.z picks the set, and the set's GEMM covers only its
// direction's R + 2N outputs.  A CTA of 256 threads computes a 64 x 32 tile: two groups of 128
// threads each sum half of every 32-channel operand tile (more warps to hide latency), each thread
// 4 tokens x 4 outputs (rows tg + 16 i, columns og + 8 j), so a warp's 128-bit shared loads touch 4
// A rows (broadcast) and 8 B rows (padded rows of 36 floats: conflict-free); the groups' partial
// sums meet in shared memory at the end, in a fixed order.  Operand tiles stream through a 3-stage
// cp.async pipeline.
constexpr int kPgM = 64, kPgN = 32, kPgK = 32, kPgPad = kPgK + 4, kPgStages = 3, kPgThreads = 256;
constexpr size_t kPgSmemBytes = (size_t)kPgStages * (kPgM + kPgN) * kPgPad * sizeof(float);

__global__ void __launch_bounds__(kPgThreads)
proj_gemm_kernel(Shape sh, const float* __restrict__ xbar, const float* __restrict__ W_x, float* __restrict__ u) {
    extern __shared__ __align__(16) float pg[];
    const int kz = blockIdx.z;                        // pooled-token set
    const int NZ = sh.NJ / sh.nx;                     // outputs of one set
    const int M = sh.B * sh.T, N = NZ, K = sh.E;
    const int m0 = blockIdx.x * kPgM, n0 = blockIdx.y * kPgN;
    const int tid = threadIdx.x, grp = tid >> 7, og = tid & 7, tg = (tid & 127) >> 3;
    float* As = pg;                                   // [stages][64][36]
    float* Bs = pg + kPgStages * kPgM * kPgPad;       // [stages][32][36]
    const int nk = (K + kPgK - 1) / kPgK;
    // the operand rows this thread copies: A rows ar and ar + 32, B row ar, channels k4 .. k4 + 3
    const int ar = tid >> 3, k4 = (tid & 7) * 4;
    const float* arow[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int m = m0 + ar + 32 * i;
        const int mm = m < M ? m : 0;
        const int b = mm / sh.T, t = mm - b * sh.T;
        arow[i] = m < M ? xbar + xbar_offset(sh, b, kz, t) : nullptr;
    }
    const float* brow = n0 + ar < N ? W_x + (size_t)(kz * NZ + n0 + ar) * K : nullptr;
    auto issue = [&](int kt) {
        const int st = kt % kPgStages, k0 = kt * kPgK;
        const bool kok = k0 + k4 < K;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const bool ok = arow[i] && kok;
            cp_async16(As + (st * kPgM + ar + 32 * i) * kPgPad + k4, ok ? (const void*)(arow[i] + k0 + k4)
                                                                        : (const void*)xbar, ok ? 16u : 0u);
        }
        const bool ok = brow && kok;
        cp_async16(Bs + (st * kPgN + ar) * kPgPad + k4, ok ? (const void*)(brow + k0 + k4) : (const void*)W_x,
                   ok ? 16u : 0u);
    };
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
#pragma unroll
    for (int s = 0; s < kPgStages - 1; ++s) {
        if (s < nk) issue(s);
        cp_async_commit();
    }
    for (int kt = 0; kt < nk; ++kt) {
        cp_async_wait<kPgStages - 2>();
        __syncthreads();  // tile kt landed for everyone; the stage refilled below is no longer read
        if (kt + kPgStages - 1 < nk) issue(kt + kPgStages - 1);
        cp_async_commit();
        const int st = kt % kPgStages;
        const float* a = As + st * kPgM * kPgPad;
        const float* bq = Bs + st * kPgN * kPgPad;
#pragma unroll
        for (int k = grp * (kPgK / 2); k < (grp + 1) * (kPgK / 2); k += 4) {
            float4 av[4], bv[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) av[i] = *reinterpret_cast<const float4*>(a + (tg + 16 * i) * kPgPad + k);
#pragma unroll
            for (int j = 0; j < 4; ++j) bv[j] = *reinterpret_cast<const float4*>(bq + (og + 8 * j) * kPgPad + k);
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    acc[i][j] = fmaf(av[i].w, bv[j].w,
                                     fmaf(av[i].z, bv[j].z, fmaf(av[i].y, bv[j].y, fmaf(av[i].x, bv[j].x, acc[i][j]))));
        }
    }
    cp_async_wait<0>();
    __syncthreads();  // the operand tiles are free: reuse them for the second group's partial sums
    float* part = pg;  // [128][16]
    if (grp == 1)
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) part[(tid - 128) * 16 + i * 4 + j] = acc[i][j];
    __syncthreads();
    if (grp == 1) return;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int m = m0 + tg + 16 * i;
        if (m >= M) continue;
        const int b = m / sh.T, t = m - b * sh.T;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int n = n0 + og + 8 * j;
            if (n < N) {
                const int ng = kz * NZ + n;
                const int k = ng / sh.J, jc = ng - k * sh.J;
                u[u_offset(sh, k, b, t) + jc] = acc[i][j] + part[tid * 16 + i * 4 + j];
            }
        }
    }
}

// ---- Staged scans: one CTA per (image, 128-channel tile, direction) ----------------------------
// DT_IN: Delta from dt_proj_kernel's buffer; else dt_proj + softplus per chunk in the scan.
// ckpt: NULL, or where the scans keep their states for the gradient (FV_FLAG_KEEP_STATES).
template <bool ZOH_EXACT, bool DT_IN>
__global__ void __launch_bounds__(kSeqThreads)
scan_seq_kernel(Shape sh, const float* __restrict__ u, const float* __restrict__ xbar,
                const float* __restrict__ A_log, const float* __restrict__ W_dt, const float* __restrict__ b_dt,
                const float* __restrict__ delta, float* __restrict__ ys, float* __restrict__ ckpt) {
    extern __shared__ __align__(16) float smem[];
    const int tiles = (sh.E + kSeqThreads - 1) / kSeqThreads;
    const int k = blockIdx.x % sh.nd;
    const int tile = (blockIdx.x / sh.nd) % tiles;
    const int b = blockIdx.x / (sh.nd * tiles);
    const int e0 = tile * kSeqThreads;
    seq_scan<kSeqThreads, 1, ZOH_EXACT, DT_IN>(sh, u, xbar, A_log, W_dt, b_dt, delta,
                                               ys + (size_t)b * sh.T * sh.E + e0, sh.E, b, e0, k, smem, ckpt);
}

// Device math self-test: out[i] = f(in[i]) for the SFU-based helpers the layer uses
// (0: softplus_fast, 1: silu_fast, 2: ex2_approx).
__global__ void math_selftest_kernel(int fn, const float* __restrict__ in, float* __restrict__ out, int n) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    const float v = in[i];
    out[i] = fn == 0 ? softplus_fast(v) : fn == 1 ? silu_fast(v) : ex2_approx(v);
}

}  // namespace fv
