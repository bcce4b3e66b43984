// fv_backward.cuh -- the gradient of the FastVim SSM layer (sm_100a, fp32).
//
// FastVim is trained end to end (gptget.net summary of arXiv 2502.00594, "实验结果": faster
// pre-training and fine-tuning); the pages give no backward rule, so these kernels compute the
// exact derivative of the forward definition (fv_scan.cuh, fv_kernels.cuh), by the chain rule in
// reverse step order:
//   bwd_gate_dense_kernel / bwd_gate_masked_kernel   gate, skip and repeat: dz, the skip part of
//                                                    dx, dD, and dys = the sum of ds over the
//                                                    tokens of each pooled row
//   bwd_ln_gate_kernel                               the same through the post-SSM LayerNorm,
//                                                    plus dln_gamma, dln_beta
//   bwd_scan_kernel                                  adjoint of both scans: dDelta, and through
//                                                    dt_proj + softplus d dt_low, dW_dt, db_dt; dB,
//                                                    dC, dA_log and the scans' share of dxbar
//   bwd_dwx_kernel, bwd_dxbar_kernel                 x_proj: dW_x (split-K partials), dxbar
//   bwd_pool_dense_kernel / bwd_pool_masked_kernel   pooling: dx += pool_scale / S dxbar of the
//                                                    token's row
// Inputs of the forward that the gradient reuses (xbar, the projections u, ys and, masked, the
// row lists) are read from the forward call's workspace.  The gate and pooling kernels stream the
// grid (HBM bound); the scan is SFU/issue bound; the GEMMs are small (< 1 GFLOP).
#pragma once

#include "fv_common.cuh"
#include "fv_kernels.cuh"

namespace fv {

constexpr int kBsCh = 64;        // channels per scan-gradient CTA
constexpr int kBsThreads = 256;  // 4 lanes per channel, 4 states per lane
constexpr int kBsChunk = 16;     // steps per staged chunk
constexpr int kBsHalf = 8;       // steps per checkpoint (two per staged chunk)

__host__ __device__ __forceinline__ int bs_nchunks(int T) { return (T + kBsChunk - 1) / kBsChunk; }
// checkpoints per scan: one every 8 steps of the scan order (the forward's kept-state layout)
__host__ __device__ __forceinline__ int bs_nckpt(int T) { return ckpt_count(T); }
static_assert(kBsChunk == 2 * kCkptSteps && kBsHalf == kCkptSteps, "checkpoint layout");
// dt_rank rounded up to whole float4s (the dt_low rows and the dW_dt sums are read as float4).
__host__ __device__ __forceinline__ int bs_r4(int R) { return (R + 3) & ~3; }
constexpr int kBsWS = 64 + 4;  // row stride of W_dt transposed, [r][channel]: float4-aligned rows
// one staged chunk: dt_low [16][R4] (zero past R), B | C [16][32], then xbar, dys, Delta [16][64]
__host__ __device__ __forceinline__ int bs_stage_floats(int R) {
    return kBsChunk * bs_r4(R) + kBsChunk * 32 + 3 * kBsChunk * kBsCh;
}
__host__ __device__ __forceinline__ size_t bs_smem_floats(int R) {
    return (size_t)R * kBsWS                  // W_dt of the CTA's channels, transposed
           + 2 * (size_t)bs_stage_floats(R)   // two staged chunks (copies of the next one in flight)
           + 3 * (size_t)kBsChunk * kBsCh     // sig(v), dv, dxbar (scan share) of the chunk
           + (size_t)(kBsThreads / 32) * kBsChunk * 32  // dB | dC sums of the chunk, one row per warp
           + (size_t)kBsCh * (bs_r4(R) + 4);  // dW_dt | db_dt sums of the CTA's channels
}

// sigmoid(v) = 1 / (1 + e^-v) on the SFU (v -> -inf gives 0, v -> +inf gives 1).
__device__ __forceinline__ float sigmoid_fast(float v) {
    return rcp_approx(1.f + ex2_approx(v * -1.4426950408889634f));
}

// ------------------------------------------------------------------------------------------
// Gate, skip and repeat
// ------------------------------------------------------------------------------------------

// One channel of one token.  y = SiLU(z) s, s = ys + Dsum x:
//   dz = dy s SiLU'(z),  SiLU'(z) = sig(z) (1 + z (1 - sig(z))),  ds = dy SiLU(z),
//   dx (skip part) = ds Dsum,  dD += ds x,  dys += ds.
__device__ __forceinline__ void gate_grad1(float x, float z, float g, float ys, float Ds, float& dz, float& dx,
                                           float& acc, float& dDa) {
    const float sg = sigmoid_fast(z);
    const float s = fmaf(Ds, x, ys);
    const float ds = g * z * sg;
    dz = g * s * sg * fmaf(z, 1.f - sg, 1.f);
    dx = ds * Ds;
    acc += ds;
    dDa = fmaf(ds, x, dDa);
}

__device__ __forceinline__ void gate_grad4(const float4& x, const float4& z, const float4& g, const float4& ys,
                                           const float4& Ds, float4& dz, float4& dx, float4& acc, float4& dDa) {
    gate_grad1(x.x, z.x, g.x, ys.x, Ds.x, dz.x, dx.x, acc.x, dDa.x);
    gate_grad1(x.y, z.y, g.y, ys.y, Ds.y, dz.y, dx.y, acc.y, dDa.y);
    gate_grad1(x.z, z.z, g.z, ys.z, Ds.z, dz.z, dx.z, acc.z, dDa.z);
    gate_grad1(x.w, z.w, g.w, ys.w, Ds.w, dz.w, dx.w, acc.w, dDa.w);
}

__device__ __forceinline__ float4 f4_zero() { return make_float4(0.f, 0.f, 0.f, 0.f); }

__device__ __forceinline__ float4 bwd_dsum4(const float* __restrict__ D, int nd, int SL, int slot) {
    const float4* D4 = reinterpret_cast<const float4*>(D);
    float4 dv = D4[slot];
    if (nd == 2) f4_add(dv, D4[SL + slot]);
    return dv;
}

// Slots (float4 columns) a thread block covers per pass and the token groups that share a slot:
// SL <= 256: one pass over all SL slots, 256 / SL groups; otherwise passes of 256 slots, one group.
__host__ __device__ __forceinline__ int bwd_slot_width(int SL) { return SL <= kThreads ? SL : kThreads; }
__host__ __device__ __forceinline__ int bwd_groups(int SL) { return kThreads / bwd_slot_width(SL); }

// Dense gate gradient, persistent over pooled rows (b, t) (grid-stride), launched with
// bwd_groups(SL) * bwd_slot_width(SL) threads.  Writes dz and the skip part of dx for every token
// of the row, dys[b][t] (the sum of ds over the row's S tokens), and the block's dD sums into row
// blockIdx.x of part_dD ([gridDim.x][E]; bwd_reduce_kernel adds the rows in block order).
// U tokens per thread in flight (3 U 128-bit loads).
template <int U>
__global__ void __launch_bounds__(kThreads)
bwd_gate_dense_kernel(Shape sh, const float* __restrict__ x, const float* __restrict__ z,
                      const float* __restrict__ dy, const float* __restrict__ ys, const float* __restrict__ D,
                      float* __restrict__ dx, float* __restrict__ dz, float* __restrict__ dys,
                      float* __restrict__ part_dD) {
    __shared__ float4 part[kThreads];
    const int SL = sh.SL, SW = bwd_slot_width(SL), G = bwd_groups(SL);
    const int ls = threadIdx.x % SW, g = threadIdx.x / SW;
    const int rows = sh.B * sh.T, S = sh.S;
    const size_t st4 = dense_stride(sh) >> 2;
    const float4* x4 = reinterpret_cast<const float4*>(x);
    const float4* z4 = reinterpret_cast<const float4*>(z);
    const float4* g4 = reinterpret_cast<const float4*>(dy);
    float4* dx4 = reinterpret_cast<float4*>(dx);
    float4* dz4 = reinterpret_cast<float4*>(dz);
    for (int s0 = 0; s0 < SL; s0 += SW) {
        const int slot = s0 + ls;
        const bool act = g < G && slot < SL;
        const float4 Ds = act ? bwd_dsum4(D, sh.nd, SL, slot) : f4_zero();
        float4 dDa = f4_zero();
        for (int bt = blockIdx.x; bt < rows; bt += gridDim.x) {
            const int b = bt / sh.T, t = bt - b * sh.T;
            float4 acc = f4_zero();
            if (act) {
                const size_t base = (dense_base(sh, b, t) >> 2) + slot;
                const float4 yv = reinterpret_cast<const float4*>(ys + (size_t)bt * sh.E)[slot];
                int s = g;
                for (; s + (U - 1) * G < S; s += U * G) {  // U tokens, 3 U loads in flight
                    float4 xv[U], zv[U], gv[U];
#pragma unroll
                    for (int u = 0; u < U; ++u) {
                        const size_t o = base + (size_t)(s + u * G) * st4;
                        xv[u] = ld_stream(x4 + o);
                        zv[u] = ld_stream(z4 + o);
                        gv[u] = ld_stream(g4 + o);
                    }
#pragma unroll
                    for (int u = 0; u < U; ++u) {
                        const size_t o = base + (size_t)(s + u * G) * st4;
                        float4 dzv, dxv;
                        gate_grad4(xv[u], zv[u], gv[u], yv, Ds, dzv, dxv, acc, dDa);
                        st_stream(dz4 + o, dzv);
                        st_stream(dx4 + o, dxv);
                    }
                }
                for (; s < S; s += G) {
                    const size_t o = base + (size_t)s * st4;
                    float4 dzv, dxv;
                    gate_grad4(ld_stream(x4 + o), ld_stream(z4 + o), ld_stream(g4 + o), yv, Ds, dzv, dxv, acc, dDa);
                    st_stream(dz4 + o, dzv);
                    st_stream(dx4 + o, dxv);
                }
            }
            part[threadIdx.x] = acc;
            __syncthreads();
            if (g == 0 && slot < SL) {
                float4 sum = part[ls];
                for (int q = 1; q < G; ++q) f4_add(sum, part[q * SW + ls]);
                reinterpret_cast<float4*>(dys + (size_t)bt * sh.E)[slot] = sum;
            }
            __syncthreads();
        }
        part[threadIdx.x] = dDa;
        __syncthreads();
        if (g == 0 && slot < SL) {  // this block's dD sums (the same for every direction)
            float4 sum = part[ls];
            for (int q = 1; q < G; ++q) f4_add(sum, part[q * SW + ls]);
            reinterpret_cast<float4*>(part_dD + (size_t)blockIdx.x * sh.E)[slot] = sum;
        }
        __syncthreads();
    }
}

// Masked layers: slots per pass and token groups, block = bwd_mgroups(SL) * bwd_mslot_width(SL)
// threads (<= 384): up to 384 slots in one pass (every thread busy at E = 1536; 56 registers,
// three blocks per SM), several token groups for narrow rows (SL <= 128), passes of 256 slots
// above 384.
__host__ __device__ __forceinline__ int bwd_mslot_width(int SL) { return SL <= 3 * kThreads / 2 ? SL : kThreads; }
__host__ __device__ __forceinline__ int bwd_mgroups(int SL) { return SL <= kThreads / 2 ? kThreads / SL : 1; }

// Masked gate gradient, persistent over pooled rows (b, t): the row's kept tokens come from the
// forward's row lists (row_off, row_tok); token group g takes the row's tokens g, g + G, .. (two
// in flight, six 128-bit loads).  dys of the row is the groups' sums added in group order (zero
// for a row without tokens), and the block's dD sums go to row blockIdx.x of part_dD.  Tokens
// whose id was rejected are in no row; bwd_pool_masked_kernel zeroes their dx and dz.
__global__ void __launch_bounds__(3 * kThreads / 2, 3)
bwd_gate_masked_kernel(Shape sh, const float* __restrict__ x, const float* __restrict__ z,
                       const float* __restrict__ dy, const float* __restrict__ ys, const float* __restrict__ D,
                       const int32_t* __restrict__ row_off, const int32_t* __restrict__ row_tok,
                       float* __restrict__ dx, float* __restrict__ dz, float* __restrict__ dys,
                       float* __restrict__ part_dD) {
    __shared__ float4 part[kThreads];  // the groups' sums (G > 1 only: then G SW <= 256)
    const int SL = sh.SL, K = sh.K, T = sh.T;
    const int SW = bwd_mslot_width(SL), G = bwd_mgroups(SL);
    const int ls = threadIdx.x % SW, g = threadIdx.x / SW;
    const int rows = sh.B * T;
    const float4* x4 = reinterpret_cast<const float4*>(x);
    const float4* z4 = reinterpret_cast<const float4*>(z);
    const float4* g4 = reinterpret_cast<const float4*>(dy);
    float4* dx4 = reinterpret_cast<float4*>(dx);
    float4* dz4 = reinterpret_cast<float4*>(dz);
    // the sum over the groups of v, in group order, to group 0 (G > 1; all threads take part)
    auto group_sum = [&](const float4& v) {
        part[threadIdx.x] = v;
        __syncthreads();
        float4 sum = part[ls];
        for (int q = 1; q < G; ++q) f4_add(sum, part[q * SW + ls]);
        __syncthreads();
        return sum;
    };
    for (int s0 = 0; s0 < SL; s0 += SW) {
        const int slot = s0 + ls;
        const bool act = g < G && slot < SL;
        const float4 Ds = act ? bwd_dsum4(D, sh.nd, SL, slot) : f4_zero();
        float4 dDa = f4_zero();
        for (int bt = blockIdx.x; bt < rows; bt += gridDim.x) {
            float4 acc = f4_zero();
            if (act) {
                const int b = bt / T, t = bt - b * T;
                const int p0 = row_off[(size_t)b * (T + 1) + t], p1 = row_off[(size_t)b * (T + 1) + t + 1];
                const int32_t* tok = row_tok + (size_t)b * K;
                const float4 yv = reinterpret_cast<const float4*>(ys + (size_t)bt * sh.E)[slot];
                int p = p0 + g;
                for (; p + G < p1; p += 2 * G) {  // two tokens, six loads in flight
                    const size_t o0 = ((size_t)b * K + tok[p]) * SL + slot;
                    const size_t o1 = ((size_t)b * K + tok[p + G]) * SL + slot;
                    const float4 xa = ld_stream(x4 + o0), za = ld_stream(z4 + o0), ga = ld_stream(g4 + o0);
                    const float4 xb = ld_stream(x4 + o1), zb = ld_stream(z4 + o1), gb = ld_stream(g4 + o1);
                    float4 dzv, dxv;
                    gate_grad4(xa, za, ga, yv, Ds, dzv, dxv, acc, dDa);
                    st_stream(dz4 + o0, dzv);
                    st_stream(dx4 + o0, dxv);
                    gate_grad4(xb, zb, gb, yv, Ds, dzv, dxv, acc, dDa);
                    st_stream(dz4 + o1, dzv);
                    st_stream(dx4 + o1, dxv);
                }
                if (p < p1) {
                    const size_t o = ((size_t)b * K + tok[p]) * SL + slot;
                    float4 dzv, dxv;
                    gate_grad4(ld_stream(x4 + o), ld_stream(z4 + o), ld_stream(g4 + o), yv, Ds, dzv, dxv, acc, dDa);
                    st_stream(dz4 + o, dzv);
                    st_stream(dx4 + o, dxv);
                }
            }
            if (G > 1) acc = group_sum(acc);
            if (g == 0 && slot < SL) reinterpret_cast<float4*>(dys + (size_t)bt * sh.E)[slot] = acc;
        }
        if (G > 1) dDa = group_sum(dDa);
        if (g == 0 && slot < SL)  // this block's sums
            reinterpret_cast<float4*>(part_dD + (size_t)blockIdx.x * sh.E)[slot] = dDa;
    }
}

// ------------------------------------------------------------------------------------------
// Gate, skip and repeat through the post-SSM LayerNorm
// ------------------------------------------------------------------------------------------

// Warps per block of the LayerNorm gate gradient: as many (up to 4) as keep its shared memory
// ((3 + 4 W) E floats) within about 100 KB.
__host__ __forceinline__ int bwd_ln_warps(int SL) {
    for (int w = 4; w > 1; w >>= 1)
        if ((size_t)(3 + 4 * w) * SL * sizeof(float4) <= (size_t)100 * 1024) return w;
    return 1;
}
__host__ __forceinline__ size_t bwd_ln_smem_bytes(int SL, int warps) {
    return (size_t)(3 + 4 * warps) * SL * sizeof(float4);
}

// Persistent over pooled rows (b, t) (grid-stride); the block's warps take the row's tokens in
// turn, one token per warp at a time.  Per token, with s = ys[t] + (sum_k D[k]) x over its E
// channels, sh = (s - mean) rstd, n = gamma sh + beta, y = SiLU(z) n:
//   dz = dy n SiLU'(z);  dn = dy SiLU(z);  gs = dn gamma;
//   ds = rstd (gs - mean(gs) - sh mean(gs sh));  dx (skip part) = ds sum_k D[k];
//   dys[t] += ds;  dgamma += dn sh;  dbeta += dn;  dD += ds x.
// Three passes over the token's channels: the statistics of s, the two means of gs, the outputs;
// the first pass reads x and the second z and dy from HBM, the repeats hit L1.  Every lane owns
// the same float4 slots in every pass, so each warp sums dys, dgamma, dbeta and dD into private
// shared-memory rows with no atomics; the rows meet, in warp order, at the end of each pooled row
// (dys) and of the kernel (the block's batch sums: row blockIdx.x of part_ln, [gridDim.x][3][E] =
// dgamma | dbeta | dD, added in block order by bwd_reduce_kernel).  Masked layers take a row's kept
// tokens from the forward's row lists; a rejected id is in no row (dx, dz zeroed by
// bwd_pool_masked_kernel).
template <bool MASKED>
__global__ void __launch_bounds__(128)
bwd_ln_gate_kernel(Shape sh, const float* __restrict__ x, const float* __restrict__ z, const float* __restrict__ dy,
                   const float* __restrict__ ys, const float* __restrict__ D, const float* __restrict__ gamma,
                   const float* __restrict__ beta, const int32_t* __restrict__ row_off,
                   const int32_t* __restrict__ row_tok, float* __restrict__ dx, float* __restrict__ dz,
                   float* __restrict__ dys, float* __restrict__ part_ln) {
    extern __shared__ float4 lgs[];
    const int SL = sh.SL, W = blockDim.x >> 5;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float4* dsum = lgs;
    float4* g4 = dsum + SL;
    float4* be4 = g4 + SL;
    float4* prow = be4 + SL;  // [W][4][SL]: dys, dgamma, dbeta, dD of each warp
    float4* pdys = prow + (size_t)warp * 4 * SL;
    float4* pdg = pdys + SL;
    float4* pdb = pdg + SL;
    float4* pdD = pdb + SL;
    for (int slot = threadIdx.x; slot < SL; slot += blockDim.x) {
        dsum[slot] = bwd_dsum4(D, sh.nd, SL, slot);
        g4[slot] = __ldg(reinterpret_cast<const float4*>(gamma) + slot);
        be4[slot] = __ldg(reinterpret_cast<const float4*>(beta) + slot);
    }
    for (int i = threadIdx.x; i < 4 * W * SL; i += blockDim.x) prow[i] = f4_zero();
    __syncthreads();
    const int T = sh.T, K = sh.K;
    const int rows = sh.B * T;
    const size_t st4 = dense_stride(sh) >> 2;
    const float invE = 1.f / (float)sh.E, eps = sh.ln_eps;
    const float4* x4 = reinterpret_cast<const float4*>(x);
    const float4* z4 = reinterpret_cast<const float4*>(z);
    const float4* gy4 = reinterpret_cast<const float4*>(dy);
    float4* dx4 = reinterpret_cast<float4*>(dx);
    float4* dz4 = reinterpret_cast<float4*>(dz);
    for (int bt = blockIdx.x; bt < rows; bt += gridDim.x) {
        const int b = bt / T, t = bt - b * T;
        int p0 = 0, ntok = sh.S;
        if (MASKED) {
            p0 = row_off[(size_t)b * (T + 1) + t];
            ntok = row_off[(size_t)b * (T + 1) + t + 1] - p0;
        }
        const float4* ys4 = reinterpret_cast<const float4*>(ys + (size_t)bt * sh.E);
        for (int i = warp; i < ntok; i += W) {
            const size_t o = MASKED ? ((size_t)b * K + row_tok[(size_t)b * K + p0 + i]) * SL
                                    : (dense_base(sh, b, t) >> 2) + (size_t)i * st4;
            // statistics of s (moments shifted by the token's first s value, the same in every lane)
            const float Ks = fmaf(dsum[0].x, __ldg(x + o * 4), __ldg(ys + (size_t)bt * sh.E));
            float m1 = 0.f, m2 = 0.f;
#pragma unroll 4
            for (int slot = lane; slot < SL; slot += 32)
                ln_accum(f4_fma(dsum[slot], __ldg(x4 + o + slot), ys4[slot]), Ks, m1, m2);
            float mean, rstd;
            ln_stats(m1, m2, Ks, invE, eps, mean, rstd);
            // the two means of gs = dy SiLU(z) gamma
            float a1 = 0.f, a2 = 0.f;
#pragma unroll 4
            for (int slot = lane; slot < SL; slot += 32) {
                const float4 sv = f4_fma(dsum[slot], __ldg(x4 + o + slot), ys4[slot]);
                const float4 zv = __ldg(z4 + o + slot), gv = __ldg(gy4 + o + slot), gm = g4[slot];
                const float sa[4] = {sv.x, sv.y, sv.z, sv.w}, za[4] = {zv.x, zv.y, zv.z, zv.w};
                const float ga[4] = {gv.x, gv.y, gv.z, gv.w}, gma[4] = {gm.x, gm.y, gm.z, gm.w};
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const float shv = (sa[c] - mean) * rstd;
                    const float gs = ga[c] * za[c] * sigmoid_fast(za[c]) * gma[c];
                    a1 += gs;
                    a2 = fmaf(gs, shv, a2);
                }
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                a1 += __shfl_xor_sync(0xffffffffu, a1, off);
                a2 += __shfl_xor_sync(0xffffffffu, a2, off);
            }
            const float mgs = a1 * invE, mgss = a2 * invE;
            // outputs
#pragma unroll 2
            for (int slot = lane; slot < SL; slot += 32) {
                const float4 xv = __ldg(x4 + o + slot), zv = __ldg(z4 + o + slot), gv = __ldg(gy4 + o + slot);
                const float4 ds4 = dsum[slot], gm = g4[slot], bm = be4[slot];
                const float4 sv = f4_fma(ds4, xv, ys4[slot]);
                const float sa[4] = {sv.x, sv.y, sv.z, sv.w}, za[4] = {zv.x, zv.y, zv.z, zv.w};
                const float ga[4] = {gv.x, gv.y, gv.z, gv.w}, xa[4] = {xv.x, xv.y, xv.z, xv.w};
                const float gma[4] = {gm.x, gm.y, gm.z, gm.w}, bma[4] = {bm.x, bm.y, bm.z, bm.w};
                const float dsa[4] = {ds4.x, ds4.y, ds4.z, ds4.w};
                float dzo[4], dxo[4], dso[4], dno[4], sho[4];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const float shv = (sa[c] - mean) * rstd;
                    const float sg = sigmoid_fast(za[c]);
                    const float dn = ga[c] * za[c] * sg;
                    const float n = fmaf(gma[c], shv, bma[c]);
                    dzo[c] = ga[c] * n * sg * fmaf(za[c], 1.f - sg, 1.f);
                    const float ds = (fmaf(dn, gma[c], -mgs) - shv * mgss) * rstd;
                    dxo[c] = ds * dsa[c];
                    dso[c] = ds;
                    dno[c] = dn;
                    sho[c] = shv;
                }
                st_stream(dz4 + o + slot, make_float4(dzo[0], dzo[1], dzo[2], dzo[3]));
                st_stream(dx4 + o + slot, make_float4(dxo[0], dxo[1], dxo[2], dxo[3]));
                f4_add(pdys[slot], make_float4(dso[0], dso[1], dso[2], dso[3]));
                f4_add(pdg[slot], make_float4(dno[0] * sho[0], dno[1] * sho[1], dno[2] * sho[2], dno[3] * sho[3]));
                f4_add(pdb[slot], make_float4(dno[0], dno[1], dno[2], dno[3]));
                f4_add(pdD[slot], make_float4(dso[0] * xa[0], dso[1] * xa[1], dso[2] * xa[2], dso[3] * xa[3]));
            }
        }
        __syncthreads();
        for (int slot = threadIdx.x; slot < SL; slot += blockDim.x) {
            float4 acc = f4_zero();
            for (int w = 0; w < W; ++w) {
                float4* r = prow + (size_t)w * 4 * SL + slot;
                f4_add(acc, *r);
                *r = f4_zero();
            }
            reinterpret_cast<float4*>(dys)[(size_t)bt * SL + slot] = acc;
        }
        __syncthreads();
    }
    for (int slot = threadIdx.x; slot < SL; slot += blockDim.x) {
        float4 sg = f4_zero(), sb = f4_zero(), sd = f4_zero();
        for (int w = 0; w < W; ++w) {
            const float4* r = prow + (size_t)w * 4 * SL;
            f4_add(sg, r[SL + slot]);
            f4_add(sb, r[2 * SL + slot]);
            f4_add(sd, r[3 * SL + slot]);
        }
        float4* row = reinterpret_cast<float4*>(part_ln + (size_t)blockIdx.x * 3 * sh.E);
        row[slot] = sg;
        row[SL + slot] = sb;
        row[2 * SL + slot] = sd;
    }
}

// The same gradient with each token's values in registers.  A group of WPT warps takes one token
// (thread gt of the group owns float4 slots gt + 32 WPT u, u < U: E <= 128 U WPT); a
// block of NG groups is persistent over pooled rows, its groups taking the row's tokens in turn.
// Per token: x, z and dy are loaded at once (one memory round trip), and the group's next token
// is prefetched into L2 meanwhile, so that its loads hit L2 (measured on B200: 0.71 -> 0.82 of the
// copy rate at E = 384, 0.66 -> 0.75 at E = 768 against a shared-memory double buffer of the next
// token, 0.56 -> 0.65 at E = 1,536; prefetching two tokens ahead measured slower); pass 1 forms s
// and its shifted moments, pass 2 the two means of gs, pass 3 writes dz, dx from the registers.  The group's sums (moments, means) go
// through a shared-memory slot per warp, added in warp order behind a named barrier of the group.
// dys of the current row and the batch sums of dgamma, dbeta, dD stay in each thread's registers;
// the groups' dys meet in shared memory at the end of each row, the batch sums at the end of the
// kernel (row blockIdx.x of part_ln, in group order).  No per-warp shared rows: occupancy is set
// by registers, and the group spans any E up to U x 32 x WPT x 4 channels.  U = 1 (three blocks
// per SM) for 513-1,024 channels, U = 2 (128 registers, two blocks) otherwise: measured on B200
// before the double buffer, E = 768 streamed at 0.60 of the copy rate with U = 1 against 0.53 with
// U = 2, E = 384 at 0.68 with U = 2 against 0.65 with U = 1.
__host__ __device__ __forceinline__ int bwd_lnr_nsl(int SL) { return (SL > 128 && SL <= 256) ? 1 : 2; }
__host__ __device__ __forceinline__ int bwd_lnr_wpt(int SL) {
    const int u = bwd_lnr_nsl(SL);
    return (SL + 32 * u - 1) / (32 * u);
}
// groups per block: about 8 warps, at most 15 (named barrier ids 1..15)
__host__ __device__ __forceinline__ int bwd_lnr_groups(int SL) {
    const int w = bwd_lnr_wpt(SL);
    const int ng = w >= 8 ? 1 : 8 / w;
    return ng > 15 ? 15 : ng;
}
__host__ __device__ __forceinline__ size_t bwd_lnr_smem_bytes(int SL) {
    const int ng = bwd_lnr_groups(SL), wpt = bwd_lnr_wpt(SL);
    return (size_t)(3 + ng) * SL * sizeof(float4)                // sum D, gamma, beta; the groups' rows
           + (size_t)ng * wpt * 4 * sizeof(float);               // the warps' partial sums
}
__device__ __forceinline__ void group_bar(int id, int threads) {
    asm volatile("bar.sync %0, %1;" : : "r"(id), "r"(threads) : "memory");
}

template <int U, bool MASKED>
__global__ void __launch_bounds__(256, U == 1 ? 3 : 2)
bwd_ln_gate_reg_kernel(Shape sh, const float* __restrict__ x, const float* __restrict__ z,
                       const float* __restrict__ dy, const float* __restrict__ ys, const float* __restrict__ D,
                       const float* __restrict__ gamma, const float* __restrict__ beta,
                       const int32_t* __restrict__ row_off, const int32_t* __restrict__ row_tok,
                       float* __restrict__ dx, float* __restrict__ dz, float* __restrict__ dys,
                       float* __restrict__ part_ln) {
    extern __shared__ float4 lrs[];
    const int SL = sh.SL, WPT = bwd_lnr_wpt(SL), NG = bwd_lnr_groups(SL), G = 32 * WPT;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int grp = warp / WPT, wig = warp - grp * WPT, gt = wig * 32 + lane;
    float4* dsum = lrs;
    float4* g4 = dsum + SL;
    float4* be4 = g4 + SL;
    float4* rows = be4 + SL;                                    // [NG][SL]
    float* red = reinterpret_cast<float*>(rows + (size_t)NG * SL) + (size_t)grp * WPT * 4;  // [WPT][4]
    for (int slot = threadIdx.x; slot < SL; slot += blockDim.x) {
        dsum[slot] = bwd_dsum4(D, sh.nd, SL, slot);
        g4[slot] = __ldg(reinterpret_cast<const float4*>(gamma) + slot);
        be4[slot] = __ldg(reinterpret_cast<const float4*>(beta) + slot);
    }
    __syncthreads();
    const bool live = grp < NG;  // warps past the last whole group only help with the row sums
    const int T = sh.T, K = sh.K, rows_n = sh.B * T;
    const size_t st4 = dense_stride(sh) >> 2;
    const float invE = 1.f / (float)sh.E, eps = sh.ln_eps;
    const float4* x4 = reinterpret_cast<const float4*>(x);
    const float4* z4 = reinterpret_cast<const float4*>(z);
    const float4* gy4 = reinterpret_cast<const float4*>(dy);
    float4* dx4 = reinterpret_cast<float4*>(dx);
    float4* dz4 = reinterpret_cast<float4*>(dz);
    bool own[U];
    float4 acc_g[U], acc_b[U], acc_d[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
        own[u] = live && gt + G * u < SL;
        acc_g[u] = acc_b[u] = acc_d[u] = f4_zero();
    }
    // sum D, gamma, beta of the thread's slots, from shared memory
    auto ds4 = [&](int u) { return own[u] ? dsum[gt + G * u] : f4_zero(); };
    auto gm = [&](int u) { return own[u] ? g4[gt + G * u] : f4_zero(); };
    auto bm = [&](int u) { return own[u] ? be4[gt + G * u] : f4_zero(); };
    // the group's sum of (a, b) over its WPT warps, in warp order; `phase` picks one of two slots
    auto group_sum2 = [&](float& a, float& b, int phase) {
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            a += __shfl_xor_sync(0xffffffffu, a, off);
            b += __shfl_xor_sync(0xffffffffu, b, off);
        }
        if (WPT == 1) return;
        if (lane == 0) {
            red[wig * 4 + 2 * phase] = a;
            red[wig * 4 + 2 * phase + 1] = b;
        }
        group_bar(1 + grp, G);
        a = red[2 * phase];
        b = red[2 * phase + 1];
        for (int w = 1; w < WPT; ++w) {
            a += red[w * 4 + 2 * phase];
            b += red[w * 4 + 2 * phase + 1];
        }
    };
    for (int bt = blockIdx.x; bt < rows_n; bt += gridDim.x) {
        const int b = bt / T, t = bt - b * T;
        int p0 = 0, ntok = sh.S;
        if (MASKED) {
            p0 = row_off[(size_t)b * (T + 1) + t];
            ntok = row_off[(size_t)b * (T + 1) + t + 1] - p0;
        }
        const float4* ys4 = reinterpret_cast<const float4*>(ys + (size_t)bt * sh.E);
        float4 yv[U], acc_y[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            yv[u] = own[u] ? ys4[gt + G * u] : f4_zero();
            acc_y[u] = f4_zero();
        }
        const float y0 = __ldg(ys + (size_t)bt * sh.E);
        // token i of the row: its float4 offset
        auto tok_off = [&](int i) -> size_t {
            return MASKED ? ((size_t)b * K + row_tok[(size_t)b * K + p0 + i]) * SL
                          : (dense_base(sh, b, t) >> 2) + (size_t)i * st4;
        };
        for (int i = grp; live && i < ntok; i += NG) {
            const size_t o = tok_off(i);
            // every load of the token at once (one memory round trip per token)
            float4 xv[U], zv[U], gv[U], sv[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                xv[u] = own[u] ? ld_stream(x4 + o + gt + G * u) : f4_zero();
                zv[u] = own[u] ? ld_stream(z4 + o + gt + G * u) : f4_zero();
                gv[u] = own[u] ? ld_stream(gy4 + o + gt + G * u) : f4_zero();
            }
            const float x0 = __ldg(x + o * 4);  // x of the token's first channel (the shift of its moments)
            if (i + NG < ntok) {  // the group's next token: into L2 while this one is processed
                const size_t on = tok_off(i + NG);
#pragma unroll
                for (int u = 0; u < U; ++u)
                    if (own[u]) {
                        prefetch_l2(x4 + on + gt + G * u);
                        prefetch_l2(z4 + on + gt + G * u);
                        prefetch_l2(gy4 + on + gt + G * u);
                    }
            }
            // pass 1: s and its moments about the token's first s value (the same in every thread)
            const float Ks = fmaf(dsum[0].x, x0, y0);
            float m1 = 0.f, m2 = 0.f;
#pragma unroll
            for (int u = 0; u < U; ++u) {
                sv[u] = f4_fma(ds4(u), xv[u], yv[u]);
                if (own[u]) ln_accum(sv[u], Ks, m1, m2);
            }
            group_sum2(m1, m2, 0);
            const float d = m1 * invE;
            const float mean = Ks + d;
            const float rstd = rsqrtf(fmaxf(m2 * invE - d * d, 0.f) + eps);
            // pass 2: the two means of gs = dy SiLU(z) gamma
            float a1 = 0.f, a2 = 0.f;
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const float sa[4] = {sv[u].x, sv[u].y, sv[u].z, sv[u].w}, za[4] = {zv[u].x, zv[u].y, zv[u].z, zv[u].w};
                const float ga[4] = {gv[u].x, gv[u].y, gv[u].z, gv[u].w};
                const float4 g = gm(u);
                const float gma[4] = {g.x, g.y, g.z, g.w};
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const float shv = (sa[c] - mean) * rstd;
                    const float gs = ga[c] * za[c] * sigmoid_fast(za[c]) * gma[c];
                    a1 += gs;
                    a2 = fmaf(gs, shv, a2);
                }
            }
            group_sum2(a1, a2, 1);
            const float mgs = a1 * invE, mgss = a2 * invE;
            // pass 3: the outputs, from registers
#pragma unroll
            for (int u = 0; u < U; ++u) {
                if (!own[u]) continue;
                const int slot = gt + G * u;
                const float sa[4] = {sv[u].x, sv[u].y, sv[u].z, sv[u].w}, za[4] = {zv[u].x, zv[u].y, zv[u].z, zv[u].w};
                const float ga[4] = {gv[u].x, gv[u].y, gv[u].z, gv[u].w}, xa[4] = {xv[u].x, xv[u].y, xv[u].z, xv[u].w};
                const float4 g = gm(u), be = bm(u), dd = ds4(u);
                const float gma[4] = {g.x, g.y, g.z, g.w}, bma[4] = {be.x, be.y, be.z, be.w};
                const float dsa[4] = {dd.x, dd.y, dd.z, dd.w};
                float dzo[4], dxo[4], dso[4], dno[4], sho[4];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const float shv = (sa[c] - mean) * rstd;
                    const float sg = sigmoid_fast(za[c]);
                    const float dn = ga[c] * za[c] * sg;
                    const float n = fmaf(gma[c], shv, bma[c]);
                    dzo[c] = ga[c] * n * sg * fmaf(za[c], 1.f - sg, 1.f);
                    const float ds = (fmaf(dn, gma[c], -mgs) - shv * mgss) * rstd;
                    dxo[c] = ds * dsa[c];
                    dso[c] = ds;
                    dno[c] = dn;
                    sho[c] = shv;
                }
                st_stream(dz4 + o + slot, make_float4(dzo[0], dzo[1], dzo[2], dzo[3]));
                st_stream(dx4 + o + slot, make_float4(dxo[0], dxo[1], dxo[2], dxo[3]));
                f4_add(acc_y[u], make_float4(dso[0], dso[1], dso[2], dso[3]));
                f4_add(acc_g[u], make_float4(dno[0] * sho[0], dno[1] * sho[1], dno[2] * sho[2], dno[3] * sho[3]));
                f4_add(acc_b[u], make_float4(dno[0], dno[1], dno[2], dno[3]));
                f4_add(acc_d[u], make_float4(dso[0] * xa[0], dso[1] * xa[1], dso[2] * xa[2], dso[3] * xa[3]));
            }
        }
        // dys of the row: the groups' sums, added in group order
#pragma unroll
        for (int u = 0; u < U; ++u)
            if (own[u]) rows[(size_t)grp * SL + gt + G * u] = acc_y[u];
        __syncthreads();
        for (int slot = threadIdx.x; slot < SL; slot += blockDim.x) {
            float4 acc = rows[slot];
            for (int q = 1; q < NG; ++q) f4_add(acc, rows[(size_t)q * SL + slot]);
            reinterpret_cast<float4*>(dys)[(size_t)bt * SL + slot] = acc;
        }
        __syncthreads();
    }
    // the block's batch sums, dgamma | dbeta | dD, each added over the groups in group order
    float4* out = reinterpret_cast<float4*>(part_ln + (size_t)blockIdx.x * 3 * sh.E);
#pragma unroll
    for (int which = 0; which < 3; ++which) {
#pragma unroll
        for (int u = 0; u < U; ++u)
            if (own[u]) rows[(size_t)grp * SL + gt + G * u] = which == 0 ? acc_g[u] : which == 1 ? acc_b[u] : acc_d[u];
        __syncthreads();
        for (int slot = threadIdx.x; slot < SL; slot += blockDim.x) {
            float4 acc = rows[slot];
            for (int q = 1; q < NG; ++q) f4_add(acc, rows[(size_t)q * SL + slot]);
            out[(size_t)which * SL + slot] = acc;
        }
        __syncthreads();
    }
}

// ------------------------------------------------------------------------------------------
// Adjoint of the scans
// ------------------------------------------------------------------------------------------

// Grid (B, nd, ceil(E / 64)), 256 threads: thread (channel c = tid / 4, lane q = tid % 4) holds
// states n = 4q .. 4q + 3 of channel e0 + c.  For direction slot k with scan order t_0, t_1, ...
// (forward t = 0..T-1, backward t = T-1..0), h_{-1} = 0:
//   forward   h_i = Abar_i h_{i-1} + q_i,  Abar_i = exp(Delta_i A),  q_i = Delta_i B_i xbar_i (Euler)
//             or (Abar_i - 1) / A B_i xbar_i (exact ZOH);  ys += C_i . h_i
//   adjoint   lam_i = C_i dys_i + Abar_{i+1} lam_{i+1}  (lam = 0 past the last step)
//             dC_i += dys_i h_i;  dAbar_i = lam_i h_{i-1};  dq_i = lam_i
// Delta comes from a buffer: the forward's (staged path, dt_rank >= 32) or the one the gradient call
// fills first with dt_proj_kernel; sig(v) = softplus'(v) = 1 - e^-Delta.
// Pass 1 runs the recurrence in scan order and stores the state entering every 8 steps
// (ckpt [B][nd][2 nchunks][E][16]); with FV_FLAG_KEEP_STATES the forward stored them (ckpt is
// then its buffer) and pass 1 is skipped.  Pass 2 walks the 16-step staged chunks in reverse, each as two
// halves of 8 steps, last half first: it recomputes the half's states from its checkpoint (8 steps
// x 4 states in registers, which keeps the kernel at two resident blocks per SM) and steps the
// adjoint back through them.  Per step: dDelta and the scans' dxbar are summed over the 4 lanes of
// a channel (written as dv = dDelta sig(v) and dxs [B][nd][T][E]); dB and dC are summed over the
// warp's 8 channels by a transposing butterfly, then over the block's 8 warps (one shared row per
// warp, added in warp order).  dA_log (= dA A) sums in registers over all steps.  dt_proj
// (v = W_dt dt_low + b_dt) is differentiated here too, from the chunk's dv and dt_low already in
// shared memory: d dt_low[t] = sum over the block's channels of W_dt[e] dv[t][e], dW_dt[e] and
// db_dt[e] = sums over the steps of dv[t][e] [dt_low[t] | 1].  No atomics: the block's du terms go
// to its own copy of du's layout in part_du (one per 64-channel tile) and its parameter terms to
// per-image slots; bwd_reduce_kernel adds tiles and images in a fixed order, so the sums are the
// same in every run.
template <bool ZOH_EXACT>
__global__ void __launch_bounds__(kBsThreads, 2)
bwd_scan_kernel(Shape sh, const float* __restrict__ u, const float* __restrict__ xbar, const float* __restrict__ dys,
                const float* __restrict__ A_log, const float* __restrict__ W_dt, const float* __restrict__ delta,
                float* __restrict__ ckpt, float* __restrict__ dxs, float* __restrict__ part_du,
                float* __restrict__ part_dA, float* __restrict__ part_wdt, float* __restrict__ part_bdt) {
    extern __shared__ float bsm[];
    const int b = blockIdx.x, k = blockIdx.y, e0 = blockIdx.z * kBsCh;
    const int T = sh.T, E = sh.E, N = sh.N, R = sh.R, J = sh.J;
    const int R4 = bs_r4(R), WA = R4 + 4;   // dt_low row stride; dW_dt | db_dt row stride
    float* swT = bsm;                         // [R][kBsWS]: W_dt transposed
    float* sstage = swT + R * kBsWS;          // [2] staged chunks, bs_stage_floats(R) each
    float* ssg = sstage + 2 * bs_stage_floats(R);  // [16][64]
    float* sdv = ssg + kBsChunk * kBsCh;      // [16][64]
    float* sdx = sdv + kBsChunk * kBsCh;      // [16][64]
    float* sred = sdx + kBsChunk * kBsCh;     // [8 warps][16][32]
    float* swacc = sred + (kBsThreads / 32) * kBsChunk * 32;  // [64][WA]: dW_dt row (R4) | db_dt
    const int tid = threadIdx.x;
    const int c = tid >> 2, q = tid & 3, lane = tid & 31;
    const int e = e0 + c;
    const bool live = e < E;
    const bool fwd = sh.nd == 2 ? k == 0 : (sh.dir_flags & 1u) != 0;
    const int nchunks = bs_nchunks(T);
    const float* ub = u + u_offset(sh, k, b, 0);
    // this CTA's share of du (dB, dC and d dt_low summed over its 64 channels): part_du holds one
    // copy of du's layout per 64-channel tile
    float* pdu = part_du + (size_t)blockIdx.z * sh.nd * sh.B * u_block_stride(T, J);
    auto ckpt_at = [&](int c) { return ckpt + ckpt_offset(sh, b, k, c, e) + 4 * q; };

    for (int i = tid; i < kBsCh * R; i += kBsThreads) {
        const int row = i / R, r = i - row * R;
        swT[r * kBsWS + row] = (e0 + row < E) ? __ldg(W_dt + ((size_t)k * E + e0 + row) * R + r) : 0.f;
    }
    for (int i = tid; i < kBsCh * WA; i += kBsThreads) swacc[i] = 0.f;

    constexpr float kLog2e = 1.4426950408889634f;
    float A2[4], An[4], Ainv[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int n = 4 * q + j;
        const float A = (live && n < N) ? -expf(__ldg(A_log + ((size_t)k * E + e) * N + n)) : 0.f;
        An[j] = A;
        A2[j] = A * kLog2e;
        Ainv[j] = A != 0.f ? 1.f / A : 0.f;
    }

    // chunk `it` in scan order: first pooled token and length; slot i <-> step t_of(i)
    auto chunk_t0 = [&](int it) { return (fwd ? it : nchunks - 1 - it) * kBsChunk; };
    auto chunk_len = [&](int it) { return min(kBsChunk, T - chunk_t0(it)); };
    auto t_of = [&](int it, int i) { return fwd ? chunk_t0(it) + i : chunk_t0(it) + chunk_len(it) - 1 - i; };

    // The chunks in the order they are used: pass 1 takes chunks 0 .. n-1 (scan order), pass 2
    // n-1 .. 0; stage number si <-> chunk si (pass 1) or 2n-1-si (pass 2).  stage(si) queues the
    // copies of the chunk's per-step inputs into buffer si & 1 (slots past the chunk and channels
    // past E read as zero): B | C, xbar and Delta (written by the forward's or this call's dt_proj
    // kernel), and in pass 2 dt_low and dys.  The next stage's copies run during a stage's steps.
    const int nstages = 2 * nchunks;
    auto chunk_of = [&](int si) { return si < nchunks ? si : nstages - 1 - si; };
    auto stage = [&](int si) {
        const int it = chunk_of(si), len = chunk_len(it);
        float* sb = sstage + (si & 1) * bs_stage_floats(R);
        float* dtl = sb;
        float* bc = dtl + kBsChunk * R4;
        float* rows = bc + kBsChunk * 32;  // xbar | dys | Delta
        if (si >= nchunks)
            for (int i = tid; i < kBsChunk * R4; i += kBsThreads) {
                const int s = i / R4, r = i - s * R4;
                const bool ok = s < len && r < R;
                cp_async4z(dtl + i, ok ? ub + (size_t)t_of(it, s) * J + r : ub, ok);
            }
        for (int i = tid; i < kBsChunk * 32; i += kBsThreads) {
            const int s = i >> 5, j = i & 31, n = j & 15;
            const bool ok = s < len && n < N;
            cp_async4z(bc + i, ok ? ub + (size_t)t_of(it, s) * J + R + (j < 16 ? n : N + n) : ub, ok);
        }
        for (int i = tid; i < 3 * kBsChunk * (kBsCh / 4); i += kBsThreads) {
            const int which = i / (kBsChunk * (kBsCh / 4)), v = i - which * (kBsChunk * (kBsCh / 4));
            const int s = v / (kBsCh / 4), c4 = 4 * (v - s * (kBsCh / 4));
            if (which == 1 && si < nchunks) continue;  // dys: pass 2 only
            const bool ok = s < len && e0 + c4 < E;
            const int t = ok ? t_of(it, s) : 0;
            const float* src = which == 0 ? xbar + ((size_t)b * T + t) * E
                               : which == 1 ? dys + ((size_t)b * T + t) * E
                                            : delta + delta_offset(sh, k, b, t);
            cp_async16(rows + (which * kBsChunk + s) * kBsCh + c4, ok ? (const void*)(src + e0 + c4) : (const void*)ub,
                       ok ? 16u : 0u);
        }
        cp_async_commit();
    };
    // wait for stage si's copies (the next stage's stay in flight) and return its buffer
    auto arrive = [&](int si) {
        if (si + 1 < nstages) {
            stage(si + 1);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        return sstage + (si & 1) * bs_stage_floats(R);
    };

    // the input term of one step and state
    auto qterm = [&](float dt, float Bn, float xv, int j) {
        return ZOH_EXACT ? expm1f(dt * An[j]) * Ainv[j] * Bn * xv : dt * Bn * xv;
    };

    // ---- pass 1: states entering each chunk (skipped when the forward kept them) ----
    stage(sh.keep ? nchunks : 0);
    float h[4] = {0.f, 0.f, 0.f, 0.f};
    for (int it = 0; it < (sh.keep ? 0 : nchunks); ++it) {
        const float* sb = arrive(it);
        const float* sbc = sb + kBsChunk * R4;
        const float* sx = sbc + kBsChunk * 32;
        const float* sdl = sx + 2 * kBsChunk * kBsCh;
        const int len = chunk_len(it);
        for (int i = 0; i < len; ++i) {
            if (live && (i == 0 || i == kBsHalf))
                *reinterpret_cast<float4*>(ckpt_at(2 * it + i / kBsHalf)) = make_float4(h[0], h[1], h[2], h[3]);
            const float dt = sdl[i * kBsCh + c], xv = sx[i * kBsCh + c];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float Bn = sbc[i * 32 + 4 * q + j];
                h[j] = fmaf(ex2_approx(dt * A2[j]), h[j], qterm(dt, Bn, xv, j));
            }
        }
        __syncthreads();  // the buffer is refilled by the stage after next
    }

    // ---- pass 2: the adjoint, chunks in reverse scan order ----
    float lam[4] = {0.f, 0.f, 0.f, 0.f}, Anext[4] = {0.f, 0.f, 0.f, 0.f}, gA[4] = {0.f, 0.f, 0.f, 0.f};
    const bool b2 = lane & 4, b3 = lane & 8, b4 = lane & 16;
    const int v_idx = (b2 ? 1 : 0) + (b3 ? 2 : 0) + (b4 ? 4 : 0);  // value this lane ends up holding
    const int red_n = 4 * q + (v_idx & 3), red_w = v_idx >> 2;       // state, and 0 = dB / 1 = dC
    for (int it = nchunks - 1; it >= 0; --it) {
        const float* sdtl = arrive(nstages - 1 - it);
        const float* sbc = sdtl + kBsChunk * R4;
        const float* sx = sbc + kBsChunk * 32;
        const float* sdy = sx + kBsChunk * kBsCh;
        const float* sdl = sdy + kBsChunk * kBsCh;
        const int len = chunk_len(it);
        // softplus'(v) = sigmoid(v) = 1 - e^-Delta (as -expm1, exact for small Delta) of the steps
        // whose dv this thread writes (steps i = q mod 4 of its channel): no barrier needed
        for (int i = q; i < len; i += 4) ssg[i * kBsCh + c] = -expm1f(-sdl[i * kBsCh + c]);
        for (int half = (len - 1) / kBsHalf; half >= 0; --half) {
            const int i0 = half * kBsHalf, hl = min(kBsHalf, len - i0);
            float hin[4] = {0.f, 0.f, 0.f, 0.f};
            if (live) {
                const float4 v = *reinterpret_cast<const float4*>(ckpt_at(2 * it + half));
                hin[0] = v.x; hin[1] = v.y; hin[2] = v.z; hin[3] = v.w;
            }
            float hist[kBsHalf][4];
            {
                float hc[4] = {hin[0], hin[1], hin[2], hin[3]};
#pragma unroll
                for (int ii = 0; ii < kBsHalf; ++ii) {
                    const int i = i0 + ii;
                    if (ii < hl) {
                        const float dt = sdl[i * kBsCh + c], xv = sx[i * kBsCh + c];
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const float Bn = sbc[i * 32 + 4 * q + j];
                            hc[j] = fmaf(ex2_approx(dt * A2[j]), hc[j], qterm(dt, Bn, xv, j));
                            hist[ii][j] = hc[j];
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < 4; ++j) hist[ii][j] = 0.f;
                    }
                }
            }
#pragma unroll
            for (int r = 0; r < kBsHalf; ++r) {
                const int ii = kBsHalf - 1 - r;
                const int i = i0 + ii;
                if (ii < hl) {
                    const float dt = sdl[i * kBsCh + c], xv = sx[i * kBsCh + c], gy = sdy[i * kBsCh + c];
                    float ddt = 0.f, dxb = 0.f, vals[8];
                    const float dtx = dt * xv;
                    float lb = 0.f;  // Euler: sum_j lam_j B_j, the shared factor of dDelta and dxbar
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const float Bn = sbc[i * 32 + 4 * q + j], Cn = sbc[i * 32 + 16 + 4 * q + j];
                        const float Ab = ex2_approx(dt * A2[j]);
                        const float hp = ii > 0 ? hist[ii > 0 ? ii - 1 : 0][j] : hin[j];
                        lam[j] = fmaf(Anext[j], lam[j], Cn * gy);
                        vals[4 + j] = gy * hist[ii][j];
                        const float t1 = lam[j] * hp * Ab;
                        ddt = fmaf(t1, An[j], ddt);
                        gA[j] = fmaf(t1, dt, gA[j]);
                        if (ZOH_EXACT) {
                            const float em = expm1f(dt * An[j]);
                            const float cf = em * Ainv[j];
                            ddt = fmaf(lam[j] * Ab, Bn * xv, ddt);
                            gA[j] = fmaf(lam[j] * Bn * xv, (dt * Ab * An[j] - em) * Ainv[j] * Ainv[j], gA[j]);
                            vals[j] = lam[j] * cf * xv;
                            dxb = fmaf(lam[j] * cf, Bn, dxb);
                        } else {
                            lb = fmaf(lam[j], Bn, lb);
                            vals[j] = lam[j] * dtx;
                        }
                        Anext[j] = Ab;
                    }
                    if (!ZOH_EXACT) {  // dDelta += xbar sum_j lam_j B_j;  dxbar = Delta sum_j lam_j B_j
                        ddt = fmaf(xv, lb, ddt);
                        dxb = dt * lb;
                    }
                    ddt += __shfl_xor_sync(0xffffffffu, ddt, 1);
                    ddt += __shfl_xor_sync(0xffffffffu, ddt, 2);
                    dxb += __shfl_xor_sync(0xffffffffu, dxb, 1);
                    dxb += __shfl_xor_sync(0xffffffffu, dxb, 2);
                    if (q == (i & 3)) {  // every lane of the channel holds the sums
                        sdv[i * kBsCh + c] = ddt * ssg[i * kBsCh + c];
                        sdx[i * kBsCh + c] = dxb;
                    }
                    // sum the 8 values over the warp's 8 channels (lane bits 2..4); each lane keeps one
                    float r1[4], r2[2];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const float send = b4 ? vals[j] : vals[j + 4];
                        const float keep = b4 ? vals[j + 4] : vals[j];
                        r1[j] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
                    }
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        const float send = b3 ? r1[j] : r1[j + 2];
                        const float keep = b3 ? r1[j + 2] : r1[j];
                        r2[j] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
                    }
                    const float send = b2 ? r2[0] : r2[1];
                    const float keep = b2 ? r2[1] : r2[0];
                    const float fin = keep + __shfl_xor_sync(0xffffffffu, send, 4);
                    if (red_n < N) sred[((tid >> 5) * kBsChunk + i) * 32 + red_w * 16 + red_n] = fin;
                }
            }
        }
        __syncthreads();
        for (int i = tid; i < len * kBsCh; i += kBsThreads) {
            const int s = i / kBsCh, cc = i - s * kBsCh;
            if (e0 + cc < E) dxs[(((size_t)b * sh.nd + k) * T + t_of(it, s)) * E + e0 + cc] = sdx[i];
        }
        for (int i = tid; i < len * 32; i += kBsThreads) {  // the warps' dB | dC rows, in warp order
            const int s = i >> 5, j = i & 31, n = j & 15;
            if (n < N) {
                float acc = sred[i];
                for (int w = 1; w < kBsThreads / 32; ++w) acc += sred[w * kBsChunk * 32 + i];
                pdu[u_offset(sh, k, b, t_of(it, s)) + R + (j < 16 ? n : N + n)] = acc;
            }
        }
        // dt_proj: d dt_low of the chunk's steps (this block's channels): one output per thread,
        // W_dt's row r and the step's dv as float4 over the 64 channels
        for (int i = tid; i < len * R; i += kBsThreads) {
            const int s = i / R, r = i - s * R;
            const float4* w4 = reinterpret_cast<const float4*>(swT + r * kBsWS);
            const float4* d4 = reinterpret_cast<const float4*>(sdv + s * kBsCh);
            float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
            for (int c4 = 0; c4 < kBsCh / 4; ++c4) {
                const float4 w = w4[c4], d = d4[c4];
                a0 = fmaf(w.x, d.x, a0);
                a1 = fmaf(w.y, d.y, a1);
                a2 = fmaf(w.z, d.z, a2);
                a3 = fmaf(w.w, d.w, a3);
            }
            pdu[u_offset(sh, k, b, t_of(it, s)) + r] = (a0 + a1) + (a2 + a3);
        }
        // dW_dt | db_dt partial sums over the chunk's steps: thread = (4 channels, 4 entries of
        // their rows; the last group is the bias), dv and dt_low read as float4: 16 FMA per pair
        // of loads
        const int ng = R4 / 4 + 1;
        for (int i = tid; i < (kBsCh / 4) * ng; i += kBsThreads) {
            const int cq = i / ng, g = i - cq * ng;
            float4* a = reinterpret_cast<float4*>(swacc + 4 * cq * WA + 4 * g);  // rows 4 cq .. 4 cq + 3
            const int aw = WA / 4;
            if (g < R4 / 4) {
                float4 acc[4] = {a[0], a[aw], a[2 * aw], a[3 * aw]};
                for (int s = 0; s < len; ++s) {
                    const float4 dv = *reinterpret_cast<const float4*>(sdv + s * kBsCh + 4 * cq);
                    const float4 d = *reinterpret_cast<const float4*>(sdtl + s * R4 + 4 * g);
                    const float dvs[4] = {dv.x, dv.y, dv.z, dv.w};
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        acc[m].x = fmaf(dvs[m], d.x, acc[m].x);
                        acc[m].y = fmaf(dvs[m], d.y, acc[m].y);
                        acc[m].z = fmaf(dvs[m], d.z, acc[m].z);
                        acc[m].w = fmaf(dvs[m], d.w, acc[m].w);
                    }
                }
#pragma unroll
                for (int m = 0; m < 4; ++m) a[m * aw] = acc[m];
            } else {  // the bias entries (column R4) of the 4 rows
                float bs[4] = {a[0].x, a[aw].x, a[2 * aw].x, a[3 * aw].x};
                for (int s = 0; s < len; ++s) {
                    const float4 dv = *reinterpret_cast<const float4*>(sdv + s * kBsCh + 4 * cq);
                    bs[0] += dv.x;
                    bs[1] += dv.y;
                    bs[2] += dv.z;
                    bs[3] += dv.w;
                }
#pragma unroll
                for (int m = 0; m < 4; ++m) a[m * aw].x = bs[m];
            }
        }
        __syncthreads();  // the buffers are refilled by the next stage(s)
    }
    // this image's dW_dt | db_dt and dA_log terms (part_wdt [B][nd][E][R], part_bdt [B][nd][E],
    // part_dA [B][nd][E][N]; bwd_reduce_kernel adds the images in order)
    const size_t img = (size_t)b * sh.nd + k;
    for (int i = tid; i < kBsCh * (R + 1); i += kBsThreads) {
        const int cc = i / (R + 1), r = i - cc * (R + 1);
        if (e0 + cc < E) {
            if (r < R) part_wdt[(img * E + e0 + cc) * R + r] = swacc[cc * WA + r];
            else part_bdt[img * E + e0 + cc] = swacc[cc * WA + R4];
        }
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int n = 4 * q + j;
        if (live && n < N) part_dA[(img * E + e) * N + n] = gA[j] * An[j];
    }
}

// ------------------------------------------------------------------------------------------
// Projection gradients (x_proj: u[k] = xbar W_x[k]^T, J = R + 2N outputs per direction)
// ------------------------------------------------------------------------------------------

constexpr int kGxM = 128, kGxE = 128, kGxK = 16;  // dxbar tile (tokens x channels) and k-step
constexpr int kGwE = 128, kGwK = 16;              // dW_x tile columns, tokens per k-step

// dxbar[m][e] = sum_k sum_jj du[k][m][jj] W_x[k][jj][e] + sum_k dxs[b][k][t][e] (m = b T + t): the
// projections' share, then the scans' share added in direction order.  Grid (ceil(M / 128),
// ceil(E / 128)), 256 threads; thread (ty, tx) = (tid / 16, tid % 16) holds 8 x 8 outputs: tokens
// 4 ty .. and 64 + 4 ty .., channels 4 tx .. and 64 + 4 tx ...  The k loop takes 16 projection
// outputs of one direction per step (zero past J) through a cp.async double buffer: du transposed
// to [16][128 tokens] by 4-byte copies (each thread copies 8 entries of one token's row), W_x rows
// [16][128 channels] by 16-byte copies.  The k order is that of the plain sum (direction, then jj).
__global__ void __launch_bounds__(kThreads, 2)
bwd_dxbar_kernel(Shape sh, const float* __restrict__ du, const float* __restrict__ W_x,
                 const float* __restrict__ dxs, float* __restrict__ dxbar) {
    __shared__ __align__(16) float As[2][kGxK][kGxM];
    __shared__ __align__(16) float Bs[2][kGxK][kGxE];
    const int T = sh.T, E = sh.E, J = sh.J, nd = sh.nd;
    const int M = sh.B * T;
    const int m0 = blockIdx.x * kGxM, e0 = blockIdx.y * kGxE;
    const int tid = threadIdx.x;
    // the token whose du entries this thread copies (k rows ck, ck + 2, ..)
    const int cm = tid & (kGxM - 1), ck = tid >> 7;
    const int gm = m0 + cm;
    const bool m_ok = gm < M;
    const int cb = m_ok ? gm / T : 0;
    const float* du_row = du + u_offset(sh, 0, cb, m_ok ? gm - cb * T : 0);  // direction 0
    const size_t ubs = u_block_stride(T, J);                                  // next direction
    const int jsteps = (J + kGxK - 1) / kGxK, nsteps = nd * jsteps;
    auto stage = [&](int si) {
        const int k = si / jsteps, jj0 = (si - k * jsteps) * kGxK, buf = si & 1;
        const float* src = du_row + k * ubs + jj0;
#pragma unroll
        for (int l = 0; l < kGxK / 2; ++l) {
            const int kk = ck + 2 * l;
            const bool ok = m_ok && jj0 + kk < J;
            cp_async4z(&As[buf][kk][cm], ok ? src + kk : du, ok);
        }
#pragma unroll
        for (int l = 0; l < 2; ++l) {
            const int idx = tid + kThreads * l;
            const int kk = idx >> 5, c4 = (idx & 31) * 4;
            const bool ok = jj0 + kk < J && e0 + c4 < E;
            const float* w = W_x + ((size_t)k * J + jj0 + kk) * E + e0 + c4;
            cp_async16(&Bs[buf][kk][c4], ok ? (const void*)w : (const void*)W_x, ok ? 16u : 0u);
        }
        cp_async_commit();
    };
    const int tx = tid & 15, ty = tid >> 4;
    float acc[8][8];
#pragma unroll
    for (int p = 0; p < 8; ++p)
#pragma unroll
        for (int r = 0; r < 8; ++r) acc[p][r] = 0.f;
    stage(0);
    for (int si = 0; si < nsteps; ++si) {
        if (si + 1 < nsteps) {
            stage(si + 1);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        const int buf = si & 1;
#pragma unroll
        for (int kk = 0; kk < kGxK; ++kk) {
            const float4 a0 = *reinterpret_cast<const float4*>(&As[buf][kk][4 * ty]);
            const float4 a1 = *reinterpret_cast<const float4*>(&As[buf][kk][64 + 4 * ty]);
            const float4 b0 = *reinterpret_cast<const float4*>(&Bs[buf][kk][4 * tx]);
            const float4 b1 = *reinterpret_cast<const float4*>(&Bs[buf][kk][64 + 4 * tx]);
            const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
            const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
            for (int p = 0; p < 8; ++p)
#pragma unroll
                for (int r = 0; r < 8; ++r) acc[p][r] = fmaf(av[p], bv[r], acc[p][r]);
        }
        __syncthreads();  // the buffer is refilled by the stage after next
    }
    // two rows at a time: their scan shares (up to 8 float4, read once: streaming loads) are all
    // requested before the first is used
#pragma unroll
    for (int p0 = 0; p0 < 8; p0 += 2) {
        float4 sv[2][2][2];
        int mrow[2];
#pragma unroll
        for (int pp = 0; pp < 2; ++pp) {
            const int p = p0 + pp;
            const int m = m0 + (p < 4 ? 4 * ty + p : 64 + 4 * ty + p - 4);
            mrow[pp] = m;
            const int b = m < M ? m / T : 0, t = m - b * T;
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                const int e = e0 + 64 * hf + 4 * tx;
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    // E is a multiple of 4: e < E covers e + 3
                    sv[pp][hf][k] = (m < M && e < E && k < nd)
                                        ? __ldcs(reinterpret_cast<const float4*>(dxs + (((size_t)b * nd + k) * T + t) * E + e))
                                        : make_float4(0.f, 0.f, 0.f, 0.f);
                }
            }
        }
#pragma unroll
        for (int pp = 0; pp < 2; ++pp) {
            const int p = p0 + pp, m = mrow[pp];
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                const int e = e0 + 64 * hf + 4 * tx;
                if (m >= M || e >= E) continue;
                float4 v = make_float4(acc[p][4 * hf], acc[p][4 * hf + 1], acc[p][4 * hf + 2], acc[p][4 * hf + 3]);
                f4_add(v, sv[pp][hf][0]);  // the directions' shares in order (+0 past nd)
                if (nd > 1) f4_add(v, sv[pp][hf][1]);
                *reinterpret_cast<float4*>(dxbar + (size_t)m * E + e) = v;
            }
        }
    }
}

// Split-K partial sums of dW_x[k][jj][e] = sum_m du[k][m][jj] xbar[m][e]: split s sums the tokens
// [s kchunk, min(M, (s + 1) kchunk)) in order into part [splits][nd][J][E] (bwd_reduce_kernel adds
// the splits in order).  Grid (ceil(E / 128), nd * splits), 256 threads, RT = ceil(J / 16): thread
// (ty, tx) = (tid / 16, tid % 16) holds rows RT ty .. RT ty + RT - 1 and channels 4 tx .. and
// 64 + 4 tx ...  Each k-step stages 16 tokens through a cp.async double buffer: their du rows
// [16][16 RT] (zero past J; 16-byte copies when VEC: J a multiple of 4, else 4-byte ones) and their
// xbar rows [16][128] (16-byte copies).
template <int RT, bool VEC>
__global__ void __launch_bounds__(kThreads)
bwd_dwx_kernel(Shape sh, const float* __restrict__ du, const float* __restrict__ xbar, float* __restrict__ part,
               int splits, int kchunk) {
    constexpr int JP = 16 * RT;
    __shared__ __align__(16) float As[2][kGwK][JP];
    __shared__ __align__(16) float Bs[2][kGwK][kGwE];
    const int T = sh.T, E = sh.E, J = sh.J;
    const int M = sh.B * T;
    const int k = blockIdx.y / splits, s = blockIdx.y - k * splits;
    const int e0 = blockIdx.x * kGwE;
    const int mbeg = s * kchunk, mend = min(M, mbeg + kchunk);
    const int nsteps = (max(mend - mbeg, 0) + kGwK - 1) / kGwK;
    const int tid = threadIdx.x;
    auto stage = [&](int si) {
        const int m0 = mbeg + si * kGwK, buf = si & 1;
        const int b0 = m0 / T, t0 = m0 - b0 * T;
        if (VEC) {  // J a multiple of 4: 16-byte copies of the du rows
            for (int idx = tid; idx < kGwK * (JP / 4); idx += kThreads) {
                const int kk = idx / (JP / 4), j4 = 4 * (idx - kk * (JP / 4));
                const bool ok = m0 + kk < mend && j4 < J;
                const float* src = du;
                if (ok) {
                    int b = b0, t = t0 + kk;
                    while (t >= T) {
                        t -= T;
                        ++b;
                    }
                    src = du + u_offset(sh, k, b, t) + j4;
                }
                cp_async16(&As[buf][kk][j4], src, ok ? 16u : 0u);
            }
        } else {
            for (int idx = tid; idx < kGwK * JP; idx += kThreads) {
                const int kk = idx / JP, jj = idx - kk * JP;
                const bool ok = m0 + kk < mend && jj < J;
                const float* src = du;
                if (ok) {
                    int b = b0, t = t0 + kk;
                    while (t >= T) {
                        t -= T;
                        ++b;
                    }
                    src = du + u_offset(sh, k, b, t) + jj;
                }
                cp_async4z(&As[buf][kk][jj], src, ok);
            }
        }
#pragma unroll
        for (int l = 0; l < 2; ++l) {
            const int idx = tid + kThreads * l;
            const int kk = idx >> 5, c4 = (idx & 31) * 4;
            const bool ok = m0 + kk < mend && e0 + c4 < E;
            const float* x = xbar + (size_t)(m0 + kk) * E + e0 + c4;
            cp_async16(&Bs[buf][kk][c4], ok ? (const void*)x : (const void*)xbar, ok ? 16u : 0u);
        }
        cp_async_commit();
    };
    const int tx = tid & 15, ty = tid >> 4;
    float acc[RT][8];
#pragma unroll
    for (int p = 0; p < RT; ++p)
#pragma unroll
        for (int r = 0; r < 8; ++r) acc[p][r] = 0.f;
    if (nsteps > 0) stage(0);
    for (int si = 0; si < nsteps; ++si) {
        if (si + 1 < nsteps) {
            stage(si + 1);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        const int buf = si & 1;
#pragma unroll
        for (int kk = 0; kk < kGwK; ++kk) {
            const float4 b0 = *reinterpret_cast<const float4*>(&Bs[buf][kk][4 * tx]);
            const float4 b1 = *reinterpret_cast<const float4*>(&Bs[buf][kk][64 + 4 * tx]);
            const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
            for (int p = 0; p < RT; ++p) {
                const float av = As[buf][kk][RT * ty + p];
#pragma unroll
                for (int r = 0; r < 8; ++r) acc[p][r] = fmaf(av, bv[r], acc[p][r]);
            }
        }
        __syncthreads();  // the buffer is refilled by the stage after next
    }
#pragma unroll
    for (int p = 0; p < RT; ++p) {
        const int jj = RT * ty + p;
        if (jj >= J) continue;
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            const int e = e0 + 64 * hf + 4 * tx;
            if (e >= E) continue;
            *reinterpret_cast<float4*>(part + (((size_t)s * sh.nd + k) * J + jj) * E + e) =
                make_float4(acc[p][4 * hf], acc[p][4 * hf + 1], acc[p][4 * hf + 2], acc[p][4 * hf + 3]);
        }
    }
}

// ------------------------------------------------------------------------------------------
// Fixed-order sums of per-block partials (reproducible batch sums)
// ------------------------------------------------------------------------------------------

// out[c * out_stride + i] = the sum over p < P of part[p][i] (partial p starts at
// part + p * part_stride) for i < L and c < copies; with blk > 0 entries whose i % blk >= valid are
// padding and get 0.
struct RedSeg {
    const float* part;
    float* out;
    long long L, part_stride, out_stride, blk, valid;
    int P, copies;
};
constexpr int kMaxRedSegs = 8;
struct RedSegs {
    RedSeg seg[kMaxRedSegs];
};
// Grid (x, number of segments): blockIdx.y picks the segment.  Up to 128 partials: one
// thread per output adds them in order.  Many: a block takes 32 consecutive outputs at a time (one
// per lane: coalesced loads) and splits the P partials over its 8 warps (warp w adds partials
// w, w + 8, ... in order); the 8 warp sums are then added in warp order.  Either grouping depends
// on nothing but P, so the result is the same in every run.
constexpr int kRedWarps = 8;
__global__ void __launch_bounds__(kRedWarps * 32)
bwd_reduce_kernel(RedSegs segs) {
    __shared__ float wsum[kRedWarps][32];
    const RedSeg g = segs.seg[blockIdx.y];
    if (g.P <= 128) {
        for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < g.L;
             i += (long long)gridDim.x * blockDim.x) {
            float acc = 0.f;
            if (g.blk == 0 || i % g.blk < g.valid)
                for (int p = 0; p < g.P; ++p) acc += g.part[(size_t)p * g.part_stride + i];
            for (int c = 0; c < g.copies; ++c) g.out[(size_t)c * g.out_stride + i] = acc;
        }
        return;
    }
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    for (long long i0 = (long long)blockIdx.x * 32; i0 < g.L; i0 += (long long)gridDim.x * 32) {
        const long long i = i0 + lane;
        float acc = 0.f;
        if (i < g.L && (g.blk == 0 || i % g.blk < g.valid)) {
#pragma unroll 4
            for (int p = w; p < g.P; p += kRedWarps) acc += g.part[(size_t)p * g.part_stride + i];
        }
        wsum[w][lane] = acc;
        __syncthreads();
        if (w == 0 && i < g.L) {
            float sum = wsum[0][lane];
            for (int q = 1; q < kRedWarps; ++q) sum += wsum[q][lane];
            for (int c = 0; c < g.copies; ++c) g.out[(size_t)c * g.out_stride + i] = sum;
        }
        __syncthreads();
    }
}

// ------------------------------------------------------------------------------------------
// Pooling
// ------------------------------------------------------------------------------------------

// One block per pooled row (b, t), launched with bwd_groups(SL) * bwd_slot_width(SL) threads:
// every token of the row gets dx += pool_scale / S * dxbar[b][t].
__global__ void __launch_bounds__(kThreads)
bwd_pool_dense_kernel(Shape sh, const float* __restrict__ dxbar, float* __restrict__ dx) {
    const int SL = sh.SL, SW = bwd_slot_width(SL), G = bwd_groups(SL);
    const int ls = threadIdx.x % SW, g = threadIdx.x / SW;
    const int bt = blockIdx.x, b = bt / sh.T, t = bt - b * sh.T;
    const int S = sh.S;
    const size_t st4 = dense_stride(sh) >> 2;
    const float scale = sh.pool_scale / (float)S;
    float4* dx4 = reinterpret_cast<float4*>(dx);
    for (int s0 = 0; s0 < SL; s0 += SW) {
        const int slot = s0 + ls;
        if (g >= G || slot >= SL) continue;
        const float4 a = f4_scale(reinterpret_cast<const float4*>(dxbar + (size_t)bt * sh.E)[slot], scale);
        const size_t base = (dense_base(sh, b, t) >> 2) + slot;
        int s = g;
        for (; s + 3 * G < S; s += 4 * G) {
            float4 v[4];
#pragma unroll
            for (int uu = 0; uu < 4; ++uu) v[uu] = ld_stream(dx4 + base + (size_t)(s + uu * G) * st4);
#pragma unroll
            for (int uu = 0; uu < 4; ++uu) {
                f4_add(v[uu], a);
                st_stream(dx4 + base + (size_t)(s + uu * G) * st4, v[uu]);
            }
        }
        for (; s < S; s += G) {
            float4 v = ld_stream(dx4 + base + (size_t)s * st4);
            f4_add(v, a);
            st_stream(dx4 + base + (size_t)s * st4, v);
        }
    }
}

// One block per kept token (b, k): dx += pool_scale / S * dxbar of its row; a token whose id was
// rejected (row_of < 0) gets dx = dz = 0.
__global__ void __launch_bounds__(kThreads)
bwd_pool_masked_kernel(Shape sh, const int32_t* __restrict__ row_of, const float* __restrict__ dxbar,
                       float* __restrict__ dx, float* __restrict__ dz) {
    const size_t bk = blockIdx.x;
    const int b = (int)(bk / sh.K);
    const int r = row_of[bk];
    const float scale = sh.pool_scale / (float)sh.S;
    float4* dx4 = reinterpret_cast<float4*>(dx) + bk * sh.SL;
    float4* dz4 = reinterpret_cast<float4*>(dz) + bk * sh.SL;
    if (r < 0) {
        for (int slot = threadIdx.x; slot < sh.SL; slot += blockDim.x) {
            dx4[slot] = f4_zero();
            dz4[slot] = f4_zero();
        }
        return;
    }
    const float4* a4 = reinterpret_cast<const float4*>(dxbar + ((size_t)b * sh.T + r) * sh.E);
    for (int slot = threadIdx.x; slot < sh.SL; slot += blockDim.x) {
        float4 v = ld_stream(dx4 + slot);
        f4_add(v, f4_scale(a4[slot], scale));
        st_stream(dx4 + slot, v);
    }
}

}  // namespace fv
