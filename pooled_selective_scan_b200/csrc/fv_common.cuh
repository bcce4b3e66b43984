// fv_common.cuh -- shared device definitions of the FastVim SSM kernels (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace fv {

constexpr int kThreads = 256;       // every kernel of the layer runs 256-thread CTAs
constexpr int kMaxN = 16;           // d_state limit: 4 lanes x 4 states in the scan
constexpr int kMaxJ = 96;           // R + 2N limit per direction

// Device status codes (the values of fv_status that kernels may record).
constexpr unsigned kStatusIndex = 4u;
constexpr unsigned kStatusTimeout = 7u;

// Everything a kernel needs to know about one call, passed by value.
struct Shape {
    int B, h, w, E, N, R;
    int T, S;          // pooled length and pooled-over length
    int nd, J, NJ;     // directions, R + 2N, nd * J
    int K;             // kept tokens per sample (masked) or 0
    int pool_axis;     // 0 = POOL_W (T = h), 1 = POOL_H (T = w)
    unsigned dir_flags;
    int zoh_exact;
    unsigned path_flags;  // FV_FLAG_PATH_* of the call
    int trace;            // FV_FLAG_TRACE: record one trace entry per fused task
    float pool_scale;
    int SL;            // float4 slots per token row: E / 4
    int ln;            // FV_FLAG_LAYERNORM: post-SSM LayerNorm before the gate
    float ln_eps;
    int dc;            // taps of the block's Conv1D in front of the layer (0: x is its output)
    int conv_silu;     // FV_FLAG_CONV_SILU: SiLU after the Conv1D
    int nx;            // pooled-token sets: nd with the Conv1D (one per direction), else 1
    int keep;          // FV_FLAG_KEEP_STATES: the scans store their states for the gradient
};

constexpr int kMaxConv = 4;  // Conv1D taps at most

// Pooled tokens of image b, set kx (the direction's own with the Conv1D, else 0): [T][E] rows.
__host__ __device__ __forceinline__ size_t xbar_offset(const Shape& sh, int b, int kx, int t) {
    return (((size_t)b * sh.nx + kx) * sh.T + t) * (size_t)sh.E;
}

// Scan states kept for the gradient (FV_FLAG_KEEP_STATES), [B][nd][2 ceil(T / 16)][E][16], zero
// for states n >= N.  Each scan walks the time axis' 16-step chunks [16 c, 16 c + 16) in its own
// order (forward c = 0, 1, ..; backward from the last, possibly shorter, chunk down); slot 2 i + h
// of (image b, direction k, channel e) holds the state entering the h-th 8-step half of the
// scan's i-th chunk (forward: the state before step 16 i + 8 h).  A chunk of at most 8 steps has
// no second slot.
constexpr int kCkptSteps = 8;
__host__ __device__ __forceinline__ int ckpt_count(int T) { return 2 * ((T + 15) / 16); }
__host__ __device__ __forceinline__ size_t ckpt_offset(const Shape& sh, int b, int k, int c, int e) {
    return ((((size_t)b * sh.nd + k) * ckpt_count(sh.T) + c) * sh.E + e) * 16;
}

// Projections u of (image b, direction k) are one block of T x J floats, image-major (so the
// blocks of a run of images are contiguous); blocks start every
// u_block_stride floats (T J rounded up to 32 floats = 128 bytes), so no cache line holds
// projections of two images.
__host__ __device__ __forceinline__ size_t u_block_stride(int T, int J) { return (((size_t)T * J + 31) / 32) * 32; }
__host__ __device__ __forceinline__ size_t u_offset(const Shape& sh, int k, int b, int t) {
    return ((size_t)b * sh.nd + k) * u_block_stride(sh.T, sh.J) + (size_t)t * sh.J;
}

// Offset (in floats) of step size row (direction k, image b, pooled token t) in the staged path's
// Delta buffer, fp32 [nd][B][T][E].
__host__ __device__ __forceinline__ size_t delta_offset(const Shape& sh, int k, int b, int t) {
    return (((size_t)k * sh.B + b) * sh.T + t) * (size_t)sh.E;
}

// Offset (in floats) of token s of pooled token (b, t) on the dense grid, and the stride
// between consecutive s.  POOL_W: token (t, s); POOL_H: token (s, t).
__host__ __device__ __forceinline__ size_t dense_base(const Shape& sh, int b, int t) {
    return sh.pool_axis == 0 ? ((size_t)b * sh.h + t) * (size_t)sh.w * sh.E
                             : ((size_t)b * sh.h * sh.w + t) * (size_t)sh.E;
}
__host__ __device__ __forceinline__ size_t dense_stride(const Shape& sh) {
    return sh.pool_axis == 0 ? (size_t)sh.E : (size_t)sh.w * sh.E;
}

// Streaming (evict-first) 128-bit accesses for data touched once.
__device__ __forceinline__ float4 ld_stream(const float4* p) { return __ldcs(p); }
__device__ __forceinline__ void st_stream(float4* p, const float4& v) { __stcs(p, v); }

// L2 eviction-priority policies (createpolicy) and 128-bit accesses that carry them.  Loads skip
// L1 allocation: every byte is used once per CTA.
__device__ __forceinline__ uint64_t l2_policy_evict_last() {
    uint64_t p;
    asm("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
    uint64_t p;
    asm("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
// For tensors that stay read-only for the whole kernel (x, z): the compiler may schedule these
// loads freely.
__device__ __forceinline__ float4 ld_nc_hint(const float4* p, uint64_t pol) {
    float4 v;
    asm("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.f32 {%0, %1, %2, %3}, [%4], %5;"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "l"(p), "l"(pol));
    return v;
}
__device__ __forceinline__ void st_hint(float4* p, const float4& v, uint64_t pol) {
    asm volatile("st.global.L1::no_allocate.L2::cache_hint.v4.f32 [%0], {%1, %2, %3, %4}, %5;"
                 :
                 : "l"(p), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w), "l"(pol)
                 : "memory");
}

// Cross-CTA handshakes inside one launch: acquire loads of counters, release increments.
__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned* p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
// A relaxed read (no ordering): for advisory flags polled between tasks.
__device__ __forceinline__ unsigned ld_relaxed_gpu(const unsigned* p) {
    unsigned v;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void red_release_gpu_add(unsigned* p, unsigned v) {
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" : : "l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ unsigned long long globaltimer_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ---- shared-memory mbarriers and TMA bulk copies (global -> shared) ----------------------------
__device__ __forceinline__ unsigned smem_u32(const void* p) {
    return static_cast<unsigned>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(unsigned long long* bar, unsigned count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" : : "r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" : : : "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" : : : "memory");
}
// One arrival that also announces `bytes` of asynchronous transfers completing on this barrier.
__device__ __forceinline__ void mbar_arrive_expect_tx(unsigned long long* bar, unsigned bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" : : "r"(smem_u32(bar)), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(unsigned long long* bar, unsigned parity) {
    unsigned ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// Bulk copy of `bytes` (multiple of 16, both addresses 16-byte aligned) into this CTA's shared
// memory, completing on `bar`, with an L2 eviction-priority policy on the global reads.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, unsigned bytes, unsigned long long* bar,
                                         uint64_t pol) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;"
        :
        : "r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(pol)
        : "memory");
}
// 2^x on the SFU (ex2.approx.ftz: results below 2^-126 flush to zero).
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// 1/x on the SFU (rcp.approx.ftz).
__device__ __forceinline__ float rcp_approx(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
// SiLU(v) = v / (1 + e^-v) with the SFU exponential and reciprocal: about 3e-7 relative error;
// v -> -inf gives -0 (e^-v overflows to inf, its reciprocal is 0).
__device__ __forceinline__ float silu_fast(float v) {
    return v * rcp_approx(1.f + ex2_approx(v * -1.4426950408889634f));
}

// 16-byte asynchronous global -> shared copies (cp.async); src_bytes = 0 fills zeros.
__device__ __forceinline__ void cp_async16(void* dst, const void* src, unsigned src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" : : "r"(smem_u32(dst)), "l"(src), "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async4(void* dst, const void* src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" : : "r"(smem_u32(dst)), "l"(src) : "memory");
}
// 4-byte copy that writes zero instead when `valid` is false (nothing is read then).
__device__ __forceinline__ void cp_async4z(void* dst, const void* src, bool valid) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;"
                 : : "r"(smem_u32(dst)), "l"(src), "r"(valid ? 4u : 0u) : "memory");
}
// Bring the line holding p into L2 (no register, no wait).
__device__ __forceinline__ void prefetch_l2(const void* p) { asm volatile("prefetch.global.L2 [%0];" : : "l"(p)); }
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" : : : "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" : : "n"(N) : "memory"); }

// softplus(v) = max(v, 0) + log1p(e), e = exp(-|v|) in (0, 1]: e from the SFU exp2, and
// log1p(e) = 2 atanh(s) with s = e / (2 + e) in (0, 1/3], summed as the odd series
// 2 (s + s^3/3 + ... + s^13/13) (truncation below s^14/15 < 2.2e-8 relative; no branch).
__device__ __forceinline__ float softplus_fast(float v) {
    const float e = ex2_approx(-fabsf(v) * 1.4426950408889634f);
    const float s = e * rcp_approx(2.f + e);
    const float s2 = s * s;
    float p = 1.f / 13.f;
    p = fmaf(p, s2, 1.f / 11.f);
    p = fmaf(p, s2, 1.f / 9.f);
    p = fmaf(p, s2, 1.f / 7.f);
    p = fmaf(p, s2, 1.f / 5.f);
    p = fmaf(p, s2, 1.f / 3.f);
    p = fmaf(p, s2, 1.f);
    return fmaxf(v, 0.f) + 2.f * s * p;
}

__device__ __forceinline__ float silu_f(float v) { return v / (1.f + expf(-v)); }

__device__ __forceinline__ void f4_add(float4& a, const float4& b) {
    a.x += b.x; a.y += b.y; a.z += b.z; a.w += b.w;
}

// ---- post-SSM LayerNorm helpers (one warp per token row) ----
__device__ __forceinline__ float4 f4_fma(const float4& a, const float4& b, const float4& c) {
    return make_float4(fmaf(a.x, b.x, c.x), fmaf(a.y, b.y, c.y), fmaf(a.z, b.z, c.z), fmaf(a.w, b.w, c.w));
}
// Adds the shifted first and second moments of v's four values to (m1, m2).
__device__ __forceinline__ void ln_accum(const float4& v, float K, float& m1, float& m2) {
    const float a = v.x - K, b = v.y - K, c = v.z - K, d = v.w - K;
    m1 += (a + b) + (c + d);
    m2 += (a * a + b * b) + (c * c + d * d);
}
// Warp totals of (m1, m2) -> mean and 1 / sqrt(var + eps).
__device__ __forceinline__ void ln_stats(float m1, float m2, float K, float invE, float eps, float& mean,
                                         float& rstd) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        m1 += __shfl_xor_sync(0xffffffffu, m1, o);
        m2 += __shfl_xor_sync(0xffffffffu, m2, o);
    }
    const float d = m1 * invE;
    mean = K + d;
    rstd = rsqrtf(fmaxf(m2 * invE - d * d, 0.f) + eps);
}
__device__ __forceinline__ float4 ln_gate4(const float4& sv, const float4& zv, const float4& gv, const float4& bv,
                                           float mean, float rstd) {
    return make_float4(silu_fast(zv.x) * fmaf(gv.x, (sv.x - mean) * rstd, bv.x),
                       silu_fast(zv.y) * fmaf(gv.y, (sv.y - mean) * rstd, bv.y),
                       silu_fast(zv.z) * fmaf(gv.z, (sv.z - mean) * rstd, bv.z),
                       silu_fast(zv.w) * fmaf(gv.w, (sv.w - mean) * rstd, bv.w));
}

// Record the first device-side error of a call; later ones keep the first code.
__device__ __forceinline__ void set_status(unsigned* st, unsigned code) { atomicCAS(st, 0u, code); }

}  // namespace fv
