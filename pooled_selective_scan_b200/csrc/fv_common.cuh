// fv_common.cuh -- shared device definitions of the FastVim SSM kernels (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace fv {

constexpr int kThreads = 256;       // every kernel of the layer runs 256-thread CTAs
constexpr int kMaxN = 16;           // d_state limit: 4 lanes x 4 states in the scan
constexpr int kMaxJ = 96;           // R + 2N limit per direction
constexpr int kProjRows = 32;       // pooled tokens per projection CTA
constexpr int kProjChunk = 32;      // channels per projection K-step
constexpr int kProjQ = (2 * kMaxJ + 7) / 8;  // outputs per thread in the projection

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
    float pool_scale;
    int SL;            // float4 slots per token row: E / 4
};

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

__device__ __forceinline__ float softplus_f(float v) { return v > 20.f ? v : log1pf(expf(v)); }
__device__ __forceinline__ float silu_f(float v) { return v / (1.f + expf(-v)); }

__device__ __forceinline__ void f4_add(float4& a, const float4& b) {
    a.x += b.x; a.y += b.y; a.z += b.z; a.w += b.w;
}

// Record the first device-side error of a call; later ones keep the first code.
__device__ __forceinline__ void set_status(unsigned* st, unsigned code) { atomicCAS(st, 0u, code); }

}  // namespace fv
