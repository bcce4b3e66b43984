// fv_dt_tc.cuh -- dt_proj + softplus of the staged path on the 5th-generation tensor cores (sm_100a:
// tcgen05.mma with the accumulators in tensor memory), at fp32 accuracy.
//
// FastVim (gptget.net summary of arXiv 2502.00594, "方法详解" item 3) after Mamba's selective SSM:
// per direction k the step sizes are Delta = softplus(W_dt[k] dt_low + b_dt[k]), dt_low the first R
// outputs of x_proj.  Over a batch this is one GEMM per direction, D[m][e] = sum_r dt_low[m][r]
// W_dt[e][r] with M = B T pooled tokens, N = E channels, K = R, followed by Delta = softplus(D + b_dt)
// written to a [nd][B][T][E] buffer that the scans read.
//
// Accuracy.  Each operand value is split into three tf32 pieces, x = x1 + x2 + x3 (x1 = x rounded to
// tf32, x2 = the remainder rounded to tf32, x3 = what is left; the remainders are exact in fp32, so
// the pieces hold all 24 bits).  Per 8-wide k-step the product x1 y1 goes into one tensor-memory
// accumulator and the five next products (x3 y1, x2 y2, x1 y3, x2 y1, x1 y2, each above 2^-33 |x y|)
// into a second one; the epilogue adds the two and the bias in fp32.  The tensor core rounds each
// MMA's addition into its accumulator towards zero, about an ulp of the running sum: the main
// accumulator takes ceil(R / 8) such additions (6 at R = 48) and the second one holds values 2^-11
// smaller, so the sum is about as accurate as an fp32 FFMA dot product of the R terms.  (A single
// accumulator fed many MMAs lets those truncations pile up: with K = E for x_proj it missed the
// layer's tolerance, which is why x_proj stays on FFMA.)
//
// CTA: 512 threads, 128 tokens x 128 channels of one direction.  Per 32-wide slice of R the operands
// are copied with cp.async (16-byte copies when R and R + 2N are multiples of 4, else 4-byte ones:
// rows of u and W_dt then need not be 16-byte aligned) into 128-byte-swizzled K-major tiles,
// zero-filled outside the layer; the threads split them into their pieces in place; one thread
// issues the MMAs and commits them to an mbarrier, which every thread waits on (with a time limit)
// before the tiles are reused or the accumulators read.  Epilogue: warp w reads tensor-memory lanes 32 (w % 4) .. + 31 (its
// tokens) and columns 32 (w / 4) .. + 31 (its channels) of both accumulators with tcgen05.ld, adds
// them and the bias and applies softplus into a shared-memory copy of the tile; the tile then leaves
// row by row, each warp store 512 contiguous bytes of a Delta row.  (Stored straight from the
// tensor-memory layout, one token row per lane, the stores took longer than the rest of the kernel.)
#pragma once

#include "fv_common.cuh"

namespace fv {

constexpr int kDtM = 128;         // pooled tokens per CTA (the MMA's M)
constexpr int kDtN = 128;         // channels per CTA (the MMA's N)
constexpr int kDtK = 32;          // entries of dt_low per slice: one 128-byte row of fp32
constexpr int kDtThreads = 512;  // 16 warps: 4 per tensor-memory lane quarter in the epilogue
constexpr int kDtPieces = 3;
constexpr uint32_t kDtTileBytes = 128u * 128u;  // one piece of A or B: 128 rows of 128 bytes
constexpr size_t kDtSmemBytes = 2 * kDtPieces * (size_t)kDtTileBytes + 1024;  // + alignment of the tiles
constexpr uint32_t kDtTmemCols = 2 * kDtN;      // main accumulator | the smaller products
constexpr int kDtOS = kDtN + 4;                 // row stride (floats) of the staged output tile
static_assert((size_t)kDtM * kDtOS * sizeof(float) <= 2 * kDtPieces * (size_t)kDtTileBytes,
              "the output tile reuses the operand tiles");

// Shared-memory matrix descriptor of a K-major operand in the 128-byte swizzle: rows of 128 bytes,
// 8-row groups 1024 bytes apart; start address 16-byte granular (advanced by 32 bytes per 8-wide
// k-step inside the swizzle row).
__device__ __forceinline__ uint64_t dt_desc(uint32_t saddr) {
    uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);  // start address
    d |= (uint64_t)1 << 16;                            // leading-dimension offset (unused here)
    d |= (uint64_t)(1024 >> 4) << 32;                  // stride between 8-row groups
    d |= (uint64_t)1 << 46;                            // descriptor version
    d |= (uint64_t)2 << 61;                            // 128-byte swizzle
    return d;
}
// Instruction descriptor: tf32 A and B (K-major), fp32 accumulator, M x N.
__host__ __device__ constexpr uint32_t dt_idesc(int M, int N) {
    return (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
__device__ __forceinline__ void dt_mma(uint32_t tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t accum) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}"
        :
        : "r"(tmem), "l"(a), "l"(b), "r"(idesc), "r"(accum)
        : "memory");
}
__device__ __forceinline__ void dt_commit(unsigned long long* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 :
                 : "r"(smem_u32(bar))
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" : : : "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" : : : "memory"); }
__device__ __forceinline__ void tmem_ld16(uint32_t addr, uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]),
          "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(addr));
}

__device__ __forceinline__ float tf32_rna(float v) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(v));
    return __uint_as_float(r);
}
// v = p1 + p2 + p3 exactly up to the last 9 bits of p3's remainder (below 2^-33 |v|).
__device__ __forceinline__ void tf32_split3(float v, float& p1, float& p2, float& p3) {
    p1 = tf32_rna(v);
    const float r1 = v - p1;
    p2 = tf32_rna(r1);
    p3 = tf32_rna(r1 - p2);
}

// Byte offset of fp32 column c (0..31) of row r in a 128-byte-swizzled tile.
__device__ __forceinline__ uint32_t dt_swz(int r, int c) {
    return (uint32_t)(r * 128 + ((((c >> 2) ^ (r & 7)) << 4) | ((c & 3) << 2)));
}

__global__ void __launch_bounds__(kDtThreads, 2)
dt_proj_kernel(Shape sh, const float* __restrict__ u, const float* __restrict__ W_dt, const float* __restrict__ b_dt,
               float* __restrict__ delta, unsigned* status) {
    extern __shared__ __align__(16) unsigned char dt_raw[];
    __shared__ __align__(8) unsigned long long mma_done;
    __shared__ uint32_t s_tmem;
    __shared__ int s_ok;
    __shared__ float s_bias[kDtN];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int k = blockIdx.z;
    const int M = sh.B * sh.T, E = sh.E, R = sh.R;
    const int m0 = blockIdx.x * kDtM, e0 = blockIdx.y * kDtN;
    const uint32_t base = (smem_u32(dt_raw) + 1023u) & ~1023u;  // swizzle atoms are 1024-byte aligned
    unsigned char* gbase = dt_raw + (base - smem_u32(dt_raw));
    // piece p of A (tokens) and of B (channels)
    auto a_pc = [&](int p) { return base + (uint32_t)p * kDtTileBytes; };
    auto b_pc = [&](int p) { return base + (uint32_t)(kDtPieces + p) * kDtTileBytes; };

    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     :
                     : "r"(smem_u32(&s_tmem)), "r"(kDtTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" : : : "memory");
    }
    if (tid == 0) {
        mbar_init(&mma_done, 1);
        fence_mbar_init();
    }
    if (tid < kDtN) s_bias[tid] = e0 + tid < E ? __ldg(b_dt + (size_t)k * E + e0 + tid) : 0.f;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_tmem;

    // thread 0 waits (bounded) for the MMAs of slice s; the verdict reaches every thread
    auto wait_mma = [&](unsigned parity) -> bool {
        if (tid == 0) {
            int ok = 1;
            if (!mbar_try_wait(&mma_done, parity)) {
                const unsigned long long t0 = globaltimer_ns();
                while (!mbar_try_wait(&mma_done, parity)) {
                    if (globaltimer_ns() - t0 > 1000000000ull) {
                        set_status(status, kStatusTimeout);
                        ok = 0;
                        break;
                    }
                }
            }
            s_ok = ok;
        }
        __syncthreads();
        return s_ok != 0;
    };
    auto split_tile = [&](uint32_t p1) {  // piece 1 in place, pieces 2 and 3 one and two tiles further
        for (uint32_t o = tid * 16u; o < kDtTileBytes; o += kDtThreads * 16u) {
            float4* q1 = reinterpret_cast<float4*>(gbase + (p1 - base) + o);
            float4* q2 = reinterpret_cast<float4*>(gbase + (p1 - base) + kDtTileBytes + o);
            float4* q3 = reinterpret_cast<float4*>(gbase + (p1 - base) + 2 * kDtTileBytes + o);
            const float4 v = *q1;
            float4 a, b, c;
            tf32_split3(v.x, a.x, b.x, c.x);
            tf32_split3(v.y, a.y, b.y, c.y);
            tf32_split3(v.z, a.z, b.z, c.z);
            tf32_split3(v.w, a.w, b.w, c.w);
            *q1 = a;
            *q2 = b;
            *q3 = c;
        }
    };

    constexpr uint32_t idesc = dt_idesc(kDtM, kDtN);
    bool ok = true;
    int slice = 0;
    for (int r0 = 0; r0 < R && ok; r0 += kDtK, ++slice) {
        if ((R & 3) == 0 && (sh.J & 3) == 0) {
            // rows of u (J floats apart) and of W_dt (R apart) start on 16 bytes: 16-byte copies,
            // 8 per 128-byte tile row
            for (int i = tid; i < kDtM * 8; i += kDtThreads) {
                const int row = i >> 3, c = i & 7, m = m0 + row;
                const bool ok = m < M && r0 + 4 * c < R;
                const float* src = u;
                if (ok) {
                    const int b = m / sh.T, t = m - b * sh.T;
                    src = u + u_offset(sh, k, b, t) + r0 + 4 * c;
                }
                cp_async16(gbase + (a_pc(0) - base) + dt_swz(row, 4 * c), src, ok ? 16u : 0u);
            }
            for (int i = tid; i < kDtN * 8; i += kDtThreads) {
                const int ee = i >> 3, c = i & 7;
                const bool ok = e0 + ee < E && r0 + 4 * c < R;
                const float* src = ok ? W_dt + ((size_t)k * E + e0 + ee) * R + r0 + 4 * c : W_dt;
                cp_async16(gbase + (b_pc(0) - base) + dt_swz(ee, 4 * c), src, ok ? 16u : 0u);
            }
        } else {
            // 4-byte copies: warp w takes rows w + 16 q of both tiles, lane = entry r0 + lane of the row
            constexpr int kW = kDtThreads / 32;
            const bool rok = r0 + lane < R;
            {
                int m = m0 + warp, b = m / sh.T, t = m - b * sh.T;
#pragma unroll 4
                for (int q = 0; q < kDtM / kW; ++q) {
                    const bool okm = rok && m < M;
                    const float* src = okm ? u + u_offset(sh, k, b, t) + r0 + lane : u;
                    cp_async4z(gbase + (a_pc(0) - base) + dt_swz(warp + kW * q, lane), src, okm);
                    m += kW;
                    for (t += kW; t >= sh.T; t -= sh.T) ++b;
                }
            }
#pragma unroll 4
            for (int q = 0; q < kDtN / kW; ++q) {
                const int ee = warp + kW * q;
                const bool oke = rok && e0 + ee < E;
                const float* src = oke ? W_dt + ((size_t)k * E + e0 + ee) * R + r0 + lane : W_dt;
                cp_async4z(gbase + (b_pc(0) - base) + dt_swz(ee, lane), src, oke);
            }
        }
        cp_async_commit();
        cp_async_wait<0>();
        __syncthreads();
        split_tile(a_pc(0));
        split_tile(b_pc(0));
        fence_proxy_async_smem();  // the pieces, written by threads, become visible to the MMAs
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            const int nkk = min(kDtK / 8, (R - r0 + 7) / 8);  // 8-wide k-steps holding entries of dt_low
            for (int kk = 0; kk < nkk; ++kk) {
                const uint32_t step = kk * 32u;  // 8 fp32 entries
                const uint64_t a1 = dt_desc(a_pc(0) + step), a2 = dt_desc(a_pc(1) + step), a3 = dt_desc(a_pc(2) + step);
                const uint64_t b1 = dt_desc(b_pc(0) + step), b2 = dt_desc(b_pc(1) + step), b3 = dt_desc(b_pc(2) + step);
                const uint32_t acc = (r0 | kk) ? 1u : 0u;
                dt_mma(tmem, a1, b1, idesc, acc);
                dt_mma(tmem + kDtN, a3, b1, idesc, acc);
                dt_mma(tmem + kDtN, a2, b2, idesc, 1u);
                dt_mma(tmem + kDtN, a1, b3, idesc, 1u);
                dt_mma(tmem + kDtN, a2, b1, idesc, 1u);
                dt_mma(tmem + kDtN, a1, b2, idesc, 1u);
            }
            dt_commit(&mma_done);
        }
        // the slice's MMAs are done before its tiles are refilled or the accumulators read
        ok = wait_mma((unsigned)(slice & 1));
    }
    tc_fence_after();
    if (ok) {
        // Delta of the tile into shared memory (the operand tiles are free: the MMAs are done),
        // [128 tokens][kDtOS] floats, then out to the Delta rows, 512 contiguous bytes per warp store
        float* out = reinterpret_cast<float*>(gbase);
        const int q = warp & 3, grp = warp >> 2;  // lane quarter, 32-column group
        const int r = 32 * q + lane;             // this thread's token (tensor-memory lane)
        const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16);
#pragma unroll 1
        for (int c0 = 32 * grp; c0 < 32 * grp + 32; c0 += 16) {
            uint32_t vm[16], vc[16];
            tmem_ld16(lane_base + (uint32_t)c0, vm);
            tmem_ld16(lane_base + (uint32_t)(kDtN + c0), vc);
            asm volatile("tcgen05.wait::ld.sync.aligned;" : : : "memory");
#pragma unroll
            for (int j4 = 0; j4 < 4; ++j4) {
                float o[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int jj = 4 * j4 + j;
                    o[j] = softplus_fast((__uint_as_float(vm[jj]) + __uint_as_float(vc[jj])) + s_bias[c0 + jj]);
                }
                *reinterpret_cast<float4*>(out + r * kDtOS + c0 + 4 * j4) = make_float4(o[0], o[1], o[2], o[3]);
            }
        }
        __syncthreads();
        const bool live = e0 + 4 * lane < E;  // E is a multiple of 4
        for (int rr = warp; rr < kDtM; rr += kDtThreads / 32) {
            const int m = m0 + rr;
            if (m >= M) break;
            const int b = m / sh.T, t = m - b * sh.T;
            if (live)
                *reinterpret_cast<float4*>(delta + delta_offset(sh, k, b, t) + e0 + 4 * lane) =
                    *reinterpret_cast<const float4*>(out + rr * kDtOS + 4 * lane);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" : : "r"(tmem), "r"(kDtTmemCols) : "memory");
}

}  // namespace fv
