// chunk_fp32_common.cuh -- building blocks of the fp32 CUDA-core chunk kernels (the fp32 forward
// in chunk_fp32.cu and the backward in chunk_bwd.cu): vectorised chunk loads, the per-channel
// decay scan, and the blocked unit-triangular solves of the WY form.
#pragma once

#include "kda_internal.cuh"

namespace kda {
namespace fp32c {

constexpr int C = kChunk;
constexpr int DK = kHeadDim;

__device__ __forceinline__ void unpack16(const uint4 &x, float *f, float)
{
    f[0] = __uint_as_float(x.x); f[1] = __uint_as_float(x.y);
    f[2] = __uint_as_float(x.z); f[3] = __uint_as_float(x.w);
}
__device__ __forceinline__ void unpack16(const uint4 &x, float *f, __nv_bfloat16)
{
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

// Loads rows s..s+63 (zero past L) of a [tokens, H, 128] tensor, columns col0..col0+W-1 of head h,
// into dst[r * ld + j] as fp32. All of a thread's 16-byte loads are issued before any is used.
// Needs 16-byte aligned rows (base aligned, 128-element rows) and col0 a multiple of 8.
template <typename T, int NT, int W>
__device__ __forceinline__ void load_rows(float *dst, int ld, const T *src, int64_t s, int L, int H, int h,
                                          int col0, int tid)
{
    constexpr int VEC = 16 / (int)sizeof(T);
    constexpr int PER_ROW = W / VEC;
    constexpr int TOTAL = C * PER_ROW;
    constexpr int NV = (TOTAL + NT - 1) / NT;
    uint4 x[NV];
#pragma unroll
    for (int it = 0; it < NV; ++it) {
        const int idx = tid + it * NT, r = idx / PER_ROW, cv = idx % PER_ROW;
        x[it] = make_uint4(0u, 0u, 0u, 0u);
        if (idx < TOTAL && r < L)
            x[it] = __ldg(reinterpret_cast<const uint4 *>(src + ((size_t)(s + r) * H + h) * DK + col0 + cv * VEC));
    }
#pragma unroll
    for (int it = 0; it < NV; ++it) {
        const int idx = tid + it * NT, r = idx / PER_ROW, cv = idx % PER_ROW;
        if (idx < TOTAL) {
            float f[VEC];
            unpack16(x[it], f, T());
#pragma unroll
            for (int e = 0; e < VEC; ++e) dst[r * ld + cv * VEC + e] = f[e];
        }
    }
}

// Loads one chunk's rows of q, k (into Qd, Kd), log_alpha (into Gd), all 64 x 128 with row stride
// ld, and the 32 columns j0.. of a value-shaped tensor (into Vd, row stride 32); rows past L are
// zero. Every 16-byte load of the thread is in flight before the first one is stored.
template <typename T, int NT>
__device__ __forceinline__ void load_chunk(float *Kd, float *Qd, float *Gd, int ld, float *Vd,
                                           const T *q, const T *k, const float *la, const T *vsrc,
                                           int64_t s, int L, int H, int h, int j0, int tid)
{
    constexpr int VT = 16 / (int)sizeof(T), PRT = DK / VT, NQ = C * PRT / NT;
    constexpr int PRF = DK / 4, NF = C * PRF / NT;
    constexpr int PRV = 32 / VT, TV = C * PRV, NV = (TV + NT - 1) / NT;
    static_assert(NQ * NT == C * PRT && NF * NT == C * PRF, "thread count must divide the tile");
    uint4 xq[NQ], xk[NQ], xl[NF], xv[NV];
    const uint4 z = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int it = 0; it < NQ; ++it) {
        const int idx = tid + it * NT, r = idx / PRT, cv = idx % PRT;
        const size_t off = ((size_t)(s + r) * H + h) * DK + cv * VT;
        xq[it] = (r < L) ? __ldg(reinterpret_cast<const uint4 *>(q + off)) : z;
        xk[it] = (r < L) ? __ldg(reinterpret_cast<const uint4 *>(k + off)) : z;
    }
#pragma unroll
    for (int it = 0; it < NF; ++it) {
        const int idx = tid + it * NT, r = idx / PRF, cv = idx % PRF;
        xl[it] = (r < L) ? __ldg(reinterpret_cast<const uint4 *>(la + ((size_t)(s + r) * H + h) * DK + cv * 4)) : z;
    }
#pragma unroll
    for (int it = 0; it < NV; ++it) {
        const int idx = tid + it * NT, r = idx / PRV, cv = idx % PRV;
        xv[it] = (idx < TV && r < L)
                     ? __ldg(reinterpret_cast<const uint4 *>(vsrc + ((size_t)(s + r) * H + h) * DK + j0 + cv * VT))
                     : z;
    }
#pragma unroll
    for (int it = 0; it < NQ; ++it) {
        const int idx = tid + it * NT, r = idx / PRT, cv = idx % PRT;
        float fq[VT], fk[VT];
        unpack16(xq[it], fq, T());
        unpack16(xk[it], fk, T());
#pragma unroll
        for (int e = 0; e < VT; ++e) { Qd[r * ld + cv * VT + e] = fq[e]; Kd[r * ld + cv * VT + e] = fk[e]; }
    }
#pragma unroll
    for (int it = 0; it < NF; ++it) {
        const int idx = tid + it * NT, r = idx / PRF, cv = idx % PRF;
        float f[4];
        unpack16(xl[it], f, 0.f);
#pragma unroll
        for (int e = 0; e < 4; ++e) Gd[r * ld + cv * 4 + e] = f[e];
    }
#pragma unroll
    for (int it = 0; it < NV; ++it) {
        const int idx = tid + it * NT, r = idx / PRV, cv = idx % PRV;
        if (idx < TV) {
            float f[VT];
            unpack16(xv[it], f, T());
#pragma unroll
            for (int e = 0; e < VT; ++e) Vd[r * 32 + cv * VT + e] = f[e];
        }
    }
}

// acc[0..N) += a * x[0..N) with 16-byte shared-memory loads (x 16-byte aligned, N a multiple of 4).
template <int N>
__device__ __forceinline__ void axpy(float *acc, float a, const float *x)
{
#pragma unroll
    for (int i = 0; i < N / 4; ++i) {
        const float4 v = reinterpret_cast<const float4 *>(x)[i];
        acc[4 * i] += a * v.x; acc[4 * i + 1] += a * v.y; acc[4 * i + 2] += a * v.z; acc[4 * i + 3] += a * v.w;
    }
}

// Cumulative log-decay per key channel over the chunk's 64 rows, split into NT / 128 row parts
// that run at once: on entry G[r * ld + c] holds log_alpha; on exit the inclusive prefix sum g.
// Returns, for the calling thread's channel c = tid % 128, g_63 (the whole chunk's sum; rows past
// the chunk's end hold zero, so this is g_{L-1}).
template <int NT>
__device__ __forceinline__ float decay_prefix(float *G, int ld, int tid)
{
    constexpr int P = NT / DK, RP = C / P;
    const int c = tid % DK, part = tid / DK, r0 = part * RP;
    float g = 0.f;
#pragma unroll 8
    for (int r = r0; r < r0 + RP; ++r) { g += G[r * ld + c]; G[r * ld + c] = g; }
    __syncthreads();
    float tot[P];
#pragma unroll
    for (int p = 0; p < P; ++p) tot[p] = G[(p * RP + RP - 1) * ld + c];
    __syncthreads();                       // every part's total is read before any row changes
    float off = 0.f, gl = 0.f;
#pragma unroll
    for (int p = 0; p < P; ++p) { off += (p < part) ? tot[p] : 0.f; gl += tot[p]; }
    if (part > 0) {
#pragma unroll 8
        for (int r = r0; r < r0 + RP; ++r) G[r * ld + c] += off;
    }
    __syncthreads();
    return gl;
}

// U <- (I + A)^{-1} U for a strictly lower A (64 x 64, row stride lda) and 32 columns of U (row
// stride 32), by 16-row blocks: the block's right-hand side minus the solved blocks above it
// (all threads), then forward substitution inside the block (one thread per column).
template <int NT>
__device__ __forceinline__ void lower_solve_32(const float *A, int lda, float *U, int tid)
{
    static_assert(NT >= 256, "two outputs per thread in the block update");
#pragma unroll 1
    for (int b = 0; b < 4; ++b) {
        if (b > 0 && tid < 256) {
            const int r = 16 * b + (tid >> 4), j = (tid & 15) * 2;
            float a0 = U[r * 32 + j], a1 = U[r * 32 + j + 1];
            for (int i = 0; i < 16 * b; ++i) {
                const float a = A[r * lda + i];
                a0 -= a * U[i * 32 + j];
                a1 -= a * U[i * 32 + j + 1];
            }
            U[r * 32 + j] = a0;
            U[r * 32 + j + 1] = a1;
        }
        __syncthreads();
        if (tid < 32) {
            const int j = tid;
            float u[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                float x = U[(16 * b + r) * 32 + j];
#pragma unroll
                for (int i = 0; i < r; ++i) x -= A[(16 * b + r) * lda + 16 * b + i] * u[i];
                u[r] = x;
                U[(16 * b + r) * 32 + j] = x;
            }
        }
        __syncthreads();
    }
}

// Y <- (I + A)^{-T} Y (A strictly lower, so I + A^T is unit upper triangular), by 16-row blocks
// from the last: the block's right-hand side minus the solved blocks below it, then back
// substitution inside the block.
template <int NT>
__device__ __forceinline__ void upper_solve_32(const float *A, int lda, float *Y, int tid)
{
    static_assert(NT >= 256, "two outputs per thread in the block update");
#pragma unroll 1
    for (int b = 3; b >= 0; --b) {
        if (b < 3 && tid < 256) {
            const int r = 16 * b + (tid >> 4), j = (tid & 15) * 2;
            float a0 = Y[r * 32 + j], a1 = Y[r * 32 + j + 1];
            for (int i = 16 * (b + 1); i < C; ++i) {
                const float a = A[i * lda + r];
                a0 -= a * Y[i * 32 + j];
                a1 -= a * Y[i * 32 + j + 1];
            }
            Y[r * 32 + j] = a0;
            Y[r * 32 + j + 1] = a1;
        }
        __syncthreads();
        if (tid < 32) {
            const int j = tid;
            float y[16];
#pragma unroll
            for (int r = 15; r >= 0; --r) {
                float x = Y[(16 * b + r) * 32 + j];
#pragma unroll
                for (int i = r + 1; i < 16; ++i) x -= A[(16 * b + i) * lda + 16 * b + r] * y[i];
                y[r] = x;
                Y[(16 * b + r) * 32 + j] = x;
            }
        }
        __syncthreads();
    }
}

// dst[r * dst_ld + j] = scale_r * src[r * 32 + j] for r < rows, 32 columns, with 16-byte accesses
// (dst and dst_ld 16-byte aligned; src rows of 32 floats). scale = nullptr means 1.
template <int NT>
__device__ __forceinline__ void store_block32(float *dst, size_t dst_ld, const float *src, int rows, int tid,
                                              const float *scale = nullptr)
{
    for (int idx = tid; idx < rows * 8; idx += NT) {
        const int r = idx >> 3, q = idx & 7;
        float4 v = *reinterpret_cast<const float4 *>(src + r * 32 + 4 * q);
        if (scale) {
            const float b = scale[r];
            v.x *= b; v.y *= b; v.z *= b; v.w *= b;
        }
        *reinterpret_cast<float4 *>(dst + (size_t)r * dst_ld + 4 * q) = v;
    }
}

}  // namespace fp32c
}  // namespace kda
