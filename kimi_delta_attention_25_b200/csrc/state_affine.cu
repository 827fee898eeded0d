// state_affine.cu -- S_out = Phi S_in + Psi per head (fp32): composing the affine state maps of
// consecutive segments of one sequence. A segment of the recurrence maps its entering state S to
// its final state as S -> Phi S + Psi (the recurrence is linear in the state: Phi is the product of
// the segment's transitions (I - beta k k^T) Diag(alpha), Psi the final state from S = 0), so a
// sequence split over several devices (context parallelism) needs only each segment's (Phi, Psi)
// to find every segment's entering state; the pages do not describe this split.
//
// Plain fp32 CUDA-core arithmetic: 2 * 128^3 flops per head, negligible next to the prefill.
// One CTA per (head, 32 x 32 output tile), Phi and S_in tiles staged in shared memory.
#include <cuda_runtime.h>

#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int TS = 32;

__global__ void __launch_bounds__(256) state_affine_kernel(const float *__restrict__ Phi, const float *__restrict__ S_in,
                                                           const float *__restrict__ Psi, float *__restrict__ S_out)
{
    const int h = blockIdx.z, r0 = blockIdx.y * TS, c0 = blockIdx.x * TS;
    const size_t base = (size_t)h * kHeadDim * kHeadDim;
    __shared__ float a[TS][TS + 1], b[TS][TS + 1];
    const int tx = threadIdx.x % TS, ty = threadIdx.x / TS;      // 32 x 8 threads, 4 rows each
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int k0 = 0; k0 < kHeadDim; k0 += TS) {
        for (int i = ty; i < TS; i += 8) {
            a[i][tx] = Phi[base + (size_t)(r0 + i) * kHeadDim + k0 + tx];
            b[i][tx] = S_in[base + (size_t)(k0 + i) * kHeadDim + c0 + tx];
        }
        __syncthreads();
#pragma unroll 8
        for (int kk = 0; kk < TS; ++kk) {
            const float bv = b[kk][tx];
#pragma unroll
            for (int u = 0; u < 4; ++u) acc[u] += a[ty + 8 * u][kk] * bv;
        }
        __syncthreads();
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const size_t o = base + (size_t)(r0 + ty + 8 * u) * kHeadDim + c0 + tx;
        S_out[o] = acc[u] + (Psi ? Psi[o] : 0.f);
    }
}

}  // namespace
}  // namespace kda

extern "C" kda_status_t kda_state_affine(const float *Phi, const float *S_in, const float *Psi, float *S_out,
                                         int H, int dk, int dv, void *stream)
{
    using namespace kda;
    if (H < 0) return KDA_ERR_INVALID_ARG;
    if (dk != kHeadDim || dv != kHeadDim) return KDA_ERR_UNSUPPORTED;
    if (H == 0) return KDA_OK;
    if (H > kMaxGridDim) return KDA_ERR_UNSUPPORTED;
    if (!Phi || !S_in || !S_out) return KDA_ERR_INVALID_ARG;
    if (S_out == S_in || S_out == Phi) return KDA_ERR_INVALID_ARG;
    const dim3 grid(kHeadDim / TS, kHeadDim / TS, H);
    state_affine_kernel<<<grid, 256, 0, (cudaStream_t)stream>>>(Phi, S_in, Psi, S_out);
    return cudaGetLastError() == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}
