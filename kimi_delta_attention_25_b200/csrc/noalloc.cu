// noalloc.cu -- kda_chunk_fwd_noalloc: the chunked prefill for callers that cannot allocate
// device memory.
//
// Who needs it: plug-ins hosted by a runtime that owns all device memory and hands out only fixed
// input/output buffers, and memory-capped serving processes that must not grow their footprint
// per request. kda_chunk_fwd asks such callers for a workspace they
// cannot provide; this entry point instead uses a small scratch array that is part of the library
// image itself.
//
// The scratch is a file-scope __device__ array of kNoAllocScratchBytes (4 KiB). Every GPU on which
// the library is loaded holds it until the process exits. Its first 256 bytes are the status
// header that the kernels write their device-side checks to (the same layout as a workspace).
// Host code cannot use the array's name as a device address (on the host it only names a shadow
// symbol); the device address is looked up once per device with cudaGetSymbolAddress, with that
// device current, on the first call made on that device, and cached.
#include <cuda_runtime.h>

#include <mutex>

#include "kda_internal.cuh"

namespace {

constexpr size_t kNoAllocScratchBytes = KDA_NOALLOC_SCRATCH_BYTES;
static_assert(kNoAllocScratchBytes >= kda::kStatusBytes, "scratch must hold the status header");

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_scratch_addr[kMaxDevices] = {};

bool aligned_to(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }

// Device address of the scratch array on the current device (looked up once per device).
kda_status_t scratch_address(void **addr)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return KDA_ERR_CUDA;
    if (dev >= kMaxDevices) return KDA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return KDA_ERR_CUDA;
        g_scratch_addr[dev] = p;
    }
    *addr = g_scratch_addr[dev];
    return KDA_OK;
}

}  // namespace

extern "C" kda_status_t kda_chunk_fwd_noalloc(const void *q, const void *k, const void *v,
                                              const float *log_alpha, const float *beta,
                                              const float *S0, const int32_t *cu_seqlens,
                                              void *out, float *S_final,
                                              int B, int T, int H, int N, int dk, int dv,
                                              kda_dtype_t dtype, kda_dtype_t out_dtype, void *stream)
{
    using namespace kda;
    // the same host-side checks as kda_chunk_fwd
    if (dtype != KDA_F32 && dtype != KDA_BF16) return KDA_ERR_INVALID_ARG;
    if (out_dtype != KDA_F32 && out_dtype != KDA_BF16) return KDA_ERR_INVALID_ARG;
    if (B < 0 || T < 0 || H <= 0 || N < 0) return KDA_ERR_INVALID_ARG;
    if (dk != kHeadDim || dv != kHeadDim) return KDA_ERR_UNSUPPORTED;
    if (H > kMaxGridDim || N > kMaxGridDim) return KDA_ERR_UNSUPPORTED;
    if (cu_seqlens) {
        if (B != 1 || !aligned_to(cu_seqlens, 4)) return KDA_ERR_INVALID_ARG;
    } else if (N != B) {
        return KDA_ERR_INVALID_ARG;
    }
    if ((long long)B * T > 0x7fffffffLL) return KDA_ERR_INVALID_ARG;
    if ((long long)B * T > 0) {
        if (!q || !k || !v || !log_alpha || !beta || !out) return KDA_ERR_INVALID_ARG;
        if (!aligned_to(q, 16) || !aligned_to(k, 16) || !aligned_to(v, 16) || !aligned_to(out, 16) ||
            !aligned_to(log_alpha, 16) || !aligned_to(beta, 4))
            return KDA_ERR_INVALID_ARG;
    }
    if ((S0 && !aligned_to(S0, 16)) || (S_final && !aligned_to(S_final, 16))) return KDA_ERR_INVALID_ARG;
    // This entry point runs the single-kernel prefill, whose only scratch is the status header;
    // a need beyond the static array is refused.
    const size_t need = kStatusBytes;
    if (need > kNoAllocScratchBytes) return KDA_ERR_UNSUPPORTED;

    void *scratch = nullptr;
    kda_status_t st = scratch_address(&scratch);
    if (st != KDA_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    // the array keeps the previous call's contents: clear the status header
    if (cudaMemsetAsync(scratch, 0, kStatusBytes, s) != cudaSuccess) return KDA_ERR_CUDA;
    if (N == 0) return KDA_OK;

    PrefillArgs a;
    a.q = q; a.k = k; a.v = v; a.log_alpha = log_alpha; a.beta = beta; a.S0 = S0;
    a.cu_seqlens = cu_seqlens; a.out = out; a.S_final = S_final;
    a.B = B; a.T = T; a.H = H; a.N = N;
    a.status = (int32_t *)scratch;
    a.scratch = (unsigned char *)scratch + kStatusBytes;
    a.scratch_bytes = kNoAllocScratchBytes - kStatusBytes;
    // bf16 inputs: the single-kernel tensor-core prefill (its decay-range check and the cu_seqlens
    // check land in the status header); fp32 inputs: the CUDA-core prefill
    const cudaError_t e = (dtype == KDA_BF16) ? launch_chunk_tc(a, out_dtype, s)
                                              : launch_chunk_fp32(a, dtype, out_dtype, s);
    return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

extern "C" kda_status_t kda_chunk_fwd_noalloc_status(void *stream, int32_t *status)
{
    if (!status) return KDA_ERR_INVALID_ARG;
    void *scratch = nullptr;
    kda_status_t st = scratch_address(&scratch);
    if (st != KDA_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    int32_t v = 0;
    cudaError_t e = cudaMemcpyAsync(&v, scratch, sizeof(v), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return KDA_ERR_CUDA;
    *status = v;
    return KDA_OK;
}
