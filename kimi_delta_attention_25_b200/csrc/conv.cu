// conv.cu -- the short causal convolution in front of the KDA recurrence (kernel size 4 per the
// layer config, short_conv_kernel_size = 4; its rolling inputs are the conv_states the cache keeps
// beside the recurrent states: lpnh.cn Kimi Linear KDA/NoPE article, sec. 3 and 6).
//
// Reading (the pages print no formula): a depthwise convolution over tokens, per channel c,
//   y_t,c = act(bias_c + sum_{j=0}^{K-1} w_c,j x_{t-K+1+j},c)      (taps oldest to newest),
// with the inputs before a sequence's first token taken from its conv state (the last K-1 inputs
// seen before, oldest first; zeros when no state is given), act = SiLU or identity. Optionally each
// head's d-vector of outputs is then L2-normalised, y / sqrt(|y|^2 + 1e-6), which is how q and k
// enter the recurrence (unit-norm keys and queries). The new conv state is the last K-1 inputs.
//
// The conv is a streaming, element-wise pass (8 bytes in and out per bf16 element, 4 flop): one
// warp per (token, head), lane = 4 consecutive channels, so every load and store of a warp is one
// contiguous 256- (bf16) or 512-byte (fp32) row segment; the K-1 earlier rows are re-read through
// L1. The state update is a second launch, one thread per (sequence, channel), so that the
// conv may read the old state while nothing has overwritten it (in-place state buffers are fine).
#include <cuda_runtime.h>

#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int KMAX = 8;         // largest kernel size taken

template <typename T>
__device__ __forceinline__ void load4(const T *p, float (&f)[4]);
template <>
__device__ __forceinline__ void load4<float>(const float *p, float (&f)[4]) {
    const float4 v = *reinterpret_cast<const float4 *>(p);
    f[0] = v.x; f[1] = v.y; f[2] = v.z; f[3] = v.w;
}
template <>
__device__ __forceinline__ void load4<__nv_bfloat16>(const __nv_bfloat16 *p, float (&f)[4]) {
    const uint2 v = *reinterpret_cast<const uint2 *>(p);
    f[0] = __uint_as_float(v.x << 16); f[1] = __uint_as_float(v.x & 0xFFFF0000u);
    f[2] = __uint_as_float(v.y << 16); f[3] = __uint_as_float(v.y & 0xFFFF0000u);
}
template <typename T>
__device__ __forceinline__ void store4(T *p, const float (&f)[4]);
template <>
__device__ __forceinline__ void store4<float>(float *p, const float (&f)[4]) {
    *reinterpret_cast<float4 *>(p) = make_float4(f[0], f[1], f[2], f[3]);
}
template <>
__device__ __forceinline__ void store4<__nv_bfloat16>(__nv_bfloat16 *p, const float (&f)[4]) {
    uint2 v;
    v.x = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(f[0])) |
          ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(f[1])) << 16);
    v.y = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(f[2])) |
          ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(f[3])) << 16);
    *reinterpret_cast<uint2 *>(p) = v;
}

__device__ __forceinline__ float silu(float x) { return x / (1.f + __expf(-x)); }

struct ConvParams {
    const void *x;
    const float *w, *bias, *state;   // w [D, K]; bias [D] or null; state [N, D, K-1] or null
    const int32_t *cu_seqlens;
    void *y;
    int B, T, D, K, N, head_dim;     // head_dim 0: no L2 normalisation
    int silu;
    int32_t *status;
};

// The sequence holding flat token index `tok` (B rows of T tokens, or packed by cu_seqlens) and
// the first token of that sequence.
__device__ __forceinline__ bool token_sequence(const ConvParams &p, long long tok, int *n, long long *first)
{
    if (!p.cu_seqlens) {
        *n = (int)(tok / p.T);
        *first = (long long)(*n) * p.T;
        return true;
    }
    int lo = 0, hi = p.N - 1;                  // largest n with cu[n] <= tok
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (p.cu_seqlens[mid] <= tok) lo = mid; else hi = mid - 1;
    }
    // skip empty sequences that start at the same token
    while (lo + 1 < p.N && p.cu_seqlens[lo + 1] <= tok) ++lo;
    *n = lo;
    *first = p.cu_seqlens[lo];
    return tok < p.cu_seqlens[lo + 1];
}

template <typename T>
__global__ void __launch_bounds__(256) short_conv_kernel(ConvParams p)
{
    const long long rows = (long long)p.B * p.T;
    const int groups = p.D / (4 * 32);        // warps per token (128 channels each)
    const long long wid = (long long)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (wid >= rows * groups) return;         // warp-uniform
    const long long tok = wid / groups;
    const int c0 = (int)(wid % groups) * 128 + 4 * lane;
    int n;
    long long first;
    if (!token_sequence(p, tok, &n, &first)) return;   // padding token past the last sequence
    const T *x = (const T *)p.x;
    float acc[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[e] = p.bias ? p.bias[c0 + e] : 0.f;
    for (int j = 0; j < p.K; ++j) {            // tap j multiplies the input K-1-j tokens back
        const long long src = tok - (p.K - 1) + j;
        float xv[4];
        if (src >= first) {
            load4(x + src * p.D + c0, xv);
        } else if (p.state) {                  // history: state slot (K-1) - (first - src)
            const int slot = (p.K - 1) - (int)(first - src);
#pragma unroll
            for (int e = 0; e < 4; ++e) xv[e] = p.state[((size_t)n * p.D + c0 + e) * (p.K - 1) + slot];
        } else {
#pragma unroll
            for (int e = 0; e < 4; ++e) xv[e] = 0.f;
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[e] += p.w[(size_t)(c0 + e) * p.K + j] * xv[e];
    }
    if (p.silu) {
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[e] = silu(acc[e]);
    }
    if (p.head_dim) {                          // head_dim 128: this warp's 128 channels are one head
        float ss = acc[0] * acc[0] + acc[1] * acc[1] + acc[2] * acc[2] + acc[3] * acc[3];
#pragma unroll
        for (int m = 16; m > 0; m >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
        const float r = rsqrtf(ss + 1e-6f);
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[e] *= r;
    }
    store4((T *)p.y + tok * p.D + c0, acc);
}

// New conv state of every sequence: the last K-1 inputs, oldest first (old state shifted in when
// the sequence is shorter than K-1). One thread per (sequence, channel), so a state buffer may be
// updated in place.
template <typename T>
__global__ void conv_state_kernel(ConvParams p, float *state_out)
{
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (long long)p.N * p.D) return;
    const int n = (int)(i / p.D), c = (int)(i % p.D);
    long long s0, s1;
    if (p.cu_seqlens) { s0 = p.cu_seqlens[n]; s1 = p.cu_seqlens[n + 1]; }
    else { s0 = (long long)n * p.T; s1 = s0 + p.T; }
    const long long L = s1 - s0;
    const int H1 = p.K - 1;
    float old[KMAX], nw[KMAX];
    for (int j = 0; j < H1; ++j) old[j] = p.state ? p.state[((size_t)n * p.D + c) * H1 + j] : 0.f;
    const T *x = (const T *)p.x;
    for (int j = 0; j < H1; ++j) {             // ext = [old, x_s0 .. x_s1-1]; new[j] = ext[L + j]
        const long long e = L + j;
        nw[j] = (e < H1) ? old[e] : to_f32(x[(s0 + e - H1) * p.D + c]);
    }
    for (int j = 0; j < H1; ++j) state_out[((size_t)n * p.D + c) * H1 + j] = nw[j];
}

// One decode step: y = act(bias + w . [state, x]) per channel (optionally L2-normalised per head),
// state <- [state[1:], x]. One warp per (sequence, 128 channels).
template <typename T>
__global__ void __launch_bounds__(256) short_conv_step_kernel(ConvParams p, float *state)
{
    const int groups = p.D / 128;
    const long long wid = (long long)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (wid >= (long long)p.N * groups) return;
    const int n = (int)(wid / groups);
    const int c0 = (int)(wid % groups) * 128 + 4 * lane;
    const int H1 = p.K - 1;
    float xv[4];
    load4((const T *)p.x + (size_t)n * p.D + c0, xv);
    float acc[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const size_t sb = ((size_t)n * p.D + c0 + e) * H1;
        float a = p.bias ? p.bias[c0 + e] : 0.f;
        for (int j = 0; j < H1; ++j) a += p.w[(size_t)(c0 + e) * p.K + j] * state[sb + j];
        a += p.w[(size_t)(c0 + e) * p.K + H1] * xv[e];
        for (int j = 0; j + 1 < H1; ++j) state[sb + j] = state[sb + j + 1];
        if (H1 > 0) state[sb + H1 - 1] = xv[e];
        acc[e] = p.silu ? silu(a) : a;
    }
    if (p.head_dim) {
        float ss = acc[0] * acc[0] + acc[1] * acc[1] + acc[2] * acc[2] + acc[3] * acc[3];
#pragma unroll
        for (int m = 16; m > 0; m >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
        const float r = rsqrtf(ss + 1e-6f);
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[e] *= r;
    }
    store4((T *)p.y + (size_t)n * p.D + c0, acc);
}

bool al(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }

kda_status_t check_conv(const void *x, const float *w, const float *bias, const void *y, int D, int K,
                        int head_dim, int silu, kda_dtype_t dtype)
{
    if (dtype != KDA_F32 && dtype != KDA_BF16) return KDA_ERR_INVALID_ARG;
    if (D <= 0 || K < 1 || silu < 0 || silu > 1) return KDA_ERR_INVALID_ARG;
    if (K > KMAX || D % 128 != 0) return KDA_ERR_UNSUPPORTED;
    if (head_dim != 0 && head_dim != kHeadDim) return KDA_ERR_UNSUPPORTED;
    if (!w || !al(w, 4) || (bias && !al(bias, 4))) return KDA_ERR_INVALID_ARG;
    if ((x && !al(x, 16)) || (y && !al(y, 16))) return KDA_ERR_INVALID_ARG;
    return KDA_OK;
}

}  // namespace
}  // namespace kda

using namespace kda;

extern "C" {

kda_status_t kda_short_conv(const void *x, const float *weight, const float *bias,
                            const float *conv_state, float *conv_state_out, const int32_t *cu_seqlens,
                            void *y, int B, int T, int N, int D, int K, int activation_silu,
                            int normalize_head_dim, kda_dtype_t dtype, void *stream)
{
    kda_status_t s = check_conv(x, weight, bias, y, D, K, normalize_head_dim, activation_silu, dtype);
    if (s != KDA_OK) return s;
    if (B < 0 || T < 0 || N < 0) return KDA_ERR_INVALID_ARG;
    if (cu_seqlens) {
        if (B != 1 || !al(cu_seqlens, 4)) return KDA_ERR_INVALID_ARG;
    } else if (N != B) {
        return KDA_ERR_INVALID_ARG;
    }
    const long long rows = (long long)B * T;
    if (rows > 0 && (!x || !y)) return KDA_ERR_INVALID_ARG;
    if ((conv_state && !al(conv_state, 4)) || (conv_state_out && !al(conv_state_out, 4))) return KDA_ERR_INVALID_ARG;
    if (rows * D > 0x7fffffffffffLL) return KDA_ERR_INVALID_ARG;
    ConvParams p;
    p.x = x; p.w = weight; p.bias = bias; p.state = conv_state; p.cu_seqlens = cu_seqlens; p.y = y;
    p.B = B; p.T = T; p.D = D; p.K = K; p.N = N; p.head_dim = normalize_head_dim; p.silu = activation_silu;
    p.status = nullptr;
    cudaStream_t st = (cudaStream_t)stream;
    const long long warps = rows * (D / 128);
    if (warps > 0) {
        const long long blocks = (warps + 7) / 8;
        if (blocks > 0x7fffffffLL) return KDA_ERR_INVALID_ARG;
        if (dtype == KDA_BF16) short_conv_kernel<__nv_bfloat16><<<(unsigned)blocks, 256, 0, st>>>(p);
        else short_conv_kernel<float><<<(unsigned)blocks, 256, 0, st>>>(p);
        if (cudaGetLastError() != cudaSuccess) return KDA_ERR_CUDA;
    }
    if (conv_state_out && N > 0 && K > 1) {    // after the conv (which reads the old state)
        const long long th = (long long)N * D;
        const unsigned blocks = (unsigned)((th + 255) / 256);
        if (dtype == KDA_BF16) conv_state_kernel<__nv_bfloat16><<<blocks, 256, 0, st>>>(p, conv_state_out);
        else conv_state_kernel<float><<<blocks, 256, 0, st>>>(p, conv_state_out);
        if (cudaGetLastError() != cudaSuccess) return KDA_ERR_CUDA;
    }
    return KDA_OK;
}

kda_status_t kda_short_conv_step(const void *x, const float *weight, const float *bias, float *conv_state,
                                 void *y, int N, int D, int K, int activation_silu, int normalize_head_dim,
                                 kda_dtype_t dtype, void *stream)
{
    kda_status_t s = check_conv(x, weight, bias, y, D, K, normalize_head_dim, activation_silu, dtype);
    if (s != KDA_OK) return s;
    if (N < 0) return KDA_ERR_INVALID_ARG;
    if (N == 0) return KDA_OK;
    if (!x || !y || (K > 1 && (!conv_state || !al(conv_state, 4)))) return KDA_ERR_INVALID_ARG;
    ConvParams p;
    p.x = x; p.w = weight; p.bias = bias; p.state = conv_state; p.cu_seqlens = nullptr; p.y = y;
    p.B = N; p.T = 1; p.D = D; p.K = K; p.N = N; p.head_dim = normalize_head_dim; p.silu = activation_silu;
    p.status = nullptr;
    const long long warps = (long long)N * (D / 128);
    const unsigned blocks = (unsigned)((warps + 7) / 8);
    cudaStream_t st = (cudaStream_t)stream;
    if (dtype == KDA_BF16) short_conv_step_kernel<__nv_bfloat16><<<blocks, 256, 0, st>>>(p, conv_state);
    else short_conv_step_kernel<float><<<blocks, 256, 0, st>>>(p, conv_state);
    return cudaGetLastError() == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

}  // extern "C"
