// layer.cu -- the KDA layer's element-wise neighbours of the recurrence: the decay-gate producer
// (A_log, dt_bias and the low-rank projection output f), the write gate from its logits, and the
// gated RMSNorm of the outputs (o_norm = FusedRMSNormGated with a sigmoid gate). The pages name
// these parts of the module (lpnh.cn Kimi Linear KDA/NoPE article, sec. 3 and 4) but print no
// formula; the readings are
//   log_alpha = -exp(A_log[h]) * softplus(f + dt_bias[h, c]),   beta = sigmoid(b),
//   y = o / sqrt(mean_c o_c^2 + eps) * w * sigmoid(g)   over the d_v channels of one head.
//
// For bf16 inputs they are fused into the prefill's two passes (chunk_prep.cu forms log_alpha and
// beta from their inputs as it loads them; chunk_scan.cu normalises in its output epilogue, the
// four warps of a token group adding their sums of squares) and into the decode kernel. This file holds the entry points and, for fp32 inputs,
// two stand-alone passes around the CUDA-core prefill: the gates into fp32 scratch, and the norm of
// the fp32 outputs.
#include <cuda_runtime.h>

#include "kda_internal.cuh"

namespace kda {
namespace {

bool aligned_to(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }

__device__ __forceinline__ float softplus_l(float x) { return x > 20.f ? x : log1pf(__expf(x)); }
__device__ __forceinline__ float sigmoid_l(float x) { return 1.f / (1.f + __expf(-x)); }

// log_alpha for 4 consecutive channels per thread; beta per (token, head).
template <typename T>
__global__ void gates_kernel(const T *__restrict__ f, const float *__restrict__ A_log, const float *__restrict__ dt_bias,
                             const T *__restrict__ b, float *__restrict__ log_alpha, float *__restrict__ beta,
                             long long rows, int H)
{
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;     // row * 32 + channel quad
    if (f && i < rows * (kHeadDim / 4)) {
        const long long row = i / (kHeadDim / 4);
        const int c = (int)(i % (kHeadDim / 4)) * 4, h = (int)(row % H);
        const float rate = expf(A_log[h]);
        float4 o;
        o.x = -rate * softplus_l(to_f32(f[row * kHeadDim + c + 0]) + dt_bias[(size_t)h * kHeadDim + c + 0]);
        o.y = -rate * softplus_l(to_f32(f[row * kHeadDim + c + 1]) + dt_bias[(size_t)h * kHeadDim + c + 1]);
        o.z = -rate * softplus_l(to_f32(f[row * kHeadDim + c + 2]) + dt_bias[(size_t)h * kHeadDim + c + 2]);
        o.w = -rate * softplus_l(to_f32(f[row * kHeadDim + c + 3]) + dt_bias[(size_t)h * kHeadDim + c + 3]);
        *reinterpret_cast<float4 *>(log_alpha + row * kHeadDim + c) = o;
    }
    if (b && i < rows) beta[i] = sigmoid_l(to_f32(b[i]));
}

// One warp per (token, head) row of d_v = 128 outputs, 4 per lane.
template <typename T, typename TO>
__global__ void gated_norm_kernel(const float *__restrict__ o, const T *__restrict__ g, const float *__restrict__ w,
                                  float eps, TO *__restrict__ out, long long rows)
{
    const long long row = (long long)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    const float4 x = *reinterpret_cast<const float4 *>(o + row * kHeadDim + 4 * lane);
    float ss = x.x * x.x + x.y * x.y + x.z * x.z + x.w * x.w;
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
    const float rinv = rsqrtf(ss * (1.f / kHeadDim) + eps);
    const float xv[4] = {x.x, x.y, x.z, x.w};
    TO *dst = out + row * kHeadDim + 4 * lane;
#pragma unroll
    for (int e = 0; e < 4; ++e)
        dst[e] = from_f32<TO>(xv[e] * rinv * w[4 * lane + e] * sigmoid_l(to_f32(g[row * kHeadDim + 4 * lane + e])));
}

bool has_any(const kda_layer_opts_t *o)
{
    return o && (o->gate_f || o->beta_logits || o->out_gate);
}

// Layer-option checks; fills the internal argument structs.
kda_status_t check_opts(const kda_layer_opts_t *o, GateArgs *gate, NormArgs *norm, bool *use_gate, bool *use_norm)
{
    *use_gate = false;
    *use_norm = false;
    if (!o) return KDA_OK;
    if (o->gate_f) {
        if (!o->A_log || !o->dt_bias) return KDA_ERR_INVALID_ARG;
        if (!aligned_to(o->gate_f, 16) || !aligned_to(o->A_log, 4) || !aligned_to(o->dt_bias, 16))
            return KDA_ERR_INVALID_ARG;
    }
    if (o->beta_logits && !aligned_to(o->beta_logits, 4)) return KDA_ERR_INVALID_ARG;
    if (o->out_gate) {
        if (!o->norm_weight || !aligned_to(o->out_gate, 16) || !aligned_to(o->norm_weight, 4))
            return KDA_ERR_INVALID_ARG;
        if (!(o->norm_eps >= 0.f) || o->norm_eps > 3.0e38f) return KDA_ERR_INVALID_ARG;
    }
    gate->f = o->gate_f;
    gate->A_log = o->A_log;
    gate->dt_bias = o->dt_bias;
    gate->beta_logits = o->beta_logits;
    norm->gate = o->out_gate;
    norm->weight = o->norm_weight;
    norm->eps = o->norm_eps;
    *use_gate = o->gate_f || o->beta_logits;
    *use_norm = o->out_gate != nullptr;
    return KDA_OK;
}

size_t align16(size_t x) { return (x + 15) & ~(size_t)15; }

// fp32-input scratch after the status prefix: [log_alpha][beta][o before the norm]
struct Fp32Scratch {
    size_t la, beta, o, total;
};
Fp32Scratch fp32_scratch(long long tokens, int H, const kda_layer_opts_t *o, kda_dtype_t out_dtype)
{
    Fp32Scratch s = {};
    size_t off = kStatusBytes;
    if (o && o->gate_f) { s.la = off; off += align16((size_t)tokens * H * kHeadDim * 4); }
    if (o && o->beta_logits) { s.beta = off; off += align16((size_t)tokens * H * 4); }
    if (o && o->out_gate && out_dtype != KDA_F32) { s.o = off; off += align16((size_t)tokens * H * kHeadDim * 4); }
    s.total = off;
    return s;
}

}  // namespace

cudaError_t launch_gates(const GateArgs &gate, float *log_alpha, float *beta, long long tokens, int H,
                         kda_dtype_t dtype, cudaStream_t stream)
{
    const long long rows = tokens * H;
    if (rows == 0) return cudaSuccess;
    const long long work = gate.f ? rows * (kHeadDim / 4) : rows;
    const unsigned blocks = (unsigned)((work + 255) / 256);
    if (dtype == KDA_BF16)
        gates_kernel<__nv_bfloat16><<<blocks, 256, 0, stream>>>(
            (const __nv_bfloat16 *)gate.f, gate.A_log, gate.dt_bias, (const __nv_bfloat16 *)gate.beta_logits,
            log_alpha, beta, rows, H);
    else
        gates_kernel<float><<<blocks, 256, 0, stream>>>((const float *)gate.f, gate.A_log, gate.dt_bias,
                                                        (const float *)gate.beta_logits, log_alpha, beta, rows, H);
    return cudaGetLastError();
}

cudaError_t launch_gated_norm(const float *o, const NormArgs &norm, void *out, long long rows,
                              kda_dtype_t dtype, kda_dtype_t out_dtype, cudaStream_t stream)
{
    if (rows == 0) return cudaSuccess;
    const unsigned blocks = (unsigned)((rows + 7) / 8);        // 8 rows (warps) per block
    using bf = __nv_bfloat16;
    if (dtype == KDA_BF16 && out_dtype == KDA_BF16)
        gated_norm_kernel<bf, bf><<<blocks, 256, 0, stream>>>(o, (const bf *)norm.gate, norm.weight, norm.eps, (bf *)out, rows);
    else if (dtype == KDA_BF16)
        gated_norm_kernel<bf, float><<<blocks, 256, 0, stream>>>(o, (const bf *)norm.gate, norm.weight, norm.eps, (float *)out, rows);
    else if (out_dtype == KDA_BF16)
        gated_norm_kernel<float, bf><<<blocks, 256, 0, stream>>>(o, (const float *)norm.gate, norm.weight, norm.eps, (bf *)out, rows);
    else
        gated_norm_kernel<float, float><<<blocks, 256, 0, stream>>>(o, (const float *)norm.gate, norm.weight, norm.eps, (float *)out, rows);
    return cudaGetLastError();
}

}  // namespace kda

using namespace kda;

extern "C" {

size_t kda_chunk_fwd_layer_workspace_size(int B, int T, int H, int N, int dk, int dv, kda_dtype_t dtype,
                                          const kda_layer_opts_t *opts)
{
    const size_t base = kda_chunk_fwd_workspace_size(B, T, H, N, dk, dv, dtype);
    if (base == 0 || dtype == KDA_BF16) return base;
    // fp32 inputs: the norm scratch depends on out_dtype; size it for a bf16 output (the larger)
    return fp32_scratch((long long)B * T, H, opts, KDA_BF16).total;
}

kda_status_t kda_chunk_fwd_layer(const void *q, const void *k, const void *v,
                                 const float *log_alpha, const float *beta,
                                 const float *S0, const int32_t *cu_seqlens,
                                 void *out, float *S_final,
                                 int B, int T, int H, int N, int dk, int dv,
                                 kda_dtype_t dtype, kda_dtype_t out_dtype,
                                 const kda_layer_opts_t *opts,
                                 void *workspace, size_t workspace_bytes, void *stream)
{
    if (!has_any(opts))
        return kda_chunk_fwd(q, k, v, log_alpha, beta, S0, cu_seqlens, out, S_final, B, T, H, N, dk, dv, dtype,
                             out_dtype, workspace, workspace_bytes, stream);
    GateArgs gate;
    NormArgs norm;
    bool use_gate, use_norm;
    kda_status_t s = check_opts(opts, &gate, &norm, &use_gate, &use_norm);
    if (s != KDA_OK) return s;
    // the produced gates stand in for log_alpha / beta in the common checks (same alignment rules)
    const float *la_chk = opts->gate_f ? (const float *)opts->gate_f : log_alpha;
    const float *be_chk = opts->beta_logits ? (const float *)opts->beta_logits : beta;
    s = check_prefill(q, k, v, la_chk, be_chk, S0, cu_seqlens, out, S_final, B, T, H, N, dk, dv, dtype, out_dtype,
                      workspace, workspace_bytes, true, true);
    if (s != KDA_OK) return s;
    const long long tokens = (long long)B * T;
    if (dtype == KDA_F32 && workspace_bytes < fp32_scratch(tokens, H, opts, out_dtype).total)
        return KDA_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    if (cudaMemsetAsync(workspace, 0, kStatusBytes, st) != cudaSuccess) return KDA_ERR_CUDA;
    if (N == 0) return KDA_OK;
    PrefillArgs a = prefill_args(q, k, v, log_alpha, beta, S0, cu_seqlens, out, S_final, B, T, H, N, workspace,
                                 workspace_bytes);
    cudaError_t e = cudaSuccess;
    if (dtype == KDA_BF16) {
        e = run_prefill_bf16(a, out_dtype, st, use_gate ? &gate : nullptr, use_norm ? &norm : nullptr);
        return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
    }
    // fp32 inputs: gates -> fp32 scratch, CUDA-core prefill, norm of its fp32 outputs
    const Fp32Scratch sc = fp32_scratch(tokens, H, opts, out_dtype);
    unsigned char *w = (unsigned char *)workspace;
    if (use_gate) {
        float *la = opts->gate_f ? (float *)(w + sc.la) : nullptr;
        float *bt = opts->beta_logits ? (float *)(w + sc.beta) : nullptr;
        e = launch_gates(gate, la, bt, tokens, H, dtype, st);
        if (la) a.log_alpha = la;
        if (bt) a.beta = bt;
    }
    float *o32 = nullptr;
    if (use_norm) {
        o32 = (out_dtype == KDA_F32) ? (float *)out : (float *)(w + sc.o);   // in place for fp32 outputs
        a.out = o32;
    }
    if (e == cudaSuccess) e = launch_chunk_fp32(a, dtype, use_norm ? KDA_F32 : out_dtype, st);
    if (e == cudaSuccess && use_norm) e = launch_gated_norm(o32, norm, out, tokens * H, dtype, out_dtype, st);
    return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

kda_status_t kda_chunk_prep_layer(const void *q, const void *k, const float *log_alpha, const float *beta,
                                  const int32_t *cu_seqlens, int B, int T, int H, int N, int dk, int dv,
                                  const kda_layer_opts_t *opts, void *workspace, size_t workspace_bytes,
                                  void *stream)
{
    GateArgs gate;
    NormArgs norm;
    bool use_gate, use_norm;
    kda_status_t s = check_opts(opts, &gate, &norm, &use_gate, &use_norm);
    if (s != KDA_OK) return s;
    const float *la_chk = (opts && opts->gate_f) ? (const float *)opts->gate_f : log_alpha;
    const float *be_chk = (opts && opts->beta_logits) ? (const float *)opts->beta_logits : beta;
    s = check_prefill(q, k, nullptr, la_chk, be_chk, nullptr, cu_seqlens, nullptr, nullptr, B, T, H, N, dk, dv,
                      KDA_BF16, KDA_BF16, workspace, workspace_bytes, true, false);
    if (s != KDA_OK) return s;
    cudaStream_t st = (cudaStream_t)stream;
    if (cudaMemsetAsync(workspace, 0, kStatusBytes, st) != cudaSuccess) return KDA_ERR_CUDA;
    if (N == 0) return KDA_OK;
    const PrefillArgs a = prefill_args(q, k, nullptr, log_alpha, beta, nullptr, cu_seqlens, nullptr, nullptr, B, T,
                                       H, N, workspace, workspace_bytes);
    return launch_chunk_prep(a, (unsigned char *)a.scratch, (int)prep_slots((long long)B * T, N), st,
                             use_gate ? &gate : nullptr) == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

kda_status_t kda_chunk_scan_layer(const void *v, const float *S0, const int32_t *cu_seqlens, void *out,
                                  float *S_final, int B, int T, int H, int N, int dk, int dv, kda_dtype_t out_dtype,
                                  const kda_layer_opts_t *opts, void *workspace, size_t workspace_bytes,
                                  void *stream)
{
    GateArgs gate;
    NormArgs norm;
    bool use_gate, use_norm;
    kda_status_t s = check_opts(opts, &gate, &norm, &use_gate, &use_norm);
    if (s != KDA_OK) return s;
    s = check_prefill(nullptr, nullptr, v, nullptr, nullptr, S0, cu_seqlens, out, S_final, B, T, H, N, dk, dv,
                      KDA_BF16, out_dtype, workspace, workspace_bytes, false, true);
    if (s != KDA_OK) return s;
    if (N == 0) return KDA_OK;
    const PrefillArgs a = prefill_args(nullptr, nullptr, v, nullptr, nullptr, S0, cu_seqlens, out, S_final, B, T,
                                       H, N, workspace, workspace_bytes);
    return launch_chunk_scan(a, (const unsigned char *)a.scratch, (int)prep_slots((long long)B * T, N), out_dtype,
                             (cudaStream_t)stream, use_norm ? &norm : nullptr) == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

kda_status_t kda_decode_step_layer(const void *q, const void *k, const void *v,
                                   const float *log_alpha, const float *beta,
                                   float *S_inout, void *out,
                                   int N, int H, int dk, int dv, kda_dtype_t dtype,
                                   kda_dtype_t out_dtype, const kda_layer_opts_t *opts, void *stream)
{
    if (!has_any(opts))
        return kda_decode_step(q, k, v, log_alpha, beta, S_inout, out, N, H, dk, dv, dtype, out_dtype, stream);
    GateArgs gate;
    NormArgs norm;
    bool use_gate, use_norm;
    kda_status_t s = check_opts(opts, &gate, &norm, &use_gate, &use_norm);
    if (s != KDA_OK) return s;
    if (dtype != KDA_F32 && dtype != KDA_BF16) return KDA_ERR_INVALID_ARG;
    if (out_dtype != KDA_F32 && out_dtype != KDA_BF16) return KDA_ERR_INVALID_ARG;
    if (N < 0 || H <= 0) return KDA_ERR_INVALID_ARG;
    if (dk != kHeadDim || dv != kHeadDim) return KDA_ERR_UNSUPPORTED;
    if (N == 0) return KDA_OK;
    if ((long long)N * H > 0x7fffffffLL) return KDA_ERR_INVALID_ARG;
    const void *la = opts->gate_f ? opts->gate_f : log_alpha;
    const void *bt = opts->beta_logits ? opts->beta_logits : beta;
    if (!q || !k || !v || !la || !bt || !S_inout || !out) return KDA_ERR_INVALID_ARG;
    if (!aligned_to(q, 16) || !aligned_to(k, 16) || !aligned_to(v, 16) || !aligned_to(out, 16) ||
        !aligned_to(la, 16) || !aligned_to(S_inout, 16) || !aligned_to(bt, 4))
        return KDA_ERR_INVALID_ARG;
    const cudaError_t e = launch_decode(q, k, v, log_alpha, beta, S_inout, out, N, H, dtype, out_dtype,
                                        (cudaStream_t)stream, use_gate ? &gate : nullptr, use_norm ? &norm : nullptr);
    return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

}  // extern "C"
