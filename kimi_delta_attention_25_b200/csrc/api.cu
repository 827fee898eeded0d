// api.cu -- the extern "C" entry points of libkda: argument checks, then kernel launches.
//
// Every check that can be made from the host is made here, before anything is enqueued, and
// reported as a status code. The one check that needs device data (the contents of cu_seqlens)
// is made by the kernels, which record it in the caller's workspace status word.
#include <cuda_runtime.h>

#include "kda_internal.cuh"

using namespace kda;

namespace {

bool aligned(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }

kda_status_t map_cuda(cudaError_t e) { return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA; }

}  // namespace

extern "C" {

int kda_version(void) { return 100; }

const char *kda_status_string(kda_status_t s)
{
    switch (s) {
    case KDA_OK: return "ok";
    case KDA_ERR_INVALID_ARG: return "invalid argument";
    case KDA_ERR_UNSUPPORTED: return "unsupported (size, or a decay outside the range)";
    case KDA_ERR_CUDA: return "CUDA error";
    case KDA_ERR_TIMEOUT: return "device wait timed out";
    case KDA_ERR_BOUNDS: return "global index out of bounds (debug build)";
    }
    return "unknown status";
}

size_t kda_chunk_fwd_workspace_size(int B, int T, int H, int N, int dk, int dv, kda_dtype_t dtype)
{
    if (B < 0 || T < 0 || H <= 0 || N < 0 || dk != kHeadDim || dv != kHeadDim) return 0;
    if (dtype != KDA_F32 && dtype != KDA_BF16) return 0;
    if (dtype == KDA_F32) return kStatusBytes;
    // bf16: prepared operands of every (chunk slot, head), then the state carried between the token
    // ranges of the pipelined prefill (when it applies)
    return kStatusBytes + (size_t)H * (size_t)prep_slots((long long)B * T, N) * kPrepBlockBytes +
           prefill_carry_bytes((long long)B * T, H, N);
}

}  // extern "C"

namespace kda {

// Host-side checks shared by the prefill entry points. `need_*` selects which tensors the caller
// passes (the two passes of the bf16 path each take a subset).
kda_status_t check_prefill(const void *q, const void *k, const void *v, const float *log_alpha,
                           const float *beta, const float *S0, const int32_t *cu_seqlens, const void *out,
                           const float *S_final, int B, int T, int H, int N, int dk, int dv,
                           kda_dtype_t dtype, kda_dtype_t out_dtype, const void *workspace,
                           size_t workspace_bytes, bool need_qk, bool need_vout)
{
    if (dtype != KDA_F32 && dtype != KDA_BF16) return KDA_ERR_INVALID_ARG;
    if (out_dtype != KDA_F32 && out_dtype != KDA_BF16) return KDA_ERR_INVALID_ARG;
    if (B < 0 || T < 0 || H <= 0 || N < 0) return KDA_ERR_INVALID_ARG;
    if (dk != kHeadDim || dv != kHeadDim) return KDA_ERR_UNSUPPORTED;
    if (H > kMaxGridDim || N > kMaxGridDim) return KDA_ERR_UNSUPPORTED;
    if (cu_seqlens) {
        if (B != 1) return KDA_ERR_INVALID_ARG;
        if (!aligned(cu_seqlens, 4)) return KDA_ERR_INVALID_ARG;
    } else if (N != B) {
        return KDA_ERR_INVALID_ARG;
    }
    if ((long long)B * T > 0x7fffffffLL) return KDA_ERR_INVALID_ARG;
    // the preparation pass launches one CTA per (chunk slot, head)
    if (dtype == KDA_BF16 && (long long)H * prep_slots((long long)B * T, N) > 0x7fffffffLL)
        return KDA_ERR_UNSUPPORTED;
    if ((long long)B * T > 0) {
        if (need_qk && (!q || !k || !log_alpha || !beta)) return KDA_ERR_INVALID_ARG;
        if (need_vout && (!v || !out)) return KDA_ERR_INVALID_ARG;
        if ((need_qk && (!aligned(q, 16) || !aligned(k, 16) || !aligned(log_alpha, 16) || !aligned(beta, 4))) ||
            (need_vout && (!aligned(v, 16) || !aligned(out, 16))))
            return KDA_ERR_INVALID_ARG;
    }
    if ((S0 && !aligned(S0, 16)) || (S_final && !aligned(S_final, 16))) return KDA_ERR_INVALID_ARG;
    const size_t need = kda_chunk_fwd_workspace_size(B, T, H, N, dk, dv, dtype);
    if (!workspace || !aligned(workspace, 16) || workspace_bytes < need) return KDA_ERR_INVALID_ARG;
    return KDA_OK;
}

PrefillArgs prefill_args(const void *q, const void *k, const void *v, const float *log_alpha,
                         const float *beta, const float *S0, const int32_t *cu_seqlens, void *out,
                         float *S_final, int B, int T, int H, int N, void *workspace, size_t workspace_bytes)
{
    PrefillArgs a;
    a.q = q; a.k = k; a.v = v; a.log_alpha = log_alpha; a.beta = beta; a.S0 = S0;
    a.cu_seqlens = cu_seqlens; a.out = out; a.S_final = S_final;
    a.B = B; a.T = T; a.H = H; a.N = N;
    a.status = (int32_t *)workspace;
    a.scratch = (unsigned char *)workspace + kStatusBytes;
    a.scratch_bytes = workspace_bytes - kStatusBytes;
    return a;
}

}  // namespace kda

extern "C" {

kda_status_t kda_chunk_fwd(const void *q, const void *k, const void *v,
                           const float *log_alpha, const float *beta,
                           const float *S0, const int32_t *cu_seqlens,
                           void *out, float *S_final,
                           int B, int T, int H, int N, int dk, int dv,
                           kda_dtype_t dtype, kda_dtype_t out_dtype,
                           void *workspace, size_t workspace_bytes, void *stream)
{
    kda_status_t s = check_prefill(q, k, v, log_alpha, beta, S0, cu_seqlens, out, S_final, B, T, H, N,
                                   dk, dv, dtype, out_dtype, workspace, workspace_bytes, true, true);
    if (s != KDA_OK) return s;
    cudaStream_t st = (cudaStream_t)stream;
    if (cudaMemsetAsync(workspace, 0, kStatusBytes, st) != cudaSuccess) return KDA_ERR_CUDA;
    if (N == 0) return KDA_OK;
    const PrefillArgs a = prefill_args(q, k, v, log_alpha, beta, S0, cu_seqlens, out, S_final,
                                       B, T, H, N, workspace, workspace_bytes);
    if (dtype == KDA_BF16) return map_cuda(run_prefill_bf16(a, out_dtype, st, nullptr, nullptr));
    return map_cuda(launch_chunk_fp32(a, dtype, out_dtype, st));
}

kda_status_t kda_chunk_prep(const void *q, const void *k, const float *log_alpha, const float *beta,
                            const int32_t *cu_seqlens, int B, int T, int H, int N, int dk, int dv,
                            void *workspace, size_t workspace_bytes, void *stream)
{
    kda_status_t s = check_prefill(q, k, nullptr, log_alpha, beta, nullptr, cu_seqlens, nullptr, nullptr,
                                   B, T, H, N, dk, dv, KDA_BF16, KDA_BF16, workspace, workspace_bytes,
                                   true, false);
    if (s != KDA_OK) return s;
    cudaStream_t st = (cudaStream_t)stream;
    if (cudaMemsetAsync(workspace, 0, kStatusBytes, st) != cudaSuccess) return KDA_ERR_CUDA;
    if (N == 0) return KDA_OK;
    const PrefillArgs a = prefill_args(q, k, nullptr, log_alpha, beta, nullptr, cu_seqlens, nullptr,
                                       nullptr, B, T, H, N, workspace, workspace_bytes);
    return map_cuda(launch_chunk_prep(a, (unsigned char *)a.scratch, (int)prep_slots((long long)B * T, N), st));
}

kda_status_t kda_chunk_scan(const void *v, const float *S0, const int32_t *cu_seqlens, void *out,
                            float *S_final, int B, int T, int H, int N, int dk, int dv,
                            kda_dtype_t out_dtype, void *workspace, size_t workspace_bytes, void *stream)
{
    kda_status_t s = check_prefill(nullptr, nullptr, v, nullptr, nullptr, S0, cu_seqlens, out, S_final,
                                   B, T, H, N, dk, dv, KDA_BF16, out_dtype, workspace, workspace_bytes,
                                   false, true);
    if (s != KDA_OK) return s;
    if (N == 0) return KDA_OK;
    const PrefillArgs a = prefill_args(nullptr, nullptr, v, nullptr, nullptr, S0, cu_seqlens, out, S_final,
                                       B, T, H, N, workspace, workspace_bytes);
    return map_cuda(launch_chunk_scan(a, (const unsigned char *)a.scratch, (int)prep_slots((long long)B * T, N), out_dtype,
                                      (cudaStream_t)stream));
}

int kda_chunk_fwd_kernel_launches(int B, int T, int H, int N, kda_dtype_t dtype)
{
    if (B < 0 || T < 0 || H <= 0 || N < 0 || (dtype != KDA_F32 && dtype != KDA_BF16)) return 0;
    if (N == 0) return 0;
    if (dtype == KDA_F32) return 1;
    return prefill_launches((long long)B * T, H, N);
}

size_t kda_chunk_bwd_workspace_size(int B, int T, int H, int N, int dk, int dv)
{
    if (B < 0 || T < 0 || H <= 0 || N < 0 || dk != kHeadDim || dv != kHeadDim) return 0;
    // S, dS'; R, U, Y; then the reverse scan's prepared operands Kp, Bk, Y0; G0; gamma and beta;
    // P for the per-chunk kernel
    const size_t per = 2 * kBwdStateFloats + 3 * kBwdRowsFloats + 3 * kBwdRowsFloats + kBwdStateFloats + 256 +
                       kBwdTriFloats;
    return kStatusBytes + (size_t)H * (size_t)prep_slots((long long)B * T, N) * per * sizeof(float);
}

}  // extern "C"

namespace {

// The backward's host checks and launches; `phases` selects which of the three kernels to enqueue
// (bit 0: forward sweep with records, also clearing the status word; bit 1: reverse scan of the
// state gradient; bit 2: per-chunk gradients).
kda_status_t chunk_bwd_impl(unsigned phases, const void *q, const void *k, const void *v,
                            const float *log_alpha, const float *beta, const float *S0,
                            const int32_t *cu_seqlens, const void *dout, const float *dS_final,
                            float *dq, float *dk_out, float *dv_out, float *dlog_alpha, float *dbeta,
                            float *dS0, int B, int T, int H, int N, int dk, int dv, kda_dtype_t dtype,
                            void *workspace, size_t workspace_bytes, void *stream)
{
    if (dtype != KDA_F32 && dtype != KDA_BF16) return KDA_ERR_INVALID_ARG;
    if (B < 0 || T < 0 || H <= 0 || N < 0) return KDA_ERR_INVALID_ARG;
    if (dk != kHeadDim || dv != kHeadDim) return KDA_ERR_UNSUPPORTED;
    if (H > kMaxGridDim || N > kMaxGridDim) return KDA_ERR_UNSUPPORTED;
    if (cu_seqlens) {
        if (B != 1 || !aligned(cu_seqlens, 4)) return KDA_ERR_INVALID_ARG;
    } else if (N != B) {
        return KDA_ERR_INVALID_ARG;
    }
    const long long total = (long long)B * T;
    if (total > 0x7fffffffLL) return KDA_ERR_INVALID_ARG;
    const long long n_slots = prep_slots(total, N);
    if ((long long)H * n_slots > 0x7fffffffLL) return KDA_ERR_UNSUPPORTED;
    if (total > 0) {
        if (!q || !k || !v || !log_alpha || !beta || !dout || !dq || !dk_out || !dv_out || !dlog_alpha || !dbeta)
            return KDA_ERR_INVALID_ARG;
        if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(log_alpha, 16) ||
            !aligned(dout, 16) || !aligned(dq, 16) || !aligned(dk_out, 16) || !aligned(dv_out, 16) ||
            !aligned(dlog_alpha, 16) || !aligned(beta, 4) || !aligned(dbeta, 4))
            return KDA_ERR_INVALID_ARG;
    }
    if ((S0 && !aligned(S0, 16)) || (dS_final && !aligned(dS_final, 16)) || (dS0 && !aligned(dS0, 16)))
        return KDA_ERR_INVALID_ARG;
    const size_t need = kda_chunk_bwd_workspace_size(B, T, H, N, dk, dv);
    if (!workspace || !aligned(workspace, 16) || workspace_bytes < need) return KDA_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    if ((phases & 1u) && cudaMemsetAsync(workspace, 0, kStatusBytes, st) != cudaSuccess) return KDA_ERR_CUDA;
    if (N == 0) return KDA_OK;

    // records: S and dS' per (head, slot), then R, U, Y
    float *base = (float *)((unsigned char *)workspace + kStatusBytes);
    const size_t hs = (size_t)H * (size_t)n_slots;
    float *ck_S = base;
    float *ck_dS = ck_S + hs * kBwdStateFloats;
    float *ck_R = ck_dS + hs * kBwdStateFloats;
    float *ck_U = ck_R + hs * kBwdRowsFloats;
    float *ck_Y = ck_U + hs * kBwdRowsFloats;
    float *ck_Kp = ck_Y + hs * kBwdRowsFloats;
    float *ck_Bk = ck_Kp + hs * kBwdRowsFloats;
    float *ck_Y0 = ck_Bk + hs * kBwdRowsFloats;
    float *ck_G0 = ck_Y0 + hs * kBwdRowsFloats;
    float *ck_gb = ck_G0 + hs * kBwdStateFloats;
    float *ck_P = ck_gb + hs * 256;

    cudaError_t e = cudaSuccess;
    // bf16 inputs take the forward records from the tensor-core passes, which write S and U but not
    // R (the per-chunk kernel forms it); their prepared blocks sit in the dS' and R areas, which
    // the reverse scan rewrites and nothing reads until then
    const bool tc = dtype == KDA_BF16;
    if (phases & 1u) {              // 1. forward sweep with records (outputs not needed)
        PrefillArgs a = prefill_args(q, k, v, log_alpha, beta, S0, cu_seqlens, nullptr, nullptr, B, T, H, N,
                                     workspace, workspace_bytes);
        a.ck_S = ck_S; a.ck_U = ck_U; a.n_slots = (int)n_slots;
        if (tc) {
            static_assert(kPrepBlockBytes <= (kBwdStateFloats + kBwdRowsFloats) * sizeof(float),
                          "prepared blocks fit the dS' and R areas");
            // the two passes as the forward runs them (pipelined over token ranges when few chains);
            // the state carried between ranges goes to the G0 area, written only later
            a.scratch = ck_dS;
            a.S_final = ck_G0;
            e = run_prefill_bf16(a, KDA_F32, st, nullptr, nullptr, /*records=*/true);
        } else {
            a.ck_R = ck_R;
            e = launch_chunk_fp32(a, dtype, KDA_F32, st);
        }
    }
    BwdArgs b;
    b.q = q; b.k = k; b.v = v; b.dout = dout;
    b.log_alpha = log_alpha; b.beta = beta; b.dS_final = dS_final;
    b.cu_seqlens = cu_seqlens;
    b.dq = dq; b.dk = dk_out; b.dv = dv_out; b.dlog_alpha = dlog_alpha; b.dbeta = dbeta; b.dS0 = dS0;
    b.ck_S = ck_S; b.ck_R = tc ? nullptr : ck_R; b.ck_U = ck_U; b.ck_dS = ck_dS; b.ck_Y = ck_Y;
    b.ck_Kp = ck_Kp; b.ck_Bk = ck_Bk; b.ck_Y0 = ck_Y0; b.ck_G0 = ck_G0; b.ck_gb = ck_gb; b.ck_P = ck_P;
    b.B = B; b.T = T; b.H = H; b.N = N; b.n_slots = (int)n_slots;
    b.status = (int32_t *)workspace;
    if (e == cudaSuccess && (phases & 2u)) e = launch_chunk_bwd_scan(b, dtype, st);   // 2. reverse scan
    if (e == cudaSuccess && (phases & 4u)) e = launch_chunk_bwd_local(b, dtype, st);  // 3. per chunk
    return map_cuda(e);
}

}  // namespace

extern "C" {

kda_status_t kda_chunk_bwd(const void *q, const void *k, const void *v,
                           const float *log_alpha, const float *beta,
                           const float *S0, const int32_t *cu_seqlens,
                           const void *dout, const float *dS_final,
                           float *dq, float *dk_out, float *dv_out,
                           float *dlog_alpha, float *dbeta, float *dS0,
                           int B, int T, int H, int N, int dk, int dv, kda_dtype_t dtype,
                           void *workspace, size_t workspace_bytes, void *stream)
{
    return chunk_bwd_impl(7u, q, k, v, log_alpha, beta, S0, cu_seqlens, dout, dS_final, dq, dk_out, dv_out,
                          dlog_alpha, dbeta, dS0, B, T, H, N, dk, dv, dtype, workspace, workspace_bytes, stream);
}

kda_status_t kda_chunk_bwd_phase(int phase, const void *q, const void *k, const void *v,
                                 const float *log_alpha, const float *beta,
                                 const float *S0, const int32_t *cu_seqlens,
                                 const void *dout, const float *dS_final,
                                 float *dq, float *dk_out, float *dv_out,
                                 float *dlog_alpha, float *dbeta, float *dS0,
                                 int B, int T, int H, int N, int dk, int dv, kda_dtype_t dtype,
                                 void *workspace, size_t workspace_bytes, void *stream)
{
    if (phase < 0 || phase > 2) return KDA_ERR_INVALID_ARG;
    return chunk_bwd_impl(1u << phase, q, k, v, log_alpha, beta, S0, cu_seqlens, dout, dS_final, dq, dk_out,
                          dv_out, dlog_alpha, dbeta, dS0, B, T, H, N, dk, dv, dtype, workspace, workspace_bytes,
                          stream);
}

kda_status_t kda_decode_step(const void *q, const void *k, const void *v,
                             const float *log_alpha, const float *beta,
                             float *S_inout, void *out,
                             int N, int H, int dk, int dv, kda_dtype_t dtype,
                             kda_dtype_t out_dtype, void *stream)
{
    if (dtype != KDA_F32 && dtype != KDA_BF16) return KDA_ERR_INVALID_ARG;
    if (out_dtype != KDA_F32 && out_dtype != KDA_BF16) return KDA_ERR_INVALID_ARG;
    if (N < 0 || H <= 0) return KDA_ERR_INVALID_ARG;
    if (dk != kHeadDim || dv != kHeadDim) return KDA_ERR_UNSUPPORTED;
    if (N == 0) return KDA_OK;
    if ((long long)N * H > 0x7fffffffLL) return KDA_ERR_INVALID_ARG;
    if (!q || !k || !v || !log_alpha || !beta || !S_inout || !out) return KDA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) ||
        !aligned(log_alpha, 16) || !aligned(S_inout, 16) || !aligned(beta, 4))
        return KDA_ERR_INVALID_ARG;
    return map_cuda(launch_decode(q, k, v, log_alpha, beta, S_inout, out, N, H, dtype, out_dtype,
                                  (cudaStream_t)stream));
}

kda_status_t kda_workspace_status(const void *workspace, void *stream, int32_t *status)
{
    if (!workspace || !status) return KDA_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    int32_t v = 0;
    cudaError_t e = cudaMemcpyAsync(&v, workspace, sizeof(v), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return KDA_ERR_CUDA;
    *status = v;
    return KDA_OK;
}

}  // extern "C"
