// kda_internal.cuh -- shared device helpers and launcher prototypes of libkda.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "libkda.h"

namespace kda {

constexpr int kHeadDim = 128;   // d_k = d_v supported by every kernel
constexpr int kChunk = 64;      // chunk length of the prefill (tokens)
constexpr size_t kStatusBytes = 256;  // workspace prefix holding the device status word
// Lowest cumulative log-decay within one chunk (per channel) that the chunked kernels take: they
// factor e^{g_r - g_i} = e^{g_r} e^{-g_i}, and e^{-g} must stay finite in fp32.
constexpr float kMinChunkLogDecay = -80.f;
constexpr int kMaxGridDim = 65535;    // heads and sequences index grid dimensions y and z of the
                                      // chunked kernels

// Two-pass bf16 prefill: per (chunk slot, head) block of prepared operands in the workspace,
// laid out as the scan pass wants them in shared memory (see chunk_prep.cu). The first 66048 bytes
// are contiguous in the same order in the scan's ring stage, so one bulk copy moves a block.
constexpr uint32_t kPrepXOff = 0;           // X = [W; Qt - M W], 128 x 128 f16, 32 KiB
constexpr uint32_t kPrepYOff = 32768;       // Y = [-Tb; M Tb], 128 x 64 f16, 16 KiB
constexpr uint32_t kPrepKEOff = 49152;      // Kend, 64 x 128 f16 (two 64-channel halves), 16 KiB
constexpr uint32_t kPrepGammaOff = 65536;   // gamma, 512 B
constexpr size_t kPrepBlockBytes = 66048;

// Chunk slots per head: slot(sequence n, chunk c) = floor(first token / 64) + n.
__host__ __device__ inline long long prep_slots(long long total_tokens, int n_seqs) {
    return total_tokens / kChunk + n_seqs + 1;
}

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// Records the first device-side error in the workspace status word.
__device__ __forceinline__ void set_status(int32_t *status, int32_t code) {
    if (status) atomicCAS(status, 0, code);
}

#ifndef KDA_DEBUG
#define KDA_DEBUG 0
#endif
// Bounds check of a global access of `n` consecutive elements starting at element `idx` of a
// buffer of `extent` elements. Debug builds (-DKDA_DEBUG=1, the library's stand-in for a memory
// checker) record KDA_ERR_BOUNDS in the status word and return false, and the caller skips the
// access (a skipped load reads zero); release builds compile the check away.
__device__ __forceinline__ bool in_bounds(int32_t *status, long long idx, long long n, long long extent) {
#if KDA_DEBUG
    if (idx < 0 || n < 0 || idx + n > extent) {
        set_status(status, KDA_ERR_BOUNDS);
        return false;
    }
#else
    (void)status; (void)idx; (void)n; (void)extent;
#endif
    return true;
}

// Resolves the token span [t0, t1) of sequence n (flat token index = b * T + t)
// and checks cu_seqlens on the device. Returns false (and flags the status word)
// when the offsets are inconsistent; the caller then skips the sequence.
__device__ __forceinline__ bool sequence_span(const int32_t *cu_seqlens, int n, int N, int T,
                                              int64_t *t0, int64_t *t1, int32_t *status) {
    if (cu_seqlens == nullptr) {
        *t0 = (int64_t)n * T;
        *t1 = *t0 + T;
        return true;
    }
    const int32_t a = cu_seqlens[n], b = cu_seqlens[n + 1];
    bool ok = (a >= 0) && (b >= a) && (b <= T);
    if (n == 0 && a != 0) ok = false;
    if (n == N - 1 && b != T) ok = false;
    if (!ok) {
        set_status(status, KDA_ERR_INVALID_ARG);
        return false;
    }
    *t0 = a;
    *t1 = b;
    return true;
}

struct PrefillArgs {
    const void *q, *k, *v;
    const float *log_alpha, *beta, *S0;
    const int32_t *cu_seqlens;
    void *out;
    float *S_final;
    int B, T, H, N;
    int32_t *status;      // device status word (workspace prefix)
    void *scratch;        // workspace after the status prefix
    size_t scratch_bytes;
    // Backward-pass records written by the fp32 chunk kernel when non-null (one block per
    // (head, chunk slot), see chunk_bwd.cu): the state entering each chunk (d_k x d_v) and the
    // chunk's R = V - Kt S and U (64 x d_v each, rows past the chunk's end zero).
    float *ck_S = nullptr, *ck_R = nullptr, *ck_U = nullptr;
    int n_slots = 0;
};

// Backward-pass record sizes (floats) per (head, chunk slot).
constexpr size_t kBwdStateFloats = (size_t)kHeadDim * kHeadDim;   // 128 x 128
constexpr size_t kBwdRowsFloats = (size_t)kChunk * kHeadDim;       // 64 x 128
constexpr size_t kBwdTriFloats = (size_t)kChunk * kChunk;          // 64 x 64

// The chunk slot of a chunk starting at absolute token s in sequence n (unique per chunk, below
// prep_slots(total_tokens, N)).
__host__ __device__ inline long long chunk_slot(int64_t s, int n) { return s / kChunk + n; }

// Inverse of chunk_slot: the sequence n, first token and length of chunk slot `slot`. Returns
// false for a slot that no chunk uses, or when cu_seqlens is inconsistent (without flagging it:
// the kernels that walk the sequences flag that).
__device__ __forceinline__ bool slot_to_chunk(const int32_t *cu_seqlens, int N, int T, int slot,
                                              int *n_out, int64_t *tok0, int *L)
{
    if (N <= 0) return false;
    int lo = 0, hi = N - 1;                 // largest n with floor(first token of n / 64) + n <= slot
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        const int64_t st = cu_seqlens ? (int64_t)cu_seqlens[mid] : (int64_t)mid * T;
        if (st / kChunk + mid <= slot) lo = mid; else hi = mid - 1;
    }
    const int n = lo;
    int64_t s0, s1;
    if (cu_seqlens) {
        s0 = cu_seqlens[n];
        s1 = cu_seqlens[n + 1];
        if (s1 < s0 || s0 < 0 || s1 > T) return false;
    } else {
        s0 = (int64_t)n * T;
        s1 = s0 + T;
    }
    const int64_t c = slot - (s0 / kChunk + n);
    if (c < 0) return false;
    *tok0 = s0 + c * kChunk;
    if (*tok0 >= s1) return false;
    *L = (s1 - *tok0 < kChunk) ? (int)(s1 - *tok0) : kChunk;
    *n_out = n;
    return true;
}

// CUDA-core fp32 chunk path (any input dtype; fp32 arithmetic throughout).
cudaError_t launch_chunk_fp32(const PrefillArgs &a, kda_dtype_t dtype, kda_dtype_t out_dtype,
                              cudaStream_t stream);

// Tensor-core (tcgen05) chunk path for bf16 q/k/v in one kernel (no workspace beyond the status).
cudaError_t launch_chunk_tc(const PrefillArgs &a, kda_dtype_t out_dtype, cudaStream_t stream);

// The layer's output norm, fused into the output epilogue when given: y = o / sqrt(mean(o^2) + eps)
// * weight * sigmoid(gate), over the d_v channels of each head (gate in the inputs' dtype).
struct NormArgs {
    const void *gate;
    const float *weight;
    float eps;
};

// The layer's gate producers: log_alpha = -exp(A_log[h]) * softplus(f + dt_bias[h, c]) (f NULL:
// log_alpha given), beta = sigmoid(beta_logits) (NULL: beta given); f and beta_logits in the inputs'
// dtype.
struct GateArgs {
    const void *f;
    const float *A_log, *dt_bias;
    const void *beta_logits;
};

// Tensor map of a [tokens][H][128] row-major tensor whose box is `box_cols` channels of the 64 token
// rows of one head, without swizzle or with the 128-byte swizzle (box_cols * elem_bytes = 128).
bool token_rows_map(CUtensorMap *m, const void *base, CUtensorMapDataType dt, uint32_t elem_bytes, int H,
                    long long tokens, uint32_t box_cols = kHeadDim, bool swizzle128 = false);

// Two-pass tensor-core chunk path for bf16 q/k/v: prepared operands go through the workspace.
// (slots [slot_lo, slot_hi) only; slot_hi < 0: to the end)
cudaError_t launch_chunk_prep(const PrefillArgs &a, unsigned char *ws, int n_slots, cudaStream_t stream,
                              const GateArgs *gate = nullptr, int slot_lo = 0, int slot_hi = -1);
// The state scan (chunk_scan.cu), one CTA per (sequence, head), over the chunks whose slots lie in
// [slot_lo, slot_hi) (slot_hi < 0: to the end); a range that does not start a sequence starts from
// S_final, which must then be given.
cudaError_t launch_chunk_scan(const PrefillArgs &a, const unsigned char *ws, int n_slots,
                              kda_dtype_t out_dtype, cudaStream_t stream, const NormArgs *norm = nullptr,
                              long long slot_lo = 0, long long slot_hi = -1);

// The same scan writing the backward pass's forward records (a.ck_S: the state entering every chunk,
// a.ck_U: each chunk's U; both per (head, chunk slot)) instead of outputs; the same slot ranges.
cudaError_t launch_chunk_scan_records(const PrefillArgs &a, const unsigned char *ws, int n_slots,
                                      cudaStream_t stream, long long slot_lo = 0, long long slot_hi = -1);

// The bf16 prefill as kda_chunk_fwd runs it (prefill.cu): with at most kPipeMaxChains (sequence,
// head) chains and enough chunk slots, a pipeline over token ranges (scan of one range beside the
// preparation of the next ones), else the two passes one after the other. The pipeline carries the
// state between ranges in S_final, or in prefill_carry_bytes of workspace after the blocks. With
// records, the scans write the backward's forward records (launch_chunk_scan_records) instead of
// outputs.
constexpr int kPipeMaxChains = 64;
constexpr int kPipeMinSlotsPerRange = 32;
bool prefill_pipelined(long long tokens, int H, int N);
size_t prefill_carry_bytes(long long tokens, int H, int N);
int prefill_launches(long long tokens, int H, int N);   // kernels run_prefill_bf16 launches
cudaError_t run_prefill_bf16(const PrefillArgs &a, kda_dtype_t out_dtype, cudaStream_t stream,
                             const GateArgs *gate, const NormArgs *norm, bool records = false);

// Backward pass (chunk_bwd.cu). Gradient pointers and the records of the forward kernel.
struct BwdArgs {
    const void *q, *k, *v, *dout;
    const float *log_alpha, *beta, *dS_final;
    const int32_t *cu_seqlens;
    float *dq, *dk, *dv, *dlog_alpha, *dbeta, *dS0;
    const float *ck_S, *ck_R, *ck_U;   // from the forward sweep
    float *ck_dS, *ck_Y;               // from the reverse scan
    // state-independent operands of the reverse scan (per (head, slot)), formed by a data-parallel
    // pass before it when given: Kp, Bk, Y0 (64 x 128), G0 (128 x 128), gamma and beta (256 floats);
    // the same pass leaves P = StrictLower(Kt Kh^T) (64 x 64) for the per-chunk kernel
    float *ck_Kp = nullptr, *ck_Bk = nullptr, *ck_Y0 = nullptr, *ck_G0 = nullptr, *ck_gb = nullptr;
    float *ck_P = nullptr;
    int B, T, H, N, n_slots;
    int32_t *status;
};
cudaError_t launch_chunk_bwd_scan(const BwdArgs &a, kda_dtype_t dtype, cudaStream_t stream);
cudaError_t launch_chunk_bwd_local(const BwdArgs &a, kda_dtype_t dtype, cudaStream_t stream);

// Decode step (memory-bound state update in place), optionally with the layer's gate producers
// and output norm.
cudaError_t launch_decode(const void *q, const void *k, const void *v, const float *log_alpha,
                          const float *beta, float *S, void *out, int N, int H,
                          kda_dtype_t dtype, kda_dtype_t out_dtype, cudaStream_t stream,
                          const GateArgs *gate = nullptr, const NormArgs *norm = nullptr);

// Stand-alone layer passes (layer.cu), used around the fp32 CUDA-core prefill: the gate producers
// into fp32 log_alpha / beta, and the gated output norm of fp32 outputs o into out.
cudaError_t launch_gates(const GateArgs &gate, float *log_alpha, float *beta, long long tokens, int H,
                         kda_dtype_t dtype, cudaStream_t stream);
cudaError_t launch_gated_norm(const float *o, const NormArgs &norm, void *out, long long rows,
                              kda_dtype_t dtype, kda_dtype_t out_dtype, cudaStream_t stream);

// Host-side argument checks of the prefill entry points (api.cu) and the launch arguments they build.
kda_status_t check_prefill(const void *q, const void *k, const void *v, const float *log_alpha,
                           const float *beta, const float *S0, const int32_t *cu_seqlens, const void *out,
                           const float *S_final, int B, int T, int H, int N, int dk, int dv,
                           kda_dtype_t dtype, kda_dtype_t out_dtype, const void *workspace,
                           size_t workspace_bytes, bool need_qk, bool need_vout);
PrefillArgs prefill_args(const void *q, const void *k, const void *v, const float *log_alpha,
                         const float *beta, const float *S0, const int32_t *cu_seqlens, void *out,
                         float *S_final, int B, int T, int H, int N, void *workspace, size_t workspace_bytes);

}  // namespace kda
