/*
 * libkda.h -- C ABI of libkda, a B200 (sm_100a) implementation of the KDA
 * (Kimi Delta Attention) layer's hot path: chunkwise prefill and the decode step.
 *
 * The operation (every head keeps a d_k x d_v state S):
 *
 *     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T ,   o_t = S_t^T q_t
 *
 * alpha_t = exp(log_alpha_t) in (0, 1]^{d_k} is the channel-wise forget gate,
 * beta_t in [0, 1] the write gate. KDA is described as Gated DeltaNet with
 * fine-grained, per-channel gates ("Kimi Linear" article (jdon.com), the
 * passage on KDA's gating; KimiLinear KDA/MLA tutorial (icman.com.cn), sec. 2:
 * fixed-size state, channel-level gating); the erase term (I - beta k k^T)
 * and the need for unit-norm keys come from the same tutorial, sec. 5. The
 * pages print no formula; the order "decay, erase and write, then read" is the
 * plainest reading of that delta-rule update. The layer hands q/k/v over as
 * "... h d" (lpnh.cn Kimi Linear KDA/NoPE article, sec. 4), so tensors here
 * are laid out token-major with heads inside, the head dimension fastest.
 *
 * General rules for every call:
 *  - All tensor pointers are DEVICE pointers owned by the caller. The library
 *    allocates no device memory; scratch comes from the caller's workspace.
 *  - Tensors are dense, row-major, last index fastest, with no padding.
 *  - q, k, v, out, log_alpha, S0, S_final, S_inout and workspace must be
 *    16-byte aligned; beta and cu_seqlens 4-byte aligned. A misaligned or
 *    NULL required pointer returns KDA_ERR_INVALID_ARG before any launch.
 *  - Only d_k = d_v = 128 is implemented; other sizes return KDA_ERR_UNSUPPORTED.
 *  - The chunked calls (prefill, its passes, its backward) take at most 65535 heads
 *    and 65535 sequences (one launch-grid dimension each); more return
 *    KDA_ERR_UNSUPPORTED. The decode step takes any N x H below 2^31.
 *  - q and k are expected to be L2-normalised per head (a precondition of the
 *    layer, not applied here). log_alpha must be finite and <= 0, beta in [0, 1];
 *    neither is checked. The chunked prefill (kda_chunk_fwd, its passes and its
 *    backward, for either input dtype) additionally needs the cumulative log-decay
 *    inside one 64-token chunk to stay at or above -80 per channel (exp of its
 *    negation must be finite in fp32). That check needs device data, so the call
 *    returns KDA_OK and a chunk outside the range writes KDA_ERR_UNSUPPORTED to the
 *    workspace status word (read it with kda_workspace_status); the outputs of such a
 *    call are not usable. kda_chunk_fwd_noalloc with bf16 inputs has a narrower range
 *    (see there). The decode step has no such limit.
 *  - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL is the
 *    legacy default stream). A KDA_ERR_CUDA return means a launch failed.
 *  - Calls are thread-safe; concurrent calls must not share output buffers
 *    or workspaces.
 *  - Errors are returned, never thrown.
 */
#ifndef LIBKDA_H
#define LIBKDA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    KDA_OK = 0,
    KDA_ERR_INVALID_ARG = 1,   /* bad pointer, size, alignment or cu_seqlens content */
    KDA_ERR_UNSUPPORTED = 2,   /* valid but not implemented: d_k, d_v != 128, more heads or
                                * sequences than a launch grid holds, or (in a status word)
                                * a chunk whose decay is outside the supported range */
    KDA_ERR_CUDA = 3,          /* a CUDA runtime call or launch failed */
    KDA_ERR_TIMEOUT = 4,       /* a bounded device-side wait gave up */
    KDA_ERR_BOUNDS = 5         /* debug builds only (libkda_debug.so): a kernel computed a global
                                * index outside its buffer and skipped that access */
} kda_status_t;

typedef enum {
    KDA_F32 = 0,               /* float32 */
    KDA_BF16 = 1               /* bfloat16 (round-to-nearest-even on output) */
} kda_dtype_t;

/* Bytes of device workspace kda_chunk_fwd needs for these sizes (always >= 256;
 * the first 256 bytes hold the device status word read by kda_workspace_status).
 * For bf16 inputs the workspace also holds the per-chunk operands that the first of the
 * two prefill passes prepares for the second: 66048 bytes per (chunk slot, head), with
 * floor(B*T/64) + N + 1 chunk slots per head (about 1 KiB per token and head), and, when
 * kda_chunk_fwd pipelines its two passes (see there), N*H*dk*dv*4 bytes that carry the state
 * between token ranges.
 * Returns 0 for sizes kda_chunk_fwd would reject. */
size_t kda_chunk_fwd_workspace_size(int B, int T, int H, int N, int dk, int dv,
                                    kda_dtype_t dtype);

/* Number of kernels one kda_chunk_fwd call with these sizes launches (for profiling and launch
 * accounting; the bf16 layer variant kda_chunk_fwd_layer launches as many). 0 for sizes the call
 * rejects or that launch nothing. */
int kda_chunk_fwd_kernel_launches(int B, int T, int H, int N, kda_dtype_t dtype);

/* Chunkwise-parallel prefill (chunk of 64 tokens): the recurrence above over
 * every sequence and head, returning every o_t and the final state.
 * Chunked form with a WY (UT) representation: KimiLinear KDA/MLA tutorial
 * (icman.com.cn), sec. 3 (chunk_size 64) and sec. 6 (chunk-parallel + WY);
 * training and long prompts use this chunk mode (lpnh.cn article, sec. 5).
 *
 *   q, k       [B, T, H, dk]  dtype           v    [B, T, H, dv] dtype
 *   (dtype is the element type of q, k and v; out_dtype that of out. An fp32
 *    out keeps the result unrounded for what follows, e.g. an output norm;
 *    a bf16 out halves the output traffic and adds one bf16 rounding.)
 *   log_alpha  [B, T, H, dk]  float32         beta [B, T, H]     float32
 *   S0         [N, H, dk, dv] float32, or NULL for a zero initial state
 *   cu_seqlens NULL: N must equal B and batch row b is one sequence of T tokens.
 *              Otherwise int32 [N+1] device array of packed offsets (B must be 1):
 *              cu_seqlens[0] = 0, non-decreasing, cu_seqlens[N] = T. Sequences may
 *              be empty (then S_final = S0). Contents are checked on the device:
 *              a violation writes KDA_ERR_INVALID_ARG to the workspace status word
 *              (read it with kda_workspace_status) and the affected sequences are
 *              skipped.
 *   out        [B, T, H, dv]  out_dtype  (written: o_t for every token)
 *   S_final    [N, H, dk, dv] float32, or NULL (not written)
 *   workspace  device buffer of kda_chunk_fwd_workspace_size(...) bytes,
 *              workspace_bytes its size. Its status word is cleared by this call.
 * S0 and S_final may alias (in-place continuation); no other buffers may overlap.
 * T = 0 or N = 0 is valid (only S_final = S0 is written).
 * For bf16 inputs with at most 64 (sequence, head) pairs and at least 64 chunk slots the two
 * passes run as a pipeline over up to 16 token ranges: the state scan of one range beside the
 * preparation of the later ones, on two library-owned streams (created on the first such call per
 * device) that fork from `stream` and join it again; everything stays ordered on `stream`. Between
 * ranges the state is carried in S_final (or the workspace when S_final is NULL). */
kda_status_t kda_chunk_fwd(const void *q, const void *k, const void *v,
                           const float *log_alpha, const float *beta,
                           const float *S0, const int32_t *cu_seqlens,
                           void *out, float *S_final,
                           int B, int T, int H, int N, int dk, int dv,
                           kda_dtype_t dtype, kda_dtype_t out_dtype,
                           void *workspace, size_t workspace_bytes, void *stream);

/* The two passes kda_chunk_fwd runs for bf16 inputs, callable one by one (the same
 * chunked form as kda_chunk_fwd; the split is this library's, the pages name no passes).
 * kda_chunk_prep does every step that does not depend on the running state, for all
 * chunks at once (decay scaling, the intra-chunk products, the triangular inverse, the
 * WY factors) and writes the results to the workspace; kda_chunk_scan then runs the
 * state recurrence over the chunks and writes out and S_final. Together they compute
 * exactly what one kda_chunk_fwd call does. A caller can run the passes of different
 * batches on different streams, or time them separately.
 *
 *   Arguments mean what they mean for kda_chunk_fwd with dtype = KDA_BF16; the
 *   workspace is sized by kda_chunk_fwd_workspace_size(..., KDA_BF16).
 *   kda_chunk_prep reads q, k, log_alpha, beta (and cu_seqlens) and clears the
 *   workspace status word before it enqueues its kernel.
 *   kda_chunk_scan reads v, S0 and the prepared workspace, writes out and S_final, and
 *   leaves the status word as it is, so that it reports errors of both passes.
 * kda_chunk_scan must follow a kda_chunk_prep with the same B, T, H, N, cu_seqlens and
 * workspace, ordered after it (same stream, or an event); it reads whatever the
 * workspace holds, so a scan without its prep returns garbage, not an error. */
kda_status_t kda_chunk_prep(const void *q, const void *k,
                            const float *log_alpha, const float *beta,
                            const int32_t *cu_seqlens,
                            int B, int T, int H, int N, int dk, int dv,
                            void *workspace, size_t workspace_bytes, void *stream);
kda_status_t kda_chunk_scan(const void *v, const float *S0, const int32_t *cu_seqlens,
                            void *out, float *S_final,
                            int B, int T, int H, int N, int dk, int dv, kda_dtype_t out_dtype,
                            void *workspace, size_t workspace_bytes, void *stream);

/* Backward pass of kda_chunk_fwd: the gradients of a scalar loss with respect to every
 * input, given its gradients with respect to every output o_t and to the final states.
 * The pages print no backward pass (training uses the chunk mode: lpnh.cn article, sec. 5);
 * these are the chain rule through the recurrence above, computed through the same chunk
 * form (chunk 64). The gradients are fp32 arithmetic on CUDA cores for either input dtype; for
 * bf16 inputs the forward records come from the tensor-core forward passes, run as
 * kda_chunk_fwd runs them (pipelined over token ranges on the library's two streams when there
 * are few (sequence, head) chains; the call stays ordered on `stream`).
 *
 *   q, k, v, log_alpha, beta, S0, cu_seqlens, B, T, H, N, dk, dv, dtype:
 *              exactly as passed to kda_chunk_fwd (the forward is recomputed here).
 *   dout       [B, T, H, dv]  dtype: dL/do_t for every token.
 *   dS_final   [N, H, dk, dv] float32: dL/dS_final, or NULL for zero.
 *   dq, dk_out, dlog_alpha  [B, T, H, dk] float32 (written)
 *   dv_out     [B, T, H, dv]  float32 (written)
 *   dbeta      [B, T, H]      float32 (written)
 *   dS0        [N, H, dk, dv] float32 (written: dL/dS0), or NULL (not computed).
 *   workspace  device buffer of kda_chunk_bwd_workspace_size(...) bytes (fp32 records
 *              of the forward and of the reverse sweep and the reverse sweep's prepared
 *              operands: 401 KiB per chunk slot and head, see kda_chunk_fwd_workspace_size
 *              for chunk slots). Its status word is
 *              cleared by this call; cu_seqlens is checked on the device as for
 *              kda_chunk_fwd.
 * Gradient buffers must not overlap each other or the inputs. Every pointer except S0,
 * dS_final and dS0 must be non-NULL when B * T > 0; alignment as for kda_chunk_fwd
 * (16 bytes; 4 for beta and dbeta). Errors: KDA_ERR_INVALID_ARG, KDA_ERR_UNSUPPORTED
 * (dk, dv other than 128, or more chunk slots times heads than one launch grid holds),
 * KDA_ERR_CUDA. */
size_t kda_chunk_bwd_workspace_size(int B, int T, int H, int N, int dk, int dv);
kda_status_t kda_chunk_bwd(const void *q, const void *k, const void *v,
                           const float *log_alpha, const float *beta,
                           const float *S0, const int32_t *cu_seqlens,
                           const void *dout, const float *dS_final,
                           float *dq, float *dk_out, float *dv_out,
                           float *dlog_alpha, float *dbeta, float *dS0,
                           int B, int T, int H, int N, int dk, int dv, kda_dtype_t dtype,
                           void *workspace, size_t workspace_bytes, void *stream);

/* The three kernels kda_chunk_bwd runs, one at a time (for timing them separately, or for
 * running the phases of different batches on different streams), with the arguments of
 * kda_chunk_bwd and the same checks:
 *   phase 0  the forward sweep, recording into the workspace the state entering every chunk
 *            and each chunk's U (and, for fp32 inputs, R = V - Kt S); clears the workspace
 *            status word first;
 *   phase 1  the reverse scan of the state gradient: a data-parallel pass forms every chunk's
 *            state-independent operands, then the scan writes dv_out and dS0, and records Y and
 *            the gradient reaching the end of every chunk;
 *   phase 2  every other gradient (dq, dk_out, dlog_alpha, dbeta), chunk by chunk.
 * Each phase reads what the earlier ones recorded, so they must run in this order on the same
 * workspace and arguments (same stream, or ordered by events); a phase run without the earlier
 * ones returns garbage, not an error. Any other phase number: KDA_ERR_INVALID_ARG. */
kda_status_t kda_chunk_bwd_phase(int phase, const void *q, const void *k, const void *v,
                                 const float *log_alpha, const float *beta,
                                 const float *S0, const int32_t *cu_seqlens,
                                 const void *dout, const float *dS_final,
                                 float *dq, float *dk_out, float *dv_out,
                                 float *dlog_alpha, float *dbeta, float *dS0,
                                 int B, int T, int H, int N, int dk, int dv, kda_dtype_t dtype,
                                 void *workspace, size_t workspace_bytes, void *stream);

/* One decode step for N independent sequences (one token each), updating the
 * state in place: the recurrent ("fused_recurrent") mode the layer uses for
 * short queries and generation (lpnh.cn article, sec. 2 and 5); the per-step
 * cost is fixed by the state size, not by the context length (KimiLinear
 * KDA/MLA tutorial (icman.com.cn), sec. 1 and 2).
 *
 *   q, k       [N, H, dk] dtype     v [N, H, dv] dtype
 *   log_alpha  [N, H, dk] float32   beta [N, H] float32
 *   S_inout    [N, H, dk, dv] float32, read as S_{t-1} and overwritten with S_t
 *   out        [N, H, dv] out_dtype, written with o_t = S_t^T q_t
 * N = 0 is valid (nothing is launched). */
kda_status_t kda_decode_step(const void *q, const void *k, const void *v,
                             const float *log_alpha, const float *beta,
                             float *S_inout, void *out,
                             int N, int H, int dk, int dv, kda_dtype_t dtype,
                             kda_dtype_t out_dtype, void *stream);

/* ---------------------------------------------------------------------------------------------
 * The KDA layer's element-wise neighbours of the recurrence, fused into its kernels.
 *
 * The pages name these parts of the Kimi Linear KDA module without printing a formula
 * (lpnh.cn Kimi Linear KDA/NoPE article, sec. 3: A_log, dt_bias and the low-rank f_a/f_b
 * projection feed the channel-wise decay through fused_kda_gate; b_proj feeds the write gate
 * beta; the output goes through o_norm = FusedRMSNormGated with the activation fixed to
 * sigmoid; sec. 4 names the decay and beta gating). The readings used here:
 *   log_alpha[t,h,c] = -exp(A_log[h]) * softplus(gate_f[t,h,c] + dt_bias[h*dk + c])
 *   beta[t,h]        = sigmoid(beta_logits[t,h])
 *   y[t,h,:]         = o[t,h,:] / sqrt(mean_c o[t,h,c]^2 + norm_eps) * norm_weight[:]
 *                      * sigmoid(out_gate[t,h,:])
 * Each group is optional: a NULL gate_f means log_alpha is passed directly, a NULL beta_logits
 * means beta is passed directly, a NULL out_gate means the raw outputs o are written.
 *   gate_f      [B,T,H,dk] (decode: [N,H,dk]) in dtype; A_log [H] and dt_bias [H*dk] float32
 *   beta_logits [B,T,H]    (decode: [N,H])    in dtype
 *   out_gate    [B,T,H,dv] (decode: [N,H,dv]) in dtype; norm_weight [dv] float32 (shared by
 *               the heads); norm_eps >= 0
 * Alignment: gate_f, out_gate, dt_bias 16 bytes; A_log, norm_weight, beta_logits 4 bytes.
 * --------------------------------------------------------------------------------------------- */
typedef struct {
    const void *gate_f;
    const float *A_log;
    const float *dt_bias;
    const void *beta_logits;
    const void *out_gate;
    const float *norm_weight;
    float norm_eps;
} kda_layer_opts_t;

/* Workspace bytes of kda_chunk_fwd_layer: that of kda_chunk_fwd, plus (fp32 inputs only) fp32
 * scratch for the produced gates and for the outputs before the norm. 0 for rejected sizes. */
size_t kda_chunk_fwd_layer_workspace_size(int B, int T, int H, int N, int dk, int dv,
                                          kda_dtype_t dtype, const kda_layer_opts_t *opts);

/* kda_chunk_fwd with the layer options above (opts NULL or all-NULL: exactly kda_chunk_fwd).
 * log_alpha / beta may be NULL when their producer inputs are given. For bf16 inputs every part
 * is fused: the decay and write gates are produced inside the preparation pass (the fp32
 * log_alpha stream is never written or read), and the output norm runs in the scan's output
 * epilogue (one CTA holds all value channels of a head). fp32 inputs run separate gate and norm passes
 * around the CUDA-core prefill. Errors as for kda_chunk_fwd; a NULL A_log/dt_bias with gate_f, or
 * a NULL norm_weight with out_gate, or norm_eps < 0 is KDA_ERR_INVALID_ARG. */
kda_status_t kda_chunk_fwd_layer(const void *q, const void *k, const void *v,
                                 const float *log_alpha, const float *beta,
                                 const float *S0, const int32_t *cu_seqlens,
                                 void *out, float *S_final,
                                 int B, int T, int H, int N, int dk, int dv,
                                 kda_dtype_t dtype, kda_dtype_t out_dtype,
                                 const kda_layer_opts_t *opts,
                                 void *workspace, size_t workspace_bytes, void *stream);

/* The two passes of kda_chunk_fwd_layer for bf16 inputs, one by one (see kda_chunk_prep and
 * kda_chunk_scan): the preparation pass with the gate producers, the scan with the output norm. */
kda_status_t kda_chunk_prep_layer(const void *q, const void *k,
                                  const float *log_alpha, const float *beta,
                                  const int32_t *cu_seqlens,
                                  int B, int T, int H, int N, int dk, int dv,
                                  const kda_layer_opts_t *opts,
                                  void *workspace, size_t workspace_bytes, void *stream);
kda_status_t kda_chunk_scan_layer(const void *v, const float *S0, const int32_t *cu_seqlens,
                                  void *out, float *S_final,
                                  int B, int T, int H, int N, int dk, int dv, kda_dtype_t out_dtype,
                                  const kda_layer_opts_t *opts,
                                  void *workspace, size_t workspace_bytes, void *stream);

/* kda_decode_step with the layer options (all fused into the decode kernel). */
kda_status_t kda_decode_step_layer(const void *q, const void *k, const void *v,
                                   const float *log_alpha, const float *beta,
                                   float *S_inout, void *out,
                                   int N, int H, int dk, int dv, kda_dtype_t dtype,
                                   kda_dtype_t out_dtype, const kda_layer_opts_t *opts, void *stream);

/* ---------------------------------------------------------------------------------------------
 * Short causal convolution in front of q, k and v, and its decode step. The layer config sets
 * short_conv_kernel_size 4 and the cache keeps conv_states beside the recurrent states (lpnh.cn
 * Kimi Linear KDA/NoPE article, sec. 3 and 6); no formula is printed. Reading used: a depthwise
 * convolution over tokens, per channel c,
 *     y[t,c] = act(bias[c] + sum_{j=0}^{K-1} weight[c,j] * x[t-K+1+j, c])   (taps oldest first)
 * with the inputs before a sequence's first token taken from its conv state, act = SiLU when
 * activation_silu is 1 (identity when 0), then, when normalize_head_dim = 128, each consecutive
 * 128-channel head vector divided by sqrt(|y|^2 + 1e-6) (the unit-norm q and k of the recurrence).
 *
 *   x, y        [B,T,D] (packed: B = 1 and cu_seqlens as for kda_chunk_fwd) in dtype; D a multiple
 *               of 128 (for example H * 128 channels of q); 16-byte aligned
 *   weight      [D,K] float32; bias [D] float32 or NULL; 1 <= K <= 8
 *   conv_state  [N,D,K-1] float32, the last K-1 inputs before each sequence, oldest first, or NULL
 *               (zeros); conv_state_out [N,D,K-1] float32 or NULL: written with the last K-1 inputs
 *               of each sequence (the old state shifted in for sequences shorter than K-1); it may
 *               be the same buffer as conv_state.
 * kda_short_conv_step: one token per sequence, x and y [N,D], conv_state [N,D,K-1] read and
 * updated in place.
 * Errors: KDA_ERR_INVALID_ARG (sizes, pointers, alignment), KDA_ERR_UNSUPPORTED (D not a multiple
 * of 128, K > 8, normalize_head_dim other than 0 or 128), KDA_ERR_CUDA. */
kda_status_t kda_short_conv(const void *x, const float *weight, const float *bias,
                            const float *conv_state, float *conv_state_out, const int32_t *cu_seqlens,
                            void *y, int B, int T, int N, int D, int K, int activation_silu,
                            int normalize_head_dim, kda_dtype_t dtype, void *stream);
kda_status_t kda_short_conv_step(const void *x, const float *weight, const float *bias,
                                 float *conv_state, void *y, int N, int D, int K, int activation_silu,
                                 int normalize_head_dim, kda_dtype_t dtype, void *stream);

/* S_out[h] = Phi[h] S_in[h] + Psi[h] for every head (float32, [H,dk,dv], Phi [H,dk,dk]; Psi may be
 * NULL for zero). A segment of the recurrence maps the state entering it to the state leaving it
 * affinely, S -> Phi S + Psi: Phi is S_final of the segment run from S0 = I with v = 0, and Psi is
 * S_final run from S0 = 0. Composing the maps of consecutive segments gives each segment's entering
 * state without running the earlier segments again: the exchange step of a sequence split across
 * devices (context-parallel prefill). The pages do not describe this split; it follows from the
 * recurrence being linear in the state. S_out must not alias S_in or Phi (KDA_ERR_INVALID_ARG). */
kda_status_t kda_state_affine(const float *Phi, const float *S_in, const float *Psi, float *S_out,
                              int H, int dk, int dv, void *stream);

/* Capacity of the library-owned scratch array used by kda_chunk_fwd_noalloc (bytes). */
#define KDA_NOALLOC_SCRATCH_BYTES 4096

/* kda_chunk_fwd without a workspace argument, for callers that cannot allocate device memory:
 * plug-ins whose host runtime owns all device memory and passes in only the input and output
 * buffers, and memory-capped servers that may not grow their footprint per call.
 * The pages describe no such entry point; it has no counterpart there.
 *
 * Arguments, layouts and results are those of kda_chunk_fwd; the caller still passes (and owns)
 * every input and output. Instead of a workspace, the library uses a static device array of
 * KDA_NOALLOC_SCRATCH_BYTES that every GPU on which the library is loaded holds until the process
 * exits. The first call on a device looks up that array's device address (with the device
 * current) and caches it. bf16 inputs run
 * the single-kernel prefill, whose only scratch is the 256-byte status header (a scratch need
 * beyond the array would be refused with KDA_ERR_UNSUPPORTED); it is slower than the two-pass
 * prefill kda_chunk_fwd runs with its workspace, and its f16 tensor-core operands narrow the
 * decay range: the cumulative log-decay inside one 64-token chunk must stay at or above -9.0 per
 * channel (fp32 inputs keep the -80 of kda_chunk_fwd). The function calls no cudaMalloc, cudaFree
 * or other allocating routine.
 * The array is shared by every call and keeps the last call's contents; each call clears its
 * status header first. Calls whose work overlaps on the GPU (for example on two streams) race
 * on that shared array: serialise them. Device-side check results (cu_seqlens contents, the
 * decay range) are written to that shared status header; read them back with
 * kda_chunk_fwd_noalloc_status. */
kda_status_t kda_chunk_fwd_noalloc(const void *q, const void *k, const void *v,
                                   const float *log_alpha, const float *beta,
                                   const float *S0, const int32_t *cu_seqlens,
                                   void *out, float *S_final,
                                   int B, int T, int H, int N, int dk, int dv,
                                   kda_dtype_t dtype, kda_dtype_t out_dtype, void *stream);

/* Waits for `stream`, then copies the status word of the shared scratch array of
 * kda_chunk_fwd_noalloc on the current device to *status: KDA_OK when every device-side check
 * of the last kda_chunk_fwd_noalloc call on this device passed, else the first failure
 * (KDA_ERR_INVALID_ARG for inconsistent cu_seqlens contents, KDA_ERR_UNSUPPORTED for a decay
 * outside the range, KDA_ERR_TIMEOUT for a device wait that gave up). The pages have no
 * counterpart. Allocates nothing. Errors: KDA_ERR_INVALID_ARG (status NULL), KDA_ERR_CUDA. */
kda_status_t kda_chunk_fwd_noalloc_status(void *stream, int32_t *status);

/* Self-test of the library's failure detection (the pages have no counterpart): every device-side
 * wait of the kernels (on an mbarrier or a copy) is bounded and, when it runs out, records
 * KDA_ERR_TIMEOUT in the workspace status word and lets the kernel return, so that the CUDA context
 * stays usable. This call launches one tiny kernel that makes such a wait on a barrier nothing
 * arrives on, with a limit of budget_cycles SM clock cycles (1 .. KDA_SELFTEST_MAX_BUDGET), so the
 * caller can read KDA_ERR_TIMEOUT back with kda_workspace_status. workspace: at least 256 bytes,
 * 16-byte aligned; its status word is cleared first. Returns KDA_ERR_INVALID_ARG for a bad
 * workspace or budget. */
#define KDA_SELFTEST_MAX_BUDGET 2000000000LL
kda_status_t kda_selftest_wait_timeout(void *workspace, size_t workspace_bytes,
                                       long long budget_cycles, void *stream);

/* Waits for `stream`, then copies the workspace status word to *status
 * (KDA_OK when every device-side check passed). */
kda_status_t kda_workspace_status(const void *workspace, void *stream, int32_t *status);

/* Static, human-readable name of a status code. */
const char *kda_status_string(kda_status_t status);

/* Library version as major*10000 + minor*100 + patch. */
int kda_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LIBKDA_H */
