// chunk_fp32.cu -- chunkwise KDA prefill on CUDA cores, fp32 arithmetic throughout.
//
// This is the exact-precision path (fp32 inputs, where bf16 tensor-core operands could not
// meet a 1e-4 relative error) and the reference-quality path for any input dtype.
//
// Chunked form (chunk C = 64; KimiLinear KDA/MLA tutorial (icman.com.cn), sec. 3 and 6 name the
// chunk size and the chunk-parallel + WY approach; the algebra is derived from the recurrence):
// for a chunk of L <= C tokens entering with state S (d_k x d_v), per key channel c,
//   g_r    = sum_{j<=r} log_alpha_j                      cumulative log-decay
//   Kt_r   = k_r e^{g_r},  Kh_r = k_r e^{-g_r},  Qt_r = q_r e^{g_r},  Ke_r = k_r e^{g_{L-1}-g_r}
//   A      = StrictLower(diag(beta) Kt Kh^T),  M = tril(Qt Kh^T)
//   U      = (I + A)^{-1} diag(beta) (V - Kt S)          (forward substitution, row by row)
//   O      = Qt S + M U
//   S     <- Diag(e^{g_{L-1}}) S + Ke^T U
// Rows past L are zero-filled (log_alpha = 0, k = q = v = 0), which leaves every result unchanged.
//
// Work split: one CTA per (sequence, head, 32-column block of d_v); the columns of S evolve
// independently, so blocks never communicate. Chunks are processed in order; everything stays
// in shared memory (about 198 KiB).
//
// For the backward pass the same kernel also records, per (head, chunk slot), the state entering
// each chunk and the chunk's R = V - Kt S and U (PrefillArgs::ck_*), and may skip the outputs.
#include "chunk_fp32_common.cuh"
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int C = kChunk;
constexpr int DK = kHeadDim;
constexpr int DVB = 32;          // value columns per CTA
constexpr int LD = DK + 1;       // padded row stride of the chunk operand tiles
constexpr int LDC = C + 1;       // padded row stride of the 64 x 64 tiles
constexpr int NT = 256;

struct Smem {
    float Kt[C * LD];
    float Kh[C * LD];
    float Qt[C * LD];
    float Ke[C * LD];
    float S[DK * DVB];
    float A[C * LDC];
    float M[C * LDC];
    float U[C * DVB];
    float R[C * DVB];
    float gam[DK];
    float beta[C];
};

template <typename T, typename TO>
__global__ void __launch_bounds__(NT, 1)
chunk_fp32_kernel(PrefillArgs a)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    Smem &sm = *reinterpret_cast<Smem *>(smem_raw);
    const int tid = threadIdx.x;
    const int j0 = blockIdx.x * DVB;
    const int h = blockIdx.y;
    const int n = blockIdx.z;
    const int H = a.H;
    const T *q = (const T *)a.q;
    const T *k = (const T *)a.k;
    const T *v = (const T *)a.v;
    TO *out = (TO *)a.out;

    int64_t t0, t1;
    if (!sequence_span(a.cu_seqlens, n, a.N, a.T, &t0, &t1, a.status)) return;

    // initial state block (every state access below stays inside this head's DK x DK block)
    const size_t sbase = ((size_t)n * H + h) * DK * DK;
    if (!in_bounds(a.status, (long long)sbase, DK * DK, (long long)a.N * H * DK * DK)) return;
    for (int idx = tid; idx < DK * DVB; idx += NT) {
        const int c = idx / DVB, j = idx % DVB;
        sm.S[idx] = a.S0 ? a.S0[sbase + (size_t)c * DK + j0 + j] : 0.f;
    }

    for (int64_t s = t0; s < t1; s += C) {
        const int L = (t1 - s < C) ? (int)(t1 - s) : C;
        // every global access of this chunk lies in its token rows [s, s + L) and, for the records,
        // in its (head, chunk slot) block
        if (!in_bounds(a.status, s, L, (long long)a.B * a.T) ||
            ((a.ck_S || a.ck_U) && !in_bounds(a.status, (long long)h * a.n_slots + chunk_slot(s, n), 1,
                                                   (long long)H * a.n_slots)))
            break;
        __syncthreads();
        // ---- load the chunk: k -> Kt, q -> Qt, log_alpha -> Kh, v block -> R
        fp32c::load_chunk<T, NT>(sm.Kt, sm.Qt, sm.Kh, LD, sm.R, q, k, a.log_alpha, v, s, L, H, h, j0, tid);
        if (tid < C) sm.beta[tid] = (tid < L) ? a.beta[(size_t)(s + tid) * H + h] : 0.f;
        // backward records of this chunk: (head, chunk slot) blocks
        const size_t rec = (size_t)h * a.n_slots + (size_t)chunk_slot(s, n);
        if (a.ck_S) fp32c::store_block32<NT>(a.ck_S + rec * kBwdStateFloats + j0, DK, sm.S, DK, tid);
        __syncthreads();

        // ---- cumulative log-decay (all threads, in row parts), then the decay-scaled operands
        {
            const float gl = fp32c::decay_prefix<NT>(sm.Kh, LD, tid);
            const int c = tid % DK, part = tid / DK, r0 = part * (C / (NT / DK));
            if (part == 0) sm.gam[c] = expf(gl);
            // e^{-g} must stay finite in fp32: outside the range the outputs are not usable
            if (part == 0 && !(gl >= kMinChunkLogDecay)) set_status(a.status, KDA_ERR_UNSUPPORTED);
#pragma unroll 4
            for (int r = r0; r < r0 + C / (NT / DK); ++r) {
                const float gr = sm.Kh[r * LD + c];
                const float kk = sm.Kt[r * LD + c];
                const float e = expf(gr);
                sm.Kt[r * LD + c] = kk * e;
                sm.Qt[r * LD + c] *= e;
                sm.Kh[r * LD + c] = kk * expf(-gr);
                sm.Ke[r * LD + c] = kk * expf(gl - gr);
            }
        }
        __syncthreads();

        // ---- A = StrictLower(diag(beta) Kt Kh^T), M = tril(Qt Kh^T); 4x4 register tiles
        {
            const int rb = tid / 16, ib = tid % 16;
            float accA[4][4], accM[4][4];
#pragma unroll
            for (int x = 0; x < 4; ++x)
#pragma unroll
                for (int y = 0; y < 4; ++y) { accA[x][y] = 0.f; accM[x][y] = 0.f; }
            if (ib <= rb && out) {
                for (int c = 0; c < DK; ++c) {
                    float kt[4], qt[4], kh[4];
#pragma unroll
                    for (int x = 0; x < 4; ++x) {
                        kt[x] = sm.Kt[(4 * rb + x) * LD + c];
                        qt[x] = sm.Qt[(4 * rb + x) * LD + c];
                        kh[x] = sm.Kh[(4 * ib + x) * LD + c];
                    }
#pragma unroll
                    for (int x = 0; x < 4; ++x)
#pragma unroll
                        for (int y = 0; y < 4; ++y) {
                            accA[x][y] += kt[x] * kh[y];
                            accM[x][y] += qt[x] * kh[y];
                        }
                }
            } else if (ib <= rb) {                 // records only: M is not needed
                for (int c = 0; c < DK; ++c) {
                    float kt[4], kh[4];
#pragma unroll
                    for (int x = 0; x < 4; ++x) {
                        kt[x] = sm.Kt[(4 * rb + x) * LD + c];
                        kh[x] = sm.Kh[(4 * ib + x) * LD + c];
                    }
#pragma unroll
                    for (int x = 0; x < 4; ++x)
#pragma unroll
                        for (int y = 0; y < 4; ++y) accA[x][y] += kt[x] * kh[y];
                }
            }
#pragma unroll
            for (int x = 0; x < 4; ++x)
#pragma unroll
                for (int y = 0; y < 4; ++y) {
                    const int r = 4 * rb + x, i = 4 * ib + y;
                    sm.A[r * LDC + i] = (i < r) ? sm.beta[r] * accA[x][y] : 0.f;
                    sm.M[r * LDC + i] = (i <= r) ? accM[x][y] : 0.f;
                }
        }
        // ---- R = diag(beta) (V - Kt S): thread -> row r, 8 columns
        {
            const int r = tid / 4, jg = (tid % 4) * 8;
            float acc[8];
#pragma unroll
            for (int x = 0; x < 8; ++x) acc[x] = 0.f;
            for (int c = 0; c < DK; ++c) fp32c::axpy<8>(acc, sm.Kt[r * LD + c], sm.S + c * DVB + jg);
            const float b = sm.beta[r];
            if (a.ck_R) {
                float4 *dst = reinterpret_cast<float4 *>(a.ck_R + rec * kBwdRowsFloats + (size_t)r * DK + j0 + jg);
                const float *rv = sm.R + r * DVB + jg;
                dst[0] = make_float4(rv[0] - acc[0], rv[1] - acc[1], rv[2] - acc[2], rv[3] - acc[3]);
                dst[1] = make_float4(rv[4] - acc[4], rv[5] - acc[5], rv[6] - acc[6], rv[7] - acc[7]);
            }
#pragma unroll
            for (int x = 0; x < 8; ++x) sm.R[r * DVB + jg + x] = b * (sm.R[r * DVB + jg + x] - acc[x]);
        }
        __syncthreads();

        // ---- U = (I + A)^{-1} R: blocked forward substitution (U starts as a copy of R)
        for (int idx = tid; idx < C * DVB; idx += NT) sm.U[idx] = sm.R[idx];
        __syncthreads();
        fp32c::lower_solve_32<NT>(sm.A, LDC, sm.U, tid);
        if (a.ck_U) fp32c::store_block32<NT>(a.ck_U + rec * kBwdRowsFloats + j0, DK, sm.U, C, tid);

        // ---- O = Qt S + M U  -> out (rows < L); skipped when only the records are wanted
        if (out) {
            const int r = tid / 4, jg = (tid % 4) * 8;
            float acc[8];
#pragma unroll
            for (int x = 0; x < 8; ++x) acc[x] = 0.f;
            for (int c = 0; c < DK; ++c) fp32c::axpy<8>(acc, sm.Qt[r * LD + c], sm.S + c * DVB + jg);
            for (int i = 0; i <= r; ++i) fp32c::axpy<8>(acc, sm.M[r * LDC + i], sm.U + i * DVB + jg);
            if (r < L) {
                TO *o = out + ((size_t)(s + r) * H + h) * DK + j0 + jg;
#pragma unroll
                for (int x = 0; x < 8; ++x) o[x] = from_f32<TO>(acc[x]);
            }
        }
        __syncthreads();

        // ---- S <- Diag(gamma) S + Ke^T U: thread -> key channel c, 16 columns
        {
            const int c = tid / 2, jh = (tid % 2) * 16;
            float acc[16];
            const float gm = sm.gam[c];
#pragma unroll
            for (int x = 0; x < 16; ++x) acc[x] = gm * sm.S[c * DVB + jh + x];
            for (int r = 0; r < C; ++r) fp32c::axpy<16>(acc, sm.Ke[r * LD + c], sm.U + r * DVB + jh);
#pragma unroll
            for (int x = 0; x < 16; ++x) sm.S[c * DVB + jh + x] = acc[x];
        }
    }
    __syncthreads();
    if (a.S_final) {
        for (int idx = tid; idx < DK * DVB; idx += NT) {
            const int c = idx / DVB, j = idx % DVB;
            a.S_final[sbase + (size_t)c * DK + j0 + j] = sm.S[idx];
        }
    }
}

}  // namespace

template <typename T, typename TO>
static cudaError_t launch_typed(const PrefillArgs &a, cudaStream_t stream)
{
    const dim3 grid(DK / DVB, a.H, a.N);
    const size_t smem = sizeof(Smem);
    cudaError_t e = cudaFuncSetAttribute(chunk_fp32_kernel<T, TO>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    chunk_fp32_kernel<T, TO><<<grid, NT, smem, stream>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_chunk_fp32(const PrefillArgs &a, kda_dtype_t dtype, kda_dtype_t out_dtype,
                              cudaStream_t stream)
{
    if (a.N == 0) return cudaSuccess;
    using bf = __nv_bfloat16;
    if (dtype == KDA_BF16 && out_dtype == KDA_BF16) return launch_typed<bf, bf>(a, stream);
    if (dtype == KDA_BF16) return launch_typed<bf, float>(a, stream);
    if (out_dtype == KDA_BF16) return launch_typed<float, bf>(a, stream);
    return launch_typed<float, float>(a, stream);
}

}  // namespace kda
