// chunk_bwd.cu -- backward pass of the chunked KDA prefill on CUDA cores, fp32 arithmetic.
//
// Forward chunk form (chunk C = 64; chunk-parallel prefill with a WY representation: KimiLinear
// KDA/MLA tutorial (icman.com.cn), sec. 3 and 6; the algebra is derived from the recurrence of
// sec. 2 and 5). For a chunk of L <= C tokens entering with state S, per key channel c,
//   g_r = sum_{j<=r} log_alpha_j,  E = e^g,  Kt = K E,  Kh = K / E,  Qt = Q E,  gamma = E_{L-1},
//   Ke = Kh gamma,  A = StrictLower(diag(beta) Kt Kh^T),  M = tril(Qt Kh^T),
//   R = V - Kt S,  U = (I + A)^{-1} diag(beta) R,  O = Qt S + M U,  S' = Diag(gamma) S + Ke^T U.
// The pages give no backward pass; the gradients are the chain rule through these lines. With dO
// the output gradient and dS' the gradient reaching the state that leaves the chunk:
//   dU  = M^T dO + Ke dS'                Y = (I + A)^{-T} dU   (back substitution)
//   dV  = diag(beta) Y                   dS = Diag(gamma) dS' + Qt^T dO - Kt^T dV
// and, with every sum over the value channels gathered into dense products,
//   dM  = tril(dO U^T)                   dA = -StrictLower(Y U^T)     dP = diag(beta) dA
//   dQt = dO S^T + dM Kh                 dKt = -diag(beta) Y S^T + dP Kh
//   dKh = dM^T Qt + dP^T Kt              dKe = U dS'^T                dgamma = rowsum(dS' * S)
//   dbeta_r = sum_v R_rv Y_rv + sum_{i<r} dA_ri (Kt Kh^T)_ri
//   dq = dQt E,  dk = dKt E + dKh / E + dKe gamma / E,
//   dg = dQt Qt + dKt Kt - dKh Kh - dKe Ke,  plus (sum_r dKe Ke + dgamma gamma) on the last row,
//   dlog_alpha = reverse cumulative sum of dg over the chunk's rows.
//
// Three launches (the host calls them in order on one stream):
//  1. the forward records: the state entering every chunk and each chunk's R and U, per (head,
//     chunk slot). For fp32 inputs the fp32 forward kernel (chunk_fp32.cu) writes all three; for
//     bf16 inputs the tensor-core passes do (chunk_prep.cu, then chunk_scan.cu in record mode),
//     writing S and U, and kernel 3 forms R = V - Kt S itself;
//  2. the state gradient, chunk by chunk from the end of each sequence, in two kernels:
//     chunk_bwd_prep_kernel (data-parallel, one CTA per (chunk slot, head)) forms every chunk's
//     state-independent operands (below) and the per-chunk kernel's StrictLower(Kt Kh^T), and
//     chunk_bwd_rscan_kernel (one CTA per (sequence,
//     head, 32 value columns); the columns are independent) runs the two state products per
//     chunk and writes dV, dS0, Y and the gradient dS' reaching the end of every chunk;
//  3. chunk_bwd_local_kernel: everything else, one CTA per (chunk slot, head), no chunk-to-chunk
//     dependence (data-parallel over the whole grid).
// Rows past a chunk's end are zero-filled (log_alpha = 0, k = q = v = dO = 0), which leaves every
// gradient of the real rows unchanged.
#include "chunk_fp32_common.cuh"
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int C = kChunk;
constexpr int DK = kHeadDim;
constexpr int DVB = 32;          // value columns per block
constexpr int LD = DK + 4;       // row stride of the 64 x 128 operand tiles (16-byte aligned rows)
constexpr int LDC = C + 1;       // padded row stride of the 64 x 64 tiles read by scalar loads
constexpr int LDC4 = C + 4;      // row stride of the 64 x 64 tiles read as float4
constexpr int LDV = DVB + 4;     // row stride of the 32-column blocks (16-byte aligned rows)

// ------------------------------------------------------------------------------------------
// 2a. backward preparation (data-parallel): the state-independent operands of the reverse scan
// ------------------------------------------------------------------------------------------
// With T = (I + A)^{-1}, the reverse scan's two lines become Y = Y0 + Kp dS' and
// dS = Diag(gamma) dS' + G0 - Bk^T Y, where per chunk
//   Kp = T^T Ke (64 x 128),  Y0 = T^T M^T dO (64 x 128),  G0 = Qt^T dO (128 x 128),  Bk = diag(beta) Kt,
// none of which depends on the state gradient. One CTA per (chunk slot, head) forms them.
constexpr int NT_BP = 512;
constexpr size_t kBwdSmallFloats = 256;   // gamma (128) then beta (64) of a chunk, per (head, slot)

constexpr int LDB = DK + 4;      // row stride of the 64 x 128 tiles: 16-byte aligned rows, 4-bank skew
struct BprepSmem {
    float Kt[C * LDB];       // Kt, then Bk
    float Qt[C * LDB];       // Qt, then M^T dO -> Y0 (solved in place)
    float Kh[C * LDB];
    float Ke[C * LDB];       // Ke -> Kp (solved in place)
    float dO[C * LDB];
    float A[C * LDC];
    float M[C * LDC];
    float beta[C];
    float gam[DK];
};

template <typename T>
__global__ void __launch_bounds__(NT_BP, 1)
chunk_bwd_prep_kernel(BwdArgs a)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    BprepSmem &sm = *reinterpret_cast<BprepSmem *>(smem_raw);
    const int tid = threadIdx.x;
    const int H = a.H;
    const int h = (int)(blockIdx.x % (unsigned)H), slot = (int)(blockIdx.x / (unsigned)H);
    int n, L;
    int64_t s;
    if (!slot_to_chunk(a.cu_seqlens, a.N, a.T, slot, &n, &s, &L)) return;
    const size_t rec = (size_t)h * a.n_slots + (size_t)slot;
    if (!in_bounds(a.status, s, L, (long long)a.B * a.T) ||
        !in_bounds(a.status, (long long)rec, 1, (long long)H * a.n_slots))
        return;
    fp32c::load_rows<T, NT_BP, DK>(sm.Kt, LDB, (const T *)a.k, s, L, H, h, 0, tid);
    fp32c::load_rows<T, NT_BP, DK>(sm.Qt, LDB, (const T *)a.q, s, L, H, h, 0, tid);
    fp32c::load_rows<float, NT_BP, DK>(sm.Kh, LDB, a.log_alpha, s, L, H, h, 0, tid);
    fp32c::load_rows<T, NT_BP, DK>(sm.dO, LDB, (const T *)a.dout, s, L, H, h, 0, tid);
    if (tid < C) sm.beta[tid] = (tid < L) ? a.beta[(size_t)(s + tid) * H + h] : 0.f;
    __syncthreads();
    {   // decay: Kt = K e^g, Qt = Q e^g, Kh = K e^-g, Ke = K e^(g_last - g)
        const float gl = fp32c::decay_prefix<NT_BP>(sm.Kh, LDB, tid);
        constexpr int RP = C / (NT_BP / DK);
        const int c = tid % DK, r0 = (tid / DK) * RP;
        if (tid < DK) sm.gam[c] = expf(gl);
        if (tid < DK && !(gl >= kMinChunkLogDecay)) set_status(a.status, KDA_ERR_UNSUPPORTED);
#pragma unroll 4
        for (int r = r0; r < r0 + RP; ++r) {
            const float gr = sm.Kh[r * LDB + c], kk = sm.Kt[r * LDB + c];
            const float e = expf(gr);
            sm.Kt[r * LDB + c] = kk * e;
            sm.Qt[r * LDB + c] *= e;
            sm.Kh[r * LDB + c] = kk * expf(-gr);
            sm.Ke[r * LDB + c] = kk * expf(gl - gr);
        }
    }
    __syncthreads();
    // G0 (threads 0-255) beside A and M (threads 256-511); per step of the sum a thread tile of
    // a x b outputs reads a + b values, so the larger tiles take fewer shared-memory wavefronts
    if (tid < 256) {
        // G0 = Qt^T dO: thread -> key channels 8 cq .. + 7, value columns 4 jq .. + 3 and 64 + 4 jq ..
        // + 3 (cq = tid / 16, jq = tid % 16: the 8 lanes of a phase read 8 distinct bank groups of dO)
        const int cq = tid >> 4, jq = tid & 15;
        float acc[8][8];
#pragma unroll
        for (int x = 0; x < 8; ++x)
#pragma unroll
            for (int y = 0; y < 8; ++y) acc[x][y] = 0.f;
#pragma unroll 2
        for (int r = 0; r < C; ++r) {
            const float4 qa = *reinterpret_cast<const float4 *>(sm.Qt + r * LDB + 8 * cq);
            const float4 qb = *reinterpret_cast<const float4 *>(sm.Qt + r * LDB + 8 * cq + 4);
            const float4 o0 = *reinterpret_cast<const float4 *>(sm.dO + r * LDB + 4 * jq);
            const float4 o1 = *reinterpret_cast<const float4 *>(sm.dO + r * LDB + 64 + 4 * jq);
            const float qt[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
            const float o[8] = {o0.x, o0.y, o0.z, o0.w, o1.x, o1.y, o1.z, o1.w};
#pragma unroll
            for (int x = 0; x < 8; ++x)
#pragma unroll
                for (int y = 0; y < 8; ++y) acc[x][y] += qt[x] * o[y];
        }
        float *g0 = a.ck_G0 + rec * kBwdStateFloats;
#pragma unroll
        for (int x = 0; x < 8; ++x) {
            float *dst = g0 + (size_t)(8 * cq + x) * DK + 4 * jq;
            *reinterpret_cast<float4 *>(dst) = make_float4(acc[x][0], acc[x][1], acc[x][2], acc[x][3]);
            *reinterpret_cast<float4 *>(dst + 64) = make_float4(acc[x][4], acc[x][5], acc[x][6], acc[x][7]);
        }
    } else {
        // [A; M] from the rows of [Kt; Qt] times Kh^T, A = StrictLower(diag(beta) Kt Kh^T),
        // M = tril(Qt Kh^T): thread -> rows rb + 16 x of [Kt; Qt] (x < 8: Kt for x < 4, Qt after),
        // columns ib + 16 y (y < 4); float4 steps along the key channels, so that the 8 lanes of a
        // phase read one X row (a broadcast) and 8 Kh rows in 8 distinct bank groups (a row stride
        // of 33 groups)
        const int t = tid - 256, rb = t >> 4, ib = t & 15;
        float acc[8][4];
#pragma unroll
        for (int x = 0; x < 8; ++x)
#pragma unroll
            for (int y = 0; y < 4; ++y) acc[x][y] = 0.f;
#pragma unroll 1
        for (int c = 0; c < DK; c += 4) {
            float4 kh[4];
#pragma unroll
            for (int y = 0; y < 4; ++y) kh[y] = *reinterpret_cast<const float4 *>(sm.Kh + (ib + 16 * y) * LDB + c);
#pragma unroll
            for (int x = 0; x < 8; ++x) {
                const float *X = x < 4 ? sm.Kt : sm.Qt;
                const float4 xr = *reinterpret_cast<const float4 *>(X + (rb + 16 * (x & 3)) * LDB + c);
#pragma unroll
                for (int y = 0; y < 4; ++y) {
                    acc[x][y] += xr.x * kh[y].x;
                    acc[x][y] += xr.y * kh[y].y;
                    acc[x][y] += xr.z * kh[y].z;
                    acc[x][y] += xr.w * kh[y].w;
                }
            }
        }
        float *gP = a.ck_P + rec * kBwdTriFloats;   // P = StrictLower(Kt Kh^T) for the per-chunk kernel
#pragma unroll
        for (int x = 0; x < 8; ++x)
#pragma unroll
            for (int y = 0; y < 4; ++y) {
                const int r = rb + 16 * (x & 3), i = ib + 16 * y;
                if (x >= 4) {
                    sm.M[r * LDC + i] = (i <= r) ? acc[x][y] : 0.f;
                } else {
                    sm.A[r * LDC + i] = (i < r) ? sm.beta[r] * acc[x][y] : 0.f;
                    gP[r * C + i] = (i < r) ? acc[x][y] : 0.f;
                }
            }
    }
    __syncthreads();                      // Qt is dead
    {   // M^T dO into Qt's place: thread -> rows 4 (tid / 32) .. + 3, columns 4 (tid % 32) .. + 3
        const int r0 = 4 * (tid >> 5), j0 = 4 * (tid & 31);
        float acc[4][4];
#pragma unroll
        for (int x = 0; x < 4; ++x)
#pragma unroll
            for (int y = 0; y < 4; ++y) acc[x][y] = 0.f;
        for (int i = r0; i < C; ++i) {
            float m[4];
#pragma unroll
            for (int x = 0; x < 4; ++x) m[x] = sm.M[i * LDC + r0 + x];       // M^T[r][i] = M[i][r]
            const float4 o4 = *reinterpret_cast<const float4 *>(sm.dO + i * LDB + j0);
            const float o[4] = {o4.x, o4.y, o4.z, o4.w};
#pragma unroll
            for (int x = 0; x < 4; ++x)
#pragma unroll
                for (int y = 0; y < 4; ++y) acc[x][y] += m[x] * o[y];
        }
#pragma unroll
        for (int x = 0; x < 4; ++x)
#pragma unroll
            for (int y = 0; y < 4; ++y) sm.Qt[(r0 + x) * LDB + j0 + y] = acc[x][y];
    }
    // Bk = diag(beta) Kt (Kt is not needed any more) and the chunk's gamma and beta
    for (int idx = tid; idx < C * DK / 4; idx += NT_BP) {
        const int r = idx / (DK / 4), c = 4 * (idx % (DK / 4));
        const float bt = sm.beta[r];
        const float4 k4 = *reinterpret_cast<const float4 *>(sm.Kt + r * LDB + c);
        *reinterpret_cast<float4 *>(a.ck_Bk + rec * kBwdRowsFloats + 4 * idx) =
            make_float4(bt * k4.x, bt * k4.y, bt * k4.z, bt * k4.w);
    }
    if (tid < DK) a.ck_gb[rec * kBwdSmallFloats + tid] = sm.gam[tid];
    else if (tid < DK + C) a.ck_gb[rec * kBwdSmallFloats + tid] = sm.beta[tid - DK];
    __syncthreads();
    // (I + A)^T X = B for B = M^T dO (in Qt) and B = Ke, 16-row blocks from the last: the block minus
    // the solved rows below it (all threads), then back substitution inside the block (a thread per
    // column, 128 columns of each matrix)
#pragma unroll 1
    for (int b = 3; b >= 0; --b) {
        if (b < 3) {   // thread -> matrix tid / 256, rows r, r + 1 of the block, columns j .. j + 3
            float *X = (tid < 256) ? sm.Qt : sm.Ke;
            const int t = tid & 255, r = 16 * b + 2 * (t >> 5), j = 4 * (t & 31);
            float4 v0 = *reinterpret_cast<const float4 *>(X + r * LDB + j);
            float4 v1 = *reinterpret_cast<const float4 *>(X + (r + 1) * LDB + j);
#pragma unroll 4
            for (int i = 16 * (b + 1); i < C; ++i) {
                const float a0 = sm.A[i * LDC + r], a1 = sm.A[i * LDC + r + 1];
                const float4 x = *reinterpret_cast<const float4 *>(X + i * LDB + j);
                v0.x -= a0 * x.x; v0.y -= a0 * x.y; v0.z -= a0 * x.z; v0.w -= a0 * x.w;
                v1.x -= a1 * x.x; v1.y -= a1 * x.y; v1.z -= a1 * x.z; v1.w -= a1 * x.w;
            }
            *reinterpret_cast<float4 *>(X + r * LDB + j) = v0;
            *reinterpret_cast<float4 *>(X + (r + 1) * LDB + j) = v1;
        }
        __syncthreads();
        if (tid < 2 * DK) {
            float *X = (tid < DK) ? sm.Qt : sm.Ke;
            const int j = tid % DK;
            float y[16];
#pragma unroll
            for (int r = 15; r >= 0; --r) {
                float v = X[(16 * b + r) * LDB + j];
#pragma unroll
                for (int i = r + 1; i < 16; ++i) v -= sm.A[(16 * b + i) * LDC + 16 * b + r] * y[i];
                y[r] = v;
                X[(16 * b + r) * LDB + j] = v;
            }
        }
        __syncthreads();
    }
    for (int idx = tid; idx < C * DK / 4; idx += NT_BP) {
        const int r = idx / (DK / 4), c = 4 * (idx % (DK / 4));
        *reinterpret_cast<float4 *>(a.ck_Y0 + rec * kBwdRowsFloats + 4 * idx) =
            *reinterpret_cast<const float4 *>(sm.Qt + r * LDB + c);
        *reinterpret_cast<float4 *>(a.ck_Kp + rec * kBwdRowsFloats + 4 * idx) =
            *reinterpret_cast<const float4 *>(sm.Ke + r * LDB + c);
    }
}

// ------------------------------------------------------------------------------------------
// 2b. reverse scan of the state gradient on the prepared operands
// ------------------------------------------------------------------------------------------
// Per chunk, from the last: record dS' (the gradient reaching the chunk's end), Y = Y0 + Kp dS',
// dV = diag(beta) Y, record Y, dS = Diag(gamma) dS' + G0 - Bk^T Y. One CTA per (sequence, head,
// 32 value columns); the next chunk's operands are copied in (cp.async, two buffers) while this
// one is computed.
constexpr int NT_RS = 256;
constexpr int LDP = DK + 4;      // row stride of the 64 x 128 operand tiles (16-byte aligned rows)

struct RscanBuf {
    float Kp[C * LDP];
    float Bk[C * LDP];
    float Y0[C * DVB];
    float G0[DK * DVB];
    float gb[kBwdSmallFloats];
};
struct RscanSmem {
    RscanBuf buf[2];
    float dS[DK * DVB];
    float Y[C * DVB];
    float Yp[C * DVB];       // the upper key-channel half's part of Kp dS'
};

// acc + a.x b.x + a.y b.y + a.z b.z + a.w b.w, added in that order
__device__ __forceinline__ float dot4acc(float acc, const float4 a, const float4 b) {
    acc += a.x * b.x;
    acc += a.y * b.y;
    acc += a.z * b.z;
    acc += a.w * b.w;
    return acc;
}

__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait0() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

template <typename T>
__global__ void __launch_bounds__(NT_RS, 1)
chunk_bwd_rscan_kernel(BwdArgs a)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    RscanSmem &sm = *reinterpret_cast<RscanSmem *>(smem_raw);
    const int tid = threadIdx.x;
    const int j0 = blockIdx.x * DVB;
    const int h = blockIdx.y;
    const int n = blockIdx.z;
    const int H = a.H;
    int64_t t0, t1;
    if (!sequence_span(a.cu_seqlens, n, a.N, a.T, &t0, &t1, a.status)) return;
    const size_t sbase = ((size_t)n * H + h) * DK * DK;
    if (!in_bounds(a.status, (long long)sbase, DK * DK, (long long)a.N * H * DK * DK)) return;
    for (int idx = tid; idx < DK * DVB; idx += NT_RS) {
        const int c = idx / DVB, j = idx % DVB;
        sm.dS[idx] = a.dS_final ? a.dS_final[sbase + (size_t)c * DK + j0 + j] : 0.f;
    }
    const int64_t n_chunks = (t1 - t0 + C - 1) / C;
    auto record_of = [&](int64_t ci) { return (size_t)h * a.n_slots + (size_t)chunk_slot(t0 + ci * C, n); };
    // copy the prepared operands of chunk ci into buffer b (16-byte pieces, 11 or 12 per thread)
    auto fetch = [&](int64_t ci, int b) {
        const size_t rec = record_of(ci);
        RscanBuf &B = sm.buf[b];
        const float *kp = a.ck_Kp + rec * kBwdRowsFloats, *bk = a.ck_Bk + rec * kBwdRowsFloats;
        for (int idx = tid; idx < C * (DK / 4); idx += NT_RS) {
            const int r = idx / (DK / 4), q = idx % (DK / 4);
            cp_async16(B.Kp + r * LDP + 4 * q, kp + (size_t)r * DK + 4 * q);
            cp_async16(B.Bk + r * LDP + 4 * q, bk + (size_t)r * DK + 4 * q);
        }
        const float *y0 = a.ck_Y0 + rec * kBwdRowsFloats + j0, *g0 = a.ck_G0 + rec * kBwdStateFloats + j0;
        for (int idx = tid; idx < C * (DVB / 4); idx += NT_RS) {
            const int r = idx / (DVB / 4), q = idx % (DVB / 4);
            cp_async16(B.Y0 + r * DVB + 4 * q, y0 + (size_t)r * DK + 4 * q);
        }
        for (int idx = tid; idx < DK * (DVB / 4); idx += NT_RS) {
            const int c = idx / (DVB / 4), q = idx % (DVB / 4);
            cp_async16(B.G0 + c * DVB + 4 * q, g0 + (size_t)c * DK + 4 * q);
        }
        if (tid < (int)(kBwdSmallFloats / 4)) cp_async16(B.gb + 4 * tid, a.ck_gb + rec * kBwdSmallFloats + 4 * tid);
        cp_async_commit();
    };
    if (n_chunks > 0) fetch(n_chunks - 1, 0);
    for (int64_t ci = n_chunks - 1; ci >= 0; --ci) {
        const int b = (int)((n_chunks - 1 - ci) & 1);
        const int64_t s = t0 + ci * C;
        const int L = (t1 - s < C) ? (int)(t1 - s) : C;
        const size_t rec = record_of(ci);
        if (!in_bounds(a.status, s, L, (long long)a.B * a.T) ||
            !in_bounds(a.status, (long long)rec, 1, (long long)H * a.n_slots))
            break;
        __syncthreads();                  // the other buffer is free (its chunk is done)
        if (ci > 0) { fetch(ci - 1, b ^ 1); cp_async_wait1(); } else { cp_async_wait0(); }
        // record dS' (the gradient reaching this chunk's end) while the operands are in use
        fp32c::store_block32<NT_RS>(a.ck_dS + rec * kBwdStateFloats + j0, DK, sm.dS, DK, tid);
        __syncthreads();
        const RscanBuf &B = sm.buf[b];
        {   // Y = Y0 + Kp dS', the key-channel sum in two halves (warps 0-3: c < 64, warps 4-7: the
            // rest, whose part goes through Yp): thread -> rows rq + 16 x (x < 4), columns 4 jq .. + 3.
            // Per channel a warp reads 4 Kp values (4 rows in 4 banks) and one 128-byte row of dS'.
            const int g = tid >> 7, t = tid & 127, rq = t >> 3, jq = t & 7;
            float acc[4][4];
#pragma unroll
            for (int x = 0; x < 4; ++x)
#pragma unroll
                for (int y = 0; y < 4; ++y) acc[x][y] = 0.f;
#pragma unroll 4
            for (int c = 64 * g; c < 64 * g + 64; ++c) {
                const float4 d4 = *reinterpret_cast<const float4 *>(sm.dS + c * DVB + 4 * jq);
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    const float kp = B.Kp[(rq + 16 * x) * LDP + c];
                    acc[x][0] += kp * d4.x; acc[x][1] += kp * d4.y; acc[x][2] += kp * d4.z; acc[x][3] += kp * d4.w;
                }
            }
            if (g == 1) {
#pragma unroll
                for (int x = 0; x < 4; ++x)
                    *reinterpret_cast<float4 *>(sm.Yp + (rq + 16 * x) * DVB + 4 * jq) =
                        make_float4(acc[x][0], acc[x][1], acc[x][2], acc[x][3]);
            }
            __syncthreads();
            if (g == 0) {
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    const int o = (rq + 16 * x) * DVB + 4 * jq;
                    const float4 y0 = *reinterpret_cast<const float4 *>(B.Y0 + o);
                    const float4 yp = *reinterpret_cast<const float4 *>(sm.Yp + o);
                    *reinterpret_cast<float4 *>(sm.Y + o) =
                        make_float4(y0.x + (acc[x][0] + yp.x), y0.y + (acc[x][1] + yp.y),
                                    y0.z + (acc[x][2] + yp.z), y0.w + (acc[x][3] + yp.w));
                }
            }
        }
        __syncthreads();
        fp32c::store_block32<NT_RS>(a.ck_Y + rec * kBwdRowsFloats + j0, DK, sm.Y, C, tid);
        fp32c::store_block32<NT_RS>(a.dv + ((size_t)s * H + h) * DK + j0, (size_t)H * DK, sm.Y, L, tid, B.gb + DK);
        {   // dS = Diag(gamma) dS' + G0 - Bk^T Y: thread -> key channels 4 cq .. + 3, columns 4 jq .. + 3
            const int cq = tid >> 3, jq = tid & 7;
            float acc[4][4];
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                const int o = (4 * cq + x) * DVB + 4 * jq;
                const float gm = B.gb[4 * cq + x];
                const float4 d4 = *reinterpret_cast<const float4 *>(sm.dS + o);
                const float4 g4 = *reinterpret_cast<const float4 *>(B.G0 + o);
                acc[x][0] = gm * d4.x + g4.x; acc[x][1] = gm * d4.y + g4.y;
                acc[x][2] = gm * d4.z + g4.z; acc[x][3] = gm * d4.w + g4.w;
            }
#pragma unroll 4
            for (int r = 0; r < C; ++r) {
                const float4 bk = *reinterpret_cast<const float4 *>(B.Bk + r * LDP + 4 * cq);
                const float4 y4 = *reinterpret_cast<const float4 *>(sm.Y + r * DVB + 4 * jq);
                const float b4[4] = {bk.x, bk.y, bk.z, bk.w};
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    acc[x][0] -= b4[x] * y4.x; acc[x][1] -= b4[x] * y4.y;
                    acc[x][2] -= b4[x] * y4.z; acc[x][3] -= b4[x] * y4.w;
                }
            }
            __syncthreads();              // every thread has read dS' (Y step and this one)
#pragma unroll
            for (int x = 0; x < 4; ++x)
                *reinterpret_cast<float4 *>(sm.dS + (4 * cq + x) * DVB + 4 * jq) =
                    make_float4(acc[x][0], acc[x][1], acc[x][2], acc[x][3]);
        }
    }
    cp_async_wait0();
    __syncthreads();
    if (a.dS0) {
        for (int idx = tid; idx < DK * DVB; idx += NT_RS) {
            const int c = idx / DVB, j = idx % DVB;
            a.dS0[sbase + (size_t)c * DK + j0 + j] = sm.dS[idx];
        }
    }
}

// ------------------------------------------------------------------------------------------
// 3. per-chunk gradients (data-parallel)
// ------------------------------------------------------------------------------------------
constexpr int NT_LOC = 512;

struct LocalSmem {
    float Kt[C * LD];
    float Kh[C * LD];        // after the last products: dg
    float Qt[C * LD];
    float E[C * LD];
    // one 32-column block of the value axis at a time; after the loop: dM, dP and their transposes
    // (64 x LDC4 each)
    float S[DK * LDV];
    float dSn[DK * LDV];
    float dO[C * LDV];       // after the last products: per-warp column sums (16 x 128)
    float U[C * LDV];
    float Y[C * LDV];
    float R[C * LDV];
    float beta[C];
    float gam[DK];
    float dgam[DK];
    float ry[C];
};
static_assert((NT_LOC / 32) * DK <= C * LDV, "per-warp column sums must fit the dO block");
static_assert(4 * C * LDC4 <= 2 * DK * LDV + 4 * C * LDV, "dM, dP and their transposes must fit the staging area");
static_assert((NT_LOC / DK) * 16 == C, "the reverse sum over rows takes quarters of 16 rows");

// COMPUTE_R: no R record (the forward records came from the bf16 state scan, which holds S and U
// but not R). R enters only dbeta, through sum_v R_rv Y_rv = sum_v V_rv Y_rv - sum_c Kt_rc (Y S^T)_rc;
// the value block of V takes R's place and Y S^T is the product this kernel forms for dKt anyway.
template <typename T, bool COMPUTE_R>
__global__ void __launch_bounds__(NT_LOC, 1)
chunk_bwd_local_kernel(BwdArgs a)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    LocalSmem &sm = *reinterpret_cast<LocalSmem *>(smem_raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int H = a.H;
    const int h = (int)(blockIdx.x % (unsigned)H), slot = (int)(blockIdx.x / (unsigned)H);
    int n, L;
    int64_t s;
    if (!slot_to_chunk(a.cu_seqlens, a.N, a.T, slot, &n, &s, &L)) return;
    const size_t rec = (size_t)h * a.n_slots + (size_t)slot;
    // every global access below lies in the token rows [s, s + L) and the (head, slot) records
    if (!in_bounds(a.status, s, L, (long long)a.B * a.T) ||
        !in_bounds(a.status, (long long)rec, 1, (long long)H * a.n_slots))
        return;
    const T *q = (const T *)a.q;
    const T *k = (const T *)a.k;
    const T *dout = (const T *)a.dout;
    const float *gS = a.ck_S + rec * kBwdStateFloats;
    const float *gdS = a.ck_dS + rec * kBwdStateFloats;
    const float *gU = a.ck_U + rec * kBwdRowsFloats;
    const float *gY = a.ck_Y + rec * kBwdRowsFloats;
    const float *gR = COMPUTE_R ? nullptr : a.ck_R + rec * kBwdRowsFloats;
    const float *gP = a.ck_P + rec * kBwdTriFloats;   // StrictLower(Kt Kh^T), from the preparation pass
    // asks L2 for the rows of value block jp (32 columns) ahead of its loads: one row segment per
    // thread (128 of S, 128 of dS', 64 each of U, Y, dO and V or R; token rows past L skipped)
    auto prefetch_block = [&](int jp) {
        const void *ptr = nullptr;
        if (tid < 128) ptr = gS + (size_t)tid * DK + jp;
        else if (tid < 256) ptr = gdS + (size_t)(tid - 128) * DK + jp;
        else if (tid < 320) ptr = gU + (size_t)(tid - 256) * DK + jp;
        else if (tid < 384) ptr = gY + (size_t)(tid - 320) * DK + jp;
        else if (tid < 448) {
            if (tid - 384 < L) ptr = dout + ((size_t)(s + tid - 384) * H + h) * DK + jp;
        } else if (tid - 448 < L) {
            if constexpr (COMPUTE_R) ptr = (const T *)a.v + ((size_t)(s + tid - 448) * H + h) * DK + jp;
            else ptr = gR + (size_t)(tid - 448) * DK + jp;
        }
        if (ptr) asm volatile("prefetch.global.L2 [%0];" ::"l"(ptr));
    };

    // ---- load q, k, log_alpha (zero past L), beta; then g = cumsum(log_alpha) in row parts
    fp32c::load_rows<T, NT_LOC, DK>(sm.Kt, LD, k, s, L, H, h, 0, tid);
    fp32c::load_rows<T, NT_LOC, DK>(sm.Qt, LD, q, s, L, H, h, 0, tid);
    fp32c::load_rows<float, NT_LOC, DK>(sm.E, LD, a.log_alpha, s, L, H, h, 0, tid);
    prefetch_block(0);
    if (tid < (int)(kBwdTriFloats / 32)) asm volatile("prefetch.global.L2 [%0];" ::"l"(gP + 32 * tid));
    if (tid < C) sm.beta[tid] = (tid < L) ? a.beta[(size_t)(s + tid) * H + h] : 0.f;
    if (tid < DK) sm.dgam[tid] = 0.f;
    if (tid < C) sm.ry[tid] = 0.f;
    __syncthreads();
    {
        const float gl = fp32c::decay_prefix<NT_LOC>(sm.E, LD, tid);
        constexpr int RP = C / (NT_LOC / DK);
        const int c = tid % DK, r0 = (tid / DK) * RP;
        if (tid < DK) sm.gam[c] = expf(gl);
        if (tid < DK && !(gl >= kMinChunkLogDecay)) set_status(a.status, KDA_ERR_UNSUPPORTED);
#pragma unroll 4
        for (int r = r0; r < r0 + RP; ++r) {
            const float g = sm.E[r * LD + c];
            const float e = expf(g), kk = sm.Kt[r * LD + c];
            sm.E[r * LD + c] = e;
            sm.Kt[r * LD + c] = kk * e;
            sm.Kh[r * LD + c] = kk * expf(-g);
            sm.Qt[r * LD + c] *= e;
        }
    }
    __syncthreads();

    // thread tile: rows 4 rb .. 4 rb + 3 (rb = warp), key columns lane + 32 x, token columns lane + 32 x
    const int rb = warp, cb = lane;

    // ---- sums over the value axis, 32 columns at a time
    float aQ[4][4], aY[4][4], aE[4][4], aM[4][2], aA[4][2];
#pragma unroll
    for (int x = 0; x < 4; ++x) {
#pragma unroll
        for (int y = 0; y < 4; ++y) { aQ[x][y] = 0.f; aY[x][y] = 0.f; aE[x][y] = 0.f; }
        aM[x][0] = aM[x][1] = aA[x][0] = aA[x][1] = 0.f;
    }
    float dgam_acc = 0.f, ry_acc = 0.f;
    for (int j0 = 0; j0 < DK; j0 += DVB) {
        __syncthreads();
        {
            // 16-byte loads, all in flight before the first store: the state blocks (128 rows of
            // 8 float4, two per thread) and the row blocks (64 rows of 8 float4, one per thread)
            float4 xs[2], xd[2], xu, xy, xr = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int it = 0; it < 2; ++it) {
                const int idx = tid + it * NT_LOC, c = idx >> 3, q4 = idx & 7;
                xs[it] = __ldg(reinterpret_cast<const float4 *>(gS + (size_t)c * DK + j0) + q4);
                xd[it] = __ldg(reinterpret_cast<const float4 *>(gdS + (size_t)c * DK + j0) + q4);
            }
            const int r = tid >> 3, q4 = tid & 7;
            xu = __ldg(reinterpret_cast<const float4 *>(gU + (size_t)r * DK + j0) + q4);
            xy = __ldg(reinterpret_cast<const float4 *>(gY + (size_t)r * DK + j0) + q4);
            if constexpr (!COMPUTE_R) xr = __ldg(reinterpret_cast<const float4 *>(gR + (size_t)r * DK + j0) + q4);
            fp32c::load_rows<T, NT_LOC, DVB>(sm.dO, LDV, dout, s, L, H, h, j0, tid);
            if constexpr (COMPUTE_R) fp32c::load_rows<T, NT_LOC, DVB>(sm.R, LDV, (const T *)a.v, s, L, H, h, j0, tid);
#pragma unroll
            for (int it = 0; it < 2; ++it) {
                const int idx = tid + it * NT_LOC, c = idx >> 3, v = (idx & 7) * 4;
                *reinterpret_cast<float4 *>(sm.S + c * LDV + v) = xs[it];
                *reinterpret_cast<float4 *>(sm.dSn + c * LDV + v) = xd[it];
            }
            const int v = q4 * 4;
            *reinterpret_cast<float4 *>(sm.U + r * LDV + v) = xu;
            *reinterpret_cast<float4 *>(sm.Y + r * LDV + v) = xy;
            if constexpr (!COMPUTE_R) *reinterpret_cast<float4 *>(sm.R + r * LDV + v) = xr;
        }
        __syncthreads();
        if (j0 + DVB < DK) prefetch_block(j0 + DVB);
        // float4 steps along the value axis: the thread's rows of dO, Y, U are broadcasts, the
        // column rows of S, dS', U fall in 8 distinct bank groups per phase (row stride 9 groups);
        // two loops, so that fewer operands are live at once
#pragma unroll 2
        for (int v = 0; v < DVB; v += 4) {
            float4 o[4], y[4];
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                o[x] = *reinterpret_cast<const float4 *>(sm.dO + (4 * rb + x) * LDV + v);
                y[x] = *reinterpret_cast<const float4 *>(sm.Y + (4 * rb + x) * LDV + v);
            }
#pragma unroll
            for (int z = 0; z < 4; ++z) {
                const float4 sv = *reinterpret_cast<const float4 *>(sm.S + (cb + 32 * z) * LDV + v);
#pragma unroll
                for (int x = 0; x < 4; ++x) { aQ[x][z] = dot4acc(aQ[x][z], o[x], sv); aY[x][z] = dot4acc(aY[x][z], y[x], sv); }
            }
#pragma unroll
            for (int z = 0; z < 2; ++z) {
                const float4 ui = *reinterpret_cast<const float4 *>(sm.U + (cb + 32 * z) * LDV + v);
#pragma unroll
                for (int x = 0; x < 4; ++x) { aM[x][z] = dot4acc(aM[x][z], o[x], ui); aA[x][z] = dot4acc(aA[x][z], y[x], ui); }
            }
        }
#pragma unroll 2
        for (int v = 0; v < DVB; v += 4) {
            float4 u[4];
#pragma unroll
            for (int x = 0; x < 4; ++x) u[x] = *reinterpret_cast<const float4 *>(sm.U + (4 * rb + x) * LDV + v);
#pragma unroll
            for (int z = 0; z < 4; ++z) {
                const float4 dv = *reinterpret_cast<const float4 *>(sm.dSn + (cb + 32 * z) * LDV + v);
#pragma unroll
                for (int x = 0; x < 4; ++x) aE[x][z] = dot4acc(aE[x][z], u[x], dv);
            }
        }
        if (tid < DK) {
#pragma unroll
            for (int v = 0; v < DVB; v += 4)
                dgam_acc = dot4acc(dgam_acc, *reinterpret_cast<const float4 *>(sm.dSn + tid * LDV + v),
                                   *reinterpret_cast<const float4 *>(sm.S + tid * LDV + v));
        } else if (tid < DK + C) {
            const int r = tid - DK;
#pragma unroll
            for (int v = 0; v < DVB; v += 4)
                ry_acc = dot4acc(ry_acc, *reinterpret_cast<const float4 *>(sm.R + r * LDV + v),
                                 *reinterpret_cast<const float4 *>(sm.Y + r * LDV + v));
        }
    }
    __syncthreads();                                   // the value blocks are dead from here on
    // dM, dP and their transposes, 64 x LDC4 each, in the staging area
    float *dM = sm.S, *dP = dM + C * LDC4, *dMT = dP + C * LDC4, *dPT = dMT + C * LDC4;
    if (tid < DK) sm.dgam[tid] = dgam_acc;
    else if (tid < DK + C) sm.ry[tid - DK] = ry_acc;
    {
        // dM = tril(dO U^T); dA = -StrictLower(Y U^T); dP = diag(beta) dA; dbeta's A part
        float part[4];
#pragma unroll
        for (int x = 0; x < 4; ++x) {
            const int r = 4 * rb + x;
            part[x] = 0.f;
#pragma unroll
            for (int z = 0; z < 2; ++z) {
                const int i = cb + 32 * z;
                const float da = (i < r) ? -aA[x][z] : 0.f;
                const float mv = (i <= r) ? aM[x][z] : 0.f, pv = sm.beta[r] * da;
                dM[r * LDC4 + i] = mv;
                dMT[i * LDC4 + r] = mv;
                dP[r * LDC4 + i] = pv;
                dPT[i * LDC4 + r] = pv;
                part[x] += da * __ldg(gP + r * C + i);
            }
            if constexpr (COMPUTE_R) {        // - sum_c Kt_rc (Y S^T)_rc over this thread's 4 columns
#pragma unroll
                for (int z = 0; z < 4; ++z) part[x] -= sm.Kt[r * LD + cb + 32 * z] * aY[x][z];
            }
        }
#pragma unroll
        for (int x = 0; x < 4; ++x) {
#pragma unroll
            for (int m = 16; m >= 1; m >>= 1) part[x] += __shfl_xor_sync(0xffffffffu, part[x], m);
        }
        __syncthreads();                               // ry, dM, dP complete
        if (lane == 0) {
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                const int r = 4 * rb + x;
                if (r < L) a.dbeta[(size_t)(s + r) * H + h] = sm.ry[r] + part[x];
            }
        }
    }

    // ---- dQt, dKt, dKh for the thread's 4 x 4 tile, then dq, dk and dg
    float dg[4][4], colp[4];
#pragma unroll
    for (int z = 0; z < 4; ++z) colp[z] = 0.f;
    {
        float dQ[4][4], dKt[4][4], dKh[4][4];
#pragma unroll
        for (int x = 0; x < 4; ++x) {
            const float br = sm.beta[4 * rb + x];
#pragma unroll
            for (int z = 0; z < 4; ++z) { dQ[x][z] = aQ[x][z]; dKt[x][z] = -br * aY[x][z]; dKh[x][z] = 0.f; }
        }
        for (int i = 0; i < C; ++i) {
            float kh[4], qt[4], kt[4];
#pragma unroll
            for (int z = 0; z < 4; ++z) {
                kh[z] = sm.Kh[i * LD + cb + 32 * z];
                qt[z] = sm.Qt[i * LD + cb + 32 * z];
                kt[z] = sm.Kt[i * LD + cb + 32 * z];
            }
            // the thread's 4 rows r of column i (dQt, dKt) and of row i (dKh): four broadcasts
            const float4 m_c = *reinterpret_cast<const float4 *>(dMT + i * LDC4 + 4 * rb);   // dM[r][i]
            const float4 p_c = *reinterpret_cast<const float4 *>(dPT + i * LDC4 + 4 * rb);   // dP[r][i]
            const float4 m_r = *reinterpret_cast<const float4 *>(dM + i * LDC4 + 4 * rb);    // dM[i][r]
            const float4 p_r = *reinterpret_cast<const float4 *>(dP + i * LDC4 + 4 * rb);    // dP[i][r]
            const float m_ri[4] = {m_c.x, m_c.y, m_c.z, m_c.w}, p_ri[4] = {p_c.x, p_c.y, p_c.z, p_c.w};
            const float m_ir[4] = {m_r.x, m_r.y, m_r.z, m_r.w}, p_ir[4] = {p_r.x, p_r.y, p_r.z, p_r.w};
#pragma unroll
            for (int x = 0; x < 4; ++x) {
#pragma unroll
                for (int z = 0; z < 4; ++z) {
                    dQ[x][z] += m_ri[x] * kh[z];
                    dKt[x][z] += p_ri[x] * kh[z];
                    dKh[x][z] += m_ir[x] * qt[z] + p_ir[x] * kt[z];
                }
            }
        }
#pragma unroll
        for (int x = 0; x < 4; ++x) {
            const int r = 4 * rb + x;
#pragma unroll
            for (int z = 0; z < 4; ++z) {
                const int c = cb + 32 * z;
                const float e = sm.E[r * LD + c], gm = sm.gam[c];
                const float ktv = sm.Kt[r * LD + c], khv = sm.Kh[r * LD + c], qtv = sm.Qt[r * LD + c];
                const float dke = aE[x][z], ke = khv * gm;
                if (r < L) {
                    const size_t off = ((size_t)(s + r) * H + h) * DK + c;
                    a.dq[off] = dQ[x][z] * e;
                    a.dk[off] = dKt[x][z] * e + (dKh[x][z] + dke * gm) / e;
                }
                dg[x][z] = dQ[x][z] * qtv + dKt[x][z] * ktv - dKh[x][z] * khv - dke * ke;
                colp[z] += dke * ke;
            }
        }
    }
    __syncthreads();                                   // Kh is free: it takes dg
#pragma unroll
    for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int z = 0; z < 4; ++z) sm.Kh[(4 * rb + x) * LD + cb + 32 * z] = dg[x][z];
    // per-warp column sums of dKe * Ke into the (now free) dO block, added in a fixed order below
#pragma unroll
    for (int z = 0; z < 4; ++z) sm.dO[rb * DK + cb + 32 * z] = colp[z];
    __syncthreads();
    // ---- dlog_alpha: reverse cumulative sum over rows, the last row also carrying the terms of
    //      g_{L-1} (through Ke and gamma)
    //      on all threads: 4 quarters of 16 rows per channel, each quarter's sum first
    {
        const int c = tid & (DK - 1), qd = tid / DK;
        float part = 0.f;
#pragma unroll
        for (int r = 16 * qd; r < 16 * qd + 16; ++r) part += sm.Kh[r * LD + c];
        float *qsum = sm.S;                            // free again (it held dM)
        qsum[qd * DK + c] = part;
        float run = 0.f;
        for (int w = 0; w < NT_LOC / 32; ++w) run += sm.dO[w * DK + c];
        run += sm.dgam[c] * sm.gam[c];
        __syncthreads();
        for (int q2 = NT_LOC / DK - 1; q2 > qd; --q2) run += qsum[q2 * DK + c];
#pragma unroll 4
        for (int r = 16 * qd + 15; r >= 16 * qd; --r) {
            run += sm.Kh[r * LD + c];
            if (r < L) a.dlog_alpha[((size_t)(s + r) * H + h) * DK + c] = run;
        }
    }
}

template <typename T>
cudaError_t launch_rscan_typed(const BwdArgs &a, cudaStream_t stream)
{
    cudaError_t e = cudaFuncSetAttribute(chunk_bwd_prep_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)sizeof(BprepSmem));
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(chunk_bwd_rscan_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)sizeof(RscanSmem));
    if (e != cudaSuccess) return e;
    chunk_bwd_prep_kernel<T><<<(unsigned)((long long)a.n_slots * a.H), NT_BP, sizeof(BprepSmem), stream>>>(a);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    chunk_bwd_rscan_kernel<T><<<dim3(DK / DVB, a.H, a.N), NT_RS, sizeof(RscanSmem), stream>>>(a);
    return cudaGetLastError();
}

template <typename T, bool COMPUTE_R>
cudaError_t launch_local_variant(const BwdArgs &a, cudaStream_t stream)
{
    const size_t smem = sizeof(LocalSmem);
    cudaError_t e = cudaFuncSetAttribute(chunk_bwd_local_kernel<T, COMPUTE_R>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const long long blocks = (long long)a.n_slots * a.H;
    chunk_bwd_local_kernel<T, COMPUTE_R><<<(unsigned)blocks, NT_LOC, smem, stream>>>(a);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_local_typed(const BwdArgs &a, cudaStream_t stream)
{
    return a.ck_R ? launch_local_variant<T, false>(a, stream) : launch_local_variant<T, true>(a, stream);
}

}  // namespace

cudaError_t launch_chunk_bwd_scan(const BwdArgs &a, kda_dtype_t dtype, cudaStream_t stream)
{
    if (a.N == 0) return cudaSuccess;
    if (!a.ck_Kp || !a.ck_Bk || !a.ck_Y0 || !a.ck_G0 || !a.ck_gb || !a.ck_P) return cudaErrorInvalidValue;
    // the data-parallel preparation of every chunk's operands, then the reverse scan
    return dtype == KDA_BF16 ? launch_rscan_typed<__nv_bfloat16>(a, stream) : launch_rscan_typed<float>(a, stream);
}

cudaError_t launch_chunk_bwd_local(const BwdArgs &a, kda_dtype_t dtype, cudaStream_t stream)
{
    if (a.N == 0 || a.n_slots == 0) return cudaSuccess;
    if (!a.ck_P) return cudaErrorInvalidValue;
    return dtype == KDA_BF16 ? launch_local_typed<__nv_bfloat16>(a, stream) : launch_local_typed<float>(a, stream);
}

}  // namespace kda
