// chunk_tc.cu -- chunkwise KDA prefill on the sm_100a tensor cores (tcgen05 + TMEM) for bf16
// q/k/v: f16 MMA operands, fp32 accumulation and an fp32 inter-chunk state.
//
// Why f16 operands: every product below rounds its operands once; with bf16's 8-bit significand
// the nine rounded operands together put the worst output 3-5% of RMS away from the exact result
// on 8K-token inputs, while f16's 11-bit significand (same MMA rate, same shared-memory size)
// keeps it near 0.4%. The price is range (see kMinChunkDecay).
//
// Chunk form (chunk C = 64 tokens; chunk-parallel prefill with a WY/UT representation, chunk_size
// 64: KimiLinear KDA/MLA tutorial (icman.com.cn), sec. 3 and sec. 6; the algebra is derived from
// the recurrence). For one chunk of L <= 64 tokens entering with state S (d_k x d_v), per key
// channel c, with g_r = sum_{j<=r} log_alpha_j:
//   f_r = e^{g_r},  b_r = e^{g_{L-1} - g_r},  gamma = e^{g_{L-1}}
//   Kt = K f,  Qt = Q f,  Kend = K b,  Kh = K b / gamma (= K e^{-g})
//   A  = StrictLower(diag(beta) Kt Kh^T),  M = tril(Qt Kh^T),  Tb = (I + A)^{-1} diag(beta)
//   W  = Tb Kt;   U = Tb V - W S;   O = Qt S + M U;   S <- Diag(gamma) S + Kend^T U
// f and b are running products of alpha = exp(log_alpha) (forward and backward within the chunk).
//
// This single-kernel form needs no workspace beyond the status word, so kda_chunk_fwd_noalloc runs
// it; kda_chunk_fwd runs the faster two-pass form (chunk_prep.cu, chunk_scan.cu, prefill.cu).
//
// Work split: one CTA per (sequence, head, 32-column block of d_v). The value columns of S evolve
// independently, so the four blocks of a head never communicate; each recomputes the
// d_v-independent part of a chunk. Inside a CTA two warp groups run a two-stage pipeline:
//
//   prep group (8 warps) for chunk c+1            scan group (4 warps) for chunk c
//   --------------------------------------        ------------------------------------------
//   coalesced loads of the chunk's rows            S1: D5 += [W; Qt] S          (M=128,N=32,K=128)
//                                                  U  = -(D5 rows 0-63) -> f16
//   decay scaling (fp32) -> Kt Qt Kh Kend (f16)    S2: D7 = Kend^T U            (M=128,N=32,K=64)
//   P1: Qt Kh^T, Kt Kh^T  (two M=64, N=64, K=128)  MU: D5 += [0; M] U           (M=128,N=32,K=64)
//   M (f16), A (fp32); T = (I + A)^{-1} (fp32,     S <- gamma S + D7 (fp32 registers), S -> f16
//     16x16 diagonal blocks + register-tiled       O = D5 rows 64-127 -> out
//     block products); Tb = T diag(beta) (f16)
//   P3: [Tb; 0] Kt -> W;  seed D5 = -[Tb; 0] V
//
// Operands produced for the scan (W, Qt, Tb, M, Kend, V and the seeded accumulator) are double
// buffered by chunk parity; `ready` hands a parity to the scan group and `free` returns it.
// Stacked operands ([W; Qt], [Tb; 0], [0; M]) are contiguous row ranges of one swizzled region so
// that one M=128 instruction covers both halves.
#include "kda_internal.cuh"
#include "sm100.cuh"

namespace kda {
namespace {

using namespace sm100;

constexpr int C = kChunk;          // 64
constexpr int DK = kHeadDim;       // 128
constexpr int DVB = 32;            // value columns per CTA
constexpr int SG_THREADS = 128;    // scan group: warps 0-3
constexpr int PG_THREADS = 256;    // prep group: warps 4-11
constexpr int NT = SG_THREADS + PG_THREADS;

// Operands are rounded to f16 (11-bit significand) for the tensor cores: the largest one, Kh =
// K e^{-g}, must stay finite and its partner Kt = K e^{g} must keep its significand (f16 numbers
// below 2^-14 are subnormal), so the decay accumulated over one chunk must keep e^{g} above 2^-13
// per channel (cumulative log-decay >= -9.0; in float64 emulation the worst output error then stays
// near 0.5% of RMS, while around -10.5 it reaches 5%). Chunks beyond that report UNSUPPORTED.
constexpr float kMinChunkDecay = 1.220703125e-04f;

// ---- shared memory plan (byte offsets from a 1024-byte aligned base)
constexpr uint32_t X_HALF = 128 * 128;                 // per 64-channel half: rows 0-63 W, 64-127 Qt
constexpr uint32_t X_BYTES = 2 * X_HALF;
constexpr uint32_t Y_BYTES = 192 * 128;                // rows 0-63 Tb, 64-127 zero, 128-191 M
constexpr uint32_t KE_BYTES = 2 * 64 * 128;            // Kend, two halves
constexpr uint32_t V_BYTES = C * DVB * 2;              // v block (f16), 64-byte rows
constexpr uint32_t OFF_X0 = 0;
constexpr uint32_t OFF_X1 = OFF_X0 + X_BYTES;
constexpr uint32_t OFF_Y0 = OFF_X1 + X_BYTES;
constexpr uint32_t OFF_Y1 = OFF_Y0 + Y_BYTES;
constexpr uint32_t OFF_KE0 = OFF_Y1 + Y_BYTES;
constexpr uint32_t OFF_KE1 = OFF_KE0 + KE_BYTES;
constexpr uint32_t OFF_V0 = OFF_KE1 + KE_BYTES;
constexpr uint32_t OFF_V1 = OFF_V0 + V_BYTES;
constexpr uint32_t OFF_KT = OFF_V1 + V_BYTES;          // Kt (f16), two halves
constexpr uint32_t OFF_KH = OFF_KT + 16384;            // Kh (f16); after P1: A^T (fp32, column-major)
constexpr int LDT = 68;                                // row stride of T (floats): conflict-free columns
constexpr uint32_t OFF_TF = OFF_KH + 16384;            // T (fp32, row-major, stride LDT)
constexpr uint32_t OFF_SB = OFF_TF + 18432;            // S (f16), 128 rows x 64 B
constexpr uint32_t OFF_UB = OFF_SB + DK * DVB * 2;     // U (f16), 64 rows x 64 B
constexpr uint32_t OFF_PS = OFF_UB + C * DVB * 2;      // block-product scratch of the inverse (fp32)
constexpr uint32_t OFF_GAM = OFF_PS + 32 * 32 * 4;     // gamma, 2 x 128 fp32
constexpr uint32_t OFF_BET = OFF_GAM + 2 * 128 * 4;    // beta, 64 fp32
constexpr uint32_t OFF_BAR = OFF_BET + 64 * 4;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 128;
constexpr uint32_t SMEM_ALLOC = SMEM_BYTES + 1024;
static_assert(SMEM_ALLOC <= 232448, "shared memory plan exceeds 227 KiB");
static_assert((OFF_Y0 | OFF_Y1 | OFF_KE0 | OFF_KE1 | OFF_KT | OFF_KH | OFF_SB | OFF_UB) % 1024 == 0,
              "swizzled operand regions must be 1024-byte aligned");

constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TM_D1A = 0;     // 64 cols, M=64 layout: Qt Kh^T
constexpr uint32_t TM_D1B = 64;    // 64 cols, M=64 layout: Kt Kh^T
constexpr uint32_t TM_D3 = 128;    // 128 cols: [Tb; 0] Kt (rows 0-63 = W)
constexpr uint32_t TM_D5 = 256;    // 2 x 32 cols: -U | O per chunk parity
constexpr uint32_t TM_D7 = 320;    // 32 cols: Kend^T U

// mbarrier slots
enum { B_READY = 0, B_FREE = 2, B_P1 = 4, B_P3 = 5, B_S1 = 6, B_S2 = 7, B_MU = 8, N_BARS = 9 };

struct TcParams {
    const __nv_bfloat16 *q, *k, *v;
    const float *log_alpha, *beta, *S0;
    const int32_t *cu_seqlens;
    void *out;
    float *S_final;
    int T, H, N;
    long long tokens;               // B * T (rows of q, k, v, log_alpha, out)
    int32_t *status;
};

__device__ __forceinline__ float bf_lo(uint32_t x) { return __uint_as_float(x << 16); }
__device__ __forceinline__ float bf_hi(uint32_t x) { return __uint_as_float(x & 0xFFFF0000u); }
__device__ __forceinline__ uint4 ldg_nc(const void *p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
    return r;
}
__device__ __forceinline__ uint2 ldg_nc_u2(const void *p) {
    uint2 r;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];" : "=r"(r.x), "=r"(r.y) : "l"(p));
    return r;
}
__device__ __forceinline__ float4 ldg_nc_f4(const float *p) {
    const uint4 r = ldg_nc(p);
    return make_float4(__uint_as_float(r.x), __uint_as_float(r.y), __uint_as_float(r.z), __uint_as_float(r.w));
}

// Unit lower-triangular inverse T = (I + A)^{-1} for a 64 x 64 strictly lower A held column-major
// (AT[c * 64 + r] = A[r][c]); T is written row-major with stride LDT. Diagonal 16 x 16 blocks by
// forward substitution in registers; then T_{b+1,b} = -T_{b+1,b+1} A_{b+1,b} T_{b,b} inside each
// 32 x 32 half, then T_{hi,lo} = -T_hi A_{hi,lo} T_lo for the off-diagonal 32 x 32 block.
// Called by the 256 prep threads (pt = 0..255); ends synchronised.
__device__ __forceinline__ void prep_inverse(int pt, const float *AT, float *Tf, float *Ps)
{
    const int pw = pt >> 5, lane = pt & 31;
    if (pw < 2) {
        // warp 0: blocks 0 and 1 (lanes 0-15 / 16-31); warp 1: blocks 2 and 3
        const int o = 16 * (2 * pw + (lane >> 4)), j = lane & 15;
        float xv[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) xv[r] = (r == j) ? 1.f : 0.f;
#pragma unroll
        for (int i = 0; i < 15; ++i) {
            float col[16];
            const float4 *cp = reinterpret_cast<const float4 *>(AT + (o + i) * 64 + o);
#pragma unroll
            for (int u = (i + 1) >> 2; u < 4; ++u) {
                const float4 t = cp[u];
                col[4 * u] = t.x; col[4 * u + 1] = t.y; col[4 * u + 2] = t.z; col[4 * u + 3] = t.w;
            }
            const float xi = xv[i];
#pragma unroll
            for (int r = i + 1; r < 16; ++r) xv[r] -= col[r] * xi;
        }
#pragma unroll
        for (int r = 0; r < 16; ++r) Tf[(o + r) * LDT + o + j] = xv[r];
    } else {
        // zero the strictly upper 16 x 16 blocks of T
        for (int e = pt - 64; e < 64 * 64; e += 192) {
            const int r = e >> 6, c = e & 63;
            if ((c >> 4) > (r >> 4)) Tf[r * LDT + c] = 0.f;
        }
    }
    named_bar_sync(1, PG_THREADS);
    // level 1a: P_b = A_{b+1,b} T_{b,b} for b = 0, 2 (two outputs per thread)
    {
        const int blk = pt >> 7, idx = pt & 127, r = idx >> 3, c0 = (idx & 7) * 2;
        const int b = 2 * blk;
        float a0 = 0.f, a1 = 0.f;
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            const float a = AT[(16 * b + k) * 64 + 16 * (b + 1) + r];
            const float2 t = *reinterpret_cast<const float2 *>(Tf + (16 * b + k) * LDT + 16 * b + c0);
            a0 += a * t.x;
            a1 += a * t.y;
        }
        *reinterpret_cast<float2 *>(Ps + blk * 256 + r * 16 + c0) = make_float2(a0, a1);
    }
    named_bar_sync(1, PG_THREADS);
    // level 1b: T_{b+1,b} = -T_{b+1,b+1} P_b
    {
        const int blk = pt >> 7, idx = pt & 127, r = idx >> 3, c0 = (idx & 7) * 2;
        const int b = 2 * blk, o = 16 * (b + 1);
        float a0 = 0.f, a1 = 0.f;
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            const float t = Tf[(o + r) * LDT + o + k];
            const float2 pv = *reinterpret_cast<const float2 *>(Ps + blk * 256 + k * 16 + c0);
            a0 += t * pv.x;
            a1 += t * pv.y;
        }
        *reinterpret_cast<float2 *>(Tf + (o + r) * LDT + 16 * b + c0) = make_float2(-a0, -a1);
    }
    named_bar_sync(1, PG_THREADS);
    // level 2a: P = A[32:64, 0:32] T[0:32, 0:32] (four outputs per thread)
    {
        const int r = pt >> 3, c0 = (pt & 7) * 4;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
        for (int k = 0; k < 32; ++k) {
            const float a = AT[k * 64 + 32 + r];
            const float4 t = *reinterpret_cast<const float4 *>(Tf + k * LDT + c0);
            acc.x += a * t.x; acc.y += a * t.y; acc.z += a * t.z; acc.w += a * t.w;
        }
        *reinterpret_cast<float4 *>(Ps + r * 32 + c0) = acc;
    }
    named_bar_sync(1, PG_THREADS);
    // level 2b: T[32:64, 0:32] = -T[32:64, 32:64] P
    {
        const int r = pt >> 3, c0 = (pt & 7) * 4;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
        for (int k = 0; k < 32; ++k) {
            const float t = Tf[(32 + r) * LDT + 32 + k];
            const float4 pv = *reinterpret_cast<const float4 *>(Ps + k * 32 + c0);
            acc.x += t * pv.x; acc.y += t * pv.y; acc.z += t * pv.z; acc.w += t * pv.w;
        }
        *reinterpret_cast<float4 *>(Tf + (32 + r) * LDT + c0) = make_float4(-acc.x, -acc.y, -acc.z, -acc.w);
    }
    named_bar_sync(1, PG_THREADS);
}

// One prep thread's share of a chunk's inputs, loaded from global memory into registers one chunk
// ahead so that the load latency overlaps the previous chunk's work: rows 8rb..8rb+7 and channels
// 4cq..4cq+3 of q, k and log_alpha (rb = pt & 7, cq = pt >> 3), eight v values (row pt >> 2,
// columns 8 (pt & 3)..+7 of the d_v block) and, for pt < 64, beta of row pt.
struct RawChunk {
    float4 la[8];
    uint2 kr[8], qr[8];
    uint4 v;
    float beta;
};

__device__ __forceinline__ void prep_load(RawChunk &R, const TcParams &p, int64_t tok0, int L, int h,
                                          int j0, int pt)
{
    const int H = p.H, cq = pt >> 3, rb = pt & 7;
#pragma unroll
    for (int x = 0; x < 8; ++x) {
        const int r = 8 * rb + x;
        const long long ext = p.tokens * H * DK;
        if (r < L && in_bounds(p.status, ((long long)(tok0 + r) * H + h) * DK + 4 * cq, 4, ext)) {
            const size_t row = ((size_t)(tok0 + r) * H + h) * DK + 4 * cq;
            R.la[x] = ldg_nc_f4(p.log_alpha + row);
            R.kr[x] = ldg_nc_u2(p.k + row);
            R.qr[x] = ldg_nc_u2(p.q + row);
        } else {
            R.la[x] = make_float4(0.f, 0.f, 0.f, 0.f);
            R.kr[x] = make_uint2(0u, 0u);
            R.qr[x] = R.kr[x];
        }
    }
    const int rv = pt >> 2;
    const long long vi = ((long long)(tok0 + rv) * H + h) * DK + j0 + 8 * (pt & 3);
    R.v = (rv < L && in_bounds(p.status, vi, 8, p.tokens * H * DK)) ? ldg_nc(p.v + vi) : make_uint4(0, 0, 0, 0);
    const long long bi = (long long)(tok0 + pt) * H + h;
    R.beta = (pt < L && pt < C && in_bounds(p.status, bi, 1, p.tokens * H)) ? p.beta[bi] : 0.f;
}

// =================================================================================== kernel
template <typename TO>
__global__ void __launch_bounds__(NT, 1)
chunk_tc_kernel(TcParams p)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int jb = blockIdx.x, h = blockIdx.y, n = blockIdx.z;
    const int j0 = jb * DVB;
    const int H = p.H;

    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + OFF_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + N_BARS);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(bars + N_BARS) + 1;
    float *gam = reinterpret_cast<float *>(sm + OFF_GAM);
    float *bet = reinterpret_cast<float *>(sm + OFF_BET);

    int64_t t0, t1;
    if (!sequence_span(p.cu_seqlens, n, p.N, p.T, &t0, &t1, p.status)) return;   // uniform
    const int nchunks = (int)((t1 - t0 + C - 1) / C);

    if (warp == 0) { tmem_alloc(tmem_slot, TMEM_COLS); tmem_relinquish(); }
    if (tid == 0) {
        for (int i = 0; i < N_BARS; ++i) mbar_init(&bars[i], 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    // zero blocks of both Y regions (rows 64-127), never written again
    for (int i = tid; i < 2 * 64 * 128 / 16; i += NT) {
        const int y = i / (64 * 128 / 16), o = i % (64 * 128 / 16);
        reinterpret_cast<uint4 *>(sm + (y ? OFF_Y1 : OFF_Y0) + 64 * 128)[o] = make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    auto fail = [&]() { set_status(p.status, KDA_ERR_TIMEOUT); *abort_flag = 1; };

    if (warp >= 4) {
        // =========================================================================== prep group
        const int pt = tid - SG_THREADS, pw = warp - 4, q4 = warp & 3, half = pw >> 2;
        float *AT = reinterpret_cast<float *>(sm + OFF_KH);
        float *Tf = reinterpret_cast<float *>(sm + OFF_TF);
        float *Ps = reinterpret_cast<float *>(sm + OFF_PS);
        uint32_t n_p1 = 0, n_p3 = 0;               // commits issued (thread 0)
        RawChunk R;
        if (nchunks > 0) prep_load(R, p, t0, (t1 - t0 < C) ? (int)(t1 - t0) : C, h, j0, pt);
        for (int c = 0; c < nchunks; ++c) {
            const int s = c & 1;
            const int64_t tok0 = t0 + (int64_t)c * C;
            unsigned char *X = sm + (s ? OFF_X1 : OFF_X0);
            unsigned char *Y = sm + (s ? OFF_Y1 : OFF_Y0);
            unsigned char *KE = sm + (s ? OFF_KE1 : OFF_KE0);
            unsigned char *Vs = sm + (s ? OFF_V1 : OFF_V0);
            if (c >= 2) {               // one thread polls; the group barrier releases the others
                if (pt == 0 && !mbar_wait(&bars[B_FREE + s], ((c >> 1) - 1) & 1)) fail();
                named_bar_sync(1, PG_THREADS);
            }
            tc_fence_after();

            // ---- beta and the v block (bf16 -> f16, 64-byte swizzled rows)
            if (pt < C) bet[pt] = R.beta;
            {
                uint4 o;
                o.x = bf16x2_to_f16x2(R.v.x); o.y = bf16x2_to_f16x2(R.v.y);
                o.z = bf16x2_to_f16x2(R.v.z); o.w = bf16x2_to_f16x2(R.v.w);
                *reinterpret_cast<uint4 *>(Vs + sw64_offset(pt >> 2, 8 * (pt & 3))) = o;
            }
            // ---- decay scaling: thread -> rows 8rb..8rb+7, channels 4cq..4cq+3; the 8 row blocks of
            //      one channel quad sit on 8 consecutive lanes
            {
                const int cq = pt >> 3, rb = pt & 7, kh = cq >> 4, lc4 = cq & 15;
                float a[8][4], pre[8][4], before[4], after[4], g[4], rg[4];
#pragma unroll
                for (int x = 0; x < 8; ++x) {
                    a[x][0] = __expf(R.la[x].x); a[x][1] = __expf(R.la[x].y);
                    a[x][2] = __expf(R.la[x].z); a[x][3] = __expf(R.la[x].w);
                }
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    float run = 1.f;
#pragma unroll
                    for (int x = 0; x < 8; ++x) { run *= a[x][e]; pre[x][e] = run; }
                    float inc = run, sfx = run;
#pragma unroll
                    for (int o = 1; o < 8; o <<= 1) {
                        const float u = __shfl_up_sync(0xffffffffu, inc, o, 8);
                        const float d = __shfl_down_sync(0xffffffffu, sfx, o, 8);
                        if (rb >= o) inc *= u;
                        if (rb + o < 8) sfx *= d;
                    }
                    const float bu = __shfl_up_sync(0xffffffffu, inc, 1, 8);
                    const float ad = __shfl_down_sync(0xffffffffu, sfx, 1, 8);
                    before[e] = (rb == 0) ? 1.f : bu;
                    after[e] = (rb == 7) ? 1.f : ad;
                    g[e] = __shfl_sync(0xffffffffu, inc, 7, 8);
                    rg[e] = __frcp_rn(g[e]);
                }
                if (rb == 0) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        gam[s * 128 + 4 * cq + e] = g[e];
                        if (g[e] < kMinChunkDecay) set_status(p.status, KDA_ERR_UNSUPPORTED);
                    }
                }
                float suf[4] = {1.f, 1.f, 1.f, 1.f};
#pragma unroll
                for (int x = 7; x >= 0; --x) {
                    const int r = 8 * rb + x;
                    const uint32_t off = r * 128 + ((((lc4 >> 1) ^ (r & 7)) & 7) << 4) + ((lc4 & 1) << 3);
                    const uint32_t kw[2] = {R.kr[x].x, R.kr[x].y};
                    const uint32_t qw[2] = {R.qr[x].x, R.qr[x].y};
                    uint32_t okt[2], oqt[2], oke[2], okh[2];
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const int e = 2 * u;
                        const float f0 = before[e] * pre[x][e], f1 = before[e + 1] * pre[x][e + 1];
                        const float b0 = suf[e] * after[e], b1 = suf[e + 1] * after[e + 1];
                        const float k0 = bf_lo(kw[u]), k1 = bf_hi(kw[u]);
                        const float q0 = bf_lo(qw[u]), q1 = bf_hi(qw[u]);
                        const float e0 = k0 * b0, e1 = k1 * b1;
                        okt[u] = pack_f16x2(k0 * f0, k1 * f1);
                        oqt[u] = pack_f16x2(q0 * f0, q1 * f1);
                        oke[u] = pack_f16x2(e0, e1);
                        okh[u] = pack_f16x2(e0 * rg[e], e1 * rg[e + 1]);
                    }
#pragma unroll
                    for (int e = 0; e < 4; ++e) suf[e] *= a[x][e];
                    *reinterpret_cast<uint2 *>(sm + OFF_KT + kh * 8192 + off) = make_uint2(okt[0], okt[1]);
                    *reinterpret_cast<uint2 *>(X + kh * X_HALF + 64 * 128 + off) = make_uint2(oqt[0], oqt[1]);
                    *reinterpret_cast<uint2 *>(KE + kh * 8192 + off) = make_uint2(oke[0], oke[1]);
                    *reinterpret_cast<uint2 *>(sm + OFF_KH + kh * 8192 + off) = make_uint2(okh[0], okh[1]);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar_sync(1, PG_THREADS);
            if (*abort_flag) break;                // uniform: read after a group barrier
            tc_fence_after();
            // ---- P1: D1A = Qt Kh^T, D1B = Kt Kh^T   (M=64, N=64, K=128)
            if (pt == 0) {
                ++n_p1;
                const uint32_t id = idesc_f16(64, 64, 0, 0);
                const uint32_t aX = smem_u32(X);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t kh = ks >> 2, ko = (ks & 3) * 32;
                    const uint64_t bd = smem_desc(sbase + OFF_KH + kh * 8192 + ko, 16, 1024, SW_128B);
                    umma_ss(tmem + TM_D1A, smem_desc(aX + kh * X_HALF + 64 * 128 + ko, 16, 1024, SW_128B), bd, id, ks > 0);
                    umma_ss(tmem + TM_D1B, smem_desc(sbase + OFF_KT + kh * 8192 + ko, 16, 1024, SW_128B), bd, id, ks > 0);
                }
                umma_commit(&bars[B_P1]);
            }
            // ---- the next chunk's inputs go out now; their latency overlaps P1, T and P3
            if (c + 1 < nchunks) {
                const int64_t nt0 = tok0 + C;
                prep_load(R, p, nt0, (t1 - nt0 < C) ? (int)(t1 - nt0) : C, h, j0, pt);
            }
            if (pt == 0 && !mbar_wait(&bars[B_P1], c & 1)) fail();
            named_bar_sync(1, PG_THREADS);
            tc_fence_after();
            // ---- P1 epilogue: half 0 -> M (f16, Y rows 128-191); half 1 -> A^T (fp32, column-major)
            {
                float v[64];
                tmem_ld64_sync(tmem + ((uint32_t)(32 * q4) << 16) + (half ? TM_D1B : TM_D1A), v);
                if (lane < 16) {
                    const int r = 16 * q4 + lane;
                    if (half == 0) {
#pragma unroll
                        for (int ch = 0; ch < 8; ++ch) {
                            uint32_t w4[4];
#pragma unroll
                            for (int u = 0; u < 4; ++u) {
                                const int i = 8 * ch + 2 * u;
                                w4[u] = pack_f16x2(i <= r ? v[i] : 0.f, i + 1 <= r ? v[i + 1] : 0.f);
                            }
                            *reinterpret_cast<uint4 *>(Y + sw128_offset(128 + r, 8 * ch)) =
                                make_uint4(w4[0], w4[1], w4[2], w4[3]);
                        }
                    } else {
                        const float br = bet[r];
#pragma unroll
                        for (int i = 0; i < 64; ++i) AT[i * 64 + r] = (i < r) ? br * v[i] : 0.f;
                    }
                }
            }
            tc_fence_before();
            named_bar_sync(1, PG_THREADS);
            if (*abort_flag) break;
            // ---- T = (I + A)^{-1};  Tb = T diag(beta) -> f16 Y rows 0-63
            prep_inverse(pt, AT, Tf, Ps);
            {
                const int r = pt >> 2, c0 = (pt & 3) * 16;
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int cb = c0 + 8 * hh;
                    const float4 t0v = *reinterpret_cast<const float4 *>(Tf + r * LDT + cb);
                    const float4 t1v = *reinterpret_cast<const float4 *>(Tf + r * LDT + cb + 4);
                    const float4 b0v = *reinterpret_cast<const float4 *>(bet + cb);
                    const float4 b1v = *reinterpret_cast<const float4 *>(bet + cb + 4);
                    const float tv[8] = {t0v.x * b0v.x, t0v.y * b0v.y, t0v.z * b0v.z, t0v.w * b0v.w,
                                         t1v.x * b1v.x, t1v.y * b1v.y, t1v.z * b1v.z, t1v.w * b1v.w};
                    uint32_t w4[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int i = cb + 2 * u;
                        w4[u] = pack_f16x2(i <= r ? tv[2 * u] : 0.f, i + 1 <= r ? tv[2 * u + 1] : 0.f);
                    }
                    *reinterpret_cast<uint4 *>(Y + sw128_offset(r, cb)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar_sync(1, PG_THREADS);
            tc_fence_after();
            // ---- P3: D3 = [Tb; 0] Kt (M=128, N=128, K=64); seed D5[s] = -[Tb; 0] V (M=128, N=32)
            if (pt == 0) {
                ++n_p3;
                const uint32_t aY = smem_u32(Y);
                const uint32_t id3 = idesc_f16(128, 128, 0, 1);
                const uint32_t ids = idesc_f16(128, 32, 0, 1) | (1u << 13);   // negate A
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    const uint64_t ad = smem_desc(aY + ks * 32, 16, 1024, SW_128B);
                    umma_ss(tmem + TM_D3, ad, smem_desc(sbase + OFF_KT + ks * 2048, 8192, 1024, SW_128B), id3, ks > 0);
                    umma_ss(tmem + TM_D5 + 32 * s, ad, smem_desc(smem_u32(Vs) + ks * 1024, 16, 512, SW_64B), ids, ks > 0);
                }
                umma_commit(&bars[B_P3]);
            }
            if (pt == 0 && !mbar_wait(&bars[B_P3], c & 1)) fail();
            named_bar_sync(1, PG_THREADS);
            tc_fence_after();
            // ---- W epilogue: rows 0-63 of D3 (TMEM lanes 0-63) -> f16 X rows 0-63
            if (q4 < 2) {
                const int r = 32 * q4 + lane;
                float w[64];
                tmem_ld64_sync(tmem + ((uint32_t)(32 * q4) << 16) + TM_D3 + 64 * half, w);
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    uint4 o;
                    o.x = pack_f16x2(w[8 * ch + 0], w[8 * ch + 1]);
                    o.y = pack_f16x2(w[8 * ch + 2], w[8 * ch + 3]);
                    o.z = pack_f16x2(w[8 * ch + 4], w[8 * ch + 5]);
                    o.w = pack_f16x2(w[8 * ch + 6], w[8 * ch + 7]);
                    *reinterpret_cast<uint4 *>(X + half * X_HALF + sw128_offset(r, 8 * ch)) = o;
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar_sync(1, PG_THREADS);
            if (*abort_flag) break;
            if (pt == 0) mbar_arrive(&bars[B_READY + s]);
        }
        if (*abort_flag && pt == 0) {      // drain this thread's MMAs still in flight (bounded)
            if (n_p1) mbar_wait(&bars[B_P1], (n_p1 - 1) & 1, 100000000LL);
            if (n_p3) mbar_wait(&bars[B_P3], (n_p3 - 1) & 1, 100000000LL);
        }
    } else {
        // =========================================================================== scan group
        const int st = tid;                      // key channel / TMEM lane
        float S[DVB];
        {
            const size_t sidx = (((size_t)n * H + h) * DK + st) * DK + j0;
#pragma unroll
            for (int j = 0; j < DVB; j += 4) {
                const float4 v = (p.S0 && in_bounds(p.status, (long long)(sidx + j), 4, (long long)p.N * H * DK * DK))
                                     ? *reinterpret_cast<const float4 *>(p.S0 + sidx + j) : make_float4(0, 0, 0, 0);
                S[j] = v.x; S[j + 1] = v.y; S[j + 2] = v.z; S[j + 3] = v.w;
            }
        }
        auto store_state = [&]() {
#pragma unroll
            for (int j = 0; j < DVB; j += 8) {
                uint4 v;
                v.x = pack_f16x2(S[j], S[j + 1]); v.y = pack_f16x2(S[j + 2], S[j + 3]);
                v.z = pack_f16x2(S[j + 4], S[j + 5]); v.w = pack_f16x2(S[j + 6], S[j + 7]);
                *reinterpret_cast<uint4 *>(sm + OFF_SB + sw64_offset(st, j)) = v;
            }
        };
        store_state();
        fence_proxy_async_smem();
        named_bar_sync(2, SG_THREADS);
        uint32_t n_s1 = 0, n_s2 = 0;               // commits issued (thread 0)
        auto issue_s1 = [&](int c) -> bool {   // scan thread 0 only
            const int s = c & 1;
            if (!mbar_wait(&bars[B_READY + s], (c >> 1) & 1)) return false;
            ++n_s1;
            tc_fence_after();
            const uint32_t aX = sbase + (s ? OFF_X1 : OFF_X0);
            const uint32_t id = idesc_f16(128, 32, 0, 1);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t kh = ks >> 2, ko = (ks & 3) * 32;
                umma_ss(tmem + TM_D5 + 32 * s, smem_desc(aX + kh * X_HALF + ko, 16, 1024, SW_128B),
                        smem_desc(sbase + OFF_SB + ks * 1024, 16, 512, SW_64B), id, 1);
            }
            umma_commit(&bars[B_S1]);
            return true;
        };
        if (st == 0 && nchunks > 0 && !issue_s1(0)) fail();
        for (int c = 0; c < nchunks; ++c) {
            const int s = c & 1;
            const int64_t tok0 = t0 + (int64_t)c * C;
            const int L = (t1 - tok0 < C) ? (int)(t1 - tok0) : C;
            const uint32_t d5 = tmem + TM_D5 + 32 * s;
            if (st == 0 && !mbar_wait(&bars[B_S1], c & 1)) fail();
            named_bar_sync(2, SG_THREADS);
            tc_fence_after();
            // U = -(D5 rows 0-63) -> f16 MN-major [token][32]
            if (warp < 2) {
                const uint32_t ta = d5 + ((uint32_t)(32 * warp) << 16);
                float u[32];
                tmem_ld32_sync(ta, u);
#pragma unroll
                for (int e = 0; e < 32; ++e) u[e] = -u[e];
#pragma unroll
                for (int j = 0; j < DVB; j += 8) {
                    uint4 o;
                    o.x = pack_f16x2(u[j], u[j + 1]); o.y = pack_f16x2(u[j + 2], u[j + 3]);
                    o.z = pack_f16x2(u[j + 4], u[j + 5]); o.w = pack_f16x2(u[j + 6], u[j + 7]);
                    *reinterpret_cast<uint4 *>(sm + OFF_UB + sw64_offset(st, j)) = o;
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar_sync(2, SG_THREADS);
            if (*abort_flag) break;                // uniform: read after a group barrier
            tc_fence_after();
            if (st == 0) {
                ++n_s2;
                const uint32_t aKE = sbase + (s ? OFF_KE1 : OFF_KE0);
                const uint32_t aY = sbase + (s ? OFF_Y1 : OFF_Y0);
                const uint32_t id2 = idesc_f16(128, 32, 1, 1);
                const uint32_t idm = idesc_f16(128, 32, 0, 1);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    umma_ss(tmem + TM_D7, smem_desc(aKE + ks * 2048, 8192, 1024, SW_128B),
                            smem_desc(sbase + OFF_UB + ks * 1024, 16, 512, SW_64B), id2, ks > 0);
                umma_commit(&bars[B_S2]);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    umma_ss(d5, smem_desc(aY + 64 * 128 + ks * 32, 16, 1024, SW_128B),
                            smem_desc(sbase + OFF_UB + ks * 1024, 16, 512, SW_64B), idm, 1);
                umma_commit(&bars[B_MU]);
            }
            if (st == 0 && !mbar_wait(&bars[B_S2], c & 1)) fail();
            named_bar_sync(2, SG_THREADS);
            tc_fence_after();
            {   // S <- gamma S + Kend^T U
                const uint32_t ta = tmem + TM_D7 + ((uint32_t)(32 * warp) << 16);
                const float g = gam[s * 128 + st];
                float d7[32];
                tmem_ld32_sync(ta, d7);
#pragma unroll
                for (int e = 0; e < 32; ++e) S[e] = g * S[e] + d7[e];
                store_state();
            }
            fence_proxy_async_smem();
            // the MU commit also guards UB and D5[s]
            if (st == 0 && !mbar_wait(&bars[B_MU], c & 1)) fail();
            named_bar_sync(2, SG_THREADS);
            tc_fence_after();
            if (warp >= 2) {                 // O = D5 rows 64-127 -> out
                const int r = st - 64;
                const uint32_t ta = d5 + ((uint32_t)(32 * warp) << 16);
                float o32[32];
                tmem_ld32_sync(ta, o32);
                if (r < L && in_bounds(p.status, ((long long)(tok0 + r) * H + h) * DK + j0, DVB, p.tokens * H * DK)) {
                    TO *dst = reinterpret_cast<TO *>(p.out) + ((size_t)(tok0 + r) * H + h) * DK + j0;
                    if constexpr (sizeof(TO) == 4) {
#pragma unroll
                        for (int j = 0; j < DVB; j += 4)
                            *reinterpret_cast<float4 *>(reinterpret_cast<float *>(dst) + j) =
                                make_float4(o32[j], o32[j + 1], o32[j + 2], o32[j + 3]);
                    } else {
#pragma unroll
                        for (int j = 0; j < DVB; j += 8) {
                            uint4 o;
                            o.x = pack_bf16x2(o32[j], o32[j + 1]); o.y = pack_bf16x2(o32[j + 2], o32[j + 3]);
                            o.z = pack_bf16x2(o32[j + 4], o32[j + 5]); o.w = pack_bf16x2(o32[j + 6], o32[j + 7]);
                            *reinterpret_cast<uint4 *>(reinterpret_cast<uint16_t *>(dst) + j) = o;
                        }
                    }
                }
            }
            tc_fence_before();
            named_bar_sync(2, SG_THREADS);
            if (*abort_flag) break;
            if (st == 0) {
                mbar_arrive(&bars[B_FREE + s]);
                if (c + 1 < nchunks && !issue_s1(c + 1)) fail();
            }
        }
        if (*abort_flag && st == 0) {      // drain this thread's MMAs still in flight (bounded)
            if (n_s1) mbar_wait(&bars[B_S1], (n_s1 - 1) & 1, 100000000LL);
            if (n_s2) {
                mbar_wait(&bars[B_S2], (n_s2 - 1) & 1, 100000000LL);
                mbar_wait(&bars[B_MU], (n_s2 - 1) & 1, 100000000LL);
            }
        }
        if (p.S_final && !*abort_flag &&
            in_bounds(p.status, (long long)((((size_t)n * H + h) * DK + st) * DK + j0), DVB, (long long)p.N * H * DK * DK)) {
            const size_t sidx = (((size_t)n * H + h) * DK + st) * DK + j0;
#pragma unroll
            for (int j = 0; j < DVB; j += 4)
                *reinterpret_cast<float4 *>(p.S_final + sidx + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, TMEM_COLS);
}

template <typename TO>
cudaError_t launch_typed(const PrefillArgs &a, cudaStream_t stream)
{
    TcParams p;
    p.q = (const __nv_bfloat16 *)a.q; p.k = (const __nv_bfloat16 *)a.k; p.v = (const __nv_bfloat16 *)a.v;
    p.log_alpha = a.log_alpha; p.beta = a.beta; p.S0 = a.S0; p.cu_seqlens = a.cu_seqlens;
    p.out = a.out; p.S_final = a.S_final; p.T = a.T; p.H = a.H; p.N = a.N; p.status = a.status;
    p.tokens = (long long)a.B * a.T;
    auto kern = chunk_tc_kernel<TO>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_ALLOC);
    if (e != cudaSuccess) return e;
    const dim3 grid(DK / DVB, a.H, a.N);
    kern<<<grid, NT, SMEM_ALLOC, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_chunk_tc(const PrefillArgs &a, kda_dtype_t out_dtype, cudaStream_t stream)
{
    if (a.N == 0) return cudaSuccess;
    if (out_dtype == KDA_BF16) return launch_typed<__nv_bfloat16>(a, stream);
    return launch_typed<float>(a, stream);
}

}  // namespace kda
