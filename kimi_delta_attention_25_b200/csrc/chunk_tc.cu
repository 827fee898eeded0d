// chunk_tc.cu -- chunkwise KDA prefill on the sm_100a tensor cores (tcgen05 + TMEM + TMA) for
// bf16 q/k/v: f16 MMA operands, fp32 accumulation and an fp32 inter-chunk state.
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
// f and b are running products of alpha = exp(log_alpha) (forward and backward within the chunk),
// so every factor is <= 1 except 1/gamma.
//
// Work split: one CTA (128 threads, one warpgroup) per (sequence, head, 32-column block of d_v).
// The value columns of S evolve independently, so the four blocks of a head never communicate;
// each recomputes the d_v-independent part of the chunk. The chunk loop is sequential per CTA:
//   TMA (q, k, v block into a 2-stage ring; log_alpha single-buffered) ->
//   elementwise decay scaling (CUDA cores, fp32) ->
//   P1: [Qt; Kt] Kh^T                   (UMMA M=128 N=64  K=128) -> A (fp32 smem), M (f16 smem)
//   T = (I + A)^{-1} by 16x16 blocks    (CUDA cores, fp32)       -> Tb (f16 smem)
//   P3: [Tb; 0] Kt                      (UMMA M=128 N=128 K=64)  -> W (f16 smem)
//   S1: [W; Qt] S - [Tb; 0] V           (UMMA M=128 N=32, K=128 then 64) -> -U | Qt S
//   S2: Kend^T U -> D7 ;  MU: [0; M] U accumulated onto Qt S  (UMMA M=128 N=32 K=64)
//   epilogue: S <- gamma S + D7 (fp32 registers, thread = key channel), O -> out
// Operand tiles use the 128-byte (64-byte for 32-wide tiles) swizzled canonical layouts; stacked
// operands ([Qt; Kt], [W; Qt], [Tb; 0], [0; M]) are contiguous row ranges of one region so that a
// single M=128 instruction covers both halves.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "kda_internal.cuh"
#include "sm100.cuh"

namespace kda {
namespace {

using namespace sm100;

constexpr int NT = 128;
constexpr int C = kChunk;          // 64
constexpr int DK = kHeadDim;       // 128
constexpr int DVB = 32;            // value columns per CTA

// ---- shared memory plan (byte offsets from a 1024-byte aligned base)
constexpr uint32_t X_REGION = 192 * 128;              // rows 0-63 W, 64-127 Qt, 128-191 Kt
constexpr uint32_t X_BYTES = 2 * X_REGION;            // two 64-channel halves
constexpr uint32_t V_BYTES = C * DVB * 2;             // 4 KiB, 64-byte rows
constexpr uint32_t OFF_X0 = 0;
constexpr uint32_t OFF_X1 = OFF_X0 + X_BYTES;         // 49152
constexpr uint32_t OFF_V0 = OFF_X1 + X_BYTES;         // 98304
constexpr uint32_t OFF_V1 = OFF_V0 + V_BYTES;
constexpr uint32_t OFF_LA = OFF_V1 + V_BYTES;         // 106496, 32 KiB log_alpha / later A, T
constexpr uint32_t LA_BYTES = 34 * 1024;
constexpr uint32_t OFF_KH = OFF_LA + LA_BYTES;        // Kh: two halves of 64 x 128 B
constexpr uint32_t OFF_KE = OFF_KH + 16384;           // Kend
constexpr uint32_t OFF_Y = OFF_KE + 16384;            // rows 0-63 Tb, 64-127 zero, 128-191 M
constexpr uint32_t OFF_SB = OFF_Y + 192 * 128;        // S f16, 128 rows x 64 B
constexpr uint32_t OFF_UB = OFF_SB + DK * DVB * 2;    // U f16, 64 rows x 64 B
constexpr uint32_t OFF_TOT = OFF_UB + C * DVB * 2;    // 8 x 128 fp32 row-block products
constexpr uint32_t OFF_GAM = OFF_TOT + 8 * 128 * 4;   // 128 fp32
constexpr uint32_t OFF_BET = OFF_GAM + 128 * 4;       // 64 fp32
constexpr uint32_t OFF_TMP = OFF_BET + 64 * 4;        // 3 x 16 x 16 fp32 scratch for the inverse
constexpr uint32_t OFF_BAR = OFF_TMP + 3 * 256 * 4;   // mbarriers
constexpr uint32_t SMEM_BYTES = OFF_BAR + 64;
constexpr uint32_t SMEM_ALLOC = SMEM_BYTES + 1024;    // alignment slack
static_assert(SMEM_ALLOC <= 232448, "shared memory plan exceeds 227 KiB");

constexpr int LDA = 65;            // fp32 row stride of A and T (in the log_alpha region)
constexpr uint32_t OFF_AF = 0;                     // within OFF_LA
constexpr uint32_t OFF_TF = 64 * LDA * 4;          // 16640

constexpr uint32_t TMEM_COLS = 256;
constexpr uint32_t TM_D1 = 0;      // 64 cols: [Qt;Kt] Kh^T
constexpr uint32_t TM_D3 = 64;     // 128 cols: [Tb;0] Kt
constexpr uint32_t TM_D5 = 192;    // 32 cols: -U | O
constexpr uint32_t TM_D7 = 224;    // 32 cols: Kend^T U

constexpr uint32_t TX_STAGE = 4 * 8192 + V_BYTES;  // q, k halves + v block
// Operands are rounded to f16 (11-bit significand) for the tensor cores: the largest one, Kh =
// K e^{-g}, must stay finite, so the decay accumulated over one chunk must keep e^{g} above
// 2^-15 per channel (cumulative log-decay >= -10.4). Chunks beyond that report UNSUPPORTED.
constexpr float kMinChunkDecay = 3.0517578125e-05f;
constexpr uint32_t TX_LA = C * DK * 4;

struct TcParams {
    const float *beta, *S0;
    const int32_t *cu_seqlens;
    void *out;
    float *S_final;
    int T, H, N;
    int32_t *status;
};

__device__ __forceinline__ float bf2f(uint16_t x) { return __uint_as_float((uint32_t)x << 16); }

// unit lower-triangular inverse T = (I + A)^{-1}, A strictly lower (fp32, row stride LDA),
// by 16 x 16 blocks: diagonal blocks by forward substitution, then block diagonals 1..3 with
// T_ij = -T_ii * sum_{k=j}^{i-1} L_ik T_kj. All 128 threads participate; ends synchronised.
__device__ void unit_lower_inverse(const float *Af, float *Tf, float *tmp, int tid)
{
    // diagonal blocks: thread -> (block b, column j)
    if (tid < 64) {
        const int b = tid >> 4, j = tid & 15, o = 16 * b;
        float x[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            float v = (r == j) ? 1.f : 0.f;
#pragma unroll
            for (int i = 0; i < r; ++i) v -= Af[(o + r) * LDA + o + i] * x[i];
            x[r] = (r < j) ? 0.f : v;
        }
#pragma unroll
        for (int r = 0; r < 16; ++r) Tf[(o + r) * LDA + o + j] = x[r];
    }
    // zero the strictly upper blocks so later full 16-term products stay exact
    for (int idx = tid; idx < 64 * 64; idx += NT) {
        const int r = idx >> 6, cidx = idx & 63;
        if ((cidx >> 4) > (r >> 4)) Tf[r * LDA + cidx] = 0.f;
    }
    __syncthreads();
    for (int d = 1; d <= 3; ++d) {
        const int nb = 4 - d;                  // blocks (i, i-d), i = d..3
        // P_i = sum_{k=i-d}^{i-1} L_ik T_k,(i-d)
        for (int e = tid; e < nb * 256; e += NT) {
            const int q = e >> 8, rr = (e >> 4) & 15, cc = e & 15;
            const int i = d + q, j = i - d;
            float acc = 0.f;
            for (int kb = j; kb < i; ++kb) {
#pragma unroll
                for (int x = 0; x < 16; ++x)
                    acc += Af[(16 * i + rr) * LDA + 16 * kb + x] * Tf[(16 * kb + x) * LDA + 16 * j + cc];
            }
            tmp[q * 256 + rr * 16 + cc] = acc;
        }
        __syncthreads();
        for (int e = tid; e < nb * 256; e += NT) {
            const int q = e >> 8, rr = (e >> 4) & 15, cc = e & 15;
            const int i = d + q, j = i - d;
            float acc = 0.f;
#pragma unroll
            for (int x = 0; x < 16; ++x)
                acc += Tf[(16 * i + rr) * LDA + 16 * i + x] * tmp[q * 256 + x * 16 + cc];
            Tf[(16 * i + rr) * LDA + 16 * j + cc] = -acc;
        }
        __syncthreads();
    }
}

template <typename T, typename TO>
__global__ void __launch_bounds__(NT, 1)
chunk_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_la,
                TcParams p)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const int tid = threadIdx.x, warp = tid >> 5;
    const int jb = blockIdx.x, h = blockIdx.y, n = blockIdx.z;
    const int j0 = jb * DVB;
    const int H = p.H;

    uint64_t *bar_full = reinterpret_cast<uint64_t *>(sm + OFF_BAR);       // [2]
    uint64_t *bar_la = bar_full + 2;
    uint64_t *bar_mma = bar_full + 3;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_full + 4);
    int *abort_flag = reinterpret_cast<int *>(bar_full + 5);
    float *tot = reinterpret_cast<float *>(sm + OFF_TOT);
    float *gam = reinterpret_cast<float *>(sm + OFF_GAM);
    float *bet = reinterpret_cast<float *>(sm + OFF_BET);
    float *Af = reinterpret_cast<float *>(sm + OFF_LA + OFF_AF);
    float *Tf = reinterpret_cast<float *>(sm + OFF_LA + OFF_TF);
    float *tmpf = reinterpret_cast<float *>(sm + OFF_TMP);
    const uint32_t sbase = smem_u32(sm);

    int64_t t0, t1;
    const bool ok_span = sequence_span(p.cu_seqlens, n, p.N, p.T, &t0, &t1, p.status);
    if (!ok_span) return;                                  // uniform across the CTA
    const int nchunks = (int)((t1 - t0 + C - 1) / C);

    if (warp == 0) { tmem_alloc(tmem_slot, TMEM_COLS); tmem_relinquish(); }
    if (tid == 0) {
        mbar_init(&bar_full[0], 1);
        mbar_init(&bar_full[1], 1);
        mbar_init(bar_la, 1);
        mbar_init(bar_mma, 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tm_q); tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v); tma_prefetch_desc(&tm_la);
    }
    // zero block of Y (rows 64-127) -- stays zero for the whole kernel
    for (int i = tid; i < 64 * 128 / 16; i += NT)
        reinterpret_cast<uint4 *>(sm + OFF_Y + 64 * 128)[i] = make_uint4(0, 0, 0, 0);
    // initial state: thread = key channel c, 32 fp32 columns in registers
    float S[DVB];
    {
        const size_t sidx = (((size_t)n * H + h) * DK + tid) * DK + j0;
#pragma unroll
        for (int j = 0; j < DVB; j += 4) {
            float4 v = p.S0 ? *reinterpret_cast<const float4 *>(p.S0 + sidx + j) : make_float4(0, 0, 0, 0);
            S[j] = v.x; S[j + 1] = v.y; S[j + 2] = v.z; S[j + 3] = v.w;
        }
    }
    auto store_state_f16 = [&]() {
        // S (f16) as the MN-major B operand of S1: row = key channel (64-byte rows, 64B swizzle)
        unsigned char *row = sm + OFF_SB;
#pragma unroll
        for (int j = 0; j < DVB; j += 8) {
            uint4 v;
            v.x = pack_f16x2(S[j], S[j + 1]); v.y = pack_f16x2(S[j + 2], S[j + 3]);
            v.z = pack_f16x2(S[j + 4], S[j + 5]); v.w = pack_f16x2(S[j + 6], S[j + 7]);
            *reinterpret_cast<uint4 *>(row + sw64_offset(tid, j)) = v;
        }
    };
    store_state_f16();
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    uint32_t mma_phase = 0;
    uint32_t n_full_issued[2] = {0u, 0u}, n_la_issued = 0u;      // meaningful in thread 0 only

    auto issue_loads = [&](int c) {        // q, k, v of chunk c into stage c & 1
        const int s = c & 1;
        const int tok = (int)(t0 + (int64_t)c * C);
        unsigned char *X = sm + (s ? OFF_X1 : OFF_X0);
        ++n_full_issued[s];
        mbar_arrive_expect_tx(&bar_full[s], TX_STAGE);
        for (int kh = 0; kh < 2; ++kh) {
            tma_load_3d(X + kh * X_REGION + 64 * 128, &tm_q, &bar_full[s], 64 * kh, h, tok);
            tma_load_3d(X + kh * X_REGION + 128 * 128, &tm_k, &bar_full[s], 64 * kh, h, tok);
        }
        tma_load_3d(sm + (s ? OFF_V1 : OFF_V0), &tm_v, &bar_full[s], j0, h, tok);
    };
    auto issue_la = [&](int c) {
        const int tok = (int)(t0 + (int64_t)c * C);
        ++n_la_issued;
        mbar_arrive_expect_tx(bar_la, TX_LA);
        tma_load_3d(sm + OFF_LA, &tm_la, bar_la, 0, h, tok);
    };
    auto fail = [&]() {
        set_status(p.status, KDA_ERR_TIMEOUT);
        *abort_flag = 1;
    };
    auto wait_mma = [&]() {
        if (!mbar_wait(bar_mma, mma_phase & 1)) fail();
        ++mma_phase;
        tc_fence_after();
    };

    if (tid == 0 && nchunks > 0) {
        issue_loads(0);
        issue_la(0);
        if (nchunks > 1) issue_loads(1);
    }

    const float LOG2E = 1.4426950408889634f;
    int c = 0;
    for (; c < nchunks; ++c) {
        const int s = c & 1;
        const int64_t tok0 = t0 + (int64_t)c * C;
        const int L = (t1 - tok0 < C) ? (int)(t1 - tok0) : C;
        unsigned char *X = sm + (s ? OFF_X1 : OFF_X0);
        unsigned char *Vs = sm + (s ? OFF_V1 : OFF_V0);
        const uint32_t aX = smem_u32(X), aV = smem_u32(Vs), aY = sbase + OFF_Y;

        if (tid < C) bet[tid] = (tid < L) ? p.beta[(size_t)(tok0 + tid) * H + h] : 0.f;
        if (!mbar_wait(&bar_full[s], (c >> 1) & 1)) fail();
        if (!mbar_wait(bar_la, c & 1)) fail();

        // ---------------- elementwise decay scaling: thread -> 8 rows x 8 channels
        {
            const int rb = tid >> 4, cc = tid & 15, kh = cc >> 3, lc = cc & 7;
            const float *LA = reinterpret_cast<const float *>(sm + OFF_LA);
            float a[8][8];
#pragma unroll
            for (int x = 0; x < 8; ++x) {
                const int r = 8 * rb + x;
                const float4 l0 = *reinterpret_cast<const float4 *>(LA + r * DK + 8 * cc);
                const float4 l1 = *reinterpret_cast<const float4 *>(LA + r * DK + 8 * cc + 4);
                const bool valid = r < L;
                a[x][0] = valid ? exp2f(l0.x * LOG2E) : 1.f; a[x][1] = valid ? exp2f(l0.y * LOG2E) : 1.f;
                a[x][2] = valid ? exp2f(l0.z * LOG2E) : 1.f; a[x][3] = valid ? exp2f(l0.w * LOG2E) : 1.f;
                a[x][4] = valid ? exp2f(l1.x * LOG2E) : 1.f; a[x][5] = valid ? exp2f(l1.y * LOG2E) : 1.f;
                a[x][6] = valid ? exp2f(l1.z * LOG2E) : 1.f; a[x][7] = valid ? exp2f(l1.w * LOG2E) : 1.f;
            }
            // local inclusive prefix and exclusive suffix products over the 8 rows
            float pre[8][8], suf[8][8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                float run = 1.f;
#pragma unroll
                for (int x = 0; x < 8; ++x) { run *= a[x][e]; pre[x][e] = run; }
                float rs = 1.f;
#pragma unroll
                for (int x = 7; x >= 0; --x) { suf[x][e] = rs; rs *= a[x][e]; }
                tot[rb * 128 + 8 * cc + e] = run;
            }
            __syncthreads();
            float before[8], after[8], rg[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                float bfr = 1.f, aft = 1.f;
                for (int y = 0; y < 8; ++y) {
                    const float tv = tot[y * 128 + 8 * cc + e];
                    if (y < rb) bfr *= tv;
                    if (y > rb) aft *= tv;
                }
                before[e] = bfr;
                after[e] = aft;
                const float g = bfr * pre[7][e] * aft;           // gamma = product over the chunk
                rg[e] = 1.f / g;
                if (rb == 0) gam[8 * cc + e] = g;
                if (g < kMinChunkDecay) set_status(p.status, KDA_ERR_UNSUPPORTED);
            }
            {   // v block: bf16 -> f16 in place (16 elements per thread; layout unchanged)
                uint4 *vv = reinterpret_cast<uint4 *>(Vs) + 2 * tid;
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    uint4 x = vv[u];
                    x.x = bf16x2_to_f16x2(x.x); x.y = bf16x2_to_f16x2(x.y);
                    x.z = bf16x2_to_f16x2(x.z); x.w = bf16x2_to_f16x2(x.w);
                    vv[u] = x;
                }
            }
            unsigned char *Xk = X + kh * X_REGION + 128 * 128;   // k -> Kt in place
            unsigned char *Xq = X + kh * X_REGION + 64 * 128;    // q -> Qt in place
            unsigned char *Kh = sm + OFF_KH + kh * 8192;
            unsigned char *Ke = sm + OFF_KE + kh * 8192;
#pragma unroll
            for (int x = 0; x < 8; ++x) {
                const int r = 8 * rb + x;
                const uint32_t off = sw128_offset(r, 8 * lc);
                const uint4 kraw = *reinterpret_cast<const uint4 *>(Xk + off);
                const uint4 qraw = *reinterpret_cast<const uint4 *>(Xq + off);
                const uint16_t *kv = reinterpret_cast<const uint16_t *>(&kraw);
                const uint16_t *qv = reinterpret_cast<const uint16_t *>(&qraw);
                const bool valid = r < L;
                float kt[8], qt[8], ke[8], kc[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float kk = valid ? bf2f(kv[e]) : 0.f;
                    const float qq = valid ? bf2f(qv[e]) : 0.f;
                    const float f = before[e] * pre[x][e];
                    const float b = suf[x][e] * after[e];
                    kt[e] = kk * f;
                    qt[e] = qq * f;
                    ke[e] = kk * b;
                    kc[e] = ke[e] * rg[e];
                }
                uint4 o;
                o.x = pack_f16x2(kt[0], kt[1]); o.y = pack_f16x2(kt[2], kt[3]);
                o.z = pack_f16x2(kt[4], kt[5]); o.w = pack_f16x2(kt[6], kt[7]);
                *reinterpret_cast<uint4 *>(Xk + off) = o;
                o.x = pack_f16x2(qt[0], qt[1]); o.y = pack_f16x2(qt[2], qt[3]);
                o.z = pack_f16x2(qt[4], qt[5]); o.w = pack_f16x2(qt[6], qt[7]);
                *reinterpret_cast<uint4 *>(Xq + off) = o;
                o.x = pack_f16x2(ke[0], ke[1]); o.y = pack_f16x2(ke[2], ke[3]);
                o.z = pack_f16x2(ke[4], ke[5]); o.w = pack_f16x2(ke[6], ke[7]);
                *reinterpret_cast<uint4 *>(Ke + off) = o;
                o.x = pack_f16x2(kc[0], kc[1]); o.y = pack_f16x2(kc[2], kc[3]);
                o.z = pack_f16x2(kc[4], kc[5]); o.w = pack_f16x2(kc[6], kc[7]);
                *reinterpret_cast<uint4 *>(Kh + off) = o;
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (*abort_flag) break;
        tc_fence_after();

        // ---------------- P1: D1 = [Qt; Kt] Kh^T  (M=128, N=64, K=128)
        if (tid == 0) {
            const uint32_t id = idesc_f16(128, 64, 0, 0);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t kh = ks >> 2, ko = (ks & 3) * 32;
                const uint64_t ad = smem_desc(aX + kh * X_REGION + 64 * 128 + ko, 16, 1024, SW_128B);
                const uint64_t bd = smem_desc(sbase + OFF_KH + kh * 8192 + ko, 16, 1024, SW_128B);
                umma_ss(tmem + TM_D1, ad, bd, id, ks > 0);
            }
            umma_commit(bar_mma);
        }
        wait_mma();
        // rows 0-63: M = tril(Qt Kh^T) -> f16 Y rows 128-191; rows 64-127: A -> fp32
        {
            float v[64];
            const uint32_t ta = tmem + ((uint32_t)(32 * warp) << 16) + TM_D1;
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
                float r16[16];
                tmem_ld16(ta + 16 * q4, r16);
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 16; ++e) v[16 * q4 + e] = r16[e];
            }
            if (tid < 64) {
                const int r = tid;
                unsigned char *row = sm + OFF_Y;
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    float m8[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) m8[e] = (8 * ch + e <= r) ? v[8 * ch + e] : 0.f;
                    uint4 o;
                    o.x = pack_f16x2(m8[0], m8[1]); o.y = pack_f16x2(m8[2], m8[3]);
                    o.z = pack_f16x2(m8[4], m8[5]); o.w = pack_f16x2(m8[6], m8[7]);
                    *reinterpret_cast<uint4 *>(row + sw128_offset(128 + r, 8 * ch)) = o;
                }
            } else {
                const int r = tid - 64;
                const float br = bet[r];
#pragma unroll
                for (int i = 0; i < 64; ++i) Af[r * LDA + i] = (i < r) ? br * v[i] : 0.f;
            }
        }
        tc_fence_before();
        __syncthreads();

        // ---------------- T = (I + A)^{-1};  Tb = T diag(beta) -> f16 Y rows 0-63
        unit_lower_inverse(Af, Tf, tmpf, tid);
        {
            const int r = tid >> 1, half = tid & 1;
            unsigned char *row = sm + OFF_Y;
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                const int c0 = 32 * half + 8 * ch;
                float t8[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) t8[e] = (c0 + e <= r) ? Tf[r * LDA + c0 + e] * bet[c0 + e] : 0.f;
                uint4 o;
                o.x = pack_f16x2(t8[0], t8[1]); o.y = pack_f16x2(t8[2], t8[3]);
                o.z = pack_f16x2(t8[4], t8[5]); o.w = pack_f16x2(t8[6], t8[7]);
                *reinterpret_cast<uint4 *>(row + sw128_offset(r, c0)) = o;
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        // log_alpha region (A, T) is free: prefetch the next chunk's log_alpha
        if (tid == 0 && c + 1 < nchunks) issue_la(c + 1);
        tc_fence_after();

        // ---------------- P3: D3 = [Tb; 0] Kt  (M=128, N=128, K=64; B = Kt MN-major)
        if (tid == 0) {
            const uint32_t id = idesc_f16(128, 128, 0, 1);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const uint64_t ad = smem_desc(aY + ks * 32, 16, 1024, SW_128B);
                const uint64_t bd = smem_desc(aX + 128 * 128 + ks * 2048, X_REGION, 1024, SW_128B);
                umma_ss(tmem + TM_D3, ad, bd, id, ks > 0);
            }
            umma_commit(bar_mma);
        }
        wait_mma();
        if (tid < 64) {                      // W rows -> f16 X rows 0-63 (both halves)
            const uint32_t ta = tmem + ((uint32_t)(32 * warp) << 16) + TM_D3;
#pragma unroll
            for (int q8 = 0; q8 < 8; ++q8) {
                float r16[16];
                tmem_ld16(ta + 16 * q8, r16);
                tmem_ld_wait();
                const int col = 16 * q8, kh = col >> 6, cl = col & 63;
                unsigned char *base = X + kh * X_REGION;
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    uint4 o;
                    o.x = pack_f16x2(r16[8 * hh + 0], r16[8 * hh + 1]);
                    o.y = pack_f16x2(r16[8 * hh + 2], r16[8 * hh + 3]);
                    o.z = pack_f16x2(r16[8 * hh + 4], r16[8 * hh + 5]);
                    o.w = pack_f16x2(r16[8 * hh + 6], r16[8 * hh + 7]);
                    *reinterpret_cast<uint4 *>(base + sw128_offset(tid, cl + 8 * hh)) = o;
                }
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        // ---------------- S1: D5 = [W; Qt] S  -  [Tb; 0] V   (M=128, N=32)
        if (tid == 0) {
            const uint32_t id = idesc_f16(128, 32, 0, 1);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t kh = ks >> 2, ko = (ks & 3) * 32;
                const uint64_t ad = smem_desc(aX + kh * X_REGION + ko, 16, 1024, SW_128B);
                const uint64_t bd = smem_desc(sbase + OFF_SB + ks * 1024, 16, 512, SW_64B);
                umma_ss(tmem + TM_D5, ad, bd, id, ks > 0);
            }
            const uint32_t idn = id | (1u << 13);            // negate A
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const uint64_t ad = smem_desc(aY + ks * 32, 16, 1024, SW_128B);
                const uint64_t bd = smem_desc(aV + ks * 1024, 16, 512, SW_64B);
                umma_ss(tmem + TM_D5, ad, bd, idn, 1);
            }
            umma_commit(bar_mma);
        }
        wait_mma();
        if (tid < 64) {                      // U = -(rows 0-63) -> f16 MN-major [token][32]
            const uint32_t ta = tmem + ((uint32_t)(32 * warp) << 16) + TM_D5;
            float u[32];
#pragma unroll
            for (int q2 = 0; q2 < 2; ++q2) {
                float r16[16];
                tmem_ld16(ta + 16 * q2, r16);
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 16; ++e) u[16 * q2 + e] = -r16[e];
            }
            unsigned char *row = sm + OFF_UB;
#pragma unroll
            for (int j = 0; j < DVB; j += 8) {
                uint4 o;
                o.x = pack_f16x2(u[j], u[j + 1]); o.y = pack_f16x2(u[j + 2], u[j + 3]);
                o.z = pack_f16x2(u[j + 4], u[j + 5]); o.w = pack_f16x2(u[j + 6], u[j + 7]);
                *reinterpret_cast<uint4 *>(row + sw64_offset(tid, j)) = o;
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        // ---------------- S2: D7 = Kend^T U ;  MU: D5 += [0; M] U
        if (tid == 0) {
            const uint32_t id2 = idesc_f16(128, 32, 1, 1);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const uint64_t ad = smem_desc(sbase + OFF_KE + ks * 2048, 8192, 1024, SW_128B);
                const uint64_t bd = smem_desc(sbase + OFF_UB + ks * 1024, 16, 512, SW_64B);
                umma_ss(tmem + TM_D7, ad, bd, id2, ks > 0);
            }
            const uint32_t idm = idesc_f16(128, 32, 0, 1);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const uint64_t ad = smem_desc(aY + 64 * 128 + ks * 32, 16, 1024, SW_128B);
                const uint64_t bd = smem_desc(sbase + OFF_UB + ks * 1024, 16, 512, SW_64B);
                umma_ss(tmem + TM_D5, ad, bd, idm, 1);
            }
            umma_commit(bar_mma);
        }
        wait_mma();
        {
            // state update: thread = key channel
            const uint32_t ta7 = tmem + ((uint32_t)(32 * warp) << 16) + TM_D7;
            const float g = gam[tid];
#pragma unroll
            for (int q2 = 0; q2 < 2; ++q2) {
                float r16[16];
                tmem_ld16(ta7 + 16 * q2, r16);
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 16; ++e) S[16 * q2 + e] = g * S[16 * q2 + e] + r16[e];
            }
            // outputs: rows 64-127 of D5 are O for tokens 0-63
            if (tid >= 64) {
                const int r = tid - 64;
                const uint32_t ta5 = tmem + ((uint32_t)(32 * warp) << 16) + TM_D5;
                float o32[32];
#pragma unroll
                for (int q2 = 0; q2 < 2; ++q2) {
                    float r16[16];
                    tmem_ld16(ta5 + 16 * q2, r16);
                    tmem_ld_wait();
#pragma unroll
                    for (int e = 0; e < 16; ++e) o32[16 * q2 + e] = r16[e];
                }
                if (r < L) {
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
            store_state_f16();
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        // stage s is free again: load chunk c + 2 into it
        if (tid == 0 && c + 2 < nchunks) issue_loads(c + 2);
        if (*abort_flag) break;
    }

    if (p.S_final && !*abort_flag) {
        const size_t sidx = (((size_t)n * H + h) * DK + tid) * DK + j0;
#pragma unroll
        for (int j = 0; j < DVB; j += 4)
            *reinterpret_cast<float4 *>(p.S_final + sidx + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
    }
    if (*abort_flag && tid == 0) {
        // drain TMA copies that may still be in flight (bounded) before the CTA exits: wait for
        // the last issued phase of every load barrier
        for (int s = 0; s < 2; ++s)
            if (n_full_issued[s]) mbar_wait(&bar_full[s], (n_full_issued[s] - 1) & 1, 100000000LL);
        if (n_la_issued) mbar_wait(bar_la, (n_la_issued - 1) & 1, 100000000LL);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, TMEM_COLS);
}

// ------------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 get_encode()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

// 3-D map over a [tokens, H, 128] tensor: dims (channel, head, token), box (bx, 1, 64).
bool make_map(CUtensorMap *m, const void *base, CUtensorMapDataType dt, int esize, int H, int ntok,
              int bx, CUtensorMapSwizzle sw)
{
    auto enc = get_encode();
    if (!enc) return false;
    cuuint64_t dims[3] = {(cuuint64_t)DK, (cuuint64_t)H, (cuuint64_t)ntok};
    cuuint64_t strides[2] = {(cuuint64_t)DK * esize, (cuuint64_t)DK * esize * H};
    cuuint32_t box[3] = {(cuuint32_t)bx, 1u, (cuuint32_t)C};
    cuuint32_t estr[3] = {1u, 1u, 1u};
    CUresult r = enc(m, dt, 3, const_cast<void *>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <typename TO>
cudaError_t launch_typed(const PrefillArgs &a, const CUtensorMap &mq, const CUtensorMap &mk,
                         const CUtensorMap &mv, const CUtensorMap &ml, cudaStream_t stream)
{
    TcParams p;
    p.beta = a.beta; p.S0 = a.S0; p.cu_seqlens = a.cu_seqlens; p.out = a.out; p.S_final = a.S_final;
    p.T = a.T; p.H = a.H; p.N = a.N; p.status = a.status;
    auto kern = chunk_tc_kernel<__nv_bfloat16, TO>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_ALLOC);
    if (e != cudaSuccess) return e;
    const dim3 grid(DK / DVB, a.H, a.N);
    kern<<<grid, NT, SMEM_ALLOC, stream>>>(mq, mk, mv, ml, p);
    return cudaGetLastError();
}

}  // namespace

bool chunk_tc_supported(const PrefillArgs &a)
{
    // TMA coordinates are 32-bit; the packed token axis must fit
    return (long long)a.B * a.T < (1LL << 31) && get_encode() != nullptr;
}

cudaError_t launch_chunk_tc(const PrefillArgs &a, kda_dtype_t out_dtype, cudaStream_t stream)
{
    if (a.N == 0) return cudaSuccess;
    const int ntok = a.B * a.T;
    if (ntok == 0) {
        // no tokens: every sequence is empty, S_final = S0 -- handled by the fp32 path
        return launch_chunk_fp32(a, KDA_BF16, out_dtype, stream);
    }
    CUtensorMap mq, mk, mv, ml;
    if (!make_map(&mq, a.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.H, ntok, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&mk, a.k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.H, ntok, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&mv, a.v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.H, ntok, DVB, CU_TENSOR_MAP_SWIZZLE_64B) ||
        !make_map(&ml, a.log_alpha, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, a.H, ntok, DK, CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    if (out_dtype == KDA_BF16) return launch_typed<__nv_bfloat16>(a, mq, mk, mv, ml, stream);
    return launch_typed<float>(a, mq, mk, mv, ml, stream);
}

}  // namespace kda
