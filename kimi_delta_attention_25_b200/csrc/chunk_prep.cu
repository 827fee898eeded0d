// chunk_prep.cu -- first pass of the two-pass bf16 prefill: everything about a 64-token chunk
// that does not depend on the running state S, for every (chunk, head) at once.
//
// Chunk form (chunk C = 64; chunk-parallel prefill with a WY/UT representation: KimiLinear
// KDA/MLA tutorial (icman.com.cn), sec. 3 and 6; algebra derived from the recurrence). With
// g_r = sum_{j<=r} log_alpha_j per key channel, f_r = e^{g_r}, b_r = e^{g_{L-1} - g_r}, gamma =
// e^{g_{L-1}}:
//   Kt = K f, Qt = Q f, Kend = K b, Kh = K b / gamma;  A = StrictLower(diag(beta) Kt Kh^T);
//   M = tril(Qt Kh^T);  Tb = (I + A)^{-1} diag(beta);  W = Tb Kt.
// With U = Tb V - W S the chunk's writes, the output O = Qt S + M U regroups as
//   O = (Qt - M W) S + (M Tb) V,
// so the scan pass never needs M itself: this pass also forms M Tb and Qt - M W. The second pass
// (chunk_scan.cu) then runs the state recurrence over chunks with these operands.
//
// The chunks are independent, so this pass is a plain data-parallel grid: one CTA (8 warps) per
// (chunk slot, head), two CTAs per SM. Results go to the workspace in exactly the byte layout the
// scan wants in shared memory (f16, 128-byte swizzled canonical UMMA tiles), so the scan moves each
// block with one bulk copy:
//   [0, 32K)    X: W (rows 0-63) and Qt - M W (rows 64-127), two 64-channel halves, K-major
//   [32K, 48K)  Y: -Tb (rows 0-63) and M Tb (rows 64-127), 64 token columns, K-major
//   [48K, 64K)  Kend, two halves of 64 tokens x 64 channels (the MN-major B of U^T Kend)
//   [64K, +512) gamma (fp32)
// A chunk slot is floor(first_token / 64) + sequence, which is unique per (sequence, chunk) and
// below floor(total_tokens / 64) + N + 1.
#include <cuda.h>
#include <cuda_fp16.h>

#include <mutex>

#include "kda_internal.cuh"
#include "sm100.cuh"

namespace kda {
namespace {

using namespace sm100;

constexpr int C = kChunk;
constexpr int DK = kHeadDim;
constexpr int NT = 256;

// The intra-chunk product P1 pairs Kt = K e^{g} with Kh = K e^{-g}: for a channel that forgets fast
// within the chunk, e^{-g} leaves the f16 range (and Kt its normal range) long before the product
// loses meaning. A chunk whose decay stays above kF16MinDecay in every channel runs P1 on f16
// operands; any other chunk runs it on tf32 operands (fp32 range, the 10-bit significand of f16).
// Every later product takes f16 operands, which only shrink toward zero there. e^{-g} must stay
// finite in fp32: the decay over one chunk must keep e^{g} above e^{-80} per channel; beyond that
// the chunk is reported UNSUPPORTED.
constexpr float kMinChunkDecay = 1.80485139e-35f;   // e^{-80}
constexpr float kF16MinDecay = 3.35462628e-04f;     // e^{-8}: Kh <= 2981 |k|, Kt >= 3.4e-4 |k|

// shared memory (1024-aligned base)
constexpr uint32_t OFF_QK = 0;               // [Qt; Kt] (f16): per 64-channel half (16 KB apart),
                                             // rows 0-63 Qt then rows 64-127 Kt, 128 B per row
constexpr uint32_t QK_HALF = 16384;
constexpr uint32_t OFF_KT = OFF_QK + 8192;   // Kt rows of half 0 (half 1 at + QK_HALF)
constexpr uint32_t OFF_TB = 32768;           // Tb (f16), 64 x 128 B; N-block 0 of [Tb | W]
constexpr uint32_t OFF_KH = 40960;           // after P1: A^T (fp32, column-major);
                                             // after P3: W (f16), N-blocks 1-2 of [Tb | W]
constexpr uint32_t OFF_M = 57344;            // M (f16), 64 x 128 B
// input staging of the chunk (bulk copies), dead once the rows are in registers: aliases the
// operand tiles above, all of which are written later
constexpr uint32_t STG_Q = 0;                // q rows, 64 x 256 B
constexpr uint32_t STG_K = 16384;            // k rows
constexpr uint32_t STG_LA = 32768;           // log_alpha rows, 64 x 512 B
// tf32 operands of P1, dead once P1 has completed (alias everything above and T): [Qt; Kt] as four
// 32-channel quarters of 128 rows x 128 B (rows 0-63 Qt, 64-127 Kt), then Kh as four quarters of
// 64 rows x 128 B; the f16 tiles above are written after P1 from registers
constexpr uint32_t OFF_QK32 = 0;
constexpr uint32_t OFF_KH32 = 65536;
constexpr int LDT = 68;
constexpr uint32_t OFF_TF = 65536;           // T (fp32, stride LDT) = 17408 B
constexpr uint32_t OFF_PS = 98304;           // 4 KB: row-block products, then inverse scratch
constexpr uint32_t OFF_BET = OFF_PS + 4096;  // 64 fp32
constexpr uint32_t OFF_BAR = OFF_BET + 256;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 64;
constexpr uint32_t SMEM_ALLOC = SMEM_BYTES + 1024;
static_assert(OFF_KH32 + 4 * 8192 <= OFF_PS && OFF_TF + 17408 <= OFF_PS, "P1 operands and T end below Ps");
static_assert(2 * (SMEM_ALLOC + 1024) <= 233472, "two CTAs per SM");

constexpr uint32_t TMEM_COLS = 256;
constexpr uint32_t TM_D1A = 0;               // [Qt; Kt] Kh^T (M=128, 64 cols), later W (cols 0-127),
                                             // then M [Tb | W] (cols 0-191)

__device__ __forceinline__ float bf_lo(uint32_t x) { return __uint_as_float(x << 16); }
__device__ __forceinline__ float bf_hi(uint32_t x) { return __uint_as_float(x & 0xFFFF0000u); }
__device__ __forceinline__ uint2 ldg_nc_u2(const void *p) {
    uint2 r;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];" : "=r"(r.x), "=r"(r.y) : "l"(p));
    return r;
}
__device__ __forceinline__ float4 ldg_nc_f4(const float *p) {
    float4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.f32 {%0,%1,%2,%3}, [%4];"
                 : "=f"(r.x), "=f"(r.y), "=f"(r.z), "=f"(r.w) : "l"(p));
    return r;
}

struct PrepParams {
    const __nv_bfloat16 *q, *k;
    const float *log_alpha, *beta;
    // gate producers (the layer's fused_kda_gate and b_proj gate): with GATE the third tensor copy
    // brings the bf16 gate input f instead of log_alpha, and log_alpha = -exp(A_log[h]) *
    // softplus(f + dt_bias[h, c]) is formed here; beta_logits (bf16) gives beta = sigmoid(b)
    const float *A_log, *dt_bias;
    const __nv_bfloat16 *beta_logits;
    const int32_t *cu_seqlens;
    unsigned char *ws;              // chunk blocks, [H][n_slots][kPrepBlockBytes]
    int T, H, N, n_slots;
    int slot_base;                  // first chunk slot of this launch (the grid covers slots from here)
    long long tokens;               // B * T (rows of q, k, log_alpha; beta has tokens * H entries)
    int prefetch_wave;              // CTAs resident at once; > 0: prefetch that many units ahead
    int32_t *status;
};

// The (sequence, chunk) of a chunk slot: slot = floor(first_token / 64) + sequence. Returns false
// for an unused slot (or for cu_seqlens that the scan pass reports as invalid).
__device__ __forceinline__ bool slot_chunk(const PrepParams &p, int slot, int64_t *tok0, int *L)
{
    int n = 0;
    int64_t s0, s1;
    if (p.cu_seqlens) {
        int lo = 0, hi = p.N - 1;                 // largest n with floor(cu[n]/64) + n <= slot
        if (hi < 0) return false;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (p.cu_seqlens[mid] / C + mid <= slot) lo = mid; else hi = mid - 1;
        }
        n = lo;
        s0 = p.cu_seqlens[n];
        s1 = p.cu_seqlens[n + 1];
        if (s1 < s0 || s0 < 0 || s1 > p.T) return false;
    } else {
        // sequence n = batch row; its first slot is (n * T) / 64 + n
        int lo = 0, hi = p.N - 1;
        if (hi < 0) return false;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if ((int)(((int64_t)mid * p.T) / C) + mid <= slot) lo = mid; else hi = mid - 1;
        }
        n = lo;
        s0 = (int64_t)n * p.T;
        s1 = s0 + p.T;
    }
    const int64_t c = slot - (s0 / C + n);
    *tok0 = s0 + c * C;
    if (c < 0 || *tok0 >= s1) return false;
    *L = (s1 - *tok0 < C) ? (int)(s1 - *tok0) : C;
    return true;
}


// Unit lower-triangular inverse (see chunk_tc.cu): A column-major in AT, T row-major stride LDT.
__device__ __forceinline__ void inverse64(int pt, const float *AT, float *Tf, float *Ps)
{
    const int pw = pt >> 5, lane = pt & 31;
    if (pw < 2) {
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
        for (int e = pt - 64; e < 64 * 64; e += NT - 64) {
            const int r = e >> 6, c = e & 63;
            if ((c >> 4) > (r >> 4)) Tf[r * LDT + c] = 0.f;
        }
    }
    __syncthreads();
    {   // T_{b+1,b} partial products, b = 0, 2
        const int blk = pt >> 7, idx = pt & 127, r = idx >> 3, c0 = (idx & 7) * 2, b = 2 * blk;
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
    __syncthreads();
    {
        const int blk = pt >> 7, idx = pt & 127, r = idx >> 3, c0 = (idx & 7) * 2, b = 2 * blk, o = 16 * (b + 1);
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
    __syncthreads();
    {   // T[32:64, 0:32] = -T_hi (A_hi,lo T_lo)
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
    __syncthreads();
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
    __syncthreads();
}

// softplus on the bf16 path: two fast special-function ops; its absolute error (~1e-7, which is
// also all that is left of softplus(x) below x = -16) is far inside what bf16 inputs carry
__device__ __forceinline__ float softplus_f(float x) { return x > 16.f ? x : __logf(1.f + __expf(x)); }

template <bool GATE>
__global__ void __launch_bounds__(NT, 2)
chunk_prep_kernel(PrepParams p, const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_la)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // head fastest: the CTAs resident at one time cover all heads of a few consecutive chunks, so
    // together they read whole [token][head][channel] rows of q, k and log_alpha (DRAM pages are
    // used in full; with one head per row window each 8 KB row would give up 256 bytes)
    const int h = (int)(blockIdx.x % (unsigned)p.H), slot = p.slot_base + (int)(blockIdx.x / (unsigned)p.H);
    const int H = p.H;

    int64_t tok0;
    int L;
    if (!slot_chunk(p, slot, &tok0, &L)) return;  // unused slot
    // every workspace store below is at a constant offset below kPrepBlockBytes inside this block
    if (!in_bounds(p.status, (long long)h * p.n_slots + slot, 1, (long long)H * p.n_slots)) return;
    unsigned char *blk = p.ws + ((size_t)h * p.n_slots + slot) * kPrepBlockBytes;

    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + OFF_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar + 1);
    float *AT = reinterpret_cast<float *>(sm + OFF_KH);
    float *Tf = reinterpret_cast<float *>(sm + OFF_TF);
    float *Ps = reinterpret_cast<float *>(sm + OFF_PS);
    float *bet = reinterpret_cast<float *>(sm + OFF_BET);

    uint64_t *bar_in = bar + 2;
    if (warp == 0) { tmem_alloc(tmem_slot, TMEM_COLS); tmem_relinquish(); }
    if (tid == 0) {
        // ---- loads: the chunk's 64 rows of q, k and log_alpha for this head, one tensor copy each
        //      (rows past the end of the tensor read as zero; rows of the next sequence are masked
        //      below); then warp w -> rows 8w..8w+7, lane -> channels 4 lane..4 lane+3 into registers
        mbar_init(bar, 1);
        mbar_init(bar_in, 1);
        fence_mbar_init();
        mbar_arrive_expect_tx(bar_in, (uint32_t)C * (2 * DK * 2 + DK * (GATE ? 2 : 4)));
        tma_load_3d(sm + STG_Q, &tm_q, bar_in, 0, h, (int)tok0);
        tma_load_3d(sm + STG_K, &tm_k, bar_in, 0, h, (int)tok0);
        tma_load_3d(sm + STG_LA, &tm_la, bar_in, 0, h, (int)tok0);
        // ask for the inputs of the unit one wave of resident CTAs ahead into L2, so that its
        // tensor copies are served from L2 instead of waiting on DRAM
        if (p.prefetch_wave > 0) {
            const long long nxt = (long long)blockIdx.x + p.prefetch_wave;
            int64_t ptok;
            int pL;
            if (nxt < (long long)gridDim.x && slot_chunk(p, p.slot_base + (int)(nxt / H), &ptok, &pL)) {
                const int ph = (int)(nxt % H);
                tma_prefetch_3d(&tm_q, 0, ph, (int)ptok);
                tma_prefetch_3d(&tm_k, 0, ph, (int)ptok);
                tma_prefetch_3d(&tm_la, 0, ph, (int)ptok);
            }
        }
    }
    __syncthreads();
    if (!mbar_wait(bar_in, 0)) {
        set_status(p.status, KDA_ERR_TIMEOUT);
        mbar_wait(bar_in, 0, 100000000LL);         // copies still landing must not outlive the CTA
    }
    const int cq = lane, kh = cq >> 4, lc4 = cq & 15;
    float4 la[8];
    uint2 kr[8], qr[8];
    float rate = 0.f, bias[4] = {0.f, 0.f, 0.f, 0.f};
    if constexpr (GATE) {
        rate = expf(p.A_log[h]);
        const float4 b4 = *reinterpret_cast<const float4 *>(p.dt_bias + (size_t)h * DK + 4 * cq);
        bias[0] = b4.x; bias[1] = b4.y; bias[2] = b4.z; bias[3] = b4.w;
    }
#pragma unroll
    for (int x = 0; x < 8; ++x) {
        const int r = 8 * warp + x;
        if (r < L) {
            if constexpr (GATE) {         // log_alpha = -exp(A_log) softplus(f + dt_bias)
                const uint2 fr = *reinterpret_cast<const uint2 *>(sm + STG_LA + r * 256 + 8 * cq);
                la[x] = make_float4(-rate * softplus_f(bf_lo(fr.x) + bias[0]), -rate * softplus_f(bf_hi(fr.x) + bias[1]),
                                    -rate * softplus_f(bf_lo(fr.y) + bias[2]), -rate * softplus_f(bf_hi(fr.y) + bias[3]));
            } else {
                la[x] = *reinterpret_cast<const float4 *>(sm + STG_LA + r * 512 + 16 * cq);
            }
            kr[x] = *reinterpret_cast<const uint2 *>(sm + STG_K + r * 256 + 8 * cq);
            qr[x] = *reinterpret_cast<const uint2 *>(sm + STG_Q + r * 256 + 8 * cq);
        } else {
            la[x] = make_float4(0.f, 0.f, 0.f, 0.f);
            kr[x] = make_uint2(0u, 0u);
            qr[x] = kr[x];
        }
    }
    if (tid < C) {
        const long long bi = (long long)(tok0 + tid) * H + h;
        float b = 0.f;
        if (tid < L && in_bounds(p.status, bi, 1, p.tokens * H))
            b = p.beta_logits ? 1.f / (1.f + __expf(-__bfloat162float(p.beta_logits[bi]))) : p.beta[bi];
        bet[tid] = b;
    }

    // ---- decay scaling: per-thread products over its 8 rows, then over the 8 warps via smem
    float a[8][4], pre[8][4];
#pragma unroll
    for (int x = 0; x < 8; ++x) {
        a[x][0] = __expf(la[x].x); a[x][1] = __expf(la[x].y);
        a[x][2] = __expf(la[x].z); a[x][3] = __expf(la[x].w);
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        float run = 1.f;
#pragma unroll
        for (int x = 0; x < 8; ++x) { run *= a[x][e]; pre[x][e] = run; }
    }
    *reinterpret_cast<float4 *>(Ps + warp * 128 + 4 * cq) = make_float4(pre[7][0], pre[7][1], pre[7][2], pre[7][3]);
    __syncthreads();
    float before[4] = {1.f, 1.f, 1.f, 1.f}, after[4] = {1.f, 1.f, 1.f, 1.f}, g[4], rg[4];
    float gall[4] = {1.f, 1.f, 1.f, 1.f};      // the same product in one fixed order in every warp
#pragma unroll
    for (int y = 0; y < 8; ++y) {
        const float4 t = *reinterpret_cast<const float4 *>(Ps + y * 128 + 4 * cq);
        const float tv[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            if (y < warp) before[e] *= tv[e];
            if (y > warp) after[e] *= tv[e];
            gall[e] *= tv[e];
        }
    }
    // tf32 operands for P1 when any channel decays below e^-8 over the chunk (bitwise the same
    // decision in every warp: each lane holds 4 channels, the lanes of a warp all 128)
    const bool wide = __any_sync(0xffffffffu, gall[0] < kF16MinDecay || gall[1] < kF16MinDecay ||
                                               gall[2] < kF16MinDecay || gall[3] < kF16MinDecay) != 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        g[e] = before[e] * pre[7][e] * after[e];
        rg[e] = __frcp_rn(g[e]);
    }
    // Workspace (global) stores of each phase are issued after that phase's proxy fence and MMA
    // issue: a fence.proxy.async would otherwise also wait for them to complete.
    uint2 kend[8], okt8[8], oqt8[8];   // f16 Kend (to the workspace), Kt and Qt (tiles after P1)
    {
        float suf[4] = {1.f, 1.f, 1.f, 1.f};
        const uint32_t qj = (uint32_t)(lane >> 3), ch16 = (uint32_t)(lane & 7);   // tf32 quarter, chunk
#pragma unroll
        for (int x = 7; x >= 0; --x) {
            const int r = 8 * warp + x;
            const uint32_t off32 = r * 128 + (((ch16 ^ (r & 7)) & 7) << 4);
            const uint32_t kw[2] = {kr[x].x, kr[x].y};
            const uint32_t qw[2] = {qr[x].x, qr[x].y};
            uint32_t okt[2], oqt[2], oke[2];
            float kt4[4], qt4[4], kh4[4];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int e = 2 * u;
                const float f0 = before[e] * pre[x][e], f1 = before[e + 1] * pre[x][e + 1];
                const float b0 = suf[e] * after[e], b1 = suf[e + 1] * after[e + 1];
                const float k0 = bf_lo(kw[u]), k1 = bf_hi(kw[u]);
                const float q0 = bf_lo(qw[u]), q1 = bf_hi(qw[u]);
                const float e0 = k0 * b0, e1 = k1 * b1;
                kt4[e] = k0 * f0; kt4[e + 1] = k1 * f1;
                qt4[e] = q0 * f0; qt4[e + 1] = q1 * f1;
                kh4[e] = e0 * rg[e]; kh4[e + 1] = e1 * rg[e + 1];
                okt[u] = pack_f16x2(kt4[e], kt4[e + 1]);
                oqt[u] = pack_f16x2(qt4[e], qt4[e + 1]);
                oke[u] = pack_f16x2(e0, e1);
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) suf[e] *= a[x][e];
            if (wide) {
                *reinterpret_cast<float4 *>(sm + OFF_QK32 + qj * 16384 + off32) =
                    make_float4(to_tf32(qt4[0]), to_tf32(qt4[1]), to_tf32(qt4[2]), to_tf32(qt4[3]));
                *reinterpret_cast<float4 *>(sm + OFF_QK32 + qj * 16384 + 8192 + off32) =
                    make_float4(to_tf32(kt4[0]), to_tf32(kt4[1]), to_tf32(kt4[2]), to_tf32(kt4[3]));
                *reinterpret_cast<float4 *>(sm + OFF_KH32 + qj * 8192 + off32) =
                    make_float4(to_tf32(kh4[0]), to_tf32(kh4[1]), to_tf32(kh4[2]), to_tf32(kh4[3]));
            } else {
                const uint32_t off = r * 128 + ((((lc4 >> 1) ^ (r & 7)) & 7) << 4) + ((lc4 & 1) << 3);
                *reinterpret_cast<uint2 *>(sm + OFF_KT + kh * QK_HALF + off) = make_uint2(okt[0], okt[1]);
                *reinterpret_cast<uint2 *>(sm + OFF_QK + kh * QK_HALF + off) = make_uint2(oqt[0], oqt[1]);
                *reinterpret_cast<uint2 *>(sm + OFF_KH + kh * 8192 + off) =
                    make_uint2(pack_f16x2(kh4[0], kh4[1]), pack_f16x2(kh4[2], kh4[3]));
            }
            kend[x] = make_uint2(oke[0], oke[1]);
            okt8[x] = make_uint2(okt[0], okt[1]);
            oqt8[x] = make_uint2(oqt[0], oqt[1]);
        }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // ---- P1: D1A = [Qt; Kt] Kh^T (M=128, N=64, K=128; f16, or tf32 for a wide decay range):
    //      rows 0-63 Qt Kh^T, rows 64-127 Kt Kh^T
    if (tid == 0) {
        if (wide) {
            const uint32_t id = idesc_tf32(128, 64, 0, 0);
#pragma unroll
            for (int ks = 0; ks < 16; ++ks) {
                const uint32_t qj = ks >> 2, ko = (ks & 3) * 32;
                umma_ss_tf32(tmem + TM_D1A, smem_desc(sbase + OFF_QK32 + qj * 16384 + ko, 16, 1024, SW_128B),
                             smem_desc(sbase + OFF_KH32 + qj * 8192 + ko, 16, 1024, SW_128B), id, ks > 0);
            }
        } else {
            const uint32_t id = idesc_f16(128, 64, 0, 0);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t k2 = ks >> 2, ko = (ks & 3) * 32;
                umma_ss(tmem + TM_D1A, smem_desc(sbase + OFF_QK + k2 * QK_HALF + ko, 16, 1024, SW_128B),
                        smem_desc(sbase + OFF_KH + k2 * 8192 + ko, 16, 1024, SW_128B), id, ks > 0);
            }
        }
        umma_commit(bar);
    }
#pragma unroll
    for (int x = 0; x < 8; ++x) {
        const int r = 8 * warp + x;
        const uint32_t off = r * 128 + ((((lc4 >> 1) ^ (r & 7)) & 7) << 4) + ((lc4 & 1) << 3);
        *reinterpret_cast<uint2 *>(blk + kPrepKEOff + kh * 8192 + off) = kend[x];
    }
    if (warp == 0) {
        float *gw = reinterpret_cast<float *>(blk + kPrepGammaOff);
        *reinterpret_cast<float4 *>(gw + 4 * cq) = make_float4(g[0], g[1], g[2], g[3]);
        if (g[0] < kMinChunkDecay || g[1] < kMinChunkDecay || g[2] < kMinChunkDecay || g[3] < kMinChunkDecay)
            set_status(p.status, KDA_ERR_UNSUPPORTED);
    }
    int32_t failed = 0;
    if (tid == 0 && !mbar_wait(bar, 0)) failed = 1;
    __syncthreads();
    tc_fence_after();
    // ---- tf32 path: its operands are dead; the f16 Kt and Qt tiles (B of P3; read by the last
    //      epilogue) take their place
    if (wide) {
#pragma unroll
        for (int x = 0; x < 8; ++x) {
            const int r = 8 * warp + x;
            const uint32_t off = r * 128 + ((((lc4 >> 1) ^ (r & 7)) & 7) << 4) + ((lc4 & 1) << 3);
            *reinterpret_cast<uint2 *>(sm + OFF_KT + kh * QK_HALF + off) = okt8[x];
            *reinterpret_cast<uint2 *>(sm + OFF_QK + kh * QK_HALF + off) = oqt8[x];
        }
    }
    // ---- P1 epilogue (M=128: lane = row): rows 0-63 -> M (f16, smem), rows 64-127 -> A^T (fp32,
    //      smem); warp w takes columns 32 (w / 4) .. +31 of its rows
    {
        const int q4 = warp & 3, half = warp >> 2;
        const int row = 32 * q4 + lane, c0 = 32 * half;
        float v[32];
        tmem_ld32_sync(tmem + ((uint32_t)(32 * q4) << 16) + TM_D1A + c0, v);
        if (q4 < 2) {
            const int r = row;
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                uint32_t w4[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int i = c0 + 8 * ch + 2 * u;
                    w4[u] = pack_f16x2(i <= r ? v[8 * ch + 2 * u] : 0.f, i + 1 <= r ? v[8 * ch + 2 * u + 1] : 0.f);
                }
                *reinterpret_cast<uint4 *>(sm + OFF_M + sw128_offset(r, c0 + 8 * ch)) =
                    make_uint4(w4[0], w4[1], w4[2], w4[3]);
            }
        } else {
            const int r = row - 64;
            const float br = bet[r];
#pragma unroll
            for (int j = 0; j < 32; ++j) AT[(c0 + j) * 64 + r] = (c0 + j < r) ? br * v[j] : 0.f;
        }
    }
    tc_fence_before();
    __syncthreads();
    // ---- T = (I + A)^{-1};  Tb = T diag(beta) -> f16 (smem for P3 and P4; -Tb to the workspace)
    inverse64(tid, AT, Tf, Ps);
    {
        const int r = tid >> 2, c0 = (tid & 3) * 16;
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
            const uint4 o = make_uint4(w4[0], w4[1], w4[2], w4[3]);
            *reinterpret_cast<uint4 *>(sm + OFF_TB + sw128_offset(r, cb)) = o;
        }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // ---- P3: W = Tb Kt (M=64, N=128, K=64; B = Kt MN-major) into columns 0-127
    if (tid == 0) {
        const uint32_t id = idesc_f16(64, 128, 0, 1);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
            umma_ss(tmem + TM_D1A, smem_desc(sbase + OFF_TB + ks * 32, 16, 1024, SW_128B),
                    smem_desc(sbase + OFF_KT + ks * 2048, QK_HALF, 1024, SW_128B), id, ks > 0);
        umma_commit(bar);
    }
    {   // -Tb to the workspace (Y rows 0-63), from its shared-memory copy
        const int r = tid >> 2, c0 = (tid & 3) * 16;
        const uint32_t sgn = 0x80008000u;            // f16 sign bits
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const uint32_t o = sw128_offset(r, c0 + 8 * hh);
            const uint4 t = *reinterpret_cast<const uint4 *>(sm + OFF_TB + o);
            *reinterpret_cast<uint4 *>(blk + kPrepYOff + o) = make_uint4(t.x ^ sgn, t.y ^ sgn, t.z ^ sgn, t.w ^ sgn);
        }
    }
    if (tid == 0 && !failed && !mbar_wait(bar, 1)) failed = 1;
    __syncthreads();
    tc_fence_after();
    // ---- W epilogue (M=64 layout: lanes 0-15 of each quadrant), warps 0-3 cols 0-63, 4-7 cols 64-127:
    //      W -> workspace (X rows 0-63) and -> smem as N-blocks 1-2 of [Tb | W] (A^T is dead by now)
    {
        const int q4 = warp & 3, half = warp >> 2;
        float w[64];
        tmem_ld64_sync(tmem + ((uint32_t)(32 * q4) << 16) + TM_D1A + 64 * half, w);
        if (lane < 16) {
            const int r = 16 * q4 + lane;
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
                uint4 o;
                o.x = pack_f16x2(w[8 * ch + 0], w[8 * ch + 1]);
                o.y = pack_f16x2(w[8 * ch + 2], w[8 * ch + 3]);
                o.z = pack_f16x2(w[8 * ch + 4], w[8 * ch + 5]);
                o.w = pack_f16x2(w[8 * ch + 6], w[8 * ch + 7]);
                *reinterpret_cast<uint4 *>(sm + OFF_KH + half * 8192 + sw128_offset(r, 8 * ch)) = o;
            }
        }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // ---- P4: M [Tb | W] (M=64, N=192, K=64; B = [Tb | W] MN-major, N-blocks 8 KiB apart) -> cols 0-191
    if (tid == 0 && !failed) {
        const uint32_t id = idesc_f16(64, 192, 0, 1);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
            umma_ss(tmem + TM_D1A, smem_desc(sbase + OFF_M + ks * 32, 16, 1024, SW_128B),
                    smem_desc(sbase + OFF_TB + ks * 2048, 8192, 1024, SW_128B), id, ks > 0);
        umma_commit(bar);
    }
    {   // W to the workspace (X rows 0-63), from its shared-memory copy
        const int q4 = warp & 3, half = warp >> 2;
        if (lane < 16) {
            const int r = 16 * q4 + lane;
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
                const uint32_t o = sw128_offset(r, 8 * ch);
                *reinterpret_cast<uint4 *>(blk + kPrepXOff + half * 16384 + o) =
                    *reinterpret_cast<const uint4 *>(sm + OFF_KH + half * 8192 + o);
            }
        }
    }
    if (tid == 0 && !failed && !mbar_wait(bar, 0)) failed = 1;
    __syncthreads();
    tc_fence_after();
    // ---- P4 epilogue (M=64 layout: lanes 0-15 of each quadrant), warps 0-3 cols 0-95, 4-7 cols
    //      96-191, in 32-column groups: M Tb (cols 0-63) -> Y rows 64-127; Qt - M W (cols 64-191,
    //      channel = col - 64) -> X rows 64-127
    {
        const int q4 = warp & 3, half = warp >> 2;
        const int r = 16 * q4 + (lane & 15);
#pragma unroll
        for (int grp = 0; grp < 3; ++grp) {
            const int c0 = 96 * half + 32 * grp;
            float m[32];
            tmem_ld32_sync(tmem + ((uint32_t)(32 * q4) << 16) + TM_D1A + c0, m);
            if (lane < 16) {
#pragma unroll
                for (int u8 = 0; u8 < 4; ++u8) {
                    const int c = c0 + 8 * u8;                 // 8 columns c .. c + 7
                    uint32_t o[4];
                    if (c < 64) {
#pragma unroll
                        for (int u = 0; u < 4; ++u) o[u] = pack_f16x2(m[8 * u8 + 2 * u], m[8 * u8 + 2 * u + 1]);
                        *reinterpret_cast<uint4 *>(blk + kPrepYOff + sw128_offset(64 + r, c)) =
                            make_uint4(o[0], o[1], o[2], o[3]);
                    } else {
                        const int kh = (c - 64) >> 6, cc = (c - 64) & 63;
                        const uint4 qv = *reinterpret_cast<const uint4 *>(sm + OFF_QK + kh * QK_HALF + sw128_offset(r, cc));
                        const uint32_t qw[4] = {qv.x, qv.y, qv.z, qv.w};
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const float2 qf = __half22float2(*reinterpret_cast<const __half2 *>(&qw[u]));
                            o[u] = pack_f16x2(qf.x - m[8 * u8 + 2 * u], qf.y - m[8 * u8 + 2 * u + 1]);
                        }
                        *reinterpret_cast<uint4 *>(blk + kPrepXOff + kh * 16384 + 64 * 128 + sw128_offset(r, cc)) =
                            make_uint4(o[0], o[1], o[2], o[3]);
                    }
                }
            }
        }
    }
    if (failed) set_status(p.status, KDA_ERR_TIMEOUT);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, TMEM_COLS);
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, []() {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(f);
    });
    return fn;
}

}  // namespace

bool token_rows_map(CUtensorMap *m, const void *base, CUtensorMapDataType dt, uint32_t elem_bytes, int H,
                    long long tokens, uint32_t box_cols, bool swizzle128)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)DK, (cuuint64_t)H, (cuuint64_t)tokens};
    const cuuint64_t strides[2] = {(cuuint64_t)DK * elem_bytes, (cuuint64_t)DK * elem_bytes * H};
    const cuuint32_t box[3] = {box_cols, 1u, (cuuint32_t)C};
    const cuuint32_t estr[3] = {1u, 1u, 1u};
    return fn(m, dt, 3, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_chunk_prep(const PrefillArgs &a, unsigned char *ws, int n_slots, cudaStream_t stream,
                              const GateArgs *gate, int slot_lo, int slot_hi)
{
    if (slot_hi < 0 || slot_hi > n_slots) slot_hi = n_slots;
    if (slot_lo < 0) slot_lo = 0;
    if (slot_lo >= slot_hi) return cudaSuccess;
    PrepParams p;
    p.q = (const __nv_bfloat16 *)a.q; p.k = (const __nv_bfloat16 *)a.k;
    p.log_alpha = a.log_alpha; p.beta = a.beta; p.cu_seqlens = a.cu_seqlens;
    const bool fgate = gate && gate->f;
    p.A_log = fgate ? gate->A_log : nullptr;
    p.dt_bias = fgate ? gate->dt_bias : nullptr;
    p.beta_logits = gate ? (const __nv_bfloat16 *)gate->beta_logits : nullptr;
    p.ws = ws; p.T = a.T; p.H = a.H; p.N = a.N; p.n_slots = n_slots; p.status = a.status;
    p.slot_base = slot_lo;
    p.tokens = (long long)a.B * a.T;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        sms = 0;
    p.prefetch_wave = 2 * sms;                    // two CTAs per SM
    const long long tokens = (long long)a.B * a.T;
    if (tokens == 0) return cudaSuccess;          // no chunk to prepare
    CUtensorMap tq, tk, tla;
    if (!token_rows_map(&tq, a.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.H, tokens) ||
        !token_rows_map(&tk, a.k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.H, tokens) ||
        !(fgate ? token_rows_map(&tla, gate->f, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.H, tokens)
                : token_rows_map(&tla, a.log_alpha, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, a.H, tokens)))
        return cudaErrorNotSupported;

    auto kern = fgate ? chunk_prep_kernel<true> : chunk_prep_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_ALLOC);
    if (e != cudaSuccess) return e;
    const dim3 grid((unsigned)(slot_hi - slot_lo) * (unsigned)a.H);
    kern<<<grid, NT, SMEM_ALLOC, stream>>>(p, tq, tk, tla);
    return cudaGetLastError();
}

}  // namespace kda
