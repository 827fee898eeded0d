// chunk_scan.cu -- second pass of the two-pass bf16 prefill: the state recurrence over chunks.
//
// For each chunk (operands from chunk_prep.cu) with S the state entering the chunk:
//   D5  = -[Tb; 0] V                      (the Tb V term; seeds the accumulator)
//   D5 += [W; Qt] S                       rows 0-63: W S - Tb V = -U,  rows 64-127: Qt S
//   D7  = Kend^T U ;   D5 += [0; M] U     rows 64-127: O = Qt S + M U
//   S  <- Diag(gamma) S + D7              (fp32, registers; thread = key channel)
// (U = Tb V - W S are the chunk's delta-rule writes; chunk-parallel form with a WY/UT
// representation, KimiLinear KDA/MLA tutorial (icman.com.cn), sec. 3 and 6.)
//
// One CTA per (sequence, head, 32-wide block of d_v): the value columns of S evolve independently.
// Warp 4 is the producer: it bulk-copies each chunk's prepared block (W/Qt, Tb, M, Kend, gamma;
// already in the swizzled shared-memory layout) into a two-stage ring with cp.async.bulk, tracked
// by mbarriers with transaction counts. Warps 0-3 run the chain; the v block of the next chunk is
// loaded into registers while the current chunk is in flight. Only the tensor-core instructions of
// the chain sit between consecutive chunks.
#include "kda_internal.cuh"
#include "sm100.cuh"

namespace kda {
namespace {

using namespace sm100;

constexpr int C = kChunk;
constexpr int DK = kHeadDim;
constexpr int DVB = 32;
constexpr int SG = 128;                       // scan threads (warps 0-3)
constexpr int NT = SG + 32;                   // + producer warp

// one ring stage (offsets inside a stage; stages are 1024-aligned)
constexpr uint32_t ST_WQ = 0;                 // 32 KB: W rows 0-63, Qt rows 64-127 (two halves)
constexpr uint32_t ST_Y = 32768;              // 24 KB: Tb (rows 0-63) | zero (64-127) | M (128-191)
constexpr uint32_t ST_KE = ST_Y + 24576;      // 16 KB: Kend
constexpr uint32_t ST_V = ST_KE + 16384;      // 4 KB: v block (f16, 64-byte rows)
constexpr uint32_t ST_G = ST_V + 4096;        // 512 B: gamma
constexpr uint32_t STAGE = 78848;             // 77 KB
constexpr uint32_t OFF_SB = 2 * STAGE;        // S (f16), 128 rows x 64 B
constexpr uint32_t OFF_UB = OFF_SB + 8192;    // U (f16), 64 rows x 64 B
constexpr uint32_t OFF_BAR = OFF_UB + 4096;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 128;
constexpr uint32_t SMEM_ALLOC = SMEM_BYTES + 1024;
static_assert(SMEM_ALLOC <= 232448, "shared memory plan exceeds 227 KiB");
static_assert(ST_G + 512 <= STAGE && STAGE % 1024 == 0, "stage layout");

constexpr uint32_t BLOCK_TX = 32768 + 8192 + 8192 + 16384 + 512;   // bytes copied per chunk

constexpr uint32_t TMEM_COLS = 64;
constexpr uint32_t TM_D5 = 0;
constexpr uint32_t TM_D7 = 32;

enum { B_FULL = 0, B_EMPTY = 2, B_S1 = 4, B_S2 = 5, B_MU = 6, N_BARS = 7 };

struct ScanParams {
    const __nv_bfloat16 *v;
    const float *S0;
    const int32_t *cu_seqlens;
    const unsigned char *ws;
    void *out;
    float *S_final;
    int T, H, N, n_slots;
    int32_t *status;
};

__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ uint4 ldg_nc(const void *p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
    return r;
}

template <typename TO>
__global__ void __launch_bounds__(NT, 1)
chunk_scan_kernel(ScanParams p)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int jb = blockIdx.x, h = blockIdx.y, n = blockIdx.z;
    const int j0 = jb * DVB, H = p.H;

    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + OFF_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + N_BARS);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(bars + N_BARS) + 1;

    int64_t t0, t1;
    if (!sequence_span(p.cu_seqlens, n, p.N, p.T, &t0, &t1, p.status)) return;   // uniform
    const int nchunks = (int)((t1 - t0 + C - 1) / C);
    const int64_t first_slot = t0 / C + n;

    if (warp == 0) { tmem_alloc(tmem_slot, TMEM_COLS); tmem_relinquish(); }
    if (tid == 0) {
        for (int i = 0; i < N_BARS; ++i) mbar_init(&bars[i], 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    for (int i = tid; i < 2 * 8192 / 16; i += NT) {      // zero rows 64-127 of both Y regions
        const int st = i / (8192 / 16), o = i % (8192 / 16);
        reinterpret_cast<uint4 *>(sm + st * STAGE + ST_Y + 8192)[o] = make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    auto fail = [&]() { set_status(p.status, KDA_ERR_TIMEOUT); *abort_flag = 1; };

    if (warp == 4) {
        // ================================================================ producer (one lane)
        if (lane == 0) {
            uint32_t issued[2] = {0u, 0u};
            for (int c = 0; c < nchunks; ++c) {
                const int s = c & 1;
                if (*abort_flag) break;
                if (c >= 2 && !mbar_wait(&bars[B_EMPTY + s], ((c >> 1) - 1) & 1)) { fail(); break; }
                const unsigned char *blk = p.ws + ((size_t)h * p.n_slots + (first_slot + c)) * kPrepBlockBytes;
                unsigned char *stg = sm + s * STAGE;
                mbar_arrive_expect_tx(&bars[B_FULL + s], BLOCK_TX);
                bulk_g2s(stg + ST_WQ, blk + kPrepWQOff, 32768, &bars[B_FULL + s]);
                bulk_g2s(stg + ST_Y, blk + kPrepTbOff, 8192, &bars[B_FULL + s]);
                bulk_g2s(stg + ST_Y + 16384, blk + kPrepMOff, 8192, &bars[B_FULL + s]);
                bulk_g2s(stg + ST_KE, blk + kPrepKEOff, 16384, &bars[B_FULL + s]);
                bulk_g2s(stg + ST_G, blk + kPrepGammaOff, 512, &bars[B_FULL + s]);
                ++issued[s];
            }
            // no copy may still be landing when the CTA exits
            for (int s = 0; s < 2; ++s)
                if (issued[s]) mbar_wait(&bars[B_FULL + s], (issued[s] - 1) & 1, 100000000LL);
        }
    } else {
        // ================================================================ scan chain
        const int st = tid;
        float S[DVB];
        {
            const size_t sidx = (((size_t)n * H + h) * DK + st) * DK + j0;
#pragma unroll
            for (int j = 0; j < DVB; j += 4) {
                const float4 v = p.S0 ? *reinterpret_cast<const float4 *>(p.S0 + sidx + j) : make_float4(0, 0, 0, 0);
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
        // v block of a chunk: thread -> row st >> 1, columns 16 (st & 1)..+15
        auto load_v = [&](int c, uint4 (&vr)[2]) {
            const int64_t tok0 = t0 + (int64_t)c * C;
            const int L = (t1 - tok0 < C) ? (int)(t1 - tok0) : C;
            const int r = st >> 1;
            if (r < L) {
                const __nv_bfloat16 *src = p.v + ((size_t)(tok0 + r) * H + h) * DK + j0 + 16 * (st & 1);
                vr[0] = ldg_nc(src);
                vr[1] = ldg_nc(src + 8);
            } else {
                vr[0] = make_uint4(0, 0, 0, 0);
                vr[1] = vr[0];
            }
        };
        store_state();
        uint4 vr[2];
        if (nchunks > 0) load_v(0, vr);
        uint32_t n_commits = 0;
        for (int c = 0; c < nchunks; ++c) {
            const int s = c & 1;
            const int64_t tok0 = t0 + (int64_t)c * C;
            const int L = (t1 - tok0 < C) ? (int)(t1 - tok0) : C;
            unsigned char *stg = sm + s * STAGE;
            const uint32_t astg = sbase + s * STAGE;
            {   // v (bf16 -> f16) into the stage
                const int r = st >> 1;
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    uint4 o;
                    o.x = bf16x2_to_f16x2(vr[u].x); o.y = bf16x2_to_f16x2(vr[u].y);
                    o.z = bf16x2_to_f16x2(vr[u].z); o.w = bf16x2_to_f16x2(vr[u].w);
                    *reinterpret_cast<uint4 *>(stg + ST_V + sw64_offset(r, 16 * (st & 1) + 8 * u)) = o;
                }
            }
            fence_proxy_async_smem();
            // every scan thread observes the stage's arrival (it reads gamma from it directly)
            if (!mbar_wait(&bars[B_FULL + s], (c >> 1) & 1)) fail();
            tc_fence_before();
            named_bar_sync(1, SG);
            if (*abort_flag) break;
            tc_fence_after();
            if (st == 0) {
                ++n_commits;
                const uint32_t ids = idesc_f16(128, 32, 0, 1) | (1u << 13);   // -[Tb; 0] V
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    umma_ss(tmem + TM_D5, smem_desc(astg + ST_Y + ks * 32, 16, 1024, SW_128B),
                            smem_desc(astg + ST_V + ks * 1024, 16, 512, SW_64B), ids, ks > 0);
                const uint32_t id = idesc_f16(128, 32, 0, 1);                  // += [W; Qt] S
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t kh = ks >> 2, ko = (ks & 3) * 32;
                    umma_ss(tmem + TM_D5, smem_desc(astg + ST_WQ + kh * 16384 + ko, 16, 1024, SW_128B),
                            smem_desc(sbase + OFF_SB + ks * 1024, 16, 512, SW_64B), id, 1);
                }
                umma_commit(&bars[B_S1]);
            }
            if (c + 1 < nchunks) load_v(c + 1, vr);
            if (st == 0 && !mbar_wait(&bars[B_S1], c & 1)) fail();
            named_bar_sync(1, SG);
            tc_fence_after();
            if (warp < 2) {                  // U = -(rows 0-63) -> f16, MN-major [token][32]
                float u[32];
                tmem_ld32_sync(tmem + TM_D5 + ((uint32_t)(32 * warp) << 16), u);
#pragma unroll
                for (int j = 0; j < DVB; j += 8) {
                    uint4 o;
                    o.x = pack_f16x2(-u[j], -u[j + 1]); o.y = pack_f16x2(-u[j + 2], -u[j + 3]);
                    o.z = pack_f16x2(-u[j + 4], -u[j + 5]); o.w = pack_f16x2(-u[j + 6], -u[j + 7]);
                    *reinterpret_cast<uint4 *>(sm + OFF_UB + sw64_offset(st, j)) = o;
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar_sync(1, SG);
            tc_fence_after();
            if (st == 0) {
                const uint32_t id2 = idesc_f16(128, 32, 1, 1);                 // Kend^T U
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    umma_ss(tmem + TM_D7, smem_desc(astg + ST_KE + ks * 2048, 8192, 1024, SW_128B),
                            smem_desc(sbase + OFF_UB + ks * 1024, 16, 512, SW_64B), id2, ks > 0);
                umma_commit(&bars[B_S2]);
                const uint32_t idm = idesc_f16(128, 32, 0, 1);                 // += [0; M] U
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    umma_ss(tmem + TM_D5, smem_desc(astg + ST_Y + 8192 + ks * 32, 16, 1024, SW_128B),
                            smem_desc(sbase + OFF_UB + ks * 1024, 16, 512, SW_64B), idm, 1);
                umma_commit(&bars[B_MU]);
            }
            if (st == 0 && !mbar_wait(&bars[B_S2], c & 1)) fail();
            named_bar_sync(1, SG);
            tc_fence_after();
            {   // S <- gamma S + Kend^T U
                const float g = reinterpret_cast<const float *>(stg + ST_G)[st];
                float d7[32];
                tmem_ld32_sync(tmem + TM_D7 + ((uint32_t)(32 * warp) << 16), d7);
#pragma unroll
                for (int e = 0; e < 32; ++e) S[e] = g * S[e] + d7[e];
                store_state();
            }
            fence_proxy_async_smem();
            if (st == 0 && !mbar_wait(&bars[B_MU], c & 1)) fail();
            tc_fence_before();
            named_bar_sync(1, SG);
            tc_fence_after();
            if (warp >= 2) {                 // O = rows 64-127 -> out
                const int r = st - 64;
                float o32[32];
                tmem_ld32_sync(tmem + TM_D5 + ((uint32_t)(32 * warp) << 16), o32);
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
            tc_fence_before();
            named_bar_sync(1, SG);
            if (*abort_flag) break;
            if (st == 0) mbar_arrive(&bars[B_EMPTY + s]);      // stage s may be refilled
        }
        if (*abort_flag && st == 0 && n_commits) {             // drain in-flight MMAs (bounded)
            mbar_wait(&bars[B_S1], (n_commits - 1) & 1, 100000000LL);
            mbar_wait(&bars[B_S2], (n_commits - 1) & 1, 100000000LL);
            mbar_wait(&bars[B_MU], (n_commits - 1) & 1, 100000000LL);
        }
        if (p.S_final && !*abort_flag) {
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
cudaError_t launch_typed(const PrefillArgs &a, const unsigned char *ws, int n_slots, cudaStream_t stream)
{
    ScanParams p;
    p.v = (const __nv_bfloat16 *)a.v; p.S0 = a.S0; p.cu_seqlens = a.cu_seqlens; p.ws = ws;
    p.out = a.out; p.S_final = a.S_final; p.T = a.T; p.H = a.H; p.N = a.N; p.n_slots = n_slots;
    p.status = a.status;
    auto kern = chunk_scan_kernel<TO>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_ALLOC);
    if (e != cudaSuccess) return e;
    const dim3 grid(DK / DVB, a.H, a.N);
    kern<<<grid, NT, SMEM_ALLOC, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_chunk_scan(const PrefillArgs &a, const unsigned char *ws, int n_slots,
                              kda_dtype_t out_dtype, cudaStream_t stream)
{
    if (out_dtype == KDA_BF16) return launch_typed<__nv_bfloat16>(a, ws, n_slots, stream);
    return launch_typed<float>(a, ws, n_slots, stream);
}

}  // namespace kda
