// chunk_scan.cu -- second pass of the two-pass bf16 prefill: the state recurrence over chunks.
//
// For each chunk (operands from chunk_prep.cu) with S the state entering the chunk:
//   D5  = Y V = [-Tb; M Tb] V             (seeds the accumulator; independent of S)
//   D5 += X S = [W; Qt - M W] S           rows 0-63: W S - Tb V = -U,  rows 64-127: the output
//                                         O = Qt S + M U = (Qt - M W) S + M Tb V
//   D7  = Kend^T U
//   S  <- Diag(gamma) S + D7              (fp32, registers; thread = key channel)
// (U = Tb V - W S are the chunk's delta-rule writes; chunk-parallel form with a WY/UT
// representation, KimiLinear KDA/MLA tutorial (icman.com.cn), sec. 3 and 6.)
//
// One CTA per (sequence, head, 32-wide block of d_v): the value columns of S evolve independently.
// Three roles, coupled only by mbarriers (no group-wide barrier inside the chunk loop):
//   warp 5 (lane 0)   issues every tcgen05.mma and commit;
//   warp 4            loader: bulk-copies each chunk's prepared block (X, Y, Kend, gamma, already
//                     in the swizzled layout) into a three-stage ring with one cp.async.bulk, and
//                     writes the v block beside it as f16 (loaded into registers one chunk ahead);
//   warps 0-3         epilogues: U (TMEM -> f16 smem), the outputs, the fp32 state update.
// Only S1 -> U -> S2 -> S sits on the serial chain; the next chunk's seed is queued behind S2 into
// the other half of the double-buffered D5, and the outputs are read while S2 runs.
//
// With the layer's output norm fused (NORM; o_norm = FusedRMSNormGated with a sigmoid gate, lpnh.cn
// Kimi Linear article, sec. 3): y = O / sqrt(mean over the head's d_v channels of O^2 + eps) * w *
// sigmoid(g). The four CTAs of a head hold 32 channels each, so they run as one 4-CTA cluster. Two
// more warps (6, 7; TMEM lanes 64-127, the output rows) own the whole output path: per chunk each
// output thread (one token) sends its partial sum of squares to all four CTAs with asynchronous
// remote stores that complete transaction bytes on the receiving CTA's barrier (no fence on the
// sending side); it finishes the previous chunk meanwhile (sums the four partials of each token from
// its own shared memory and writes the normalised, gated outputs), so one exchange is always in
// flight. Each CTA re-arms a slot once both output warps have read it and tells the senders (a
// relaxed remote arrive) that it may be written again; four slots give the senders slack. Warps 0-3
// keep only the U epilogue and the state update, so the exchange never sits on the serial chain; a
// six D5 buffers let the output warps trail the chain by up to five chunks.
#include "kda_internal.cuh"
#include "sm100.cuh"

namespace kda {
namespace {

using namespace sm100;

constexpr int C = kChunk;
constexpr int DK = kHeadDim;
constexpr int DVB = 32;
constexpr int NT = 192;                       // warps 0-3 epilogue, 4 loader, 5 MMA issuer
constexpr int NT_NORM = 256;                  // with the output norm: warps 6-7 the output path

// one ring stage (offsets inside a stage; stages are 1024-aligned). [0, 66048) is a copy of the
// workspace block.
constexpr uint32_t ST_X = kPrepXOff;          // 32 KB: W rows 0-63, Qt - M W rows 64-127 (two halves)
constexpr uint32_t ST_Y = kPrepYOff;          // 16 KB: -Tb rows 0-63, M Tb rows 64-127
constexpr uint32_t ST_KE = kPrepKEOff;        // 16 KB: Kend
constexpr uint32_t ST_G = kPrepGammaOff;      // 512 B: gamma
constexpr uint32_t ST_V = 66560;              // 4 KB: v block (f16, 64-byte rows)
constexpr uint32_t STAGE = ST_V + 4096;       // 69 KB
constexpr int NSTAGE = 3;
constexpr uint32_t OFF_SB = NSTAGE * STAGE;   // S (f16), 128 rows x 64 B
constexpr uint32_t OFF_UB = OFF_SB + 8192;    // U (f16), 64 rows x 64 B
constexpr uint32_t OFF_BAR = OFF_UB + 4096;
constexpr uint32_t OFF_RED = OFF_BAR + 512;   // output norm: partial sums [4 slots][4 CTAs][64 tokens]
constexpr uint32_t OFF_NW = OFF_RED + 4096;   // output norm: the weight of this CTA's 32 channels
constexpr uint32_t RED_TX = 4 * 64 * 4;      // bytes of partials one chunk brings to a CTA
constexpr uint32_t SMEM_BYTES = OFF_NW + 128;
constexpr uint32_t SMEM_ALLOC = SMEM_BYTES + 1024;
static_assert(SMEM_ALLOC <= 232448, "shared memory plan exceeds 227 KiB");
static_assert(kPrepBlockBytes <= ST_V && STAGE % 1024 == 0 && kPrepBlockBytes % 16 == 0, "stage layout");

// The blocks come from DRAM (the workspace is far larger than L2) and the ring holds three chunks,
// so with copies issued only as stages free up the DRAM latency divided by the ring depth would set
// the chunk rate. Each block is also asked into L2 this many chunks ahead.
constexpr int PREFETCH_AHEAD = 6;

constexpr uint32_t TM_D5 = 0;                 // 2 (6 with the output norm) x 32 columns: [-U; O], by chunk
constexpr int CLUSTER = 4;                    // output norm: the CTAs of one head (d_v / 32)

// mbarriers. A barrier that one role waits on never runs two phases ahead of that role: every
// arrival on it depends, through another barrier, on the waiter having consumed the previous phase.
enum {
    B_FULL = 0,      // [3] by stage: block copied (tx bytes) + loader's v arrival               count 2
    B_EMPTY = 3,     // [3] by stage: consumed (S2 commit + 128 epilogue threads, gamma read)    count 129
    B_D5FREE = 6,    // [6] by D5 buffer: read by the U and output epilogues (128 threads)       count 128
    B_SREADY = 12,   // state of the next chunk in smem (128 epilogue threads)                   count 128
    B_UREADY = 13,   // U in smem (64 epilogue threads)                                          count 64
    B_S1 = 14, B_S2 = 15,   // MMA completions (commit)                                          count 1
    B_DRAIN = 16,    // every MMA of the CTA complete (final commit)                             count 1
    B_REDFULL = 17,  // [4] output norm, by slot (chunk % 4): the 4 x 64 partials have landed here
                     //     (this CTA's own expect_tx arrival + 1024 transaction bytes)          count 1
    B_REDEMPTY = 21, // [4] output norm, by slot: the 4 CTAs have read and re-armed their slot,
                     //     this CTA may send again (one arrival per CTA)                        count 4
    B_S1X = 25,      // [6] output norm, by D5 buffer: D5 complete (commit), for the output warps count 1
    B_REDREAD = 31,  // [4] output norm, by slot: both output warps have read the slot           count 2
    N_BARS = 35
};
static_assert(N_BARS * 8 + 8 <= 512, "barrier area");
constexpr int RSLOTS = 4;                     // output norm: partial-sum slots

struct ScanParams {
    const __nv_bfloat16 *v;
    const float *S0;
    const int32_t *cu_seqlens;
    const unsigned char *ws;
    void *out;
    float *S_final;
    int T, H, N, n_slots;
    long long tokens;               // B * T (rows of v and out)
    int32_t *status;
    const __nv_bfloat16 *gate;      // output norm: g [tokens, H, d_v]
    const float *norm_w;            // output norm: w [d_v]
    float eps;
};

__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void prefetch_l2(const void *p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}
__device__ __forceinline__ uint4 ldg_nc(const void *p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
    return r;
}

// The logistic function as 1/2 + tanh(x/2)/2 with the hardware tanh approximation (one
// special-function op; absolute error below 2.5e-4, under the bf16 rounding of the outputs this
// path writes or reads).
__device__ __forceinline__ float sigmoid_fast(float x) {
    float t;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * x));
    return fmaf(0.5f, t, 0.5f);
}

// 32 consecutive outputs of one token (fp32 or bf16, round to nearest even).
template <typename TO>
__device__ __forceinline__ void store_row32(TO *dst, const float (&y)[32])
{
    if constexpr (sizeof(TO) == 4) {
#pragma unroll
        for (int j = 0; j < 32; j += 4)
            *reinterpret_cast<float4 *>(reinterpret_cast<float *>(dst) + j) = make_float4(y[j], y[j + 1], y[j + 2], y[j + 3]);
    } else {
#pragma unroll
        for (int j = 0; j < 32; j += 8) {
            uint4 o;
            o.x = pack_bf16x2(y[j], y[j + 1]); o.y = pack_bf16x2(y[j + 2], y[j + 3]);
            o.z = pack_bf16x2(y[j + 4], y[j + 5]); o.w = pack_bf16x2(y[j + 6], y[j + 7]);
            *reinterpret_cast<uint4 *>(reinterpret_cast<uint16_t *>(dst) + j) = o;
        }
    }
}

template <typename TO, bool NORM>
__global__ void __launch_bounds__(NORM ? NT_NORM : NT, 1)
chunk_scan_kernel(ScanParams p)
{
    constexpr int ND5 = NORM ? 6 : 2;         // D5 buffers (with the norm: the output warps may trail by 5)
    constexpr uint32_t TMEM_COLS = NORM ? 256 : 128;
    constexpr uint32_t TM_D7 = TM_D5 + 32 * ND5;   // 32 columns: Kend^T U
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
        for (int i = 0; i < NSTAGE; ++i) {
            mbar_init(&bars[B_FULL + i], 2);
            mbar_init(&bars[B_EMPTY + i], 129);
        }
        for (int i = 0; i < ND5; ++i) mbar_init(&bars[B_D5FREE + i], 128);
        if (NORM) {
            for (int i = 0; i < RSLOTS; ++i) {
                mbar_init(&bars[B_REDFULL + i], 1);
                mbar_init(&bars[B_REDEMPTY + i], CLUSTER);
                mbar_init(&bars[B_REDREAD + i], 2);
            }
            for (int i = 0; i < ND5; ++i) mbar_init(&bars[B_S1X + i], 1);
        }
        mbar_init(&bars[B_SREADY], 128);
        mbar_init(&bars[B_UREADY], 64);
        mbar_init(&bars[B_S1], 1);
        mbar_init(&bars[B_S2], 1);
        mbar_init(&bars[B_DRAIN], 1);
        *abort_flag = 0;
        fence_mbar_init();
        if (NORM)               // arm the partial-sum slots of chunks 0-3 before any CTA can send
            for (int i = 0; i < RSLOTS; ++i) mbar_arrive_expect_tx(&bars[B_REDFULL + i], RED_TX);
    }
    if (NORM && tid < 32)
        reinterpret_cast<float *>(sm + OFF_NW)[tid] =
            in_bounds(p.status, j0 + tid, 1, DK) ? p.norm_w[j0 + tid] : 0.f;
    tc_fence_before();
    __syncthreads();
    if constexpr (NORM) cluster_sync_all();   // every CTA's barriers are initialised before any remote arrival
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    auto fail = [&]() { set_status(p.status, KDA_ERR_TIMEOUT); *abort_flag = 1; };
    // a wait whose outcome is the same for the whole (converged) warp, so that warp-collective
    // tcgen05.ld never runs with some lanes gone
    auto warp_wait = [&](uint64_t *bar, uint32_t parity) {
        return __all_sync(0xffffffffu, mbar_wait(bar, parity)) != 0;
    };
    auto warp_abort = [&]() { return __any_sync(0xffffffffu, *abort_flag != 0) != 0; };

    if (warp == 5) {
        // ======================================================================== MMA issuer
        if (lane == 0) {
            uint32_t n_issued = 0;
            const uint32_t id_seed = idesc_f16(128, 32, 0, 1);                // Y V
            const uint32_t id_s1 = idesc_f16(128, 32, 0, 1);                  // X S
            const uint32_t id_s2 = idesc_f16(128, 32, 1, 1);                  // Kend^T U
            for (int c = 0; c < nchunks && !*abort_flag; ++c) {
                const int s = c % NSTAGE, d = c % ND5;
                const uint32_t astg = sbase + s * STAGE;
                const uint32_t d5 = tmem + TM_D5 + 32 * d;
                if (!mbar_wait(&bars[B_FULL + s], (c / NSTAGE) & 1)) { fail(); break; }
                ++n_issued;
                if (c >= ND5 && !mbar_wait(&bars[B_D5FREE + d], ((c / ND5) - 1) & 1)) { fail(); break; }
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    umma_ss(d5, smem_desc(astg + ST_Y + ks * 32, 16, 1024, SW_128B),
                            smem_desc(astg + ST_V + ks * 1024, 16, 512, SW_64B), id_seed, ks > 0);
                if (!mbar_wait(&bars[B_SREADY], c & 1)) { fail(); break; }
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t kh = ks >> 2, ko = (ks & 3) * 32;
                    umma_ss(d5, smem_desc(astg + ST_X + kh * 16384 + ko, 16, 1024, SW_128B),
                            smem_desc(sbase + OFF_SB + ks * 1024, 16, 512, SW_64B), id_s1, 1);
                }
                umma_commit(&bars[B_S1]);
                if (NORM) umma_commit(&bars[B_S1X + d]);
                if (!mbar_wait(&bars[B_UREADY], c & 1)) { fail(); break; }
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    umma_ss(tmem + TM_D7, smem_desc(astg + ST_KE + ks * 2048, 8192, 1024, SW_128B),
                            smem_desc(sbase + OFF_UB + ks * 1024, 16, 512, SW_64B), id_s2, ks > 0);
                umma_commit(&bars[B_S2]);
                umma_commit(&bars[B_EMPTY + s]);      // every MMA reading stage s is complete
            }
            if (n_issued) {                           // every MMA complete before TMEM is freed
                umma_commit(&bars[B_DRAIN]);
                if (!mbar_wait(&bars[B_DRAIN], 0, 100000000LL)) set_status(p.status, KDA_ERR_TIMEOUT);
            }
        }
    } else if (warp == 4) {
        // ============================================================================ loader
        // v block of chunk c in registers: lane -> rows 2 lane, 2 lane + 1 (32 columns each)
        uint4 vr[2][4];
        auto load_v = [&](int c) {
            const int64_t tok0 = t0 + (int64_t)c * C;
            const int L = (t1 - tok0 < C) ? (int)(t1 - tok0) : C;
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) {
                const int r = 2 * lane + rr;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const long long vi = ((long long)(tok0 + r) * H + h) * DK + j0 + 8 * u;
                    vr[rr][u] = (r < L && in_bounds(p.status, vi, 8, p.tokens * H * DK)) ? ldg_nc(p.v + vi)
                                                                                        : make_uint4(0, 0, 0, 0);
                }
            }
        };
        if (nchunks > 0) load_v(0);
        auto block_of = [&](int c) {
            return p.ws + ((size_t)h * p.n_slots + (first_slot + c)) * kPrepBlockBytes;
        };
        // one CTA of the four that share a head's blocks asks for them into L2
        if (jb == 0 && lane == 0)
            for (int c = 0; c < PREFETCH_AHEAD && c < nchunks; ++c) prefetch_l2(block_of(c), (uint32_t)kPrepBlockBytes);
        int n_loaded = 0;
        for (int c = 0; c < nchunks; ++c) {
            const int s = c % NSTAGE;
            unsigned char *stg = sm + s * STAGE;
            if (jb == 0 && lane == 0 && c + PREFETCH_AHEAD < nchunks)
                prefetch_l2(block_of(c + PREFETCH_AHEAD), (uint32_t)kPrepBlockBytes);
            if (warp_abort()) break;
            int ok = 1;
            if (c >= NSTAGE && lane == 0) ok = mbar_wait(&bars[B_EMPTY + s], ((c / NSTAGE) - 1) & 1);
            if (!__shfl_sync(0xffffffffu, ok, 0)) { if (lane == 0) fail(); break; }
            if (!__shfl_sync(0xffffffffu, (int)in_bounds(p.status, (long long)h * p.n_slots + first_slot + c, 1,
                                                         (long long)H * p.n_slots), 0)) {
                if (lane == 0) *abort_flag = 1;        // KDA_ERR_BOUNDS recorded; every role stops
                break;
            }
            if (lane == 0) {
                const unsigned char *blk = block_of(c);
                mbar_arrive_expect_tx(&bars[B_FULL + s], (uint32_t)kPrepBlockBytes);
                bulk_g2s(stg, blk, (uint32_t)kPrepBlockBytes, &bars[B_FULL + s]);
            }
            n_loaded = c + 1;
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) {
                const int r = 2 * lane + rr;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    uint4 o;
                    o.x = bf16x2_to_f16x2(vr[rr][u].x); o.y = bf16x2_to_f16x2(vr[rr][u].y);
                    o.z = bf16x2_to_f16x2(vr[rr][u].z); o.w = bf16x2_to_f16x2(vr[rr][u].w);
                    *reinterpret_cast<uint4 *>(stg + ST_V + sw64_offset(r, 8 * u)) = o;
                }
            }
            if (c + 1 < nchunks) load_v(c + 1);      // lands while the loader waits for a free stage
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[B_FULL + s]);
        }
        if (lane == 0)       // no copy may still be landing when the CTA exits
            for (int c = (n_loaded > NSTAGE ? n_loaded - NSTAGE : 0); c < n_loaded; ++c)
                mbar_wait(&bars[B_FULL + c % NSTAGE], (c / NSTAGE) & 1, 100000000LL);
    } else if (warp < 4) {
        // ========================================================================= epilogues
        const int st = tid;                   // key channel / TMEM lane
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
        mbar_arrive(&bars[B_SREADY]);
        for (int c = 0; c < nchunks; ++c) {
            const int s = c % NSTAGE, d = c % ND5;
            const int64_t tok0 = t0 + (int64_t)c * C;
            const int L = (t1 - tok0 < C) ? (int)(t1 - tok0) : C;
            const uint32_t d5 = tmem + TM_D5 + 32 * d;
            if (warp_abort()) break;
            // gamma of this chunk (read from the stage after observing its arrival directly)
            if (!warp_wait(&bars[B_FULL + s], (c / NSTAGE) & 1)) { fail(); break; }
            const float g = reinterpret_cast<const float *>(sm + s * STAGE + ST_G)[st];
            if (!warp_wait(&bars[B_S1], c & 1)) { fail(); break; }
            tc_fence_after();
            float x[32];
            if (!NORM || warp < 2) tmem_ld32_sync(d5 + ((uint32_t)(32 * warp) << 16), x);
            if (warp < 2) {                   // U = -(D5 rows 0-63) -> f16, MN-major [token][32]
#pragma unroll
                for (int j = 0; j < DVB; j += 8) {
                    uint4 o;
                    o.x = pack_f16x2(-x[j], -x[j + 1]); o.y = pack_f16x2(-x[j + 2], -x[j + 3]);
                    o.z = pack_f16x2(-x[j + 4], -x[j + 5]); o.w = pack_f16x2(-x[j + 6], -x[j + 7]);
                    *reinterpret_cast<uint4 *>(sm + OFF_UB + sw64_offset(st, j)) = o;
                }
                fence_proxy_async_smem();
                tc_fence_before();
                mbar_arrive(&bars[B_UREADY]);
                mbar_arrive(&bars[B_D5FREE + d]);
            } else if (!NORM) {               // O = D5 rows 64-127, stored after the state update
                tc_fence_before();
                mbar_arrive(&bars[B_D5FREE + d]);
            }                                 // (with the output norm, warps 6-7 read the outputs)
            // S <- gamma S + Kend^T U, then hand the new state to the next chunk's S1
            if (!warp_wait(&bars[B_S2], c & 1)) { fail(); break; }
            tc_fence_after();
            float d7[32];
            tmem_ld32_sync(tmem + TM_D7 + ((uint32_t)(32 * warp) << 16), d7);
#pragma unroll
            for (int e = 0; e < 32; ++e) S[e] = g * S[e] + d7[e];
            store_state();
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&bars[B_SREADY]);
            mbar_arrive(&bars[B_EMPTY + s]);          // gamma of stage s has been read
            // outputs of this chunk (kept off the chain: global stores here overlap the next S1)
            if (!NORM && warp >= 2 && st - 64 < L &&
                in_bounds(p.status, ((long long)(tok0 + st - 64) * H + h) * DK + j0, DVB, p.tokens * H * DK)) {
                store_row32(reinterpret_cast<TO *>(p.out) + ((size_t)(tok0 + st - 64) * H + h) * DK + j0, x);
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
    if constexpr (NORM) {
        if (warp >= 6) {
            // ================================================ output path with the norm (warps 6-7)
            const int t = tid - 192;          // token row of the chunk = TMEM lane - 64
            const uint32_t lanes = (uint32_t)(32 * (warp & 3)) << 16;
            const uint32_t rank = cluster_ctarank();
            const float *red = reinterpret_cast<const float *>(sm + OFF_RED);
            float nw[32];                     // the norm weight of this CTA's 32 channels
#pragma unroll
            for (int j = 0; j < 32; ++j) nw[j] = reinterpret_cast<const float *>(sm + OFF_NW)[j];
            // finish chunk cc: gather the four partials of each token, release the slot, write the
            // normalised, gated outputs (x and the gate bits held since chunk cc was read)
            auto finish = [&](int cc, const float (&xv)[32], const uint4 (&gv)[4]) -> bool {
                const int slot = cc % RSLOTS;
                const int64_t tok = t0 + (int64_t)cc * C + t;
                if (!warp_wait(&bars[B_REDFULL + slot], (cc / RSLOTS) & 1)) return false;
                float ss = 0.f;
#pragma unroll
                for (int k = 0; k < CLUSTER; ++k) ss += red[(slot * CLUSTER + k) * 64 + t];
                // once both output warps have read the slot: re-arm it for chunk cc + RSLOTS and let
                // the senders go (a bounded wait, so that a warp that gave up cannot stall the other)
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[B_REDREAD + slot]);
                if (warp == 6 && lane == 0) {
                    if (mbar_wait(&bars[B_REDREAD + slot], (cc / RSLOTS) & 1)) {
                        mbar_arrive_expect_tx(&bars[B_REDFULL + slot], RED_TX);
#pragma unroll
                        for (uint32_t k = 0; k < CLUSTER; ++k)
                            mbar_arrive_remote_relaxed(mapa_shared(smem_u32(&bars[B_REDEMPTY + slot]), k));
                    } else {
                        fail();
                    }
                }
                const float rinv = rsqrtf(ss * (1.f / DK) + p.eps);
                float y[32];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const uint32_t gw[4] = {gv[u].x, gv[u].y, gv[u].z, gv[u].w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int j = 8 * u + 2 * e;
                        const float g0 = __uint_as_float(gw[e] << 16), g1 = __uint_as_float(gw[e] & 0xFFFF0000u);
                        y[j] = xv[j] * rinv * nw[j] * sigmoid_fast(g0);
                        y[j + 1] = xv[j + 1] * rinv * nw[j + 1] * sigmoid_fast(g1);
                    }
                }
                const long long gi = ((long long)tok * H + h) * DK + j0;
                if (tok < t1 && in_bounds(p.status, gi, DVB, p.tokens * H * DK))
                    store_row32(reinterpret_cast<TO *>(p.out) + gi, y);
                return true;
            };
            float xp[32];
            uint4 gp[4];
            bool ok = true;
            for (int c = 0; c < nchunks; ++c) {
                const int d = c % ND5, slot = c % RSLOTS;
                const int64_t tok = t0 + (int64_t)c * C + t;
                const bool live = tok < t1;
                if (warp_abort()) { ok = false; break; }
                if (!__all_sync(0xffffffffu, mbar_wait_sleepy(&bars[B_S1X + d], (c / ND5) & 1))) {
                    fail();
                    ok = false;
                    break;
                }
                tc_fence_after();
                float x[32];
                tmem_ld32_sync(tmem + TM_D5 + 32 * d + lanes, x);
                tc_fence_before();
                mbar_arrive(&bars[B_D5FREE + d]);
                const long long gi = ((long long)tok * H + h) * DK + j0;
                const bool gok = live && in_bounds(p.status, gi, DVB, p.tokens * H * DK);
                uint4 gr[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) gr[u] = gok ? ldg_nc(p.gate + gi + 8 * u) : make_uint4(0, 0, 0, 0);
                float part = 0.f;
                if (live) {
#pragma unroll
                    for (int j = 0; j < DVB; ++j) part += x[j] * x[j];
                }
                // send this chunk's partial: every CTA has read and re-armed the slot since chunk
                // c - RSLOTS
                if (c >= RSLOTS && !warp_wait(&bars[B_REDEMPTY + slot], ((c / RSLOTS) - 1) & 1)) {
                    fail();
                    ok = false;
                    break;
                }
                // lane l sends tokens 4 (l % 8) .. +3 of this warp to CTA l / 8: one 16-byte remote store
                // per lane, 32 in parallel per warp
                {
                    const int g4 = (lane & 7) * 4;
                    const float p0 = __shfl_sync(0xffffffffu, part, g4), p1 = __shfl_sync(0xffffffffu, part, g4 + 1);
                    const float p2 = __shfl_sync(0xffffffffu, part, g4 + 2), p3 = __shfl_sync(0xffffffffu, part, g4 + 3);
                    const uint32_t k = (uint32_t)(lane >> 3);
                    const uint32_t dst = smem_u32(red + (slot * CLUSTER + (int)rank) * 64 + (t - lane) + g4);
                    st_async_remote_v4(mapa_shared(dst, k), p0, p1, p2, p3,
                                       mapa_shared(smem_u32(&bars[B_REDFULL + slot]), k));
                }
                // meanwhile finish the previous chunk
                if (c >= 1 && !finish(c - 1, xp, gp)) { fail(); ok = false; break; }
#pragma unroll
                for (int j = 0; j < 32; ++j) xp[j] = x[j];
#pragma unroll
                for (int u = 0; u < 4; ++u) gp[u] = gr[u];
            }
            if (ok && nchunks > 0 && !finish(nchunks - 1, xp, gp)) fail();
        }
    }
    tc_fence_before();
    __syncthreads();
    // no CTA of the cluster may leave while another can still store into its shared memory or arrive
    // on its barriers
    if constexpr (NORM) cluster_sync_all();
    if (warp == 0) tmem_dealloc(tmem, TMEM_COLS);
}

template <typename TO, bool NORM>
cudaError_t launch_typed(const PrefillArgs &a, const unsigned char *ws, int n_slots, const NormArgs *norm,
                         cudaStream_t stream)
{
    ScanParams p;
    p.v = (const __nv_bfloat16 *)a.v; p.S0 = a.S0; p.cu_seqlens = a.cu_seqlens; p.ws = ws;
    p.out = a.out; p.S_final = a.S_final; p.T = a.T; p.H = a.H; p.N = a.N; p.n_slots = n_slots;
    p.status = a.status;
    p.tokens = (long long)a.B * a.T;
    p.gate = norm ? (const __nv_bfloat16 *)norm->gate : nullptr;
    p.norm_w = norm ? norm->weight : nullptr;
    p.eps = norm ? norm->eps : 0.f;
    auto kern = chunk_scan_kernel<TO, NORM>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_ALLOC);
    if (e != cudaSuccess) return e;
    const dim3 grid(DK / DVB, a.H, a.N);
    if constexpr (!NORM) {
        kern<<<grid, NT, SMEM_ALLOC, stream>>>(p);
    } else {                           // the four value blocks of a head form one cluster
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = grid;
        cfg.blockDim = dim3(NT_NORM);
        cfg.dynamicSmemBytes = SMEM_ALLOC;
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = CLUSTER;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, kern, p);
        if (e != cudaSuccess) return e;
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_chunk_scan(const PrefillArgs &a, const unsigned char *ws, int n_slots,
                              kda_dtype_t out_dtype, cudaStream_t stream, const NormArgs *norm)
{
    static_assert(DK / DVB == CLUSTER, "one cluster per head");
    if (norm) {
        if (out_dtype == KDA_BF16) return launch_typed<__nv_bfloat16, true>(a, ws, n_slots, norm, stream);
        return launch_typed<float, true>(a, ws, n_slots, norm, stream);
    }
    if (out_dtype == KDA_BF16) return launch_typed<__nv_bfloat16, false>(a, ws, n_slots, nullptr, stream);
    return launch_typed<float, false>(a, ws, n_slots, nullptr, stream);
}

}  // namespace kda
