// chunk_scan.cu -- second pass of the two-pass bf16 prefill, one CTA per (sequence, head): the state
// recurrence over chunks for all 128 value columns at once, in transposed form.
//
// Per chunk (operands from chunk_prep.cu), with S the state entering it and value channel j = row:
//   D5^T  = V^T Y^T                   Y = [-Tb; M Tb]      (seeds the accumulator; no S)
//   D5^T += S^T X^T                   X = [W; Qt - M W]    columns 0-63: -U^T, 64-127: O^T
//   D7^T  = U^T Kend
//   S^T  <- S^T Diag(gamma) + D7^T   (fp32, registers)
// U = Tb V - W S are the chunk's delta-rule writes and O = (Qt - M W) S + M Tb V its outputs
// (chunk-parallel form with a WY/UT representation, KimiLinear KDA/MLA tutorial (icman.com.cn),
// sec. 3 and 6.)
//
// S^T and U^T, the operands that the recurrence itself produces, stay in tensor memory as the A
// operands of their products (written by the epilogue threads with tcgen05.st), so every product
// reads only its prepared B operand from shared memory, each prepared block is copied once per
// head, and a head's chain holds one SM: with one long sequence the preparation pass of later token
// ranges runs on the other SMs (prefill.cu).
// Roles, coupled only by mbarriers:
//   warps 0-15   epilogues; warp w owns value rows j = 32 (w % 4) + lane (= tensor-memory lane) and
//                the column group b = w / 4: tokens 16 b .. + 15 of -U^T (to the f16 A operand of
//                D7) and of O^T (outputs), key columns 32 b .. + 31 of S^T (state update).
//   warp 16      loader: the block's three operand tiles by one bulk copy each into rings of two
//                slots freed by the product that last reads them (Y by the seed, X by S1, Kend|gamma
//                by D7 and the state update), so that the next chunk's seed can run behind D7; v by
//                two tensor copies per chunk (bf16, 128-byte swizzle) into a three-slot ring,
//                converted in place to f16 by the epilogue warps two chunks ahead, after their state
//                update (rows past the chunk's end zeroed): one warp converting a chunk's 16 KB
//                alone set the chunk period.
// Per chunk the epilogue warps run U (on the chain), the outputs (beside D7), the state update (on
// the chain), then the v conversion (beside the next chunk's S1). With the output norm only the sums
// of squares run beside D7; the normalised outputs follow the state update.
//   warp 17      MMA issuer (lane 0).
//   warp 18      output store (lane 0): a full chunk's bf16 outputs are staged as a [token][value]
//                tile and leave by two tensor stores; with the output norm it also brings each
//                chunk's gate tile into that tile by two tensor copies.
// Ragged chunks and fp32 outputs are stored by the epilogue threads directly (a warp's store covers
// 64 or 128 contiguous bytes of one token row).
//
// Output norm (NORM; o_norm = FusedRMSNormGated with a sigmoid gate, lpnh.cn Kimi Linear article,
// sec. 3): y = O / sqrt(mean over the 128 value channels of O^2 + eps) * w * sigmoid(g). Each warp
// sums the squares of its 16 tokens over its 32 value rows with a 16-shuffle reduce-scatter; the four
// warps of a token group then add their sums through shared memory behind a four-arrival mbarrier.
//
// Backward records (REC): instead of outputs, the scan writes what the backward pass needs of the
// forward one (chunk_bwd.cu): the fp32 state entering every chunk and the chunk's U, per (head, chunk
// slot), in the layout the CUDA-core forward writes them.
//
// Token ranges: a launch may cover only the chunks whose slots lie in [slot_lo, slot_hi). A chunk
// range that does not start a sequence starts from S_final (the state the previous range left
// there); every launch leaves its state in S_final.
#include "kda_internal.cuh"
#include "sm100.cuh"

namespace kda {
namespace {

using namespace sm100;

constexpr int C = kChunk;
constexpr int DK = kHeadDim;
constexpr int NEPI = 16;                      // epilogue warps
constexpr int W_LOAD = 16, W_MMA = 17, W_STORE = 18;
constexpr int NT = 19 * 32;

// rings (two slots each) of the block's tiles: X 32 KB, Y 16 KB, Kend (16 KB) with gamma (512 B) after it
constexpr int NR = 2;
constexpr uint32_t X_BYTES = 32768, Y_BYTES = 16384;
constexpr uint32_t KG_BYTES = (uint32_t)(kPrepBlockBytes - kPrepKEOff);   // Kend + gamma, 16896
constexpr uint32_t KG_SLOT = 17408;
constexpr uint32_t KG_G = kPrepGammaOff - kPrepKEOff;                      // gamma inside a Kend slot
constexpr uint32_t OFF_X = 0;
constexpr uint32_t OFF_Y = OFF_X + NR * X_BYTES;
constexpr uint32_t OFF_KG = OFF_Y + NR * Y_BYTES;
constexpr uint32_t OFF_V = OFF_KG + NR * KG_SLOT;   // v ring: two 64-column halves, 64 token rows x 128 B
constexpr uint32_t V_BYTES = 16384;
constexpr int NV = 3;
constexpr uint32_t OFF_OST = OFF_V + NV * V_BYTES;   // output / gate staging by chunk parity: 2 x (two
                                                     // halves, 64 rows x 128 B)
constexpr uint32_t OST_BYTES = 16384;
constexpr uint32_t OFF_RED = OFF_OST + 2 * OST_BYTES; // output norm: [parity][group b][warp q][16 tokens]
constexpr uint32_t OFF_NW = OFF_RED + 2048;   // output norm weight (128 fp32)
constexpr uint32_t OFF_BAR = OFF_NW + 512;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 512;
constexpr uint32_t SMEM_ALLOC = SMEM_BYTES + 1024;
static_assert(SMEM_ALLOC <= 232448, "shared memory plan exceeds 227 KiB");
static_assert(kPrepXOff == 0 && kPrepYOff == X_BYTES && kPrepKEOff == X_BYTES + Y_BYTES &&
              KG_BYTES <= KG_SLOT && KG_SLOT % 1024 == 0 && OFF_V % 1024 == 0 && OFF_OST % 1024 == 0,
              "ring layout");

constexpr int PREFETCH_AHEAD = 6;
constexpr uint32_t kSuspendHintNs = 1000000;             // blocks (and v tiles) asked into L2 this many chunks ahead

constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TM_D5 = 0;                 // 2 x 128: [-U^T | O^T], by chunk parity
constexpr uint32_t TM_D7 = 256;               // 128: U^T Kend
constexpr uint32_t TM_S = 384;                // 64: S^T (f16 pairs), A of S1
constexpr uint32_t TM_U = 448;                // 32: U^T (f16 pairs), A of S2

enum {
    B_XFULL = 0,     // [2] by X slot: landed (tx)                                                count 1
    B_XEMPTY = 2,    // [2] by X slot: read by S1 (commit)                                        count 1
    B_YFULL = 4,     // [2] by Y slot: landed (tx)                                                count 1
    B_YEMPTY = 6,    // [2] by Y slot: read by the seed (commit)                                  count 1
    B_KFULL = 8,     // [2] by Kend slot: landed (tx)                                             count 1
    B_KEMPTY = 10,   // [2] by Kend slot: read by D7 (commit) and gamma by 16 epilogue warps      count 17
    B_VLAND = 12,    // [3] by v slot: v tiles landed (tx)                                        count 1
    B_VCONV = 15,    // [3] by v slot: converted to f16 (16 epilogue warps)                       count 16
    B_VEMPTY = 18,   // [3] by v slot: read by the seed product (commit)                          count 1
    B_D5FREE = 21,   // [2] by D5 buffer: read by the 16 epilogue warps                           count 16
    B_SREADY = 23,   // S^T of the next chunk in tensor memory (16 warps)                         count 16
    B_UREADY = 24,   // U^T in tensor memory (16 warps)                                           count 16
    B_S1 = 25, B_S2 = 26, B_DRAIN = 27,   // MMA completions                                      count 1
    B_OST = 28,      // [2] by staging tile: outputs staged / stored (16 warps)                   count 16
    B_OFREE = 30,    // [2] by staging tile: free again (store warp)                              count 1
    B_GATE = 32,     // [2] by staging tile, output norm: gate tile landed (tx)                   count 1
    B_RED = 34,      // [2][4] output norm, by (chunk parity, token group b): 4 warps' sums       count 4
    N_BARS = 42
};
static_assert(N_BARS * 8 + 8 <= 512, "barrier area");

struct WideParams {
    const float *S0;
    const int32_t *cu_seqlens;
    const unsigned char *ws;
    void *out;
    float *S_final;
    int T, H, N, n_slots;
    long long tokens;
    long long slot_lo, slot_hi;     // chunk-slot range of this launch
    int32_t *status;
    const float *norm_w;
    float eps;
    float *ck_S, *ck_U;             // backward records (REC)
};

__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void prefetch_l2(const void *p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}
__device__ __forceinline__ float sigmoid_fast(float x) {   // 1/2 + tanh(x/2)/2, hardware tanh
    float t;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * x));
    return fmaf(0.5f, t, 0.5f);
}
// byte offset of element (token t, value column j) of a [64 tokens][128 values] 16-bit tile stored as
// two 64-column halves 8 KB apart, 128-byte rows, 128-byte swizzle (the tensor-copy box layout)
__device__ __forceinline__ uint32_t tile_off(int t, int j) {
    return (uint32_t)(j >> 6) * 8192u + (uint32_t)t * 128u +
           ((uint32_t)((((j & 63) >> 3) ^ (t & 7)) & 7) << 4) + (uint32_t)(j & 7) * 2u;
}

template <typename TO, bool NORM, bool REC>
__global__ void __launch_bounds__(NT, 1)
chunk_scan_kernel(WideParams p, const __grid_constant__ CUtensorMap tm_v,
                       const __grid_constant__ CUtensorMap tm_out, const __grid_constant__ CUtensorMap tm_gate)
{
    constexpr bool STAGED = sizeof(TO) == 2 && !REC;   // bf16 outputs of full chunks leave by tensor stores
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int h = blockIdx.x, n = blockIdx.y, H = p.H;

    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + OFF_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + N_BARS);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(bars + N_BARS) + 1;

    int64_t t0, t1;
    if (!sequence_span(p.cu_seqlens, n, p.N, p.T, &t0, &t1, p.status)) return;   // uniform
    const int nchunks = (int)((t1 - t0 + C - 1) / C);
    const long long first_slot = t0 / C + n;
    // chunks of this launch: slots in [slot_lo, slot_hi); an empty sequence belongs to the launch
    // that holds its first slot
    long long cb = p.slot_lo - first_slot, ce = p.slot_hi - first_slot;
    cb = cb < 0 ? 0 : cb;
    ce = ce > nchunks ? nchunks : ce;
    if (nchunks == 0 ? (first_slot < p.slot_lo || first_slot >= p.slot_hi) : cb >= ce) return;   // uniform
    const int c_begin = (int)cb, nk = nchunks == 0 ? 0 : (int)(ce - cb);
    const float *S_in = c_begin == 0 ? p.S0 : p.S_final;

    if (warp == 0) { tmem_alloc(tmem_slot, TMEM_COLS); tmem_relinquish(); }
    if (tid == 0) {
        for (int i = 0; i < NR; ++i) {
            mbar_init(&bars[B_XFULL + i], 1);
            mbar_init(&bars[B_XEMPTY + i], 1);
            mbar_init(&bars[B_YFULL + i], 1);
            mbar_init(&bars[B_YEMPTY + i], 1);
            mbar_init(&bars[B_KFULL + i], 1);
            mbar_init(&bars[B_KEMPTY + i], NEPI + 1);
            mbar_init(&bars[B_D5FREE + i], NEPI);
        }
        for (int i = 0; i < NV; ++i) {
            mbar_init(&bars[B_VLAND + i], 1);
            mbar_init(&bars[B_VCONV + i], NEPI);
            mbar_init(&bars[B_VEMPTY + i], 1);
        }
        mbar_init(&bars[B_SREADY], NEPI);
        mbar_init(&bars[B_UREADY], NEPI);
        mbar_init(&bars[B_S1], 1);
        mbar_init(&bars[B_S2], 1);
        mbar_init(&bars[B_DRAIN], 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bars[B_OST + i], NEPI);
            mbar_init(&bars[B_OFREE + i], 1);
            mbar_init(&bars[B_GATE + i], 1);
        }
        for (int i = 0; i < 8; ++i) mbar_init(&bars[B_RED + i], 4);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (NORM && tid < DK)
        reinterpret_cast<float *>(sm + OFF_NW)[tid] = in_bounds(p.status, tid, 1, DK) ? p.norm_w[tid] : 0.f;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    auto fail = [&]() { set_status(p.status, KDA_ERR_TIMEOUT); *abort_flag = 1; };
    // a wait whose outcome is the same for the whole (converged) warp, so that warp-collective
    // tcgen05.ld / st never run with some lanes gone
    // Waiting warps suspend in the barrier instruction (a long suspend-time hint; the phase completing
    // wakes them): sixteen epilogue warps polling would take the issue slots of the loader and the
    // MMA issuer, which share their schedulers.
    auto warp_wait = [&](uint64_t *bar, uint32_t parity) {
        return __all_sync(0xffffffffu, mbar_wait_sleepy(bar, parity, kSuspendHintNs)) != 0;
    };
    auto warp_abort = [&]() { return __any_sync(0xffffffffu, *abort_flag != 0) != 0; };
    auto chunk_tok0 = [&](int k) { return t0 + (int64_t)(c_begin + k) * C; };
    auto chunk_len = [&](int k) {
        const int64_t a = chunk_tok0(k);
        return (t1 - a < C) ? (int)(t1 - a) : C;
    };

    if (warp == W_MMA) {
        // ======================================================================== MMA issuer
        if (lane == 0) {
            uint32_t n_issued = 0;
            const uint32_t id_seed = idesc_f16(128, 128, 1, 0);   // A = V^T (MN-major), B = Y (K-major)
            const uint32_t id_s1 = idesc_f16(128, 128, 0, 0);     // A = S^T (tensor memory), B = X
            const uint32_t id_s2 = idesc_f16(128, 128, 0, 1);     // A = U^T (tensor memory), B = Kend (MN)
            for (int k = 0; k < nk && !*abort_flag; ++k) {
                const int r = k % NR, d = k & 1, vs = k % NV;
                const uint32_t rph = (k / NR) & 1;
                const uint32_t d5 = tmem + TM_D5 + 128 * d;
                const uint32_t vslot = sbase + OFF_V + vs * V_BYTES;
                const uint32_t yslot = sbase + OFF_Y + r * Y_BYTES, xslot = sbase + OFF_X + r * X_BYTES;
                const uint32_t kslot = sbase + OFF_KG + r * KG_SLOT;
                if (!mbar_wait(&bars[B_YFULL + r], rph)) { fail(); break; }
                ++n_issued;
                if (!mbar_wait(&bars[B_VCONV + vs], (k / NV) & 1)) { fail(); break; }
                if (k >= 2 && !mbar_wait(&bars[B_D5FREE + d], ((k >> 1) - 1) & 1)) { fail(); break; }
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    umma_ss(d5, smem_desc(vslot + ks * 2048, 8192, 1024, SW_128B),
                            smem_desc(yslot + ks * 32, 16, 1024, SW_128B), id_seed, ks > 0);
                umma_commit(&bars[B_VEMPTY + vs]);
                umma_commit(&bars[B_YEMPTY + r]);
                if (!mbar_wait(&bars[B_SREADY], k & 1)) { fail(); break; }
                if (!mbar_wait(&bars[B_XFULL + r], rph)) { fail(); break; }
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    umma_ts(d5, tmem + TM_S + 8 * ks,
                            smem_desc(xslot + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024, SW_128B), id_s1, 1);
                umma_commit(&bars[B_S1]);
                umma_commit(&bars[B_XEMPTY + r]);
                if (!mbar_wait(&bars[B_UREADY], k & 1)) { fail(); break; }
                if (!mbar_wait(&bars[B_KFULL + r], rph)) { fail(); break; }
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    umma_ts(tmem + TM_D7, tmem + TM_U + 8 * ks,
                            smem_desc(kslot + ks * 2048, 8192, 1024, SW_128B), id_s2, ks > 0);
                umma_commit(&bars[B_S2]);
                umma_commit(&bars[B_KEMPTY + r]);
            }
            if (n_issued) {
                umma_commit(&bars[B_DRAIN]);
                if (!mbar_wait(&bars[B_DRAIN], 0, 100000000LL)) set_status(p.status, KDA_ERR_TIMEOUT);
            }
        }
    } else if (warp == W_LOAD) {
        // ============================================================================ loader
        auto block_of = [&](int k) {
            return p.ws + ((size_t)h * p.n_slots + (size_t)(first_slot + c_begin + k)) * kPrepBlockBytes;
        };
        if (lane == 0) {
            tma_prefetch_desc(&tm_v);
            for (int k = 0; k < PREFETCH_AHEAD && k < nk; ++k) {
                prefetch_l2(block_of(k), (uint32_t)kPrepBlockBytes);
                tma_prefetch_3d(&tm_v, 0, h, (int)chunk_tok0(k));
                tma_prefetch_3d(&tm_v, 64, h, (int)chunk_tok0(k));
            }
        }
        int v_issued = 0, y_issued = 0, x_issued = 0, k_issued = 0;   // copies issued (lane 0)
        for (int k = 0; k < nk; ++k) {
            const int r = k % NR, vs = k % NV;
            const uint32_t eph = ((k / NR) - 1) & 1;     // phase of the slot's previous use
            if (warp_abort()) break;
            if (!__shfl_sync(0xffffffffu, (int)in_bounds(p.status, (long long)h * p.n_slots + first_slot + c_begin + k,
                                                         1, (long long)H * p.n_slots), 0)) {
                if (lane == 0) *abort_flag = 1;
                break;
            }
            int ok = 1;
            if (lane == 0) {
                const int64_t tok0 = chunk_tok0(k);
                if (k + PREFETCH_AHEAD < nk) {
                    prefetch_l2(block_of(k + PREFETCH_AHEAD), (uint32_t)kPrepBlockBytes);
                    tma_prefetch_3d(&tm_v, 0, h, (int)chunk_tok0(k + PREFETCH_AHEAD));
                    tma_prefetch_3d(&tm_v, 64, h, (int)chunk_tok0(k + PREFETCH_AHEAD));
                }
                // v of chunk k (its slot was last read by the seed of chunk k - 3)
                if (k >= NV) ok = mbar_wait_sleepy(&bars[B_VEMPTY + vs], ((k / NV) - 1) & 1, kSuspendHintNs);
                if (ok) {
                    unsigned char *vdst = sm + OFF_V + vs * V_BYTES;
                    mbar_arrive_expect_tx(&bars[B_VLAND + vs], V_BYTES);
                    tma_load_3d(vdst, &tm_v, &bars[B_VLAND + vs], 0, h, (int)tok0);
                    tma_load_3d(vdst + 8192, &tm_v, &bars[B_VLAND + vs], 64, h, (int)tok0);
                    v_issued = k + 1;
                }
                // the block's tiles of chunk k, each into the slot its product of chunk k - 2 released
                const unsigned char *blk = block_of(k);
                if (ok && k >= NR) ok = mbar_wait_sleepy(&bars[B_YEMPTY + r], eph, kSuspendHintNs);
                if (ok) {
                    mbar_arrive_expect_tx(&bars[B_YFULL + r], Y_BYTES);
                    bulk_g2s(sm + OFF_Y + r * Y_BYTES, blk + kPrepYOff, Y_BYTES, &bars[B_YFULL + r]);
                    y_issued = k + 1;
                }
                if (ok && k >= NR) ok = mbar_wait_sleepy(&bars[B_XEMPTY + r], eph, kSuspendHintNs);
                if (ok) {
                    mbar_arrive_expect_tx(&bars[B_XFULL + r], X_BYTES);
                    bulk_g2s(sm + OFF_X + r * X_BYTES, blk + kPrepXOff, X_BYTES, &bars[B_XFULL + r]);
                    x_issued = k + 1;
                }
                if (ok && k >= NR) ok = mbar_wait_sleepy(&bars[B_KEMPTY + r], eph, kSuspendHintNs);
                if (ok) {
                    mbar_arrive_expect_tx(&bars[B_KFULL + r], KG_BYTES);
                    bulk_g2s(sm + OFF_KG + r * KG_SLOT, blk + kPrepKEOff, KG_BYTES, &bars[B_KFULL + r]);
                    k_issued = k + 1;
                }
            }
            if (!__shfl_sync(0xffffffffu, ok, 0)) { if (lane == 0) fail(); break; }
        }
        if (lane == 0) {     // no copy may still be landing when the CTA exits
            for (int k = (v_issued > NV ? v_issued - NV : 0); k < v_issued; ++k)
                mbar_wait(&bars[B_VLAND + k % NV], (k / NV) & 1, 100000000LL);
            for (int k = (y_issued > NR ? y_issued - NR : 0); k < y_issued; ++k)
                mbar_wait(&bars[B_YFULL + k % NR], (k / NR) & 1, 100000000LL);
            for (int k = (x_issued > NR ? x_issued - NR : 0); k < x_issued; ++k)
                mbar_wait(&bars[B_XFULL + k % NR], (k / NR) & 1, 100000000LL);
            for (int k = (k_issued > NR ? k_issued - NR : 0); k < k_issued; ++k)
                mbar_wait(&bars[B_KFULL + k % NR], (k / NR) & 1, 100000000LL);
        }
    } else if (warp == W_STORE) {
        // ======================================================================= output store
        if (lane == 0 && (STAGED || NORM)) {
            if (NORM) tma_prefetch_desc(&tm_gate);
            if (STAGED) tma_prefetch_desc(&tm_out);
            // the gate tile of chunk k goes to staging tile k % 2, two chunks ahead of its use
            int gates_issued = 0;
            auto load_gate = [&](int k) {
                unsigned char *dst = sm + OFF_OST + (k & 1) * OST_BYTES;
                mbar_arrive_expect_tx(&bars[B_GATE + (k & 1)], 16384u);
                tma_load_3d(dst, &tm_gate, &bars[B_GATE + (k & 1)], 0, h, (int)chunk_tok0(k));
                tma_load_3d(dst + 8192, &tm_gate, &bars[B_GATE + (k & 1)], 64, h, (int)chunk_tok0(k));
                gates_issued = k + 1;
            };
            if (NORM)
                for (int k = 0; k < 2 && k < nk; ++k) load_gate(k);
            for (int k = 0; k < nk; ++k) {
                const int ob = k & 1;
                if (*abort_flag) break;
                if (!mbar_wait_sleepy(&bars[B_OST + ob], (k >> 1) & 1, kSuspendHintNs)) { fail(); break; }
                if (STAGED && chunk_len(k) == C) {
                    const int64_t tok0 = chunk_tok0(k);
                    tma_store_3d(&tm_out, sm + OFF_OST + ob * OST_BYTES, 0, h, (int)tok0);
                    tma_store_3d(&tm_out, sm + OFF_OST + ob * OST_BYTES + 8192, 64, h, (int)tok0);
                    bulk_commit_group();
                    bulk_wait_group_read0();
                }
                if (NORM && k + 2 < nk) load_gate(k + 2);
                mbar_arrive(&bars[B_OFREE + ob]);
            }
            bulk_wait_group_read0();
            // gate copies still landing must not outlive the CTA
            for (int k = (gates_issued > 2 ? gates_issued - 2 : 0); k < gates_issued; ++k)
                mbar_wait(&bars[B_GATE + (k & 1)], (k >> 1) & 1, 100000000LL);
        }
    } else {
        // ========================================================================= epilogues
        const int q = warp & 3, b = warp >> 2;
        const int j = 32 * q + lane;          // value channel = tensor-memory lane
        const uint32_t lanes = (uint32_t)(32 * q) << 16;
        const int kc0 = 32 * b;               // key columns of S^T
        const int tk0 = 16 * b;               // tokens of -U^T and O^T
        const bool odd = (lane & 1) != 0;
        float S[32];                          // S^T[j][kc0 + i] = S[kc0 + i][j]
        {
            const size_t sidx = (((size_t)n * H + h) * DK + kc0) * DK + j;
#pragma unroll
            for (int i = 0; i < 32; ++i)
                S[i] = (S_in && in_bounds(p.status, (long long)(sidx + (size_t)i * DK), 1, (long long)p.N * H * DK * DK))
                           ? S_in[sidx + (size_t)i * DK] : 0.f;
        }
        auto store_state = [&]() {            // S^T columns kc0.. -> f16 pairs, tensor memory
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) pk[i] = pack_f16x2(S[2 * i], S[2 * i + 1]);
            tmem_st16u(tmem + lanes + TM_S + 16 * b, pk);
            tmem_st_wait();
        };
        // v of chunk kk: this warp's 64 of the slot's 1024 16-byte units, bf16 -> f16 in place; rows
        // past the chunk's end (the next sequence, or the fill past the tensor's end) become zero
        auto convert_v = [&](int kk) -> bool {
            const int vs = kk % NV;
            if (!warp_wait(&bars[B_VLAND + vs], (kk / NV) & 1)) return false;
            const int L = chunk_len(kk);
            uint4 *vu = reinterpret_cast<uint4 *>(sm + OFF_V + vs * V_BYTES);
            uint4 x[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) x[u] = vu[warp * 64 + u * 32 + lane];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int row = ((warp * 64 + u * 32 + lane) >> 3) & 63;   // unit: half, row, chunk
                uint4 y = make_uint4(0u, 0u, 0u, 0u);
                if (row < L) {
                    y.x = bf16x2_to_f16x2(x[u].x); y.y = bf16x2_to_f16x2(x[u].y);
                    y.z = bf16x2_to_f16x2(x[u].z); y.w = bf16x2_to_f16x2(x[u].w);
                }
                vu[warp * 64 + u * 32 + lane] = y;
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[B_VCONV + vs]);
            return true;
        };
        // one warp's outputs of a chunk: 16 tokens x 32 value columns, to the staging tile (bf16, full
        // chunk) or straight to global memory
        auto emit = [&](const float (&o)[16], unsigned char *ost, int64_t tok0, int L) {
            if (STAGED && L == C) {
                // pairs of neighbouring value columns: the even lane keeps tokens tk0 + i, the odd
                // lane tokens tk0 + 8 + (i + 4) % 8 (rows four apart mod 8, so the two row pieces
                // of one store land in different banks)
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int ie = i, io = 8 + ((i + 4) & 7);
                    const float send = odd ? o[ie] : o[io];
                    const float got = __shfl_xor_sync(0xffffffffu, send, 1);
                    const int t = tk0 + (odd ? io : ie);
                    const uint32_t v2 = odd ? pack_bf16x2(got, o[io]) : pack_bf16x2(o[ie], got);
                    *reinterpret_cast<uint32_t *>(ost + tile_off(t, j & ~1)) = v2;
                }
                fence_proxy_async_smem();
            } else if constexpr (sizeof(TO) == 4) {
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const long long oi = ((long long)(tok0 + tk0 + i) * H + h) * DK + j;
                    if (tk0 + i < L && in_bounds(p.status, oi, 1, p.tokens * H * DK))
                        reinterpret_cast<float *>(p.out)[oi] = o[i];
                }
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int ie = i, io = 8 + i;
                    const float send = odd ? o[ie] : o[io];
                    const float got = __shfl_xor_sync(0xffffffffu, send, 1);
                    const int t = tk0 + (odd ? io : ie);
                    const uint32_t v2 = odd ? pack_bf16x2(got, o[io]) : pack_bf16x2(o[ie], got);
                    const long long oi = ((long long)(tok0 + t) * H + h) * DK + (j & ~1);
                    if (t < L && in_bounds(p.status, oi, 2, p.tokens * H * DK))
                        *reinterpret_cast<uint32_t *>(reinterpret_cast<uint16_t *>(p.out) + oi) = v2;
                }
            }
        };
        store_state();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[B_SREADY]);
        // v is converted two chunks ahead of its seed product (after the state update of the chunk
        // before, while the tensor cores run the next chunk's S1)
        for (int kk = 0; kk < 2 && kk < nk; ++kk)
            if (!convert_v(kk)) { fail(); break; }
        const float wj = NORM ? reinterpret_cast<const float *>(sm + OFF_NW)[j] : 1.f;
        for (int k = 0; k < nk; ++k) {
            const int r = k % NR, d = k & 1;
            const int64_t tok0 = chunk_tok0(k);
            const int L = chunk_len(k);
            const uint32_t d5 = tmem + lanes + TM_D5 + 128 * d;
            unsigned char *ost = sm + OFF_OST + d * OST_BYTES;   // staging tile of this chunk
            if (warp_abort()) break;
            const size_t rec = (size_t)h * p.n_slots + (size_t)(first_slot + c_begin + k);
            if constexpr (REC) {              // the state entering this chunk, [key channel][value]
                float *dst = p.ck_S + rec * (size_t)(DK * DK) + (size_t)kc0 * DK + j;
#pragma unroll
                for (int i = 0; i < 32; ++i) dst[(size_t)i * DK] = S[i];
            }
            if (!warp_wait(&bars[B_S1], k & 1)) { fail(); break; }
            tc_fence_after();
            {   // U^T = -(D5^T columns tk0..) -> f16 pairs, the A operand of D7
                float x[16];
                uint32_t pk[8];
                tmem_ld16_sync(d5 + tk0, x);
#pragma unroll
                for (int i = 0; i < 8; ++i) pk[i] = pack_f16x2(-x[2 * i], -x[2 * i + 1]);
                if constexpr (REC) {          // U of this chunk, [token][value]; rows past its end are 0
                    float *dst = p.ck_U + rec * (size_t)(C * DK) + (size_t)tk0 * DK + j;
#pragma unroll
                    for (int i = 0; i < 16; ++i) dst[(size_t)i * DK] = -x[i];
                }
                tmem_st8u(tmem + lanes + TM_U + 8 * b, pk);
                tmem_st_wait();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[B_UREADY]);
            // outputs O^T[j][tk0 + i] = O[tk0 + i][j]
            if constexpr (REC) {              // records only: no outputs
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[B_D5FREE + d]);
            } else if constexpr (!NORM) {
                float o[16];
                tmem_ld16_sync(d5 + 64 + tk0, o);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[B_D5FREE + d]);
                if (STAGED && k >= 2 && !warp_wait(&bars[B_OFREE + d], ((k >> 1) - 1) & 1)) { fail(); break; }
                emit(o, ost, tok0, L);
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[B_OST + d]);
            } else {
                // the norm's sum of squares now (while D7 runs); the rest after the state update
                float o[16];
                tmem_ld16_sync(d5 + 64 + tk0, o);
                // sum over the 32 value rows of this warp, 16 tokens: reduce-scatter by lane bits
                // 4, 3, 2, 1, then lane bit 0; lane 2 i ends with token i
                float r[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) r[i] = o[i] * o[i];
#pragma unroll
                for (int i = 0; i < 8; ++i) {         // keep tokens 8 bit4 + i
                    const bool hi = (lane & 16) != 0;
                    const float send = hi ? r[i] : r[i + 8];
                    const float keep = hi ? r[i + 8] : r[i];
                    r[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
                }
#pragma unroll
                for (int i = 0; i < 4; ++i) {         // keep 8 bit4 + 4 bit3 + i
                    const bool hi = (lane & 8) != 0;
                    const float send = hi ? r[i] : r[i + 4];
                    const float keep = hi ? r[i + 4] : r[i];
                    r[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
                }
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const bool hi = (lane & 4) != 0;
                    const float send = hi ? r[i] : r[i + 2];
                    const float keep = hi ? r[i + 2] : r[i];
                    r[i] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
                }
                {
                    const bool hi = (lane & 2) != 0;
                    const float send = hi ? r[0] : r[1];
                    const float keep = hi ? r[1] : r[0];
                    r[0] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
                }
                r[0] += __shfl_xor_sync(0xffffffffu, r[0], 1);
                // the four warps of this token group (q = 0..3) add their sums after the state update
                float *red = reinterpret_cast<float *>(sm + OFF_RED) + (d * 4 + b) * 64;
                if (!odd) red[q * 16 + (lane >> 1)] = r[0];
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[B_RED + d * 4 + b]);
            }
            // S^T <- S^T Diag(gamma) + D7^T, then hand the new state to the next chunk's S1
            if (!warp_wait(&bars[B_KFULL + r], (k / NR) & 1)) { fail(); break; }
            if (!warp_wait(&bars[B_S2], k & 1)) { fail(); break; }
            tc_fence_after();
            {
                float x[32];
                tmem_ld32_sync(tmem + lanes + TM_D7 + kc0, x);
                const float4 *g4 = reinterpret_cast<const float4 *>(sm + OFF_KG + r * KG_SLOT + KG_G) + (kc0 >> 2);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float4 gv = g4[i];
                    S[4 * i] = gv.x * S[4 * i] + x[4 * i];
                    S[4 * i + 1] = gv.y * S[4 * i + 1] + x[4 * i + 1];
                    S[4 * i + 2] = gv.z * S[4 * i + 2] + x[4 * i + 2];
                    S[4 * i + 3] = gv.w * S[4 * i + 3] + x[4 * i + 3];
                }
            }
            store_state();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) { mbar_arrive(&bars[B_SREADY]); mbar_arrive(&bars[B_KEMPTY + r]); }
            if constexpr (NORM) {
                // normalised, gated outputs of chunk k (its D5 half stays untouched until the seed of
                // chunk k + 2, which waits for the arrival below)
                const float *red = reinterpret_cast<const float *>(sm + OFF_RED) + (d * 4 + b) * 64;
                bool good = warp_wait(&bars[B_RED + d * 4 + b], (k >> 1) & 1);
                const int ti = lane >> 1;
                const float ss = red[ti] + red[16 + ti] + red[32 + ti] + red[48 + ti];
                const float rinv_mine = rsqrtf(ss * (1.f / DK) + p.eps);
                good = good && warp_wait(&bars[B_GATE + d], (k >> 1) & 1);
                if (!good) { fail(); break; }
                float o[16];
                tmem_ld16_sync(d5 + 64 + tk0, o);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[B_D5FREE + d]);
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float ri = __shfl_sync(0xffffffffu, rinv_mine, 2 * i);
                    const float gv = __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(ost + tile_off(tk0 + i, j)));
                    o[i] = o[i] * ri * wj * sigmoid_fast(gv);
                }
                __syncwarp();                         // every gate value read before the tile is rewritten
                emit(o, ost, tok0, L);
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[B_OST + d]);
            }
            // v of chunk k + 2 while the tensor cores run S1 of chunk k + 1
            if (k + 2 < nk && !convert_v(k + 2)) { fail(); break; }
        }
        if (p.S_final && !*abort_flag) {
            const size_t sidx = (((size_t)n * H + h) * DK + kc0) * DK + j;
#pragma unroll
            for (int i = 0; i < 32; ++i)
                if (in_bounds(p.status, (long long)(sidx + (size_t)i * DK), 1, (long long)p.N * H * DK * DK))
                    p.S_final[sidx + (size_t)i * DK] = S[i];
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, TMEM_COLS);
}

template <typename TO, bool NORM, bool REC = false>
cudaError_t launch_typed(const PrefillArgs &a, const unsigned char *ws, int n_slots, const NormArgs *norm,
                         long long slot_lo, long long slot_hi, cudaStream_t stream)
{
    WideParams p;
    p.S0 = a.S0; p.cu_seqlens = a.cu_seqlens; p.ws = ws;
    p.out = a.out; p.S_final = a.S_final; p.T = a.T; p.H = a.H; p.N = a.N; p.n_slots = n_slots;
    p.status = a.status;
    p.tokens = (long long)a.B * a.T;
    p.slot_lo = slot_lo; p.slot_hi = slot_hi;
    p.norm_w = norm ? norm->weight : nullptr;
    p.eps = norm ? norm->eps : 0.f;
    p.ck_S = a.ck_S; p.ck_U = a.ck_U;
    if (a.N == 0) return cudaSuccess;
    // with no token at all no CTA touches a tensor map (every sequence is empty); the maps stay zero
    CUtensorMap tv = {}, to = {}, tg = {};
    if (p.tokens > 0) {
        if (!token_rows_map(&tv, a.v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.H, p.tokens, 64, true))
            return cudaErrorNotSupported;
        if (sizeof(TO) == 2 && !REC &&
            !token_rows_map(&to, a.out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.H, p.tokens, 64, true))
            return cudaErrorNotSupported;
        if (NORM && !token_rows_map(&tg, norm->gate, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.H, p.tokens, 64, true))
            return cudaErrorNotSupported;
    }
    auto kern = chunk_scan_kernel<TO, NORM, REC>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_ALLOC);
    if (e != cudaSuccess) return e;
    kern<<<dim3(a.H, a.N), NT, SMEM_ALLOC, stream>>>(p, tv, to, tg);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_chunk_scan(const PrefillArgs &a, const unsigned char *ws, int n_slots,
                              kda_dtype_t out_dtype, cudaStream_t stream, const NormArgs *norm,
                              long long slot_lo, long long slot_hi)
{
    if (slot_hi < 0) slot_hi = n_slots;
    if (norm) {
        if (out_dtype == KDA_BF16)
            return launch_typed<__nv_bfloat16, true>(a, ws, n_slots, norm, slot_lo, slot_hi, stream);
        return launch_typed<float, true>(a, ws, n_slots, norm, slot_lo, slot_hi, stream);
    }
    if (out_dtype == KDA_BF16)
        return launch_typed<__nv_bfloat16, false>(a, ws, n_slots, nullptr, slot_lo, slot_hi, stream);
    return launch_typed<float, false>(a, ws, n_slots, nullptr, slot_lo, slot_hi, stream);
}

cudaError_t launch_chunk_scan_records(const PrefillArgs &a, const unsigned char *ws, int n_slots,
                                      cudaStream_t stream, long long slot_lo, long long slot_hi)
{
    if (!a.ck_S || !a.ck_U) return cudaErrorInvalidValue;
    if (slot_hi < 0) slot_hi = n_slots;
    return launch_typed<float, false, true>(a, ws, n_slots, nullptr, slot_lo, slot_hi, stream);
}

}  // namespace kda
