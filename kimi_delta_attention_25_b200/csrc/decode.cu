// decode.cu -- one KDA decode step for N sequences x H heads, state updated in place.
//
// Per (sequence, head), with S the 128 x 128 fp32 state (key channel i = row, value j = column):
//   S'  = Diag(alpha) S                 alpha = exp(log_alpha), one decay per key channel
//   w   = S'^T k ,  p = S'^T q
//   u   = beta (v - w)
//   S   = S' + k u^T                    == (I - beta k k^T) S' + beta k v^T
//   o   = S^T q = p + (q . k) u
// i.e. the recurrent mode of the layer (lpnh.cn Kimi Linear KDA/NoPE article, sec. 2/5), whose
// cost per step is one read and one write of the fixed-size state (KimiLinear KDA/MLA tutorial
// (icman.com.cn), sec. 1-2: the state does not grow with the context).
//
// The step is bound by HBM: 64 KiB of state read and written per head against ~4 flop per
// element. One CTA of 256 threads owns one head: warp w holds rows 16w..16w+15 and lane l the
// four columns 4l..4l+3 as float4 registers, so each warp-wide load or store moves one 512-byte
// state row (fully coalesced, 128-bit per thread). The reductions over rows for w and p are done
// in registers, then across the 8 warps through shared memory. The state is touched exactly once
// in each direction, with streaming (evict-first) cache hints since it is far larger than L2.
//
// With the layer options (GATE, NORM; the gate producers and the output norm of the KDA module,
// lpnh.cn Kimi Linear article, sec. 3): alpha = exp(-exp(A_log[h]) softplus(f + dt_bias)) and
// beta = sigmoid(b) are formed from their inputs as they are loaded, and the output becomes
// o / sqrt(mean(o^2) + eps) * w * sigmoid(g), its sum of squares reduced across the four warps that
// hold o at the barrier the state update already waits on.
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int kDecThreads = 256;
constexpr int kRowsPerWarp = kHeadDim / (kDecThreads / 32);   // 16

// Layer options of the decode step (pointers NULL when unused; f, b, g in the inputs' dtype).
template <typename T>
struct DecodeLayer {
    const T *f;                 // decay gate input [N, H, dk]
    const float *A_log;         // [H]
    const float *dt_bias;       // [H * dk]
    const T *b;                 // write gate logits [N, H]
    const T *g;                 // output gate [N, H, dv]
    const float *w;             // norm weight [dv]
    float eps;
    int H;
};

__device__ __forceinline__ float softplus_d(float x) { return x > 20.f ? x : log1pf(__expf(x)); }
__device__ __forceinline__ float sigmoid_d(float x) { return 1.f / (1.f + __expf(-x)); }

template <typename T, typename TO, bool GATE, bool NORM>
__global__ void __launch_bounds__(kDecThreads, 2)
decode_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
              const float *__restrict__ log_alpha, const float *__restrict__ beta,
              float *__restrict__ S, TO *__restrict__ out, DecodeLayer<T> lay)
{
    const int nh = blockIdx.x;                      // flat (sequence, head)
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    __shared__ float s_a[kHeadDim], s_k[kHeadDim], s_q[kHeadDim];
    __shared__ __align__(16) float s_u[kHeadDim];
    __shared__ __align__(16) float s_red[2][kDecThreads / 32][kHeadDim];
    __shared__ float s_qk;
    __shared__ float s_ss[kHeadDim / 32];

    float *Sh = S + (size_t)nh * kHeadDim * kHeadDim;
    const int row0 = warp * kRowsPerWarp;

    // The state loads go out first: they are the long pole.
    float4 st[kRowsPerWarp];
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r)
        st[r] = __ldcs(reinterpret_cast<const float4 *>(Sh + (size_t)(row0 + r) * kHeadDim) + lane);

    const size_t vec = (size_t)nh * kHeadDim;
    if (tid < kHeadDim) {
        if constexpr (GATE) {
            const int h = nh % lay.H;
            s_a[tid] = expf(-expf(lay.A_log[h]) * softplus_d(to_f32(lay.f[vec + tid]) + lay.dt_bias[(size_t)h * kHeadDim + tid]));
        } else {
            s_a[tid] = expf(log_alpha[vec + tid]);
        }
        s_k[tid] = to_f32(k[vec + tid]);
        s_q[tid] = to_f32(q[vec + tid]);
    }
    __syncthreads();
    if (warp == 0) {
        float d = 0.f;
#pragma unroll
        for (int i = lane; i < kHeadDim; i += 32) d += s_q[i] * s_k[i];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
        if (lane == 0) s_qk = d;
    }

    float4 wk = make_float4(0.f, 0.f, 0.f, 0.f), wq = wk;
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r) {
        const int i = row0 + r;
        const float a = s_a[i], ki = s_k[i], qi = s_q[i];
        st[r].x *= a; st[r].y *= a; st[r].z *= a; st[r].w *= a;        // S' = Diag(alpha) S
        wk.x += ki * st[r].x; wk.y += ki * st[r].y; wk.z += ki * st[r].z; wk.w += ki * st[r].w;
        wq.x += qi * st[r].x; wq.y += qi * st[r].y; wq.z += qi * st[r].z; wq.w += qi * st[r].w;
    }
    reinterpret_cast<float4 *>(s_red[0][warp])[lane] = wk;
    reinterpret_cast<float4 *>(s_red[1][warp])[lane] = wq;
    __syncthreads();

    float o = 0.f;
    if (tid < kHeadDim) {
        float w = 0.f, p = 0.f;
#pragma unroll
        for (int x = 0; x < kDecThreads / 32; ++x) { w += s_red[0][x][tid]; p += s_red[1][x][tid]; }
        const float bt = lay.b ? sigmoid_d(to_f32(lay.b[nh])) : beta[nh];
        const float u = bt * (to_f32(v[vec + tid]) - w);
        s_u[tid] = u;
        o = p + s_qk * u;
        if constexpr (NORM) {
            float ss = o * o;
#pragma unroll
            for (int m = 16; m > 0; m >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
            if (lane == 0) s_ss[warp] = ss;
        } else {
            out[vec + tid] = from_f32<TO>(o);
        }
    }
    __syncthreads();
    if constexpr (NORM) {
        if (tid < kHeadDim) {
            const float rinv = rsqrtf((s_ss[0] + s_ss[1] + s_ss[2] + s_ss[3]) * (1.f / kHeadDim) + lay.eps);
            out[vec + tid] = from_f32<TO>(o * rinv * lay.w[tid] * sigmoid_d(to_f32(lay.g[vec + tid])));
        }
    }

    const float4 u4 = reinterpret_cast<const float4 *>(s_u)[lane];
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r) {
        const float ki = s_k[row0 + r];
        float4 x = st[r];
        x.x += ki * u4.x; x.y += ki * u4.y; x.z += ki * u4.z; x.w += ki * u4.w;
        __stcs(reinterpret_cast<float4 *>(Sh + (size_t)(row0 + r) * kHeadDim) + lane, x);
    }
}

}  // namespace

template <typename T, typename TO>
static void launch_typed(const void *q, const void *k, const void *v, const float *log_alpha,
                         const float *beta, float *S, void *out, unsigned blocks, int H,
                         const GateArgs *gate, const NormArgs *norm, cudaStream_t stream)
{
    DecodeLayer<T> lay = {};
    lay.H = H;
    if (gate) {
        lay.f = (const T *)gate->f; lay.A_log = gate->A_log; lay.dt_bias = gate->dt_bias;
        lay.b = (const T *)gate->beta_logits;
    }
    if (norm) { lay.g = (const T *)norm->gate; lay.w = norm->weight; lay.eps = norm->eps; }
    const bool fg = lay.f != nullptr, nm = norm != nullptr;
    auto args = [&](auto kern) {
        kern<<<blocks, kDecThreads, 0, stream>>>((const T *)q, (const T *)k, (const T *)v, log_alpha, beta, S,
                                                 (TO *)out, lay);
    };
    if (fg && nm) args(decode_kernel<T, TO, true, true>);
    else if (fg) args(decode_kernel<T, TO, true, false>);
    else if (nm) args(decode_kernel<T, TO, false, true>);
    else args(decode_kernel<T, TO, false, false>);
}

cudaError_t launch_decode(const void *q, const void *k, const void *v, const float *log_alpha,
                          const float *beta, float *S, void *out, int N, int H,
                          kda_dtype_t dtype, kda_dtype_t out_dtype, cudaStream_t stream,
                          const GateArgs *gate, const NormArgs *norm)
{
    const long long blocks = (long long)N * H;
    if (blocks == 0) return cudaSuccess;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
    const unsigned nb = (unsigned)blocks;
    using bf = __nv_bfloat16;
    if (dtype == KDA_BF16 && out_dtype == KDA_BF16)
        launch_typed<bf, bf>(q, k, v, log_alpha, beta, S, out, nb, H, gate, norm, stream);
    else if (dtype == KDA_BF16)
        launch_typed<bf, float>(q, k, v, log_alpha, beta, S, out, nb, H, gate, norm, stream);
    else if (out_dtype == KDA_BF16)
        launch_typed<float, bf>(q, k, v, log_alpha, beta, S, out, nb, H, gate, norm, stream);
    else
        launch_typed<float, float>(q, k, v, log_alpha, beta, S, out, nb, H, gate, norm, stream);
    return cudaGetLastError();
}

}  // namespace kda
