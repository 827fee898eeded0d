// prefill.cu -- how kda_chunk_fwd (and its layer variant) runs the two passes of the bf16 prefill.
//
// The preparation pass (chunk_prep.cu) is data-parallel over every (chunk, head); the scan
// (chunk_scan.cu) is one serial chain of chunks per (sequence, head) and holds one SM per chain.
// With few chains (one long sequence: 32 heads hold 32 of the 148 SMs for the whole scan) the two
// passes run as a pipeline over token ranges: the scan of range r runs while the preparation of the
// later ranges fills the other SMs. Each range's scan waits for its own preparation only; a range
// that does not start a sequence starts from the state the previous range left in the carry (S_final,
// or a workspace area when the caller passes none). The scans go to a library stream of the highest
// priority and the preparations to one of the lowest, so that the SMs a finished scan range frees
// go to the next scan range before queued preparation blocks. Both streams fork from the caller's
// stream and join it again, so the call stays ordered on that stream.
// With many chains the scan alone fills the GPU; the passes then run one after the other on the
// caller's stream.
#include <mutex>

#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int kMaxRanges = 16;

struct PipeStreams {
    bool ready = false;
    cudaStream_t scan = nullptr, prep = nullptr;
    cudaEvent_t fork = nullptr, join = nullptr;
    cudaEvent_t prepped[kMaxRanges];
};
constexpr int kMaxDevices = 64;
PipeStreams g_pipe[kMaxDevices];
std::mutex g_pipe_mu;

// Streams and events of the current device, created on first use (guarded by g_pipe_mu).
PipeStreams *pipe_streams()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    PipeStreams &ps = g_pipe[dev];
    if (ps.ready) return &ps;
    int lo = 0, hi = 0;                           // least and greatest priority
    if (cudaDeviceGetStreamPriorityRange(&lo, &hi) != cudaSuccess) return nullptr;
    if (cudaStreamCreateWithPriority(&ps.scan, cudaStreamNonBlocking, hi) != cudaSuccess) return nullptr;
    if (cudaStreamCreateWithPriority(&ps.prep, cudaStreamNonBlocking, lo) != cudaSuccess) return nullptr;
    if (cudaEventCreateWithFlags(&ps.fork, cudaEventDisableTiming) != cudaSuccess) return nullptr;
    if (cudaEventCreateWithFlags(&ps.join, cudaEventDisableTiming) != cudaSuccess) return nullptr;
    for (int i = 0; i < kMaxRanges; ++i)
        if (cudaEventCreateWithFlags(&ps.prepped[i], cudaEventDisableTiming) != cudaSuccess) return nullptr;
    ps.ready = true;
    return &ps;
}

// token ranges of the pipeline over n_slots chunk slots
// chunk slots of a prefill's workspace
int n_slots_of(const PrefillArgs &a) { return (int)prep_slots((long long)a.B * a.T, a.N); }

int pipe_ranges(int n_slots)
{
    const int R = n_slots / kPipeMinSlotsPerRange;
    return R < 2 ? 2 : (R > kMaxRanges ? kMaxRanges : R);
}

}  // namespace

bool prefill_pipelined(long long tokens, int H, int N)
{
    return (long long)N * H <= kPipeMaxChains && prep_slots(tokens, N) >= 2 * kPipeMinSlotsPerRange;
}

int prefill_launches(long long tokens, int H, int N)
{
    return prefill_pipelined(tokens, H, N) ? 2 * pipe_ranges((int)prep_slots(tokens, N)) : 2;
}

size_t prefill_carry_bytes(long long tokens, int H, int N)
{
    return prefill_pipelined(tokens, H, N) ? (size_t)N * H * kHeadDim * kHeadDim * sizeof(float) : 0;
}

cudaError_t run_prefill_bf16(const PrefillArgs &a_in, kda_dtype_t out_dtype, cudaStream_t st,
                             const GateArgs *gate, const NormArgs *norm, bool records)
{
    auto scan = [&](const PrefillArgs &a, cudaStream_t s, long long lo, long long hi) {
        return records ? launch_chunk_scan_records(a, (const unsigned char *)a.scratch, n_slots_of(a), s, lo, hi)
                       : launch_chunk_scan(a, (const unsigned char *)a.scratch, n_slots_of(a), out_dtype, s, norm, lo, hi);
    };
    const long long tokens = (long long)a_in.B * a_in.T;
    const int n_slots = (int)prep_slots(tokens, a_in.N);
    unsigned char *blocks = (unsigned char *)a_in.scratch;
    if (!prefill_pipelined(tokens, a_in.H, a_in.N)) {
        cudaError_t e = launch_chunk_prep(a_in, blocks, n_slots, st, gate);
        if (e == cudaSuccess) e = scan(a_in, st, 0, n_slots);
        return e;
    }
    PrefillArgs a = a_in;
    if (!a.S_final)                               // the carry between ranges: after the blocks
        a.S_final = (float *)(blocks + (size_t)a.H * n_slots * kPrepBlockBytes);
    const int R = pipe_ranges(n_slots);
    std::lock_guard<std::mutex> lock(g_pipe_mu);
    PipeStreams *ps = pipe_streams();
    if (!ps) return cudaErrorNotReady;
    cudaError_t e = cudaEventRecord(ps->fork, st);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(ps->prep, ps->fork, 0);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(ps->scan, ps->fork, 0);
    // ranges of slots: the first half as long (its preparation runs with no scan beside it) and, with
    // eight ranges or more, the last a quarter as long (its scan runs after every preparation has
    // finished; with fewer ranges a quarter range is too short to pay for its launch)
    int bounds[kMaxRanges + 1];
    {
        const double unit = (double)n_slots / (R >= 8 ? R - 1.25 : R - 0.5);
        bounds[0] = 0;
        for (int r = 1; r < R; ++r) bounds[r] = (int)((r - 0.5) * unit);
        bounds[R] = n_slots;
    }
    for (int r = 0; r < R && e == cudaSuccess; ++r) {
        e = launch_chunk_prep(a, blocks, n_slots, ps->prep, gate, bounds[r], bounds[r + 1]);
        if (e == cudaSuccess) e = cudaEventRecord(ps->prepped[r], ps->prep);
    }
    for (int r = 0; r < R && e == cudaSuccess; ++r) {
        e = cudaStreamWaitEvent(ps->scan, ps->prepped[r], 0);
        if (e == cudaSuccess) e = scan(a, ps->scan, bounds[r], bounds[r + 1]);
    }
    // join: the caller's stream waits for both library streams (on an error too, so that nothing the
    // call enqueued can still run unordered with the caller's later work)
    cudaError_t j = cudaEventRecord(ps->join, ps->scan);
    if (j == cudaSuccess) j = cudaStreamWaitEvent(st, ps->join, 0);
    if (j == cudaSuccess) j = cudaEventRecord(ps->join, ps->prep);
    if (j == cudaSuccess) j = cudaStreamWaitEvent(st, ps->join, 0);
    return e != cudaSuccess ? e : j;
}

}  // namespace kda
