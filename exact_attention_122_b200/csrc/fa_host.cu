// fa_host.cu -- exact attention forward on host-resident tensors, with the
// host <-> device transfers overlapped with the computation.
//
// The B*H heads are cut into chunks of whole heads (contiguous in the
// [B][H][N][d] layout).  Chunk c goes through device slot c % 2 of the
// caller's workspace on three internal streams: copy in (Q, K, V), attention
// (the persistent forward kernel with its dynamic schedule), copy out (O,
// LSE).  Events order the slot reuse, so chunk c+1's inputs cross PCIe while
// chunk c is computed and chunk c-1's outputs come back.  With pinned host
// memory the step is bound by the larger of the two transfer directions.

#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "fa.h"
#include "fa_internal.h"

namespace {

constexpr int kMaxDevices = 64;   // current_device() accepts indices below this
constexpr int kSlots = 2;
constexpr long long kTargetChunks = 16;
constexpr long long kUnitRows = 256;   // rows per work unit of the forward kernel

// Internal streams and events of one device, created on first use; calls on
// the device are serialised while they enqueue (the work itself runs
// asynchronously).
struct HostPipe {
    std::once_flag once;
    std::mutex mu;
    cudaError_t err = cudaSuccess;
    cudaStream_t s_in = nullptr, s_cmp = nullptr, s_out = nullptr;
    cudaEvent_t start = nullptr, end = nullptr;
    cudaEvent_t in_done[kSlots] = {}, cmp_done[kSlots] = {}, out_done[kSlots] = {};
};
HostPipe g_pipe[kMaxDevices];

struct Chunking {
    long long hc = 0, nchunks = 0;          // heads per chunk, chunks
    size_t off_k = 0, off_v = 0, off_o = 0, off_l = 0, off_ctr = 0, slot_bytes = 0;
};

size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

Chunking chunking(long long BH, int N, int d) {
    Chunking c;
    c.hc = (BH + kTargetChunks - 1) / kTargetChunks;
    c.nchunks = (BH + c.hc - 1) / c.hc;
    const size_t t = size_t(c.hc) * size_t(N) * size_t(d) * 2;   // one bf16 tensor of a chunk
    c.off_k = up256(t);
    c.off_v = c.off_k + up256(t);
    c.off_o = c.off_v + up256(t);
    c.off_l = c.off_o + up256(t);
    c.off_ctr = c.off_l + up256(size_t(c.hc) * size_t(N) * 4);
    c.slot_bytes = c.off_ctr + FA_DYNAMIC_WORKSPACE_BYTES;
    return c;
}

cudaError_t make_pipe(HostPipe& p) {
    cudaError_t e = cudaSuccess;
    for (cudaStream_t* s : {&p.s_in, &p.s_cmp, &p.s_out})
        if (e == cudaSuccess) e = cudaStreamCreateWithFlags(s, cudaStreamNonBlocking);
    for (cudaEvent_t* ev : {&p.start, &p.end})
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming);
    for (int i = 0; i < kSlots && e == cudaSuccess; ++i) {
        e = cudaEventCreateWithFlags(&p.in_done[i], cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&p.cmp_done[i], cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&p.out_done[i], cudaEventDisableTiming);
    }
    return e;
}

bool aligned(const void* p, uintptr_t a) { return reinterpret_cast<uintptr_t>(p) % a == 0; }

fa_status launch_error(cudaError_t e) {
    fa_internal::set_last_cuda_error(int(e));
    return FA_ERR_LAUNCH;
}

// Makes `s` wait for everything queued so far on the three internal streams
// (each wait takes the event's latest record, so one event serves all three).
cudaError_t join(HostPipe& p, cudaStream_t s) {
    cudaError_t e = cudaSuccess;
    for (cudaStream_t x : {p.s_in, p.s_cmp, p.s_out}) {
        if (e == cudaSuccess) e = cudaEventRecord(p.end, x);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(s, p.end, 0);
    }
    return e;
}

// A failure after the first enqueue: the caller's stream still waits for the
// copies already queued, so freeing the buffers after synchronising it is safe.
fa_status fail_after_enqueue(HostPipe& p, cudaStream_t s, int status, cudaError_t e) {
    if (e != cudaSuccess) fa_internal::set_last_cuda_error(int(e));   // else already recorded
    join(p, s);
    return static_cast<fa_status>(status);
}

}  // namespace

extern "C" {

size_t fa_fwd_host_workspace_bytes(int B, int H, int N, int d) {
    if (B < 1 || H < 1 || N < 1 || (d != 64 && d != 128)) return 0;
    if ((long long)B * H > 0x7fffffffLL || N > (1 << 30)) return 0;
    if ((N + kUnitRows - 1) / kUnitRows * ((long long)B * H) > (1LL << 30)) return 0;
    return size_t(kSlots) * chunking((long long)B * H, N, d).slot_bytes;
}

fa_status fa_fwd_host(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                      int H, int N, int d, int causal, float scale, void* workspace,
                      size_t workspace_bytes, void* stream) {
    if (!q || !k || !v || !o || !lse || !workspace) return FA_ERR_INVALID_ARG;
    if (B < 1 || H < 1 || N < 1) return FA_ERR_INVALID_ARG;
    if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
    if (!std::isfinite(scale) || !(scale > 0.f)) return FA_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
    const long long BH = (long long)B * H;
    if (BH > 0x7fffffffLL || N > (1 << 30)) return FA_ERR_UNSUPPORTED;
    // Every chunk passes the forward's own checks when the whole problem
    // does, so no chunk fails after earlier ones were enqueued.
    if ((N + kUnitRows - 1) / kUnitRows * BH > (1LL << 30)) return FA_ERR_UNSUPPORTED;
    if (workspace_bytes < fa_fwd_host_workspace_bytes(B, H, N, d)) return FA_ERR_INVALID_ARG;
    if (!aligned(workspace, 256)) return FA_ERR_MISALIGNED;

    int dev = -1, sm_count = 0;
    const int ds = fa_internal::current_device(&dev, &sm_count);
    if (ds != FA_OK) return static_cast<fa_status>(ds);
    HostPipe& p = g_pipe[dev];
    std::call_once(p.once, [&] { p.err = make_pipe(p); });
    if (p.err != cudaSuccess) return launch_error(p.err);
    std::lock_guard<std::mutex> lk(p.mu);

    const Chunking c = chunking(BH, N, d);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    unsigned char* ws = static_cast<unsigned char*>(workspace);
    const size_t head_bytes = size_t(N) * size_t(d) * 2;
    // Work already queued on the caller's stream comes first.
    cudaError_t e = cudaEventRecord(p.start, s);
    for (cudaStream_t x : {p.s_in, p.s_cmp, p.s_out})
        if (e == cudaSuccess) e = cudaStreamWaitEvent(x, p.start, 0);
    if (e != cudaSuccess) return launch_error(e);

    for (long long ci = 0; ci < c.nchunks; ++ci) {
        const int slot = int(ci % kSlots);
        const long long h0 = ci * c.hc;
        const long long hn = (BH - h0) < c.hc ? (BH - h0) : c.hc;
        const size_t bytes = size_t(hn) * head_bytes;
        const size_t lbytes = size_t(hn) * size_t(N) * 4;
        unsigned char* base = ws + size_t(slot) * c.slot_bytes;
        const size_t src = size_t(h0) * head_bytes;
        // copy in: the slot's inputs are free once the attention of chunk ci-2 ran
        if (ci >= kSlots) e = cudaStreamWaitEvent(p.s_in, p.cmp_done[slot], 0);
        if (e == cudaSuccess)
            e = cudaMemcpyAsync(base, static_cast<const unsigned char*>(q) + src, bytes,
                                cudaMemcpyDefault, p.s_in);
        if (e == cudaSuccess)
            e = cudaMemcpyAsync(base + c.off_k, static_cast<const unsigned char*>(k) + src, bytes,
                                cudaMemcpyDefault, p.s_in);
        if (e == cudaSuccess)
            e = cudaMemcpyAsync(base + c.off_v, static_cast<const unsigned char*>(v) + src, bytes,
                                cudaMemcpyDefault, p.s_in);
        if (e == cudaSuccess) e = cudaEventRecord(p.in_done[slot], p.s_in);
        // attention: after the inputs, and after chunk ci-2's outputs left the slot
        if (e == cudaSuccess) e = cudaStreamWaitEvent(p.s_cmp, p.in_done[slot], 0);
        if (e == cudaSuccess && ci >= kSlots) e = cudaStreamWaitEvent(p.s_cmp, p.out_done[slot], 0);
        if (e != cudaSuccess) return fail_after_enqueue(p, s, FA_ERR_LAUNCH, e);
        const int st = fa_internal::forward_qk(base, base + c.off_k, base + c.off_v,
                                               base + c.off_o,
                                               reinterpret_cast<float*>(base + c.off_l), 1,
                                               int(hn), N, N, d, causal, scale,
                                               reinterpret_cast<int*>(base + c.off_ctr), p.s_cmp);
        if (st != FA_OK) return fail_after_enqueue(p, s, st, cudaSuccess);
        e = cudaEventRecord(p.cmp_done[slot], p.s_cmp);
        // copy out
        if (e == cudaSuccess) e = cudaStreamWaitEvent(p.s_out, p.cmp_done[slot], 0);
        if (e == cudaSuccess)
            e = cudaMemcpyAsync(static_cast<unsigned char*>(o) + src, base + c.off_o, bytes,
                                cudaMemcpyDefault, p.s_out);
        if (e == cudaSuccess)
            e = cudaMemcpyAsync(reinterpret_cast<unsigned char*>(lse) + size_t(h0) * N * 4,
                                base + c.off_l, lbytes, cudaMemcpyDefault, p.s_out);
        if (e == cudaSuccess) e = cudaEventRecord(p.out_done[slot], p.s_out);
        if (e != cudaSuccess) return fail_after_enqueue(p, s, FA_ERR_LAUNCH, e);
    }
    // The caller's stream waits for the last copy out, which follows every
    // other operation of the call.
    e = cudaEventRecord(p.end, p.s_out);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s, p.end, 0);
    if (e != cudaSuccess) return fail_after_enqueue(p, s, FA_ERR_LAUNCH, e);
    return FA_OK;
}

}  // extern "C"
