// workspace.cu -- per-(device, stream) scratch of the kernels that split K
// across CTAs through global memory (the small-M tensor-core kernel's
// stream-K, the M <= 4 CUDA-core kernel, the fp32 FFMA kernel when tiles are
// fewer than SMs, and the CTA-pair kernel's split last wave).
#include "launch.h"

#include <cuda_runtime.h>

#include <map>
#include <mutex>
#include <thread>
#include <tuple>

namespace tg {

namespace {

// One workspace per (device, stream): calls on one stream run in order, so
// they can share it; calls on different streams get their own.  The handle
// cudaStreamPerThread names a different stream on every host thread, so for
// it the calling thread is part of the key.  Layout:
// [tickets: ticket_cap ints, zeroed][partials: partial_cap bytes].  Tickets
// return to zero at the end of every complete call; a call that timed out
// can leave them dirty, so a device-status read that reports a timeout marks
// the device's workspaces for re-zeroing before their next use.
struct Workspace {
    void* base = nullptr;
    long long ticket_cap = 0;      // ints
    long long partial_cap = 0;     // bytes
    bool dirty = false;
};

using WsKey = std::tuple<int, void*, std::thread::id>;

std::mutex g_ws_mu;
std::map<WsKey, Workspace> g_ws;

WsKey ws_key(int dev, void* stream) {
    const bool per_thread = stream == static_cast<void*>(cudaStreamPerThread);
    return WsKey(dev, stream, per_thread ? std::this_thread::get_id() : std::thread::id());
}

}  // namespace

bool stream_workspace(int dev, void* stream, long long tickets, long long partial_bytes,
                      int** tk, float** part) {
    std::lock_guard<std::mutex> lk(g_ws_mu);
    Workspace& w = g_ws[ws_key(dev, stream)];
    if (!w.base || w.ticket_cap < tickets || w.partial_cap < partial_bytes) {
        // a stream being captured into a graph cannot allocate (and a failed
        // allocation there would invalidate the capture): report "none"
        cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
        if (cudaStreamIsCapturing(static_cast<cudaStream_t>(stream), &cs) != cudaSuccess ||
            cs != cudaStreamCaptureStatusNone)
            return false;
        if (w.base) {
            cudaFree(w.base);     // synchronises the device: no kernel still uses it
            w.base = nullptr;
        }
        const long long tcap = tickets < 4096 ? 4096 : tickets;
        const long long pcap = partial_bytes < (8ll << 20) ? (8ll << 20) : partial_bytes;
        const long long tcap_bytes = (tcap * 4 + 255) / 256 * 256;
        if (cudaMalloc(&w.base, tcap_bytes + pcap) != cudaSuccess) {
            w.base = nullptr;
            return false;
        }
        w.ticket_cap = tcap;
        w.partial_cap = pcap;
        w.dirty = true;
    }
    if (w.dirty) {
        const long long tcap_bytes = (w.ticket_cap * 4 + 255) / 256 * 256;
        if (cudaMemsetAsync(w.base, 0, tcap_bytes, static_cast<cudaStream_t>(stream)) != cudaSuccess)
            return false;
        w.dirty = false;
    }
    *tk = static_cast<int*>(w.base);
    *part = reinterpret_cast<float*>(static_cast<char*>(w.base) +
                                     (w.ticket_cap * 4 + 255) / 256 * 256);
    return true;
}

void mark_workspaces_dirty(int dev) {
    std::lock_guard<std::mutex> lk(g_ws_mu);
    for (auto& kv : g_ws)
        if (std::get<0>(kv.first) == dev) kv.second.dirty = true;
}

}  // namespace tg
