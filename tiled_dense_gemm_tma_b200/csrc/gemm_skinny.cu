// gemm_skinny.cu -- launchers of the weight-streaming (small-M) kernel and the
// per-stream workspace that holds its split-K partials and tile tickets.
#include "gemm_skinny.cuh"
#include "host.cuh"
#include "launch.h"

#include <map>
#include <mutex>
#include <utility>

namespace tg {

namespace {

// ----------------------------------------------------------------- workspace
// One workspace per (device, stream): calls on one stream run in order, so
// they can share it; calls on different streams get their own.  Layout:
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

std::mutex g_ws_mu;
std::map<std::pair<int, void*>, Workspace> g_ws;

}  // namespace

bool stream_workspace(int dev, void* stream, long long tickets, long long partial_bytes,
                      int** tk, float** part) {
    std::lock_guard<std::mutex> lk(g_ws_mu);
    Workspace& w = g_ws[{dev, stream}];
    const long long tbytes = (tickets * 4 + 255) / 256 * 256;
    if (!w.base || w.ticket_cap < tickets || w.partial_cap < partial_bytes) {
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
    (void)tbytes;
    *tk = static_cast<int*>(w.base);
    *part = reinterpret_cast<float*>(static_cast<char*>(w.base) +
                                     (w.ticket_cap * 4 + 255) / 256 * 256);
    return true;
}

namespace {

long long begin_of(long long c, long long U, long long G) { return c * U / G; }

long long owner_of(long long u, long long U, long long G) {
    long long c = u * G / U;
    while (c + 1 < G && begin_of(c + 1, U, G) <= u) ++c;
    while (c > 0 && begin_of(c, U, G) > u) --c;
    return c;
}

template <WKind W, int MPAD>
int run(const GemmArgs& a) {
    using Cfg = SkCfg<W, MPAD>;
    int dev = 0;
    const DeviceInfo* di = current_device(&dev);
    if (!di) return kNoDevice;
    const long long T = (a.N + Cfg::GN - 1) / Cfg::GN;
    const long long KB = (a.K + Cfg::BK - 1) / Cfg::BK;
    const long long U = T * KB;
    if (U > 0x7fffffffll) return kUnsupported;
    const long long G = U < di->num_sms ? U : di->num_sms;
    long long J = 1;
    for (long long t = 0; t < T; ++t) {
        const long long n = owner_of(t * KB + KB - 1, U, G) - owner_of(t * KB, U, G) + 1;
        if (n > J) J = n;
    }
    int* tickets = nullptr;
    float* ws = nullptr;
    if (!stream_workspace(dev, a.stream, T, T * J * MPAD * Cfg::GN * 4, &tickets, &ws))
        return kCudaError;

    CUtensorMap tW, tS, tX;
    if constexpr (Cfg::Q4) {
        if (!tensor_map_2d(&tW, a.B, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (a.N + 1) / 2, a.K, a.ldb,
                           Cfg::GN / 2, Cfg::BK, SWZ_128))
            return kCudaError;
        if (!tensor_map_2d(&tS, a.scales, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, a.N, a.K / 128,
                           a.lds * 2, Cfg::GN, 1, SWZ_NONE))
            return kCudaError;
    } else {
        const CUtensorMapDataType dt = W == WKind::BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                         : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
        if (!tensor_map_2d(&tW, a.B, dt, 2, a.N, a.K, a.ldb * 2, 64, Cfg::BK, SWZ_128))
            return kCudaError;
        tS = tW;                                   // unused
    }
    const CUtensorMapDataType xt = W == WKind::BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                     : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    if (!tensor_map_2d(&tX, a.A, xt, 2, a.K, a.M, a.lda * 2, 64, MPAD, SWZ_128))
        return kCudaError;

    auto kern = skinny_kernel<Cfg>;
    const int slot = 16 + static_cast<int>(W) * 4 + (MPAD == 16 ? 0 : MPAD == 32 ? 1 : MPAD == 64 ? 2 : 3);
    if (set_smem_attr(reinterpret_cast<const void*>(kern), Cfg::SMEM_BYTES, slot) != cudaSuccess)
        return kCudaError;
    SkParams p;
    p.M = static_cast<int>(a.M);
    p.N = static_cast<int>(a.N);
    p.K = static_cast<int>(a.K);
    p.relu = a.relu;
    p.T = static_cast<int>(T);
    p.KB = static_cast<int>(KB);
    p.U = static_cast<int>(U);
    p.J = static_cast<int>(J);
    p.timeout_ns = wait_limit_ns();
    p.status = device_status_ptr();
    p.C = a.C;
    p.ldc = a.ldc;
    p.ws = ws;
    p.tickets = tickets;
    if (!p.status) return kCudaError;
    kern<<<static_cast<int>(G), Cfg::THREADS, Cfg::SMEM_BYTES, static_cast<cudaStream_t>(a.stream)>>>(
        tW, tS, tX, p);
    return cudaGetLastError() == cudaSuccess ? kOk : kCudaError;
}

template <WKind W>
int dispatch(const GemmArgs& a) {
    if (a.M <= 16) return run<W, 16>(a);
    if (a.M <= 32) return run<W, 32>(a);
    if (a.M <= 64) return run<W, 64>(a);
    return run<W, 128>(a);
}

}  // namespace

int launch_skinny_bf16(const GemmArgs& a) { return dispatch<WKind::BF16>(a); }
int launch_skinny_f16(const GemmArgs& a) { return dispatch<WKind::F16>(a); }
int launch_skinny_w4a16(const GemmArgs& a) { return dispatch<WKind::INT4>(a); }

void mark_workspaces_dirty(int dev) {
    std::lock_guard<std::mutex> lk(g_ws_mu);
    for (auto& kv : g_ws)
        if (kv.first.first == dev) kv.second.dirty = true;
}

}  // namespace tg
