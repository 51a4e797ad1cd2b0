// host.cu -- device facts, tensor-map encoding and its cache, debug knobs.
#include "host.cuh"

#include <atomic>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <unordered_map>

namespace tg {

namespace {

constexpr int kMaxDevices = 64;
DeviceInfo g_dev[kMaxDevices];
std::once_flag g_dev_once[kMaxDevices];

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;
std::once_flag g_encode_once;

struct MapKey {
    uint64_t base, cols, rows, ld;
    uint32_t box_cols, box_rows;
    int dtype, swz;
    bool operator==(const MapKey& o) const {
        return base == o.base && cols == o.cols && rows == o.rows && ld == o.ld &&
               box_cols == o.box_cols && box_rows == o.box_rows && dtype == o.dtype &&
               swz == o.swz;
    }
};
struct MapKeyHash {
    size_t operator()(const MapKey& k) const {
        uint64_t h = k.base * 0x9E3779B97F4A7C15ull;
        h ^= (k.cols + 0x7F4A7C15ull) * 0xBF58476D1CE4E5B9ull;
        h ^= (k.rows + (h << 6) + (h >> 2)) * 0x94D049BB133111EBull;
        h ^= k.ld + (static_cast<uint64_t>(k.box_cols) << 32) + k.box_rows + (k.dtype << 3) + k.swz;
        return static_cast<size_t>(h ^ (h >> 31));
    }
};
std::mutex g_map_mu;
std::unordered_map<MapKey, CUtensorMap, MapKeyHash> g_maps;
constexpr size_t kMaxCachedMaps = 4096;

std::atomic<unsigned long long> g_attr_done[kMaxDevices][kMaxSlots / 64];
std::atomic<const void*> g_attr_func[kMaxDevices][kMaxSlots];   // the kernel that owns each slot

}  // namespace

const DeviceInfo* current_device(int* dev_out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    // A host thread that has made no runtime call that binds a context (for
    // example the autograd engine's worker thread) has no context current,
    // and the driver-level tensor-map encoder then fails: make the device's
    // primary context current on this thread once.
    static thread_local int bound = -1;
    if (bound != dev) {
        if (cudaSetDevice(dev) != cudaSuccess) return nullptr;
        bound = dev;
    }
    std::call_once(g_dev_once[dev], [dev] {
        cudaDeviceProp prop;
        DeviceInfo info{0, 0};
        if (cudaGetDeviceProperties(&prop, dev) == cudaSuccess) {
            info.ok = (prop.major == 10);
            info.num_sms = prop.multiProcessorCount;
        }
        g_dev[dev] = info;
    });
    if (dev_out) *dev_out = dev;
    return g_dev[dev].ok ? &g_dev[dev] : nullptr;
}

bool tensor_map_2d(CUtensorMap* out, const void* base, CUtensorMapDataType dtype,
                   int elem_bytes, uint64_t cols, uint64_t rows, uint64_t ld_bytes,
                   uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swz) {
    std::call_once(g_encode_once, [] {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
                cudaSuccess && q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    });
    if (!g_encode) return false;
    // A map over a 1-row / 1-column matrix still needs a legal stride.
    if (rows < 1) rows = 1;
    if (cols < 1) cols = 1;
    MapKey key{reinterpret_cast<uint64_t>(base), cols, rows, ld_bytes, box_cols, box_rows,
               static_cast<int>(dtype), static_cast<int>(swz)};
    {
        std::lock_guard<std::mutex> lk(g_map_mu);
        auto it = g_maps.find(key);
        if (it != g_maps.end()) { *out = it->second; return true; }
    }
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {ld_bytes};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUtensorMap m;
    std::memset(&m, 0, sizeof m);
    CUresult r = g_encode(&m, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE,
                          swz,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return false;
    (void)elem_bytes;
    {
        std::lock_guard<std::mutex> lk(g_map_mu);
        if (g_maps.size() >= kMaxCachedMaps) g_maps.clear();
        g_maps.emplace(key, m);
    }
    *out = m;
    return true;
}

unsigned long long wait_limit_ns() {
    static const unsigned long long v = [] {
        const char* e = std::getenv("TG_DEBUG_TIMEOUT_US");
        unsigned long long us = e ? std::strtoull(e, nullptr, 10) : 0ull;
        return us ? us * 1000ull : 4000000000ull;   // default 4 s
    }();
    return v;
}

int inject_mode() {
    static const int v = [] {
        const char* e = std::getenv("TG_INJECT");
        return e ? std::atoi(e) : 0;
    }();
    static std::atomic<int> taken{0};
    if (v == 0) return 0;
    return taken.exchange(1) == 0 ? v : 0;      // the first launch only
}

bool pair_kernels_disabled() {
    static const bool v = [] {
        const char* e = std::getenv("TG_NO_PAIR");
        return e != nullptr && std::atoi(e) != 0;
    }();
    return v;
}

cudaError_t set_smem_attr(const void* func, int bytes, int slot) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices || slot < 0 || slot >= kMaxSlots) return cudaErrorInvalidValue;
    std::atomic<unsigned long long>& done = g_attr_done[dev][slot / 64];
    const unsigned long long bit = 1ull << (slot % 64);
    // a slot already set for another kernel is a collision between two
    // kernels' slot numbers: refuse rather than launch without the attribute
    if (done.load(std::memory_order_acquire) & bit)
        return g_attr_func[dev][slot].load(std::memory_order_relaxed) == func ? cudaSuccess
                                                                             : cudaErrorInvalidValue;
    e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) {
        g_attr_func[dev][slot].store(func, std::memory_order_relaxed);
        done.fetch_or(bit, std::memory_order_acq_rel);
    }
    return e;
}

namespace {
// -1: not asked yet; indexed [device][slot][log2 S - 1]
std::atomic<int> g_max_clusters[kMaxDevices][kMaxSlots][3];
std::once_flag g_max_clusters_once;
}  // namespace

int max_active_clusters(const void* func, int slot, int S, int threads, int smem_bytes) {
    std::call_once(g_max_clusters_once, [] {
        for (auto& d : g_max_clusters)
            for (auto& sl : d)
                for (auto& v : sl) v.store(-1, std::memory_order_relaxed);
    });
    int dev = 0;
    const int si = S == 2 ? 0 : S == 4 ? 1 : S == 8 ? 2 : -1;
    if (si < 0 || slot < 0 || slot >= kMaxSlots || cudaGetDevice(&dev) != cudaSuccess || dev < 0 ||
        dev >= kMaxDevices)
        return 0;
    std::atomic<int>& cached = g_max_clusters[dev][slot][si];
    int n = cached.load(std::memory_order_acquire);
    if (n >= 0) return n;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(S, 1, 1);
    cfg.blockDim = dim3(threads, 1, 1);
    cfg.dynamicSmemBytes = smem_bytes;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = S;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, func, &cfg) != cudaSuccess) {
        cudaGetLastError();                        // clear: treated as "no clusters"
        n = 0;
    }
    cached.store(n, std::memory_order_release);
    return n;
}

}  // namespace tg
