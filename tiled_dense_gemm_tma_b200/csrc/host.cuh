// host.cuh -- host-side helpers shared by the launchers: device facts,
// tensor-map (TMA descriptor) encoding with a cache, debug knobs.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace tg {

struct DeviceInfo {
    int ok;            // 1 if an sm_100 device
    int num_sms;
};

// Facts about the current device (cached per device).  Returns nullptr if
// no device is current or it is not sm_100.
const DeviceInfo* current_device(int* dev_out);

// Encode (or fetch from the cache) a 2-D tiled tensor map over a row-major
// matrix: `cols` x `rows` elements, row pitch `ld_bytes`, box `box_cols` x
// `box_rows`, shared-memory swizzle `swz`.  Returns false on failure.
bool tensor_map_2d(CUtensorMap* out, const void* base, CUtensorMapDataType dtype,
                   int elem_bytes, uint64_t cols, uint64_t rows, uint64_t ld_bytes,
                   uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swz);

constexpr CUtensorMapSwizzle SWZ_NONE = CU_TENSOR_MAP_SWIZZLE_NONE;
constexpr CUtensorMapSwizzle SWZ_64 = CU_TENSOR_MAP_SWIZZLE_64B;
constexpr CUtensorMapSwizzle SWZ_128 = CU_TENSOR_MAP_SWIZZLE_128B;
constexpr CUtensorMapSwizzle SWZ_128_32B = CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B;

// Bounded-wait limit for kernels, in ns (TG_DEBUG_TIMEOUT_US overrides).
unsigned long long wait_limit_ns();

// Debug fault injection (TG_INJECT, default 0 = off), read once per process.
// With TG_INJECT=1 the first kernel launch of the process (and only that
// one) has the TMA producer of CTA 0 (of CTA pair 0's leader) skip arming its
// first ring slot: that CTA's consumers wait on a barrier nothing completes,
// run into the bounded-wait limit, report TG_ERR_TIMEOUT and return, while
// the other CTAs finish (leaving split-K tickets incomplete).  Launchers
// call this once per launch.
int inject_mode();
// Debug: TG_NO_PAIR=1 makes every CTA-pair launch report "unsupported", so
// the calls take the one-CTA kernels (the path used when a cluster launch is
// refused).  Read once per process.
bool pair_kernels_disabled();

// Device address of the current device's status word (nullptr on error).
int* device_status_ptr();

// Allow `func` to use `bytes` of dynamic shared memory (once per device).
// `slot` (0..kMaxSlots-1) names the kernel in a per-device bitmask of done
// calls; each kernel instantiation needs its own:
//    0-4   gemm_tc.cu        one-CTA bf16/f16/tf32, CTA-pair bf16/f16
//   54-55  gemm_tc.cu        CTA-pair bf16/f16 with a 4-slot ring (tuning table)
//    5, 11-15 gemm_tc.cu     CTA-pair with transposed operands
//    8     gemm_ffma.cu      9  gemm_w4a16.cu     10  gemm_w4a16_pair.cu
//    6, 7  gemm_w4a16.cu, gemm_w4a16_pair.cu (FP4 weights)
//   16-27  gemm_skinny.cu    28-35  gemm_skinny.cu (weights stored transposed)
//   36-39  gemm_skinny.cu (FP4 weights)
//   40-48  gemv.cu           58-60  gemv.cu (FP4 weights)
//   50-53  gemm_skinny_static.cu
//   56-57  gemm_sp24.cu (one CTA)   61-62  gemm_sp24.cu (CTA pairs)
//   64-67  gemm_tc.cu        CTA-pair bf16/f16 with the operands swapped (M <= 128)
//   68     gemm_tc.cu        CTA-pair TF32
constexpr int kMaxSlots = 128;
cudaError_t set_smem_attr(const void* func, int bytes, int slot);

// Clusters of S CTAs (threads and dynamic shared memory bytes each) of the
// kernel in attribute slot `slot` that the current device holds at once
// (cudaOccupancyMaxActiveClusters), cached per device, slot and S; 0 if the
// query fails.  The slot's shared-memory attribute must be set first.
int max_active_clusters(const void* func, int slot, int S, int threads, int smem_bytes);

}  // namespace tg
