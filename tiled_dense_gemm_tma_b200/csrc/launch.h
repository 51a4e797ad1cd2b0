// launch.h -- internal interface between the C ABI shim and the launchers.
// Arguments arrive here already validated (sizes, pointers, alignment).
#pragma once
#include <cstdint>

#include "tune.h"

namespace tg {

// Internal status values; identical to the tg_status codes.
enum : int { kOk = 0, kInvalidArg = 1, kAlignment = 2, kUnsupported = 3, kCudaError = 4,
             kTimeout = 5, kNoDevice = 6 };

struct GemmArgs {
    int64_t M, N, K;
    const void* A; int64_t lda;      // elements
    const void* B; int64_t ldb;      // elements (bytes for packed 4-bit weights)
    void* C; int64_t ldc;            // elements
    const void* scales; int64_t lds; // 4-bit paths only (lds: elements, bytes for E8M0 scales)
    int group;                       // 4-bit paths only
    int relu;
    void* stream;
    // launch shape from the tuning table (tune.h); 0 = the launcher's default
    int path;                        // TunePath: kernel family
    int ctas;                        // persistent CTAs (CTA pairs), stream-K ranges
    int group_m;                     // raster band height in tiles
    int splits;                      // fp32 FFMA split-K ranges
    int stages;                      // 16-bit CTA-pair ring depth (4 or 6)
};

// The arguments with a tuning rule's launch-shape fields.
inline GemmArgs with_rule(GemmArgs a, const TuneRule& r) {
    a.path = r.path;
    a.ctas = r.ctas;
    a.group_m = r.group_m;
    a.splits = r.splits;
    a.stages = r.stages;
    return a;
}

// Persistent grid size: `units` of work over at most `cap` CTAs (the rule's
// CTA count when set, else all of `cap`).
inline long long persistent_grid(long long units, int cap, int ctas) {
    const long long c = ctas > 0 && ctas < cap ? ctas : cap;
    return units < c ? units : c;
}

int launch_tc_bf16(const GemmArgs& a);
int launch_tc_f16(const GemmArgs& a);
int launch_tc_tf32(const GemmArgs& a);
int launch_tc_trans(const GemmArgs& a, int bf16, int trans_a, int trans_b);
int launch_ffma_f32(const GemmArgs& a);
int launch_w4a16(const GemmArgs& a);
int launch_w4a16_large(const GemmArgs& a);
int launch_w4a16_pair(const GemmArgs& a);
// FP4 (E2M1 + E8M0) weights, bf16 activations: scales / lds in bytes.
int launch_wfp4(const GemmArgs& a);
int launch_wfp4_large(const GemmArgs& a);
int launch_wfp4_pair(const GemmArgs& a);
int launch_skinny_wfp4(const GemmArgs& a);
// 2:4 sparse A: a.A / a.lda are the compressed values, E / lde the codes.
int launch_sp24(const GemmArgs& a, const void* E, int64_t lde, int bf16);
int launch_skinny_bf16(const GemmArgs& a);
int launch_skinny_f16(const GemmArgs& a);
int launch_skinny_w4a16(const GemmArgs& a);
// 16-bit weights stored transposed (B is N x K): the weight-streaming kernel
// reading K-major weight tiles.
int launch_skinny_trans_b(const GemmArgs& a, int bf16);
int launch_gemv_bf16(const GemmArgs& a);
int launch_gemv_f16(const GemmArgs& a);
int launch_gemv_w4a16(const GemmArgs& a);
int launch_gemv_wfp4(const GemmArgs& a);
void mark_workspaces_dirty(int dev);
// The argument checks every 16-bit and fp32 entry point runs before any CUDA
// call (sizes, pointers, leading dimensions, the row-pitch bound, alignment)
// for elements of `eb` bytes; returns a tg_status value.
int check_gemm_args(int64_t M, int64_t N, int64_t K, const void* A, int64_t lda, const void* B,
                    int64_t ldb, const void* C, int64_t ldc, int epilogue, int eb);
// Per-(device, stream) scratch of the split-K paths: `tickets` ints (zero
// between calls) and `partial_bytes` of fp32 partials.
bool stream_workspace(int dev, void* stream, long long tickets, long long partial_bytes,
                      int** tk, float** part);

// Activation rows up to which the CUDA-core kernel is used.
constexpr long long kGemvMaxM = 4;
// Activation rows up to which the weight-streaming kernel is used.
constexpr long long kSkinnyMaxM = 128;

}  // namespace tg
