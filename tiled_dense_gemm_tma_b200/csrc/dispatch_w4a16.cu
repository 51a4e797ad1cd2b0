// Dispatch of the 4-bit-weight GEMMs by the number of activation rows.
#include "launch.h"
namespace tg {
// The tuning rule's path (a.path) wins; by default M <= 4 takes the CUDA-core
// kernel, M <= 128 the weight-streaming kernel, larger M the CTA-pair kernel
// (the one-CTA kernel if a cluster launch is refused).
int launch_w4a16(const GemmArgs& a) {
    int path = a.path;
    if (path == PATH_AUTO)
        path = a.M <= kGemvMaxM ? PATH_CUDA_CORE : a.M <= kSkinnyMaxM ? PATH_SMALL_M : PATH_CTA_PAIR;
    if (path == PATH_CUDA_CORE) return launch_gemv_w4a16(a);
    if (path == PATH_SMALL_M) return launch_skinny_w4a16(a);
    if (path == PATH_ONE_CTA) return launch_w4a16_large(a);
    const int r = launch_w4a16_pair(a);
    return r == kUnsupported ? launch_w4a16_large(a) : r;
}
// FP4 weights: the same choice as for the 4-bit integers.
int launch_wfp4(const GemmArgs& a) {
    int path = a.path;
    if (path == PATH_AUTO)
        path = a.M <= kGemvMaxM ? PATH_CUDA_CORE : a.M <= kSkinnyMaxM ? PATH_SMALL_M : PATH_CTA_PAIR;
    if (path == PATH_CUDA_CORE) return launch_gemv_wfp4(a);
    if (path == PATH_SMALL_M) return launch_skinny_wfp4(a);
    if (path == PATH_ONE_CTA) return launch_wfp4_large(a);
    const int r = launch_wfp4_pair(a);
    return r == kUnsupported ? launch_wfp4_large(a) : r;
}
}
