// Dispatch of the 4-bit-weight GEMMs by the number of activation rows.
#include "launch.h"
namespace tg {
int launch_w4a16(const GemmArgs& a) {
    if (a.M <= kGemvMaxM) return launch_gemv_w4a16(a);
    if (a.M <= kSkinnyMaxM) return launch_skinny_w4a16(a);
    const int r = launch_w4a16_pair(a);
    return r == kUnsupported ? launch_w4a16_large(a) : r;
}
// FP4 weights: the weight-streaming kernel for every M <= 128 (no CUDA-core
// variant), the CTA-pair kernel above, the one-CTA kernel if a cluster
// launch is refused.
int launch_wfp4(const GemmArgs& a) {
    if (a.M <= kSkinnyMaxM) return launch_skinny_wfp4(a);
    const int r = launch_wfp4_pair(a);
    return r == kUnsupported ? launch_wfp4_large(a) : r;
}
}
