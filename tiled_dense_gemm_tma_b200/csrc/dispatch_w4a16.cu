// Dispatch of the 4-bit-weight GEMM by the number of activation rows.
#include "launch.h"
namespace tg {
int launch_w4a16(const GemmArgs& a) {
    if (a.M <= kGemvMaxM) return launch_gemv_w4a16(a);
    if (a.M <= kSkinnyMaxM) return launch_skinny_w4a16(a);
    const int r = launch_w4a16_pair(a);
    return r == kUnsupported ? launch_w4a16_large(a) : r;
}
}
