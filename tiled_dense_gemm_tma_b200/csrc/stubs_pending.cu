// Temporary: paths not yet implemented report TG_ERR_UNSUPPORTED.
#include "launch.h"
namespace tg {
int launch_w4a16(const GemmArgs&) { return kUnsupported; }
}
