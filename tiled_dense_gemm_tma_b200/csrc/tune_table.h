// tune_table.h -- built-in tuning rules (see tune.h).  Written by
// `python bench.py --sweep` on one B200 from the timings in
// profiles/tune_sweep.md; a class without a rule keeps every default.
#pragma once
#include "tune.h"

namespace tg {

constexpr TuneRule kBuiltinRules[] = {
    {0, 3, 65, 128, 4096, 0x7fffffffffffffffll, 0, 0, 0, 0},   // bf16 M 65..128: path=cta_pair (0.779 of the default)
    {2, 2, 5, 128, 4096, 0x7fffffffffffffffll, 128, 0, 0, 0},   // w4a16 M 5..128: path=small_m, ctas=128 (0.967 of the default)
    {-1, 0, 0, 0, 0, 0, 0, 0, 0, 0},   // end: matches nothing
};

}  // namespace tg
