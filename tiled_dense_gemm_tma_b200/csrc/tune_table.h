// tune_table.h -- built-in tuning rules (see tune.h).  Written by
// `python bench.py --sweep`; an empty table keeps every default.
#pragma once
#include "tune.h"

namespace tg {

constexpr TuneRule kBuiltinRules[] = {
    {-1, 0, 0, 0, 0, 0, 0, 0, 0, 0},   // placeholder: matches nothing
};

}  // namespace tg
