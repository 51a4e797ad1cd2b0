// tune.h -- the library's tuning table: for each operation and range of M
// (rows of C) and N, which kernel family runs and with which launch shape.
//
// The pages tune kernels by searching a parameter space (the autotuner of
// "TileLang架构深度剖析", 自动调优系统, and the tuning configuration of the
// gtnt.cn tutorial, section 3.3).  Here the kernels are compiled ahead of
// time; what stays open at run time is the kernel family, the number of
// persistent CTAs (the stream-K split of the small-M kernels), the raster
// band height, the fp32 split-K factor and the CTA-pair kernel's ring depth.
// An offline sweep (bench.py --sweep) times those choices on the device and
// writes the built-in rules (tune_table.h); callers may install their own
// rules at run time (tg_tune_set), which are consulted first.
#pragma once
#include <cstdint>

namespace tg {

enum TuneOp : int { OP_BF16 = 0, OP_F16 = 1, OP_W4A16 = 2, OP_WFP4 = 3, OP_F32_FFMA = 4,
                    OP_F32_TF32 = 5, OP_COUNT = 6 };
enum TunePath : int { PATH_AUTO = 0, PATH_CUDA_CORE = 1, PATH_SMALL_M = 2, PATH_CTA_PAIR = 3,
                      PATH_ONE_CTA = 4 };

// One rule; fields left 0 keep the library's default choice.  The same
// fields, in the same order, as tg_tune_rule of the C ABI.
struct TuneRule {
    int32_t op, path;
    int64_t m_lo, m_hi, n_lo, n_hi;     // inclusive ranges of M and N the rule covers
    int32_t ctas;                        // persistent CTAs (CTA pairs for the pair kernels)
    int32_t group_m;                     // raster band height, in tiles (pair tiles)
    int32_t splits;                      // fp32 FFMA: k ranges per output tile
    int32_t stages;                      // 16-bit CTA-pair kernel: ring depth, 4 or 6
};

// The first rule that covers (op, M, N): the run-time rules, then the
// built-in ones; a rule of all-default fields when none does.
TuneRule tune_lookup(int op, int64_t M, int64_t N);

// Whether a rule is well-formed: op and path known, the path serves the op
// and the whole M range (CUDA-core kernels M <= 4 and not FP4 weights,
// small-M kernels M <= 128, fp32 paths only their own), ranges ordered and
// the knobs in range.
bool tune_rule_valid(const TuneRule& r);

}  // namespace tg
