// tune.cu -- the tuning table's storage, lookup and C ABI (tune.h).
#include "tune.h"
#include "tune_table.h"
#include "../../include/tg_gemm.h"

#include <mutex>

namespace tg {

namespace {

constexpr int kMaxRuntimeRules = 64;
std::mutex g_tune_mu;
TuneRule g_rules[kMaxRuntimeRules];
int g_nrules = 0;

bool covers(const TuneRule& r, int op, int64_t M, int64_t N) {
    return r.op == op && r.m_lo <= M && M <= r.m_hi && r.n_lo <= N && N <= r.n_hi;
}

TuneRule from_c(const tg_tune_rule& c) {
    TuneRule r;
    r.op = c.op; r.path = c.path;
    r.m_lo = c.m_lo; r.m_hi = c.m_hi; r.n_lo = c.n_lo; r.n_hi = c.n_hi;
    r.ctas = c.ctas; r.group_m = c.group_m; r.splits = c.splits; r.stages = c.stages;
    return r;
}

void to_c(const TuneRule& r, tg_tune_rule* c) {
    c->op = r.op; c->path = r.path;
    c->m_lo = r.m_lo; c->m_hi = r.m_hi; c->n_lo = r.n_lo; c->n_hi = r.n_hi;
    c->ctas = r.ctas; c->group_m = r.group_m; c->splits = r.splits; c->stages = r.stages;
}

}  // namespace

bool tune_rule_valid(const TuneRule& r) {
    if (r.op < 0 || r.op >= OP_COUNT) return false;
    if (r.m_lo < 1 || r.m_hi < r.m_lo || r.n_lo < 1 || r.n_hi < r.n_lo) return false;
    if (r.ctas < 0 || r.ctas > 4096 || r.group_m < 0 || r.group_m > 256) return false;
    if (r.splits < 0 || r.splits > 8) return false;
    if (r.stages != 0 && r.stages != 4 && r.stages != 6) return false;
    const bool fp32 = r.op == OP_F32_FFMA || r.op == OP_F32_TF32;
    if (r.splits != 0 && r.op != OP_F32_FFMA) return false;
    if (r.stages != 0 && !((r.op == OP_BF16 || r.op == OP_F16) &&
                           (r.path == PATH_AUTO || r.path == PATH_CTA_PAIR)))
        return false;
    switch (r.path) {
        case PATH_AUTO: return true;
        case PATH_CUDA_CORE: return !fp32 && r.m_hi <= 4;
        case PATH_SMALL_M: return !fp32 && r.m_hi <= 128;
        case PATH_CTA_PAIR: return r.op != OP_F32_FFMA;
        case PATH_ONE_CTA: return r.op != OP_F32_FFMA;
        default: return false;
    }
}

TuneRule tune_lookup(int op, int64_t M, int64_t N) {
    {
        std::lock_guard<std::mutex> lk(g_tune_mu);
        for (int i = 0; i < g_nrules; ++i)
            if (covers(g_rules[i], op, M, N)) return g_rules[i];
    }
    for (const TuneRule& r : kBuiltinRules)
        if (covers(r, op, M, N)) return r;
    TuneRule none{};
    none.op = op;
    return none;
}

}  // namespace tg

extern "C" {

tg_status tg_tune_set(const tg_tune_rule* rules, int count) {
    if (count < 0 || count > tg::kMaxRuntimeRules || (count > 0 && !rules)) return TG_ERR_INVALID_ARG;
    tg::TuneRule tmp[tg::kMaxRuntimeRules];
    for (int i = 0; i < count; ++i) {
        tmp[i] = tg::from_c(rules[i]);
        if (!tg::tune_rule_valid(tmp[i])) return TG_ERR_INVALID_ARG;
    }
    std::lock_guard<std::mutex> lk(tg::g_tune_mu);
    for (int i = 0; i < count; ++i) tg::g_rules[i] = tmp[i];
    tg::g_nrules = count;
    return TG_OK;
}

int tg_tune_builtin(tg_tune_rule* out, int capacity) {
    int n = 0;
    for (const tg::TuneRule& r : tg::kBuiltinRules) {
        if (r.op < 0) continue;                     // the empty table's placeholder
        if (out && n < capacity) tg::to_c(r, &out[n]);
        ++n;
    }
    return n;
}

tg_status tg_tune_query(int op, int64_t M, int64_t N, tg_tune_rule* out) {
    if (!out || op < 0 || op >= tg::OP_COUNT || M < 1 || N < 1) return TG_ERR_INVALID_ARG;
    tg::to_c(tg::tune_lookup(op, M, N), out);
    return TG_OK;
}

}  // extern "C"
