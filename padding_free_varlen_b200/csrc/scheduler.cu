// Dynamic batching of a request queue (host runtime, no device code).
//
// The QbitAI article's "Serving" section and the EnergonAI README's "Batching"
// section: queued requests are packed into batches as the machine's performance
// suits best, and the batch of highest priority - from the waiting time, the
// batch size and the batch's length after padding - runs first, which keeps the
// GPU busy without starving anyone; the method follows TurboTransformer's
// dynamic-programming batch scheduler and is compared against FIFO packing.
//
// The pages give no formula; this file implements one reading of them:
//   packing  requests sorted by (length, arrival, index) are cut into consecutive
//            groups of at most max_batch, the cut minimising the summed cost of
//            the groups, cost(b, s) read from a table measured on the machine
//            (b sequences padded to s tokens);
//   priority (tokens in the group) / cost(size, longest length)
//            * (1 + waiting time of the oldest request / age_scale);
//   ties     the scan over group starts keeps the first minimum (the larger last
//            group); equal priorities keep ascending group order.
// Every double is formed in the same order as the statement of the method, so the
// decisions are reproducible bit for bit.
#include <algorithm>
#include <cmath>
#include <vector>

#include "energon_rce.h"

namespace energon {
void record_error(int code, const char* msg);
}

namespace {

int bad(const char* msg) {
    energon::record_error(ENERGON_ERR_INVALID_ARGUMENT, msg);
    return ENERGON_ERR_INVALID_ARGUMENT;
}

}  // namespace

extern "C" int energon_sched_plan(const energon_request* reqs, int n, double now_s, int max_batch,
                                  const double* cost_table, int table_max_len, double age_scale_s,
                                  int32_t* group_of, int32_t* n_groups, int32_t* order) {
    energon::record_error(ENERGON_OK, "");
    if (n < 0 || !n_groups || (n > 0 && (!reqs || !group_of || !order || !cost_table)))
        return bad("sched_plan: NULL pointer or negative count");
    if (max_batch < 1 || table_max_len < 1) return bad("sched_plan: max_batch and table_max_len must be >= 1");
    if (!(age_scale_s > 0.0) || !std::isfinite(now_s)) return bad("sched_plan: age_scale must be > 0, now finite");
    *n_groups = 0;
    if (n == 0) return ENERGON_OK;
    for (int i = 0; i < n; ++i) {
        if (reqs[i].length < 1 || reqs[i].length > table_max_len)
            return bad("sched_plan: a request length is outside [1, table_max_len]");
        if (!std::isfinite(reqs[i].arrival_s)) return bad("sched_plan: a request arrival time is not finite");
    }
    const int used_b = std::min(max_batch, n);
    for (int64_t k = 0; k < (int64_t)used_b * table_max_len; ++k)
        if (!(cost_table[k] > 0.0) || !std::isfinite(cost_table[k]))
            return bad("sched_plan: cost table entries must be finite and > 0");
    auto cost = [&](int b, int s) { return cost_table[(int64_t)(b - 1) * table_max_len + (s - 1)]; };

    // length order
    std::vector<int> idx(n);
    for (int i = 0; i < n; ++i) idx[i] = i;
    std::sort(idx.begin(), idx.end(), [&](int a, int b) {
        if (reqs[a].length != reqs[b].length) return reqs[a].length < reqs[b].length;
        if (reqs[a].arrival_s != reqs[b].arrival_s) return reqs[a].arrival_s < reqs[b].arrival_s;
        return a < b;
    });
    // DP over cuts: best[j] = cheapest packing of the first j requests in length order
    std::vector<double> best(n + 1, 0.0);
    std::vector<int> cut(n + 1, 0);
    for (int j = 1; j <= n; ++j) {
        bool set = false;
        const int s = reqs[idx[j - 1]].length;  // the group's padded length
        for (int i = std::max(0, j - max_batch); i < j; ++i) {
            const double c = best[i] + cost(j - i, s);
            if (!set || c < best[j]) {
                best[j] = c;
                cut[j] = i;
                set = true;
            }
        }
    }
    std::vector<std::pair<int, int>> groups;
    for (int j = n; j > 0; j = cut[j]) groups.emplace_back(cut[j], j);
    std::reverse(groups.begin(), groups.end());
    const int ng = (int)groups.size();
    std::vector<double> prio(ng);
    for (int g = 0; g < ng; ++g) {
        const int a = groups[g].first, b = groups[g].second;
        int64_t tokens = 0;
        double oldest = reqs[idx[a]].arrival_s;
        for (int k = a; k < b; ++k) {
            group_of[idx[k]] = g;
            tokens += reqs[idx[k]].length;
            oldest = std::min(oldest, reqs[idx[k]].arrival_s);
        }
        const double wait = now_s - oldest;
        prio[g] = (double)tokens / cost(b - a, reqs[idx[b - 1]].length) * (1.0 + wait / age_scale_s);
    }
    for (int g = 0; g < ng; ++g) order[g] = g;
    std::sort(order, order + ng, [&](int32_t a, int32_t b) {
        if (prio[a] != prio[b]) return prio[a] > prio[b];
        return a < b;
    });
    *n_groups = ng;
    return ENERGON_OK;
}

extern "C" int energon_sched_fifo(const energon_request* reqs, int n, int max_batch, int32_t* group_of,
                                  int32_t* n_groups) {
    energon::record_error(ENERGON_OK, "");
    if (n < 0 || !n_groups || (n > 0 && (!reqs || !group_of))) return bad("sched_fifo: NULL pointer or negative count");
    if (max_batch < 1) return bad("sched_fifo: max_batch must be >= 1");
    for (int i = 0; i < n; ++i)
        if (!std::isfinite(reqs[i].arrival_s)) return bad("sched_fifo: a request arrival time is not finite");
    std::vector<int> idx(n);
    for (int i = 0; i < n; ++i) idx[i] = i;
    std::sort(idx.begin(), idx.end(), [&](int a, int b) {
        if (reqs[a].arrival_s != reqs[b].arrival_s) return reqs[a].arrival_s < reqs[b].arrival_s;
        return a < b;
    });
    for (int k = 0; k < n; ++k) group_of[idx[k]] = k / max_batch;
    *n_groups = (n + max_batch - 1) / max_batch;
    return ENERGON_OK;
}
