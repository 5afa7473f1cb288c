// Host-side partition of one global batch of jagged sequences across data-
// parallel ranks.
//
// Sequences are independent in the forward and the backward, so a batch
// shards across GPUs with no collective on the data path; what matters is
// that every rank gets about the same work.  Removing padding exposes rank
// imbalance ("Meta GEM Training Efficiency: Why LLM-Scale Recommenders Need a
// Different Stack", section "Bottleneck move 4: memory relief to load
// balance": the heaviest rank ran ~15% above the average, and a global
// rebalance would cost an all-to-all every step).  Two rules, both computed
// identically on every rank from the lengths alone, so no rank needs to talk
// to another:
//
//   JFA_PARTITION_LPT  longest processing time first: sequences by cost
//                      (visible (query, key) pairs) descending, ties by
//                      index, each to the currently least-loaded rank (ties:
//                      lowest rank).
//   JFA_PARTITION_BBS  base batch shuffling as that section describes it:
//                      the batch is cut into sub-batches of `sub_batch`
//                      consecutive sequences, the sub-batches are sorted by
//                      total sequence length (sum of n_q + n_kv, descending,
//                      ties by sub-batch index) and dealt to the ranks in
//                      snake order (0..R-1, R-1..0, ...), which pairs the
//                      heavy sub-batches of one round with the light ones of
//                      the next.
#include <algorithm>
#include <numeric>
#include <queue>
#include <vector>

#include "jfa_common.cuh"

namespace {

// Visible (query, key) pairs of one sequence; bottom-right causal: query i
// sees keys j <= i + n_kv - n_q; a sliding window w > 0 keeps the keys with
// p - j < w (and, without the causal rule, j - p < w), p = i + n_kv - n_q.
int64_t visible_pairs(int64_t nq, int64_t nkv, int causal, int32_t window) {
    if (nq <= 0 || nkv <= 0) return 0;
    if (window > 0) {
        int64_t c = 0;
        for (int64_t i = 0; i < nq; ++i) {
            const int64_t p = i + nkv - nq;
            const int64_t hi = std::min(nkv - 1, causal ? p : p + window - 1);
            const int64_t lo = std::max<int64_t>(0, p - window + 1);
            c += hi >= lo ? hi - lo + 1 : 0;
        }
        return c;
    }
    if (!causal) return nq * nkv;
    const int64_t s = nkv - nq;
    if (s >= 0) return nq * (nq + 1) / 2 + nq * s;
    return nkv * (nkv + 1) / 2;  // the first -s query rows see no key
}

}  // namespace

extern "C" jfa_status jfa_partition(int32_t batch, const int32_t* q_lens, const int32_t* kv_lens,
                                    int causal, int32_t window, int32_t ranks, int method,
                                    int32_t sub_batch, int32_t* rank_of, int64_t* rank_cost) {
    if (batch < 0 || ranks < 1 || window < 0)
        return jfa::set_last_error(JFA_ERR_INVALID_ARGUMENT, "batch, window must be >= 0 and ranks >= 1");
    if (batch > 0 && (!q_lens || !kv_lens || !rank_of))
        return jfa::set_last_error(JFA_ERR_INVALID_ARGUMENT, "NULL lengths or rank_of");
    if (method != JFA_PARTITION_LPT && method != JFA_PARTITION_BBS)
        return jfa::set_last_error(JFA_ERR_INVALID_ARGUMENT, "bad partition method %d", method);
    if (method == JFA_PARTITION_BBS && sub_batch < 1)
        return jfa::set_last_error(JFA_ERR_INVALID_ARGUMENT, "sub_batch must be >= 1");
    std::vector<int64_t> cost(batch);
    for (int32_t b = 0; b < batch; ++b) {
        if (q_lens[b] < 0 || kv_lens[b] < 0)
            return jfa::set_last_error(JFA_ERR_INVALID_ARGUMENT, "negative length at %d", b);
        cost[b] = visible_pairs(q_lens[b], kv_lens[b], causal, window);
    }
    std::vector<int64_t> load(ranks, 0);
    if (method == JFA_PARTITION_LPT) {
        std::vector<int32_t> order(batch);
        std::iota(order.begin(), order.end(), 0);
        std::stable_sort(order.begin(), order.end(),
                         [&](int32_t x, int32_t y) { return cost[x] > cost[y]; });
        // min-heap of (load, rank)
        typedef std::pair<int64_t, int32_t> Slot;
        std::priority_queue<Slot, std::vector<Slot>, std::greater<Slot>> heap;
        for (int32_t r = 0; r < ranks; ++r) heap.push(Slot(0, r));
        for (int32_t b : order) {
            Slot s = heap.top();
            heap.pop();
            rank_of[b] = s.second;
            s.first += cost[b];
            heap.push(s);
        }
    } else {
        const int32_t n_sub = (batch + sub_batch - 1) / sub_batch;
        std::vector<int64_t> len(n_sub, 0);
        for (int32_t b = 0; b < batch; ++b) len[b / sub_batch] += (int64_t)q_lens[b] + kv_lens[b];
        std::vector<int32_t> order(n_sub);
        std::iota(order.begin(), order.end(), 0);
        std::stable_sort(order.begin(), order.end(),
                         [&](int32_t x, int32_t y) { return len[x] > len[y]; });
        for (int32_t pos = 0; pos < n_sub; ++pos) {
            const int32_t round = pos / ranks, c = pos % ranks;
            const int32_t r = (round & 1) ? ranks - 1 - c : c;
            const int32_t g = order[pos];
            for (int32_t b = g * sub_batch; b < std::min(batch, (g + 1) * sub_batch); ++b) rank_of[b] = r;
        }
    }
    for (int32_t b = 0; b < batch; ++b) load[rank_of[b]] += cost[b];
    if (rank_cost)
        for (int32_t r = 0; r < ranks; ++r) rank_cost[r] = load[r];
    return JFA_OK;
}
