// Jagged tile scheduler.
//
// Removing padding leaves short and long samples finishing at different times,
// so tile scheduling becomes the exposed bottleneck ("Meta GEM Training
// Efficiency: Why LLM-Scale Recommenders Need a Different Stack", section
// "Bottleneck move 1: dense-sequence kernels to jagged execution").
//
// Query-tile schedule (forward): every (sequence, head, tile) work item
// longest-first (cost = (query, key) pairs the tile computes; ties by
// sequence, tile, head ascending), so that a grid or a persistent queue that
// takes items in order runs the long causal tiles first and fills the tail
// with short ones.
//
// Short query sequences (every n_q <= 64, one item per (sequence, head)):
// the kernels stream the item's key/value tiles, each costing the same HBM
// bytes whatever n_q is, so these items are ranked by their 128-key tiles
// first (pairs only break ties): ranking them by pairs alone spreads the key
// tiles unevenly over the CTAs.
//
// Key-tile schedule (backward): the items of one (sequence, head) are kept
// together, so that the key tiles that read the same query / dO tiles and add
// into the same dQ rows run at the same time and share them through L2.
// Sequences longest-first (cost = the sequence's (query, key) pairs; ties by
// sequence), then heads ascending, then key tiles ascending (for causal
// attention the first key tile is the longest).
//
// Two kernels:
//   sched_prepare  one CTA: validates the offsets, enumerates the
//                  (sequence, tile) pairs with their costs, and (dense bias)
//                  the int64 start of each sequence's bias block.
//   sched_rank     one thread per pair: rank = number of pairs that precede
//                  it in the total order; writes H items at rank * H.
#include "jfa_common.cuh"

namespace jfa {

namespace {

constexpr int kPrepThreads = 1024;

// Pairs (query, key) computed by rows [lo, hi) of a query tile.
__device__ int64_t query_tile_cost(int lo, int hi, int nq, int nkv, int causal, int window) {
    if (!causal && window <= 0) return (int64_t)(hi - lo) * nkv;
    int64_t c = 0;
    for (int i = lo; i < hi; ++i) {
        const int vis = vis_key_hi(causal, window, i, nq, nkv) - vis_key_lo(window, i, nq, nkv) + 1;
        c += vis > 0 ? vis : 0;
    }
    return c;
}

// Pairs computed by key rows [lo, hi) of a key/value tile.
__device__ int64_t key_tile_cost(int lo, int hi, int nq, int nkv, int causal, int window) {
    if (!causal && window <= 0) return (int64_t)(hi - lo) * nq;
    int64_t c = 0;
    for (int j = lo; j < hi; ++j) {
        const int cnt = vis_query_hi(window, j, nq, nkv) - vis_query_lo(causal, window, j, nq, nkv) + 1;
        c += cnt > 0 ? cnt : 0;
    }
    return c;
}

__global__ void __launch_bounds__(kPrepThreads)
sched_prepare(const int32_t* __restrict__ q_off, const int32_t* __restrict__ kv_off, int B, int H,
              int max_q, int max_kv, int64_t total_q, int64_t total_kv, int causal, int window,
              int backward,
              int tile, int64_t pairs_cap, int want_dense, WsHeader* hdr, int64_t* dense_off,
              int2* pair_bt, int64_t* pair_cost, int32_t* pair_count_out, int reset_err,
              int64_t* seq_tmp, int64_t* seq_start, int wait_limit_us, int cost_tiles) {
    __shared__ int s_bad;
    __shared__ int64_t s_scan[kPrepThreads];
    __shared__ int64_t s_dscan[kPrepThreads];
    const int tid = threadIdx.x;
    if (tid == 0) {
        s_bad = 0;
        if (backward) hdr->kv_queue = 0;   // work-item counter of the persistent backward
        if (reset_err) {
            hdr->err = 0;
            hdr->wait_limit_us = wait_limit_us;
        }
    }
    __syncthreads();
    // 1. validation of both offset arrays
    for (int b = tid; b <= B; b += kPrepThreads) {
        int bad = 0;
        if (b == 0) bad |= (q_off[0] != 0) | (kv_off[0] != 0);
        if (b == B) bad |= ((int64_t)q_off[B] != total_q) | ((int64_t)kv_off[B] != total_kv);
        if (b < B) {
            int nq = q_off[b + 1] - q_off[b], nkv = kv_off[b + 1] - kv_off[b];
            bad |= (nq < 0) | (nkv < 0) | (nq > max_q) | (nkv > max_kv);
        }
        if (bad) atomicOr(&s_bad, 1);
    }
    __syncthreads();
    if (s_bad) {
        if (tid == 0) {
            set_error(hdr, JFA_ERR_BAD_OFFSETS);
            *pair_count_out = 0;
        }
        return;
    }
    // 2. enumerate pairs: exclusive scan of ceil(n/tile) over sequences, in
    //    chunks of kPrepThreads with a running carry
    int64_t carry = 0, dcarry = 0;
    for (int base = 0; base < B; base += kPrepThreads) {
        int b = base + tid;
        int64_t nt = 0, dn = 0;
        int nq = 0, nkv = 0;
        if (b < B) {
            nq = q_off[b + 1] - q_off[b];
            nkv = kv_off[b + 1] - kv_off[b];
            int rows = backward ? nkv : nq;
            nt = (rows + tile - 1) / tile;
            dn = (int64_t)H * nq * nkv;
        }
        s_scan[tid] = nt;
        s_dscan[tid] = dn;
        __syncthreads();
        for (int off = 1; off < kPrepThreads; off <<= 1) {  // Hillis-Steele inclusive scan
            int64_t x = tid >= off ? s_scan[tid - off] : 0;
            int64_t y = tid >= off ? s_dscan[tid - off] : 0;
            __syncthreads();
            s_scan[tid] += x;
            s_dscan[tid] += y;
            __syncthreads();
        }
        int64_t first = carry + s_scan[tid] - nt;
        if (b < B) {
            if (want_dense) dense_off[b] = dcarry + s_dscan[tid] - dn;
            if (seq_start != nullptr) seq_start[b] = first;   // the sequence's first pair (step 4)
            for (int64_t t = 0; t < nt && first + t < pairs_cap; ++t)
                pair_bt[first + t] = make_int2(b, (int)t);
        }
        int64_t chunk_total = s_scan[kPrepThreads - 1], dchunk = s_dscan[kPrepThreads - 1];
        __syncthreads();
        carry += chunk_total;
        dcarry += dchunk;
    }
    if (tid == 0) {
        if (want_dense) dense_off[B] = dcarry;
        *pair_count_out = (int32_t)(carry < pairs_cap ? carry : pairs_cap);
    }
    __syncthreads();
    // 3. cost of each pair
    const int64_t npairs = carry < pairs_cap ? carry : pairs_cap;
    for (int64_t p = tid; p < npairs; p += kPrepThreads) {
        int2 bt = pair_bt[p];
        int nq = q_off[bt.x + 1] - q_off[bt.x], nkv = kv_off[bt.x + 1] - kv_off[bt.x];
        int rows = backward ? nkv : nq;
        int lo = bt.y * tile, hi = min(rows, lo + tile);
        int64_t c = backward ? key_tile_cost(lo, hi, nq, nkv, causal, window)
                             : query_tile_cost(lo, hi, nq, nkv, causal, window);
        if (cost_tiles) {
            // 128-key tiles of the item's visible key range, then its pairs
            // (the short-query kernels run only without a window)
            int kv_end = causal ? min(nkv, hi + (nkv - nq)) : nkv;
            kv_end = kv_end < 0 ? 0 : kv_end;
            c = ((int64_t)((kv_end + 127) / 128) << 32) | (c < 0xffffffffll ? c : 0xffffffffll);
        }
        pair_cost[p] = c;
    }
    if (seq_start == nullptr) return;
    // 4. sequence order of the grouped (key-tile) schedule: seq_start[b] =
    //    tiles of the sequences ranked before b (cost descending, then b);
    //    a sequence's cost is the sum of its pairs' costs from step 3
    __syncthreads();
    for (int b = tid; b < B; b += kPrepThreads) {
        const int rows = backward ? kv_off[b + 1] - kv_off[b] : q_off[b + 1] - q_off[b];
        const int64_t first = seq_start[b];
        const int64_t last = min(first + (rows + tile - 1) / tile, npairs);
        int64_t c = 0;
        for (int64_t p = first; p < last; ++p) c += pair_cost[p];
        seq_tmp[b] = c;
    }
    __syncthreads();
    for (int b = tid; b < B; b += kPrepThreads) {
        const int64_t mine = seq_tmp[b];
        int64_t rank = 0;
        for (int o = 0; o < B; ++o) {
            const int64_t c = seq_tmp[o];
            rank += (c > mine) | ((c == mine) & (o < b));
        }
        seq_start[b] = rank;
    }
    __syncthreads();
    for (int b = tid; b < B; b += kPrepThreads) {
        const int rows = backward ? kv_off[b + 1] - kv_off[b] : q_off[b + 1] - q_off[b];
        seq_tmp[seq_start[b]] = (rows + tile - 1) / tile;
    }
    __syncthreads();
    carry = 0;   // exclusive scan of the tile counts in rank order
    for (int base = 0; base < B; base += kPrepThreads) {
        const int i = base + tid;
        const int64_t v = i < B ? seq_tmp[i] : 0;
        s_scan[tid] = v;
        __syncthreads();
        for (int off = 1; off < kPrepThreads; off <<= 1) {
            int64_t x = tid >= off ? s_scan[tid - off] : 0;
            __syncthreads();
            s_scan[tid] += x;
            __syncthreads();
        }
        if (i < B) seq_tmp[i] = carry + s_scan[tid] - v;
        const int64_t chunk_total = s_scan[kPrepThreads - 1];
        __syncthreads();
        carry += chunk_total;
    }
    __syncthreads();
    for (int b = tid; b < B; b += kPrepThreads) seq_start[b] = seq_tmp[seq_start[b]];
}

constexpr int kRankThreads = 256;
constexpr int kRankChunk = 2048;

__global__ void __launch_bounds__(kRankThreads)
sched_rank(const int2* __restrict__ pair_bt, const int64_t* __restrict__ pair_cost,
           const int32_t* __restrict__ pair_count, int H, int4* __restrict__ items,
           int32_t* __restrict__ item_count, const int64_t* __restrict__ seq_start,
           const int32_t* __restrict__ rows_off, int tile) {
    __shared__ int64_t s_cost[kRankChunk];
    const int n = *pair_count;
    const int p = blockIdx.x * kRankThreads + threadIdx.x;
    if (p == 0) *item_count = n * H;
    if (blockIdx.x * kRankThreads >= n) return;
    if (seq_start != nullptr) {  // grouped: (sequence, head) blocks of consecutive tiles
        if (p < n) {
            const int2 bt = pair_bt[p];
            const int64_t mine = pair_cost[p];
            const int cost32 = mine > 0x7fffffff ? 0x7fffffff : (int)mine;
            const int nt = (rows_off[bt.x + 1] - rows_off[bt.x] + tile - 1) / tile;
            const int64_t first = seq_start[bt.x] * H;
            for (int h = 0; h < H; ++h) items[first + (int64_t)h * nt + bt.y] = make_int4(bt.x, h, bt.y, cost32);
        }
        return;
    }
    const int64_t mine = p < n ? pair_cost[p] : 0;
    int rank = 0;
    for (int base = 0; base < n; base += kRankChunk) {
        int cnt = min(kRankChunk, n - base);
        __syncthreads();
        for (int t = threadIdx.x; t < cnt; t += kRankThreads) s_cost[t] = pair_cost[base + t];
        __syncthreads();
        if (p < n) {
            for (int t = 0; t < cnt; ++t) {
                int64_t c = s_cost[t];
                rank += (c > mine) | ((c == mine) & (base + t < p));
            }
        }
    }
    if (p < n) {
        int2 bt = pair_bt[p];
        int cost32 = mine > 0x7fffffff ? 0x7fffffff : (int)mine;
        for (int h = 0; h < H; ++h) items[(int64_t)rank * H + h] = make_int4(bt.x, h, bt.y, cost32);
    }
}

}  // namespace

// Builds the schedule on `stream`.  Returns a CUDA error code (0 on success).
cudaError_t build_schedule(const jfa_problem& pb, const int32_t* q_off, const int32_t* kv_off,
                           int causal, int backward, int tile, WsHeader* hdr, int64_t* dense_off,
                           int2* pair_bt, int64_t* pair_cost, int64_t pairs_cap, int4* items,
                           int32_t* item_count, int32_t* pair_count, int reset_err,
                           int64_t* seq_tmp, int64_t* seq_start, cudaStream_t stream,
                           int wait_limit_us, int cost_tiles) {
    int want_dense = (pb.bias_kind == JFA_BIAS_DENSE_JAGGED && dense_off != nullptr) ? 1 : 0;
    prof_begin(stream);
    sched_prepare<<<1, kPrepThreads, 0, stream>>>(
        q_off, kv_off, pb.batch, pb.heads, pb.max_q_len, pb.max_kv_len, pb.total_q, pb.total_kv,
        causal, pb.window, backward, tile, pairs_cap, want_dense, hdr, dense_off, pair_bt, pair_cost,
        pair_count, reset_err, seq_tmp, seq_start, wait_limit_us, cost_tiles);
    prof_end(stream, K_SCHED_PREPARE);
    int64_t bound = pairs_bound(pb.batch, backward ? pb.max_kv_len : pb.max_q_len,
                                backward ? pb.total_kv : pb.total_q, tile);
    if (bound > pairs_cap) bound = pairs_cap;
    int grid = (int)((bound + kRankThreads - 1) / kRankThreads);
    if (grid < 1) grid = 1;
    prof_begin(stream);
    sched_rank<<<grid, kRankThreads, 0, stream>>>(pair_bt, pair_cost, pair_count, pb.heads, items,
                                                  item_count, seq_start, backward ? kv_off : q_off,
                                                  tile);
    prof_end(stream, K_SCHED_RANK);
    return cudaGetLastError();
}

}  // namespace jfa
