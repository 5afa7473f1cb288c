// BlockAttention as jagged attention over blocks.
//
// BlockAttention turns long-sequence self-attention into attention inside
// independent fixed-size blocks ("Meta GEM Training Efficiency: Why
// LLM-Scale Recommenders Need a Different Stack", section "Bottleneck move 1";
// "Meta Enhances GEM Training Efficiency with Advanced LLM-Scale
// Innovations", "Exploring the Customized Kernel Library" -> "BlockAttention":
// quadratic to linear cost over the user history).  On a jagged batch that is
// exactly plain jagged attention over the sequences cut into blocks of W
// rows: query i of a sequence sees the keys of block floor(i / W) only, the
// relative-position bias depends on i - j alone, and the GDPA normaliser is
// the block's key count.  So BlockAttention needs no kernel of its own: this
// kernel rewrites the offsets, and the longest-first schedule and the
// attention kernels then skip every tile outside the blocks by construction.
//
// One CTA builds the block offsets: per sequence ceil(n / W) blocks (an
// exclusive scan over the sequences in chunks of the CTA size), then empty
// blocks up to the fixed count batch + total / W, so that the host can size
// the problem without reading anything back.
#include "jfa_common.cuh"

namespace jfa {
namespace {

constexpr int kThreads = 1024;

__global__ void __launch_bounds__(kThreads) block_offsets_kernel(const int32_t* __restrict__ off,
                                                                 int batch, int64_t total, int W,
                                                                 int32_t* __restrict__ out,
                                                                 int64_t n_out) {
    __shared__ int32_t warp_sum[kThreads / 32];
    __shared__ int bad;
    const int t = threadIdx.x, lane = t & 31, w = t >> 5;
    if (t == 0) bad = (off[0] != 0 || (int64_t)off[batch] != total) ? 1 : 0;
    __syncthreads();
    int64_t carry = 0;   // blocks of the sequences before this chunk
    for (int base = 0; base < batch; base += kThreads) {
        const int b = base + t;
        int n = 0, cnt = 0;
        if (b < batch) {
            n = off[b + 1] - off[b];
            if (n < 0) bad = 1;
            cnt = n > 0 ? (n + W - 1) / W : 0;
        }
        // exclusive scan of cnt over the chunk
        int x = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) warp_sum[w] = x;
        __syncthreads();
        if (w == 0) {
            int s = warp_sum[lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, s, o);
                if (lane >= o) s += y;
            }
            warp_sum[lane] = s;   // inclusive over warps
        }
        __syncthreads();
        const int64_t start = carry + (w > 0 ? warp_sum[w - 1] : 0) + (x - cnt);
        const int64_t chunk_total = warp_sum[kThreads / 32 - 1];
        if (b < batch && n > 0)
            for (int c = 0; c < cnt && start + c < n_out; ++c) out[start + c] = off[b] + c * W;
        carry += chunk_total;
        __syncthreads();   // warp_sum is rewritten by the next chunk
    }
    // empty blocks up to the fixed count, and the closing offset
    for (int64_t s = carry + t; s <= n_out; s += kThreads) out[s] = (int32_t)total;
    __syncthreads();
    if (t == 0 && (bad || carry > n_out)) out[0] = -1;   // the attention call reports it
}

}  // namespace
}  // namespace jfa

extern "C" jfa_status jfa_block_offsets(const int32_t* offsets, int32_t batch, int64_t total,
                                        int32_t block, int32_t* block_offsets,
                                        jfa_stream_t stream) {
    if (batch < 0 || total < 0 || block < 1 || !offsets || !block_offsets)
        return jfa::set_last_error(JFA_ERR_INVALID_ARGUMENT,
                                   "block_offsets: bad batch, total, block or NULL pointer");
    const int64_t n_out = (int64_t)batch + total / block;
    if (n_out >= ((int64_t)1 << 31) - 1 || total >= ((int64_t)1 << 31))
        return jfa::set_last_error(JFA_ERR_INVALID_ARGUMENT, "block count must fit int32");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    jfa::block_offsets_kernel<<<1, jfa::kThreads, 0, st>>>(offsets, batch, total, block,
                                                           block_offsets, n_out);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess)
        return jfa::set_last_error(JFA_ERR_CUDA, "block_offsets: %s", cudaGetErrorString(e));
    return JFA_OK;
}
