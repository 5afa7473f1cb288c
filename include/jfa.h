/*
 * jfa.h -- C ABI of libjfa: jagged (offsets-indexed, unpadded) attention
 * forward and backward for NVIDIA B200 (sm_100a).
 *
 * What it computes.  Attention run directly on variable-length user-sequence
 * tensors stored as values plus offsets, with custom additive biases and
 * asymmetric query / key-value lengths ("Meta GEM Training Efficiency: Why
 * LLM-Scale Recommenders Need a Different Stack", section "Bottleneck move 1:
 * dense-sequence kernels to jagged execution", and its FAQ "What is a jagged
 * tensor?"); the GDPA variant that replaces softmax with a pointwise SiLU or
 * GELU (same section); asymmetric shapes as in "GEM Training: How Meta
 * Doubled the Efficiency of Its LLM-Scale Ads Foundation Model", "Challenge 1:
 * Achieving High Per-GPU Utilization"; and MXFP8 attention (same page, opening
 * summary) with the OCP MX v1.0 E4M3 element / E8M0 scale formats.
 *
 * For sequence b, query rows are [q_offsets[b], q_offsets[b+1]) and key/value
 * rows [kv_offsets[b], kv_offsets[b+1]); n_q(b), n_kv(b) are their counts.
 * With tau = scale (<= 0 selects 1/sqrt(head_dim)) and beta the bias:
 *   s_ij  = tau * <q_i, k_j> + beta_h(i, j)
 *   valid = !causal || j <= i + n_kv(b) - n_q(b)      (bottom-right aligned)
 *   softmax: o_i = sum_valid softmax_j(s_ij) v_j,  lse_i = log sum_valid e^{s_ij}
 *   GDPA   : o_i = sum_valid act(s_ij) / n_kv(b) * v_j           (no lse)
 * A query row with no valid key gets o_i = 0 and lse_i = -inf; its gradients
 * are 0.  jfa_backward leaves the bias alone; jfa_backward_dbias also returns
 * its gradient.
 *
 * Layouts (all row-major, head_dim contiguous):
 *   q, out, dout, dq : [total_q ][heads][head_dim]
 *   k, v, dk, dv     : [total_kv][heads][head_dim]
 *   lse              : [total_q ][heads]  fp32, natural log
 *   bias RELPOS      : fp32 [heads][relpos_len], beta_h(i,j) =
 *                      table[h][clamp(i - j, -C, C) + C], C = (relpos_len-1)/2
 *   bias DENSE_JAGGED: element type of q; for each sequence in order a block
 *                      [heads][n_q(b)][n_kv(b)] (keys contiguous); blocks are
 *                      concatenated, so block b starts at
 *                      sum_{b'<b} heads * n_q(b') * n_kv(b') (int64).
 * Element type: JFA_F32 -> float; JFA_BF16 and JFA_MXFP8 -> bfloat16 (MXFP8
 * quantises Q, K and V to E4M3 with E8M0 scales per 32 inside the call and
 * runs block-scaled E4M3 MMAs; outputs stay bf16).
 *
 * Conventions shared by every entry point:
 *  - Ownership: the caller owns every buffer.  All tensor, offset and
 *    workspace pointers are DEVICE pointers (cudaMalloc / torch); the problem
 *    descriptor is a HOST pointer read during the call only.  The library
 *    allocates nothing and keeps no state between calls.
 *  - Inputs are never written.  Outputs are written only on valid rows of
 *    their own sequences.
 *  - Streams: all work is enqueued on `stream` (NULL = legacy default stream);
 *    there is no host synchronisation.  max_q_len / max_kv_len / total_* come
 *    from the host so that no device->host copy is needed to size grids.
 *    So the compute calls (forward, backward, quantisers, schedule) can be
 *    captured in a CUDA graph and replayed on new data written into the same
 *    buffers (the work-item counters and the error word are reset by each
 *    call's schedule); jfa_check_error() synchronises and is not for capture.
 *  - Alignment: tensors 16-byte aligned.
 *  - Errors are returned, never thrown; nothing aborts or traps.  Argument
 *    errors are detected on the host before anything is enqueued.  Offsets
 *    are validated ON THE DEVICE (off[0] == 0, non-decreasing, last == total,
 *    lengths <= max_*_len); a bad batch enqueues no work on invalid rows and
 *    leaves JFA_ERR_BAD_OFFSETS in the workspace's error word, which
 *    jfa_check_error() reads.  Asynchronous CUDA faults surface as
 *    JFA_ERR_CUDA.  jfa_last_error() describes the last non-OK status of the
 *    calling thread.
 */
#ifndef JFA_H_
#define JFA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t. */
typedef struct CUstream_st* jfa_stream_t;

typedef enum {
    JFA_OK = 0,
    JFA_ERR_INVALID_ARGUMENT = 1, /* null pointer, bad size or enum */
    JFA_ERR_UNSUPPORTED = 2,      /* valid but not implemented (e.g. head_dim 96) */
    JFA_ERR_WORKSPACE = 3,        /* workspace smaller than jfa_workspace_bytes() */
    JFA_ERR_CUDA = 4,             /* a CUDA launch or runtime call failed */
    JFA_ERR_TIMEOUT = 5,          /* a bounded on-device wait gave up */
    JFA_ERR_BAD_OFFSETS = 6       /* offsets failed the on-device validation */
} jfa_status;

typedef enum { JFA_F32 = 0, JFA_BF16 = 1, JFA_MXFP8 = 2 } jfa_dtype;

typedef enum { JFA_ACT_SOFTMAX = 0, JFA_ACT_SILU = 1, JFA_ACT_GELU_TANH = 2 } jfa_act;

typedef enum { JFA_BIAS_NONE = 0, JFA_BIAS_RELPOS = 1, JFA_BIAS_DENSE_JAGGED = 2 } jfa_bias_kind;

/* Problem descriptor (host memory).  head_dim in {32, 64, 128}; the bf16
 * tensor-core kernels need head_dim == 128, other sizes run on the CUDA-core
 * kernels. */
typedef struct {
    int32_t batch;       /* number of sequences B >= 0 */
    int32_t heads;       /* H >= 1 (query and key/value heads are equal) */
    int32_t head_dim;    /* d */
    int32_t max_q_len;   /* >= every n_q(b) */
    int32_t max_kv_len;  /* >= every n_kv(b) */
    int64_t total_q;     /* q_offsets[B] */
    int64_t total_kv;    /* kv_offsets[B] */
    jfa_dtype dtype;
    float scale;         /* tau; <= 0 selects 1/sqrt(head_dim) */
    jfa_bias_kind bias_kind;
    int32_t relpos_len;  /* odd table length for JFA_BIAS_RELPOS, else ignored */
    int32_t window;      /* sliding-window width w >= 0; 0 = no window (below) */
} jfa_problem;

/* Masks.  Query i of a sequence sits at the bottom-right aligned key position
 * p = i + n_kv - n_q (p = i for self-attention).  causal = 1: key j is
 * visible only when j <= p.  Sliding window (windowed attention: "Meta
 * Enhances GEM Training Efficiency with Advanced LLM-Scale Innovations",
 * "Exploring the Customized Kernel Library" -> "BlockAttention", windows
 * instead of full attention over long user histories): with window = w > 0
 * key j is visible only when p - j < w, and, without the causal rule, also
 * when j - p < w (a band of 2w - 1 keys around p).  Causal with w keeps the
 * w most recent positions up to p.  Only the key tiles inside the band are
 * computed; GDPA still divides by n_kv.  A query row that sees no key gets a
 * zero output and LSE = -inf.  A negative window is
 * JFA_ERR_INVALID_ARGUMENT. */

/* Bytes of device workspace that jfa_forward (backward = 0) or jfa_backward
 * (backward = 1) needs for this problem; 0 if the descriptor is invalid.
 * The workspace holds the tile schedule, the error word and, for the
 * backward, the fp32 dQ accumulator and the row terms D = rowsum(dO * O). */
size_t jfa_workspace_bytes(const jfa_problem* problem, int backward);

/* Forward pass.  q, k, v: device tensors as above; q_offsets, kv_offsets:
 * device int32 [batch + 1]; bias: device pointer in the layout of
 * problem->bias_kind (NULL for JFA_BIAS_NONE); act: softmax or GDPA
 * activation; causal: 0/1; out: device [total_q][heads][head_dim] in the
 * element type; lse: device fp32 [total_q][heads] for softmax (may be NULL if
 * not needed), ignored for GDPA; workspace: device buffer of ws_bytes >=
 * jfa_workspace_bytes(problem, 0), 16-byte aligned. */
jfa_status jfa_forward(const jfa_problem* problem, const void* q, const void* k, const void* v,
                       const int32_t* q_offsets, const int32_t* kv_offsets, const void* bias,
                       jfa_act act, int causal, void* out, float* lse, void* workspace,
                       size_t ws_bytes, jfa_stream_t stream);

/* MXFP8 forward on operands that their producer has already quantised (a
 * normalisation or projection kernel that writes MX directly, such as
 * jfa_norm_quantize_mxfp8), so that no separate cast pass runs ("Meta GEM
 * Training Efficiency: Why LLM-Scale Recommenders Need a Different Stack",
 * "Bottleneck move 2": scale generation and casting must not eat the
 * low-precision gain).  Softmax attention with block-scaled E4M3 MMAs, P
 * quantised per 32 keys in the kernel; problem->dtype must be JFA_MXFP8 and
 * head_dim 128 (else JFA_ERR_UNSUPPORTED).  Device inputs, in the layouts of
 * jfa_quantize_mxfp8:
 *   q8, k8, v8         E4M3 codes [rows][heads][128]
 *   q_scales, k_scales E8M0 [rows][heads][4], blocks of 32 along d
 *   v_scales           E8M0 [blocks][heads][128], blocks of 32 keys of each
 *                      sequence counted from its first key (along_rows = 1)
 * Everything else (offsets, bias, causal, out bf16, lse, workspace of
 * jfa_workspace_bytes(problem, 0), stream, errors) is as for jfa_forward. */
jfa_status jfa_forward_mxfp8(const jfa_problem* problem, const uint8_t* q8, const uint8_t* q_scales,
                             const uint8_t* k8, const uint8_t* k_scales, const uint8_t* v8,
                             const uint8_t* v_scales, const int32_t* q_offsets,
                             const int32_t* kv_offsets, const void* bias, int causal, void* out,
                             float* lse, void* workspace, size_t ws_bytes, jfa_stream_t stream);

/* Backward pass: gradients of <dout, out> with respect to q, k and v.
 * out and lse are the forward's results (softmax needs both; GDPA needs
 * neither and accepts NULL); dout: device like out.  dq/dk/dv: device
 * outputs in the element type (every valid row is written).  workspace:
 * >= jfa_workspace_bytes(problem, 1). */
jfa_status jfa_backward(const jfa_problem* problem, const void* q, const void* k,
                        const void* v, const void* out, const float* lse, const void* dout,
                        const int32_t* q_offsets, const int32_t* kv_offsets, const void* bias,
                        jfa_act act, int causal, void* dq, void* dk, void* dv, void* workspace,
                        size_t ws_bytes, jfa_stream_t stream);

/* Backward pass that also returns the gradient of the additive bias
 * ("custom biases", "Meta GEM Training Efficiency: Why LLM-Scale Recommenders
 * Need a Different Stack", section "Bottleneck move 1": a trainable bias needs
 * one).  With s_ij = tau <q_i, k_j> + beta_h(i, j) the gradient of a bias
 * entry is the sum of the score gradients ds_ij of the valid pairs that read
 * it:
 *   JFA_BIAS_RELPOS      : dbias fp32 [heads][relpos_len] (the table's
 *                          layout), dbias[h][clamp(i - j, -C, C) + C] =
 *                          sum of ds_ij over every sequence; overwritten.
 *   JFA_BIAS_DENSE_JAGGED: dbias in the bias's layout and element type: ds_ij
 *                          at each valid pair, 0 at each masked pair of the
 *                          sequence's [heads][n_q][n_kv] block.
 * dbias is a device pointer, 16-byte aligned; NULL gives jfa_backward.  The
 * other arguments, outputs and errors are those of jfa_backward; a problem
 * with JFA_BIAS_NONE and a non-NULL dbias is JFA_ERR_INVALID_ARGUMENT. */
jfa_status jfa_backward_dbias(const jfa_problem* problem, const void* q, const void* k,
                              const void* v, const void* out, const float* lse, const void* dout,
                              const int32_t* q_offsets, const int32_t* kv_offsets,
                              const void* bias, jfa_act act, int causal, void* dq, void* dk,
                              void* dv, void* dbias, void* workspace, size_t ws_bytes,
                              jfa_stream_t stream);

/* MX (OCP v1.0) quantisation of a bf16 tensor x [rows][heads][d] to E4M3
 * codes [rows][heads][d] (same layout, one byte each) and E8M0 scales: the
 * MXFP8 attention operands ("GEM Training: How Meta Doubled the Efficiency of
 * Its LLM-Scale Ads Foundation Model", opening summary: MXFP8 attention;
 * "Meta GEM Training Efficiency: Why LLM-Scale Recommenders Need a Different
 * Stack", "Bottleneck move 2": block-scaled low precision with the scales
 * generated on the device).
 * Shared exponent X = floor(log2(amax of the block)) - 8, clamped to
 * [-127, 127] (-127 for an all-zero block); codes = RNE(x * 2^-X) saturated
 * to +-448; scale byte = X + 127.
 *   along_rows == 0: blocks are 32 consecutive elements of d (d % 32 == 0);
 *                    scales [rows][heads][d/32]; offsets may be NULL.
 *   along_rows == 1: blocks are 32 consecutive rows of one sequence, counted
 *                    from its first row (offsets: device int32 [batch+1]);
 *                    the last block of a sequence is zero-padded; scales
 *                    [n_blocks][heads][d] with sequence b's blocks starting
 *                    at sum_{b'<b} ceil(n(b')/32).  The caller sizes scales
 *                    for rows/32 + batch blocks (an upper bound); max_len
 *                    bounds every sequence length (it sizes the grid).
 * Bit-exact with the OCP rounding rules. */
jfa_status jfa_quantize_mxfp8(const void* x_bf16, int64_t rows, int32_t heads, int32_t d,
                              const int32_t* offsets, int32_t batch, int32_t max_len,
                              int along_rows, uint8_t* codes, uint8_t* scales,
                              jfa_stream_t stream);

/* jfa_quantize_mxfp8 that, in the same pass, also writes every element's
 * dequantised value code * 2^X (exact in bf16: three mantissa bits times a
 * power of two) to dequant_bf16, a device tensor [rows][heads][d], 16-byte
 * aligned, owned by the caller.  For the producer of an MXFP8 training step
 * ("Meta GEM Training Efficiency: Why LLM-Scale Recommenders Need a Different
 * Stack", "Bottleneck move 2": casting belongs in the kernel that makes the
 * tensor, not in extra passes): the codes feed jfa_forward_mxfp8 and the
 * dequantised tensors a bf16 jfa_backward, which is then the MXFP8 backward
 * (bf16 gradients on the operands the forward's block-scaled MMAs saw, the
 * quantiser passed straight through) without a second quantisation pass.
 * Arguments, layouts and errors otherwise as jfa_quantize_mxfp8; a NULL
 * dequant_bf16 with rows > 0 is JFA_ERR_INVALID_ARGUMENT. */
jfa_status jfa_quantize_mxfp8_dequant(const void* x_bf16, int64_t rows, int32_t heads, int32_t d,
                                      const int32_t* offsets, int32_t batch, int32_t max_len,
                                      int along_rows, uint8_t* codes, uint8_t* scales,
                                      void* dequant_bf16, jfa_stream_t stream);

/* Normalisation fused with MX quantisation, for the producer of MXFP8
 * operands ("Meta Enhances GEM Training Efficiency with Advanced LLM-Scale
 * Innovations", "Implementing Ultra-Low-Precision Methods"; "Meta GEM
 * Training Efficiency: Why LLM-Scale Recommenders Need a Different Stack",
 * "Bottleneck move 2": scale generation and casting fused into the kernel
 * that produces the tensor, not a separate pass).  For each of `rows` rows of
 * D elements (bf16 x, device, [rows][D], 16-byte aligned):
 *   layernorm == 0 (RMSNorm): y = x * gamma / sqrt(mean(x^2) + eps)
 *   layernorm != 0          : y = (x - mean) * gamma / sqrt(var + eps) + beta
 * computed in fp32, then MX-quantised along the row in blocks of 32 exactly
 * as jfa_quantize_mxfp8 (along_rows = 0): codes E4M3 [rows][D], scales E8M0
 * [rows][D / 32].  gamma, beta: device fp32 [D], NULL for 1 and 0.  With
 * rows = tokens x heads and D = head_dim this is a per-head Q or K norm
 * whose outputs are jfa_forward_mxfp8's q8 / q_scales (or k8 / k_scales).
 * D a multiple of 32 in [32, 16384], eps > 0, else JFA_ERR_INVALID_ARGUMENT. */
jfa_status jfa_norm_quantize_mxfp8(const void* x, int64_t rows, int32_t D, const float* gamma,
                                   const float* beta, float eps, int layernorm, uint8_t* codes,
                                   uint8_t* scales, jfa_stream_t stream);

/* The longest-first tile schedule that jfa_forward (backward = 0: items are
 * query tiles) or jfa_backward (backward = 1: items are key/value tiles) runs
 * over the jagged batch, so that short and long samples balance across SMs
 * ("GEM Training: How Meta Doubled the Efficiency of Its LLM-Scale Ads
 * Foundation Model", "Challenge 1: Achieving High Per-GPU Utilization": work
 * per sample varies with its sequence length),
 * written to items (device int32 [capacity][4] = {sequence, head, tile,
 * cost}) and its length to *count (device int32).  cost = number of (query,
 * key) pairs the tile computes; order = cost descending, then sequence, tile,
 * head ascending.  tile is the tile height in rows (16..256, multiple of 16).
 * Exposed so that the schedule can be checked; the passes build their own.
 * workspace: >= jfa_workspace_bytes(problem, backward). */
jfa_status jfa_schedule(const jfa_problem* problem, const int32_t* q_offsets,
                        const int32_t* kv_offsets, int causal, int backward, int tile,
                        int32_t* items, int64_t capacity, int32_t* count, void* workspace,
                        size_t ws_bytes, jfa_stream_t stream);

/* BlockAttention ("Meta Enhances GEM Training Efficiency with Advanced
 * LLM-Scale Innovations", "Exploring the Customized Kernel Library" ->
 * "BlockAttention": windows instead of full attention over long user
 * histories; "Meta GEM Training Efficiency: Why LLM-Scale Recommenders Need a
 * Different Stack", "Bottleneck move 1": long-sequence attention as
 * independent fixed-size blocks).  With block length W, query i of a
 * self-attention sequence sees only the keys j with floor(j / W) ==
 * floor(i / W) (and j <= i when causal); GDPA divides by the block's key
 * count.  That is jagged attention over the sequences cut into blocks, so this
 * call only rewrites the offsets (on the device, enqueued on `stream`):
 *   offsets        : device int32 [batch + 1], the sequences' offsets
 *   total          : offsets[batch] (host value)
 *   block_offsets  : device int32 [batch + total / block + 1] out: the blocks
 *                    [c W, min((c + 1) W, n)) of every sequence in order,
 *                    then empty blocks up to that fixed count
 * Then jfa_forward / jfa_backward / jfa_backward_dbias with q_offsets =
 * kv_offsets = block_offsets and a problem of batch' = batch + total / block,
 * max_q_len' = max_kv_len' = min(block, max_len), the same totals, compute
 * BlockAttention; only tiles inside the blocks are scheduled.  A dense bias
 * is then laid out per block ([heads][n][n] for each block in order).  Bad
 * offsets (offsets[0] != 0, decreasing, offsets[batch] != total) make
 * block_offsets[0] = -1, which the attention call reports as
 * JFA_ERR_BAD_OFFSETS.  JFA_ERR_INVALID_ARGUMENT for block < 1 or a NULL
 * pointer. */
jfa_status jfa_block_offsets(const int32_t* offsets, int32_t batch, int64_t total,
                             int32_t block, int32_t* block_offsets, jfa_stream_t stream);

/* Data-parallel split of one global batch across ranks (HOST function: every
 * pointer is host memory, nothing touches a GPU).  Sequences are independent,
 * so each rank runs jfa_forward / jfa_backward on its own sequences with no
 * collective; the split only has to balance the work, which jagged batches
 * make uneven ("Meta GEM Training Efficiency: Why LLM-Scale Recommenders Need
 * a Different Stack", section "Bottleneck move 4: memory relief to load
 * balance": heaviest rank ~15% above the average; base batch shuffling
 * pairs heavy and light sub-batches without cross-rank communication).
 * Every rank computes the same split from the lengths alone.
 *   q_lens, kv_lens : int32 [batch] sequence lengths (>= 0)
 *   causal, window  : cost = visible (query, key) pairs under the masks of
 *                     jfa_problem (bottom-right causal; sliding window w > 0,
 *                     0 = none; negative is JFA_ERR_INVALID_ARGUMENT)
 *   method          : JFA_PARTITION_LPT -- sequences by cost descending (ties
 *                     by index), each to the least-loaded rank (ties: lowest);
 *                     JFA_PARTITION_BBS -- sub-batches of `sub_batch`
 *                     consecutive sequences sorted by total length (sum of
 *                     n_q + n_kv, descending, ties by index) and dealt in
 *                     snake order 0..R-1, R-1..0, ...
 *   rank_of         : int32 [batch] out, the rank of each sequence
 *   rank_cost       : int64 [ranks] out (may be NULL), visible pairs per rank
 *                     (per head)
 * Returns JFA_ERR_INVALID_ARGUMENT for a bad size, pointer or method. */
typedef enum { JFA_PARTITION_LPT = 0, JFA_PARTITION_BBS = 1 } jfa_partition_method;
jfa_status jfa_partition(int32_t batch, const int32_t* q_lens, const int32_t* kv_lens, int causal,
                         int32_t window, int32_t ranks, int method, int32_t sub_batch,
                         int32_t* rank_of, int64_t* rank_cost);

/* Synchronises `stream`, then reads and clears the workspace's device error
 * word: JFA_OK, JFA_ERR_BAD_OFFSETS or JFA_ERR_TIMEOUT. */
jfa_status jfa_check_error(void* workspace, jfa_stream_t stream);

/* Thread-local message for the last non-OK status returned to this thread. */
const char* jfa_last_error(void);

/* Kernel timing for measurement tools.  jfa_profile_enable(1) starts a fresh
 * record on the calling thread: from then on every kernel that jfa_forward,
 * jfa_backward, jfa_schedule or jfa_quantize_mxfp8 launches from this thread
 * is bracketed by two CUDA events recorded on the call's stream (the events
 * are created by the library and reused; no device memory is allocated).
 * jfa_profile_enable(0) stops recording and keeps the record.
 * jfa_profile_read() waits for the recorded events and writes, for up to
 * `capacity` launches in launch order, the duration in milliseconds and the
 * kernel id; it returns the number of recorded launches (which may exceed
 * capacity) or -1 on a CUDA error.  jfa_kernel_name() names a kernel id. */
jfa_status jfa_profile_enable(int enable);
int jfa_profile_read(float* ms, int32_t* kernel_ids, int32_t capacity);
const char* jfa_kernel_name(int32_t kernel_id);

/* Forward pass for callers that cannot allocate device memory.
 *
 * No counterpart in the source pages: this is a deployment convenience.
 * Same operation, arguments, layouts and errors as jfa_forward, minus the
 * workspace.  Some callers have no way to obtain a workspace: a plugin
 * inside a host framework that owns the whole device memory pool and exposes
 * no allocator, or a serving loop that forbids allocation after start-up.
 * This entry point allocates nothing (no cudaMalloc, cudaFree or allocating
 * library call); its scratch is a fixed 8 MiB __device__ array inside the
 * library, held by every GPU that loads the library until the process exits.
 *  - The first call on a device looks up that array's device address with
 *    that device current (cudaGetSymbolAddress) and caches it; make that
 *    first call before any stream capture.
 *  - Problems whose jfa_workspace_bytes(problem, 0) exceeds 8 MiB are
 *    rejected with JFA_ERR_WORKSPACE before anything is launched.  That
 *    count is the tile schedule (about 16 * heads bytes per 16 query rows,
 *    plus 16 bytes per 16 rows and 8 per sequence), the relative-position
 *    table prepared for the kernels (16 * heads * max(relpos_len, 384)
 *    bytes) and, for JFA_MXFP8, the quantised operands: so bf16 batches of a
 *    few hundred thousand query rows fit, MXFP8 only small ones.
 *  - Every call shares the one array and it keeps the last call's contents;
 *    calls whose work overlaps on the GPU (other streams, other host threads)
 *    race on it and must be serialised by the caller.
 *  - The on-device error word lives in that array too, out of reach of
 *    jfa_check_error().  Bad offsets (or a timed-out device wait) still
 *    return JFA_OK here and leave the outputs of the affected rows
 *    unwritten, so a caller that needs to detect them pre-fills out and lse
 *    with NaN and treats any row still NaN afterwards as a failed call. */
jfa_status jfa_forward_fixed_scratch(const jfa_problem* problem, const void* q, const void* k,
                                     const void* v, const int32_t* q_offsets,
                                     const int32_t* kv_offsets, const void* bias, jfa_act act,
                                     int causal, void* out, float* lse, jfa_stream_t stream);

/* Failure injection for tests of the bounded device waits (no GPU fault is
 * made: a load is left out and the waits on it give up).  what =
 * JFA_TEST_FWD_SKIP_LOAD arms the calling thread's NEXT jfa_forward that runs
 * the tensor-core kernel: CTA 0 skips its first key-tile load and the waits
 * give up after 5 ms instead of 1 s, so the call ends with JFA_ERR_TIMEOUT in
 * the workspace's error word (jfa_check_error) while every copy the kernel
 * did issue completes.  what = 0 disarms.  The hook is used up by that call
 * (or by any jfa_forward on the CUDA-core path).  JFA_ERR_INVALID_ARGUMENT
 * for another value. */
enum { JFA_TEST_FWD_SKIP_LOAD = 1 };
jfa_status jfa_test_inject(int what);

/* Which kernel family jfa_forward / jfa_backward will use for this problem:
 * 0 = CUDA-core (fp32 arithmetic), 1 = tcgen05 tensor-core. */
int jfa_path(const jfa_problem* problem, jfa_act act, int backward);

#ifdef __cplusplus
}
#endif

#endif /* JFA_H_ */
