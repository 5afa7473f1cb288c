/*
 * jfa_oracle.c -- plain fp64 CPU oracle for jagged attention (test infrastructure).
 *
 * THIS FILE IS TEST INFRASTRUCTURE.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg load it.  It shares no code, header or constant
 * with the CUDA library; it is the written-out definition of what the library
 * computes, slow on purpose, so that a reader can check it against the sources
 * by eye:
 *
 *  [JT]  "Meta GEM Training Efficiency: Why LLM-Scale Recommenders Need a
 *        Different Stack", FAQ "What is a jagged tensor?": samples are stored
 *        packed, values plus offsets, with no padding.
 *  [JFA] same page, "Bottleneck move 1: dense-sequence kernels to jagged
 *        execution": attention computed directly on variable-length tensors,
 *        with custom (additive) biases and asymmetric query / key-value lengths.
 *  [GDPA] same section: attention-like modules whose softmax is replaced by a
 *        pointwise GELU or SiLU.
 *  [ASYM] "GEM Training: How Meta Doubled the Efficiency of Its LLM-Scale Ads
 *        Foundation Model", "Challenge 1: Achieving High Per-GPU Utilization":
 *        long-query/short-kv and short-query/long-kv shapes.
 *  [MX]  "GEM Training ...", opening summary, and "Meta Enhances GEM Training
 *        Efficiency ...", "Leveraging Compute Efficiency through Customized
 *        Kernels": MXFP8 attention.  The element and scale formats follow the
 *        OCP Microscaling Formats (MX) v1.0 specification (E4M3 elements, one
 *        E8M0 power-of-two scale per 32 elements), which the pages only name.
 *
 * Everything the pages leave open is fixed by the readings listed in the
 * design notes of this repository (scale 1/sqrt(d), bias added after scaling,
 * bottom-right causal alignment, GDPA divided by the sequence's kv length,
 * empty rows give zero output and LSE = -inf, natural-log LSE).
 *
 * Layouts: Q, O, dQ, dO are [total_q][H][d]; K, V, dK, dV are [total_kv][H][d];
 * LSE is [total_q][H]; sequence b owns query rows [q_off[b], q_off[b+1]) and
 * key/value rows [kv_off[b], kv_off[b+1]).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORC_ACT_SOFTMAX = 0, ORC_ACT_SILU = 1, ORC_ACT_GELU_TANH = 2 };
enum { ORC_BIAS_NONE = 0, ORC_BIAS_RELPOS = 1, ORC_BIAS_DENSE = 2 };

/* SiLU(x) = x * sigmoid(x) (Elfwing et al., 2018). */
static double silu(double x) { return x / (1.0 + exp(-x)); }

static double silu_grad(double x) {
    double sg = 1.0 / (1.0 + exp(-x));
    return sg * (1.0 + x * (1.0 - sg));
}

/* tanh-approximated GELU (Hendrycks & Gimpel, "Gaussian Error Linear Units",
 * 2016): 0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3))). */
static double gelu_tanh(double x) {
    double c = sqrt(2.0 / M_PI);
    double t = tanh(c * (x + 0.044715 * x * x * x));
    return 0.5 * x * (1.0 + t);
}

static double gelu_tanh_grad(double x) {
    double c = sqrt(2.0 / M_PI);
    double t = tanh(c * (x + 0.044715 * x * x * x));
    return 0.5 * (1.0 + t) + 0.5 * x * (1.0 - t * t) * c * (1.0 + 3.0 * 0.044715 * x * x);
}

static double act_value(int act, double x) {
    return act == ORC_ACT_SILU ? silu(x) : gelu_tanh(x);
}

static double act_derivative(int act, double x) {
    return act == ORC_ACT_SILU ? silu_grad(x) : gelu_tanh_grad(x);
}

/* Causal validity with bottom-right alignment: query i may see key j when
 * j <= i + (n_kv - n_q); for self-attention (n_q == n_kv) this is j <= i. */
static int causal_ok(int causal, int i, int j, int nq, int nkv) {
    if (!causal) return 1;
    return (long)j <= (long)i + (long)(nkv - nq);
}

/* BlockAttention ("Meta Enhances GEM Training Efficiency ...", "Exploring the
 * Customized Kernel Library" -> "BlockAttention": windows instead of full
 * attention over the user history; "Meta GEM Training Efficiency ...",
 * "Bottleneck move 1": long-sequence attention as independent fixed-size
 * blocks).  With block length W > 0 the keys of a sequence form blocks
 * [c W, (c + 1) W) and query i, at the bottom-right aligned position
 * p = i + n_kv - n_q (p = i for self-attention), sees only the keys of block
 * floor(p / W) (none when p < 0); the causal rule applies on top. */
static int block_of(int W, int i, int nq, int nkv) {
    long p = (long)i + (long)(nkv - nq);
    return p < 0 ? -1 : (int)(p / W);
}

/* Windowed (sliding-window) attention ("Meta Enhances GEM Training Efficiency
 * ...", "Exploring the Customized Kernel Library" -> "BlockAttention":
 * windows instead of full attention over long user histories).  With window
 * w > 0 query i, at the bottom-right aligned position p = i + n_kv - n_q,
 * sees key j only when p - j < w (the w most recent positions up to p under
 * the causal rule) and, without the causal rule, also j - p < w (a band of
 * half-width w - 1 around p). */
static int window_ok(int w, int causal, int i, int j, int nq, int nkv) {
    if (w <= 0) return 1;
    long p = (long)i + (long)(nkv - nq);
    if (p - (long)j >= (long)w) return 0;
    if (!causal && (long)j - p >= (long)w) return 0;
    return 1;
}



/* Additive bias beta_h(i, j).
 *  RELPOS: table[h][clamp(i - j, -C, C) + C], table length T = 2C + 1.
 *  DENSE : block [H][n_q][n_kv] of sequence b, blocks concatenated in b order
 *          starting at element dense_off (int64, computed by the caller loop). */
static double bias_value(int kind, const double* bias, int relpos_len, int H, int h,
                         int64_t dense_off, int nq, int nkv, int i, int j) {
    (void)nq;
    if (kind == ORC_BIAS_RELPOS) {
        int C = (relpos_len - 1) / 2;
        long r = (long)i - (long)j;
        if (r < -C) r = -C;
        if (r > C) r = C;
        return bias[(int64_t)h * relpos_len + (r + C)];
    }
    if (kind == ORC_BIAS_DENSE) {
        (void)H;
        return bias[dense_off + ((int64_t)h * nq + i) * nkv + j];
    }
    return 0.0;
}

static int64_t* dense_offsets(int B, int H, const int32_t* q_off, const int32_t* kv_off) {
    int64_t* off = (int64_t*)malloc(sizeof(int64_t) * (size_t)(B + 1));
    off[0] = 0;
    for (int b = 0; b < B; ++b) {
        int64_t nq = q_off[b + 1] - q_off[b];
        int64_t nkv = kv_off[b + 1] - kv_off[b];
        off[b + 1] = off[b] + (int64_t)H * nq * nkv;
    }
    return off;
}

/* OCP MX v1.0 E4M3 element encoding, round-to-nearest-even, saturating to the
 * largest finite magnitude 448 = 1.75 * 2^8.  E4M3: 1 sign, 4 exponent bits
 * (bias 7), 3 mantissa bits; exponent field 0 holds subnormals m * 2^-9; the
 * pattern S.1111.111 is NaN and is never produced here. */
uint8_t jfa_oracle_e4m3_encode(double y) {
    uint8_t sign = (y < 0.0 || (y == 0.0 && signbit(y))) ? 0x80 : 0x00;
    double a = fabs(y);
    if (isnan(y)) return 0x7F;
    if (a >= 448.0) return sign | 0x7E;
    if (a == 0.0) return sign;
    int E;
    frexp(a, &E);              /* a = f * 2^E with f in [0.5, 1) */
    int e = E - 1;             /* floor(log2 a) */
    if (e < -6) e = -6;        /* below the smallest normal the quantum is fixed */
    double quantum = ldexp(1.0, e - 3);
    double n = nearbyint(a / quantum); /* default rounding mode: ties to even */
    /* n * quantum is the rounded value; n in [0, 16] */
    if (e == -6 && n < 8.0) {
        return sign | (uint8_t)n; /* subnormal (or zero) */
    }
    if (n >= 16.0) { n = 8.0; e += 1; }
    int code = ((e + 7) << 3) | ((int)n - 8);
    if (code > 0x7E) code = 0x7E;
    return sign | (uint8_t)code;
}

double jfa_oracle_e4m3_decode(uint8_t c) {
    int s = c >> 7, ex = (c >> 3) & 15, m = c & 7;
    double v;
    if (ex == 15 && m == 7) return NAN;
    if (ex == 0) v = ldexp((double)m, -9);
    else v = ldexp((double)(8 + m), ex - 10);
    return s ? -v : v;
}

/* MX block quantisation of n_blocks contiguous blocks of 32 values.
 * Shared exponent X = floor(log2(amax)) - 8 (8 = largest E4M3 exponent),
 * clamped to the E8M0 range [-127, 127]; an all-zero block takes X = -127.
 * Each element becomes E4M3(x * 2^-X); the scale byte is X + 127. */
void jfa_oracle_quantize_mx(const double* x, int64_t n_blocks, uint8_t* codes, uint8_t* scales) {
    for (int64_t blk = 0; blk < n_blocks; ++blk) {
        const double* xb = x + blk * 32;
        double amax = 0.0;
        for (int t = 0; t < 32; ++t) amax = fmax(amax, fabs(xb[t]));
        int X;
        if (amax == 0.0) {
            X = -127;
        } else {
            int E;
            frexp(amax, &E);
            X = (E - 1) - 8;
            if (X < -127) X = -127;
            if (X > 127) X = 127;
        }
        scales[blk] = (uint8_t)(X + 127);
        for (int t = 0; t < 32; ++t) codes[blk * 32 + t] = jfa_oracle_e4m3_encode(ldexp(xb[t], -X));
    }
}

/* Dequantise: value = E4M3(code) * 2^(scale - 127). */
void jfa_oracle_dequantize_mx(const uint8_t* codes, const uint8_t* scales, int64_t n_blocks, double* out) {
    for (int64_t blk = 0; blk < n_blocks; ++blk)
        for (int t = 0; t < 32; ++t)
            out[blk * 32 + t] = ldexp(jfa_oracle_e4m3_decode(codes[blk * 32 + t]), (int)scales[blk] - 127);
}

/* One query row of one (sequence, head): scores s_j for all keys, the softmax
 * (or activation) weights w_j, and the row's output.  Returns the number of
 * valid keys.  Work arrays s and w have n_kv entries. */
typedef struct {
    int B, H, d;
    const int32_t *q_off, *kv_off;
    const double *q, *k, *v;
    int bias_kind;
    const double* bias;
    int relpos_len;
    const int64_t* dense_off;
    int act, causal;
    double scale;
    int quant_p; /* MXFP8: quantise exp(s - m) per 32 keys before P.V */
    int block;   /* BlockAttention block length; 0 = full attention */
    int window;  /* sliding-window width; 0 = no window */
} orc_problem;

static int is_valid(const orc_problem* P, int i, int j, int nq, int nkv) {
    if (!causal_ok(P->causal, i, j, nq, nkv)) return 0;
    if (P->block > 0 && block_of(P->block, i, nq, nkv) != j / P->block) return 0;
    if (!window_ok(P->window, P->causal, i, j, nq, nkv)) return 0;
    return 1;
}

/* The GDPA normaliser: the sequence's n_kv, or with BlockAttention the
 * number of keys in the query's block. */
static double gdpa_norm(const orc_problem* P, int i, int nq, int nkv) {
    if (P->block <= 0) return (double)nkv;
    int c = block_of(P->block, i, nq, nkv);
    if (c < 0) return 1.0;  /* the row sees no key; nothing is divided */
    int n = nkv - c * P->block;
    return (double)(n < P->block ? n : P->block);
}

static const double* row_ptr(const double* base, int64_t row, int H, int h, int d) {
    return base + (row * H + h) * (int64_t)d;
}

/* Computes s_j and the normalised weights p_j (softmax) or a_j (GDPA) of query
 * row i.  For softmax also returns m (max) and l (sum of exp(s - m)); for a row
 * without a valid key m = -inf and l = 0.  pv_weight receives the weights that
 * multiply V in the forward output (equal to w unless P is quantised). */
static void row_weights(const orc_problem* P, int b, int h, int i, double* s, double* w,
                        double* pv_weight, double* m_out, double* l_out) {
    int nq = P->q_off[b + 1] - P->q_off[b];
    int nkv = P->kv_off[b + 1] - P->kv_off[b];
    const double* qi = row_ptr(P->q, P->q_off[b] + i, P->H, h, P->d);
    double m = -INFINITY;
    for (int j = 0; j < nkv; ++j) {
        const double* kj = row_ptr(P->k, P->kv_off[b] + j, P->H, h, P->d);
        double dot = 0.0;
        for (int c = 0; c < P->d; ++c) dot += qi[c] * kj[c];
        s[j] = P->scale * dot +
               bias_value(P->bias_kind, P->bias, P->relpos_len, P->H, h,
                          P->dense_off ? P->dense_off[b] : 0, nq, nkv, i, j);
        if (is_valid(P, i, j, nq, nkv) && s[j] > m) m = s[j];
    }
    if (P->act == ORC_ACT_SOFTMAX) {
        double l = 0.0;
        for (int j = 0; j < nkv; ++j)
            w[j] = is_valid(P, i, j, nq, nkv) ? exp(s[j] - m) : 0.0;
        for (int j = 0; j < nkv; ++j) l += w[j];
        if (pv_weight) {
            if (P->quant_p) {
                /* MXFP8 P: the weights 2^(x_j - R), x_j = s_j log2(e), with the
                 * integer reference R = ceil(max_j x_j), are quantised in blocks
                 * of 32 consecutive keys counted from the sequence's first key;
                 * l sums the unquantised weights.  A power-of-two reference makes
                 * the codes independent of which integer R a kernel uses. */
                double xmax = -INFINITY;
                for (int j = 0; j < nkv; ++j)
                    if (is_valid(P, i, j, nq, nkv) && s[j] * M_LOG2E > xmax) xmax = s[j] * M_LOG2E;
                const double R = ceil(xmax);
                double* w2 = (double*)malloc(sizeof(double) * (size_t)(nkv > 0 ? nkv : 1));
                double l2 = 0.0;
                for (int j = 0; j < nkv; ++j) {
                    w2[j] = is_valid(P, i, j, nq, nkv) ? exp2(s[j] * M_LOG2E - R) : 0.0;
                    l2 += w2[j];
                }
                for (int j0 = 0; j0 < nkv; j0 += 32) {
                    double blk[32];
                    uint8_t codes[32], sc;
                    for (int t = 0; t < 32; ++t) blk[t] = (j0 + t < nkv) ? w2[j0 + t] : 0.0;
                    jfa_oracle_quantize_mx(blk, 1, codes, &sc);
                    double deq[32];
                    jfa_oracle_dequantize_mx(codes, &sc, 1, deq);
                    for (int t = 0; t < 32 && j0 + t < nkv; ++t)
                        pv_weight[j0 + t] = (l2 > 0.0) ? deq[t] / l2 : 0.0;
                }
                free(w2);
            } else {
                for (int j = 0; j < nkv; ++j) pv_weight[j] = (l > 0.0) ? w[j] / l : 0.0;
            }
        }
        for (int j = 0; j < nkv; ++j) w[j] = (l > 0.0) ? w[j] / l : 0.0;
        *m_out = m;
        *l_out = l;
    } else {
        for (int j = 0; j < nkv; ++j)
            w[j] = is_valid(P, i, j, nq, nkv) ? act_value(P->act, s[j]) / gdpa_norm(P, i, nq, nkv) : 0.0;
        if (pv_weight)
            for (int j = 0; j < nkv; ++j) pv_weight[j] = w[j];
        *m_out = m;
        *l_out = 0.0;
    }
}

static void forward_item(const orc_problem* P, int b, int h, double* out, double* lse) {
    int nq = P->q_off[b + 1] - P->q_off[b];
    int nkv = P->kv_off[b + 1] - P->kv_off[b];
    int n = nkv > 0 ? nkv : 1;
    double* s = (double*)malloc(sizeof(double) * n);
    double* w = (double*)malloc(sizeof(double) * n);
    double* pw = (double*)malloc(sizeof(double) * n);
    for (int i = 0; i < nq; ++i) {
        double m, l;
        row_weights(P, b, h, i, s, w, pw, &m, &l);
        double* oi = out + ((int64_t)(P->q_off[b] + i) * P->H + h) * P->d;
        for (int c = 0; c < P->d; ++c) oi[c] = 0.0;
        for (int j = 0; j < nkv; ++j) {
            if (pw[j] == 0.0) continue;
            const double* vj = row_ptr(P->v, P->kv_off[b] + j, P->H, h, P->d);
            for (int c = 0; c < P->d; ++c) oi[c] += pw[j] * vj[c];
        }
        if (lse && P->act == ORC_ACT_SOFTMAX)
            lse[(int64_t)(P->q_off[b] + i) * P->H + h] = (l > 0.0) ? m + log(l) : -INFINITY;
    }
    free(s);
    free(w);
    free(pw);
}

/* Analytic gradients of the forward above for one (sequence, head).
 * softmax: D_i = dO_i . o_i, dp_ij = dO_i . v_j, ds_ij = p_ij (dp_ij - D_i)
 * GDPA   : ds_ij = dp_ij act'(s_ij) / n_kv on valid (i, j), 0 elsewhere
 * both   : dV_j += w_ij dO_i, dQ_i += scale sum_j ds_ij k_j,
 *          dK_j += scale ds_ij q_i.
 * Bias ("custom biases", [JFA]): s_ij = scale q_i.k_j + beta_h(i, j), so the
 * gradient of an additive bias entry is the sum of ds_ij over the pairs that
 * read it:
 *   DENSE : dbias at the pair's own position = ds_ij (0 for a masked pair);
 *   RELPOS: dtable[h][clamp(i - j, -C, C) + C] += ds_ij over valid pairs.
 * The RELPOS partial sums of this item go to dtab_item (relpos_len entries,
 * summed over items by the caller in item order); the DENSE gradient goes
 * straight into dbias_dense (blocks of different items are disjoint).
 * For MXFP8 the quantisers are straight-through estimators: the gradients
 * are those of the unquantised weights on the dequantised operands, with D
 * taken from the forward's saved output when out_for_d is given. */
static void backward_item(const orc_problem* P, int b, int h, const double* dout,
                          const double* out_for_d, double* dq, double* dk, double* dv,
                          double* dtab_item, double* dbias_dense) {
    int nq = P->q_off[b + 1] - P->q_off[b];
    int nkv = P->kv_off[b + 1] - P->kv_off[b];
    int H = P->H, d = P->d;
    int n = nkv > 0 ? nkv : 1;
    double* s = (double*)malloc(sizeof(double) * n);
    double* w = (double*)malloc(sizeof(double) * n);
    double* o = (double*)malloc(sizeof(double) * d);
    for (int j = 0; j < nkv; ++j) {
        double* dkj = dk + ((int64_t)(P->kv_off[b] + j) * H + h) * d;
        double* dvj = dv + ((int64_t)(P->kv_off[b] + j) * H + h) * d;
        for (int c = 0; c < d; ++c) dkj[c] = 0.0, dvj[c] = 0.0;
    }
    double* dbias_blk = NULL;
    if (dbias_dense) {
        dbias_blk = dbias_dense + P->dense_off[b] + (int64_t)h * nq * nkv;
        for (int64_t e = 0; e < (int64_t)nq * nkv; ++e) dbias_blk[e] = 0.0;
    }
    for (int i = 0; i < nq; ++i) {
        double m, l;
        row_weights(P, b, h, i, s, w, NULL, &m, &l);
        const double* qi = row_ptr(P->q, P->q_off[b] + i, H, h, d);
        const double* doi = dout + ((int64_t)(P->q_off[b] + i) * H + h) * d;
        double* dqi = dq + ((int64_t)(P->q_off[b] + i) * H + h) * d;
        for (int c = 0; c < d; ++c) dqi[c] = 0.0;
        double Di = 0.0;
        if (P->act == ORC_ACT_SOFTMAX) {
            if (out_for_d) {
                /* D from the forward's saved output (MXFP8: the output computed
                 * with quantised P), as a training step uses it */
                const double* oi = row_ptr(out_for_d, P->q_off[b] + i, H, h, d);
                for (int c = 0; c < d; ++c) o[c] = oi[c];
            } else {
                for (int c = 0; c < d; ++c) o[c] = 0.0;
                for (int j = 0; j < nkv; ++j) {
                    const double* vj = row_ptr(P->v, P->kv_off[b] + j, H, h, d);
                    for (int c = 0; c < d; ++c) o[c] += w[j] * vj[c];
                }
            }
            for (int c = 0; c < d; ++c) Di += doi[c] * o[c];
        }
        for (int j = 0; j < nkv; ++j) {
            if (!is_valid(P, i, j, nq, nkv)) continue;
            const double* kj = row_ptr(P->k, P->kv_off[b] + j, H, h, d);
            const double* vj = row_ptr(P->v, P->kv_off[b] + j, H, h, d);
            double* dkj = dk + ((int64_t)(P->kv_off[b] + j) * H + h) * d;
            double* dvj = dv + ((int64_t)(P->kv_off[b] + j) * H + h) * d;
            double dp = 0.0;
            for (int c = 0; c < d; ++c) dp += doi[c] * vj[c];
            double ds;
            if (P->act == ORC_ACT_SOFTMAX) ds = w[j] * (dp - Di);
            else ds = dp * act_derivative(P->act, s[j]) / gdpa_norm(P, i, nq, nkv);
            if (dbias_blk) dbias_blk[(int64_t)i * nkv + j] = ds;
            if (dtab_item) {
                int C = (P->relpos_len - 1) / 2;
                long r = (long)i - (long)j;
                if (r < -C) r = -C;
                if (r > C) r = C;
                dtab_item[r + C] += ds;
            }
            for (int c = 0; c < d; ++c) {
                dvj[c] += w[j] * doi[c];
                dqi[c] += P->scale * ds * kj[c];
                dkj[c] += P->scale * ds * qi[c];
            }
        }
    }
    free(s);
    free(w);
    free(o);
}

static void fill_problem(orc_problem* P, int B, int H, int d, const int32_t* q_off,
                         const int32_t* kv_off, const double* q, const double* k, const double* v,
                         int bias_kind, const double* bias, int relpos_len, int act, int causal,
                         double scale, int quant_p, int block, int window) {
    P->B = B; P->H = H; P->d = d;
    P->q_off = q_off; P->kv_off = kv_off;
    P->q = q; P->k = k; P->v = v;
    P->bias_kind = bias_kind; P->bias = bias; P->relpos_len = relpos_len;
    P->dense_off = (bias_kind == ORC_BIAS_DENSE) ? dense_offsets(B, H, q_off, kv_off) : NULL;
    P->act = act; P->causal = causal;
    P->scale = scale > 0.0 ? scale : 1.0 / sqrt((double)d);
    P->quant_p = quant_p;
    P->block = block;
    P->window = window;
}

/* Forward over all (sequence b, head h) items with item_mask == NULL or
 * item_mask[b * H + h] != 0.  Skipped items are left untouched in out / lse. */
int jfa_oracle_forward(int B, int H, int d, const int32_t* q_off, const int32_t* kv_off,
                       const double* q, const double* k, const double* v, int bias_kind,
                       const double* bias, int relpos_len, int act, int causal, double scale,
                       int quant_p, int block, int window, const int32_t* item_mask, double* out,
                       double* lse, int nthreads) {
    orc_problem P;
    fill_problem(&P, B, H, d, q_off, kv_off, q, k, v, bias_kind, bias, relpos_len, act, causal,
                 scale, quant_p, block, window);
    long n_items = (long)B * H;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (long it = 0; it < n_items; ++it) {
        int b = (int)(it / H), h = (int)(it % H);
        if (item_mask && !item_mask[it]) continue;
        forward_item(&P, b, h, out, lse);
    }
    free((void*)P.dense_off);
    (void)nthreads;
    return 0;
}

/* dbias (may be NULL): DENSE -> same layout as bias; RELPOS -> [H][relpos_len],
 * overwritten with the sum over the computed items (item order). */
int jfa_oracle_backward(int B, int H, int d, const int32_t* q_off, const int32_t* kv_off,
                        const double* q, const double* k, const double* v, int bias_kind,
                        const double* bias, int relpos_len, int act, int causal, double scale,
                        int block, int window, const int32_t* item_mask, const double* dout,
                        const double* out_for_d, double* dq, double* dk, double* dv,
                        double* dbias, int nthreads) {
    orc_problem P;
    fill_problem(&P, B, H, d, q_off, kv_off, q, k, v, bias_kind, bias, relpos_len, act, causal,
                 scale, 0, block, window);
    long n_items = (long)B * H;
    const int want_tab = dbias && bias_kind == ORC_BIAS_RELPOS;
    double** parts = want_tab ? (double**)calloc((size_t)(n_items > 0 ? n_items : 1), sizeof(double*)) : NULL;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (long it = 0; it < n_items; ++it) {
        int b = (int)(it / H), h = (int)(it % H);
        if (item_mask && !item_mask[it]) continue;
        if (want_tab) parts[it] = (double*)calloc((size_t)relpos_len, sizeof(double));
        backward_item(&P, b, h, dout, out_for_d, dq, dk, dv, want_tab ? parts[it] : NULL,
                      (dbias && bias_kind == ORC_BIAS_DENSE) ? dbias : NULL);
    }
    if (want_tab) {
        for (long e = 0; e < (long)H * relpos_len; ++e) dbias[e] = 0.0;
        for (long it = 0; it < n_items; ++it) {
            if (!parts[it]) continue;
            int h = (int)(it % H);
            for (int c = 0; c < relpos_len; ++c) dbias[(long)h * relpos_len + c] += parts[it][c];
            free(parts[it]);
        }
        free(parts);
    }
    free((void*)P.dense_off);
    (void)nthreads;
    return 0;
}

int jfa_oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
