"""Oracle for jagged attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The CUDA
library never calls it and shares no code with it: the oracle is the plain
fp64 definition of what the library computes (``jfa_oracle.c``), plus a plain
Python restatement of the longest-first tile schedule, written from:

* "Meta GEM Training Efficiency: Why LLM-Scale Recommenders Need a Different
  Stack", section "Bottleneck move 1: dense-sequence kernels to jagged
  execution" (jagged attention with custom biases and asymmetric q/kv lengths;
  GDPA = GELU/SiLU instead of softmax; short and long samples finishing at
  different times, which makes tile scheduling the exposed bottleneck) and its
  FAQ "What is a jagged tensor?" (values plus offsets).
* "GEM Training: How Meta Doubled the Efficiency of Its LLM-Scale Ads
  Foundation Model", "Challenge 1" (asymmetric query / key-value shapes) and
  its summary (MXFP8 attention); element/scale formats from the OCP MX v1.0
  specification.

Inputs are passed in (seeded generators live in their own module); this
package draws no random numbers.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "jfa_oracle.c")
_SO = os.path.join(_HERE, "libjfa_oracle.so")
_LOCK = threading.Lock()
_LIB = None

ACT = {"softmax": 0, "silu": 1, "gelu_tanh": 2}
BIAS = {"none": 0, "relpos": 1, "dense": 2}


def build(force: bool = False) -> str:
    """Compile jfa_oracle.c with gcc (IEEE fp64, no fast-math, no contraction)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-shared",
               "-fPIC", "-o", _SO, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
    return _SO


def _lib():
    global _LIB
    with _LOCK:
        if _LIB is None:
            build()
            lib = ctypes.CDLL(_SO)
            P = ctypes.c_void_p
            i32, f64 = ctypes.c_int, ctypes.c_double
            lib.jfa_oracle_forward.argtypes = [i32, i32, i32, P, P, P, P, P, i32, P, i32, i32,
                                               i32, f64, i32, i32, i32, P, P, P, i32]
            lib.jfa_oracle_backward.argtypes = [i32, i32, i32, P, P, P, P, P, i32, P, i32, i32,
                                                i32, f64, i32, i32, P, P, P, P, P, P, P, i32]
            lib.jfa_oracle_quantize_mx.argtypes = [P, ctypes.c_int64, P, P]
            lib.jfa_oracle_dequantize_mx.argtypes = [P, P, ctypes.c_int64, P]
            lib.jfa_oracle_e4m3_encode.argtypes = [f64]
            lib.jfa_oracle_e4m3_encode.restype = ctypes.c_uint8
            lib.jfa_oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
            lib.jfa_oracle_e4m3_decode.restype = f64
            lib.jfa_oracle_max_threads.restype = i32
            _LIB = lib
    return _LIB


def max_threads() -> int:
    return int(_lib().jfa_oracle_max_threads())


def _f64(a) -> np.ndarray:
    """Exact widening of a stored tensor (fp32 / bf16 torch or numpy) to fp64."""
    try:
        import torch
        if isinstance(a, torch.Tensor):
            return np.ascontiguousarray(a.detach().to("cpu", torch.float64).numpy())
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _i32(a) -> np.ndarray:
    try:
        import torch
        if isinstance(a, torch.Tensor):
            a = a.detach().cpu().numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _item_mask(seq_mask, B, H):
    """Per-(sequence, head) mask from a per-sequence [B] or per-item [B*H] mask."""
    if seq_mask is None:
        return None
    m = _i32(seq_mask).reshape(-1)
    if m.size == B:
        m = np.repeat(m, H)
    assert m.size == B * H
    return np.ascontiguousarray(m.astype(np.int32))


def forward(q_off, kv_off, q, k, v, *, bias=None, bias_kind="none", relpos_len=0,
            act="softmax", causal=False, scale=0.0, quant_p=False, seq_mask=None,
            block=0, window=0, nthreads=0):
    """fp64 forward.  Returns (out [total_q,H,d], lse [total_q,H] or None).

    ``seq_mask`` ([B] per sequence or [B*H] per (sequence, head)) selects what
    is computed; everything else is NaN in the result.  ``block`` > 0:
    BlockAttention, each query sees only the keys of its own block of
    ``block`` consecutive positions (GDPA then divides by the block's key
    count).  ``window`` > 0: sliding window, query i (aligned position
    p = i + n_kv - n_q) sees key j only when p - j < window, and without the
    causal rule also when j - p < window (GDPA still divides by n_kv)."""
    q_off, kv_off = _i32(q_off), _i32(kv_off)
    q64, k64, v64 = _f64(q), _f64(k), _f64(v)
    B = len(q_off) - 1
    total_q, H, d = q64.shape
    b64 = _f64(bias) if bias is not None else None
    out = np.full((total_q, H, d), np.nan)
    lse = np.full((total_q, H), np.nan)
    mask = _item_mask(seq_mask, B, H)
    _lib().jfa_oracle_forward(B, H, d, _ptr(q_off), _ptr(kv_off), _ptr(q64), _ptr(k64),
                              _ptr(v64), BIAS[bias_kind], _ptr(b64), int(relpos_len),
                              ACT[act], int(bool(causal)), float(scale), int(bool(quant_p)),
                              int(block), int(window), _ptr(mask), _ptr(out), _ptr(lse),
                              int(nthreads))
    return out, (lse if act == "softmax" else None)


def backward(q_off, kv_off, q, k, v, dout, *, bias=None, bias_kind="none", relpos_len=0,
             act="softmax", causal=False, scale=0.0, seq_mask=None, out_for_d=None,
             dbias=False, block=0, window=0, nthreads=0):
    """fp64 analytic gradients (dq, dk, dv), and with ``dbias`` also the bias
    gradient as a fourth result: for a dense bias an array like ``bias``
    (ds of each valid pair, 0 at masked pairs, NaN in items not computed),
    for a relative-position bias the table gradient [H, relpos_len] summed
    over the computed items.

    ``out_for_d``: the forward output whose rows give D = rowsum(dO * O)
    (the MXFP8 forward's output); by default O is recomputed exactly."""
    q_off, kv_off = _i32(q_off), _i32(kv_off)
    q64, k64, v64, do64 = _f64(q), _f64(k), _f64(v), _f64(dout)
    B = len(q_off) - 1
    total_q, H, d = q64.shape
    total_kv = k64.shape[0]
    b64 = _f64(bias) if bias is not None else None
    dq = np.full((total_q, H, d), np.nan)
    dk = np.full((total_kv, H, d), np.nan)
    dv = np.full((total_kv, H, d), np.nan)
    mask = _item_mask(seq_mask, B, H)
    o64 = _f64(out_for_d) if out_for_d is not None else None
    db = None
    if dbias and bias_kind == "dense":
        db = np.full(b64.shape, np.nan)
    elif dbias and bias_kind == "relpos":
        db = np.zeros((H, int(relpos_len)))
    _lib().jfa_oracle_backward(B, H, d, _ptr(q_off), _ptr(kv_off), _ptr(q64), _ptr(k64),
                               _ptr(v64), BIAS[bias_kind], _ptr(b64), int(relpos_len),
                               ACT[act], int(bool(causal)), float(scale), int(block),
                               int(window), _ptr(mask), _ptr(do64), _ptr(o64), _ptr(dq), _ptr(dk), _ptr(dv),
                               _ptr(db), int(nthreads))
    if dbias:
        return dq, dk, dv, db
    return dq, dk, dv


def e4m3_encode(y: float) -> int:
    return int(_lib().jfa_oracle_e4m3_encode(float(y)))


def e4m3_decode(c: int) -> float:
    return float(_lib().jfa_oracle_e4m3_decode(int(c)))


def quantize_mx(x) -> tuple[np.ndarray, np.ndarray]:
    """MX (OCP v1.0) quantisation of consecutive blocks of 32 values.

    ``x`` has a multiple of 32 elements (flattened in C order).  Returns
    (codes uint8 same shape, scales uint8 [n/32])."""
    x64 = _f64(x)
    flat = x64.reshape(-1)
    assert flat.size % 32 == 0
    n_blocks = flat.size // 32
    codes = np.zeros(flat.size, np.uint8)
    scales = np.zeros(n_blocks, np.uint8)
    _lib().jfa_oracle_quantize_mx(_ptr(flat), n_blocks, _ptr(codes), _ptr(scales))
    return codes.reshape(x64.shape), scales


def dequantize_mx(codes, scales) -> np.ndarray:
    codes = np.ascontiguousarray(np.asarray(codes, np.uint8))
    scales = np.ascontiguousarray(np.asarray(scales, np.uint8))
    out = np.zeros(codes.size, np.float64)
    _lib().jfa_oracle_dequantize_mx(_ptr(codes), _ptr(scales), scales.size, _ptr(out))
    return out.reshape(codes.shape)


def quantize_mx_along_d(x):
    """Q/K layout: blocks of 32 consecutive elements of the head dimension.

    x [rows, H, d] -> codes [rows, H, d], scales [rows, H, d/32]."""
    x64 = _f64(x)
    rows, H, d = x64.shape
    codes, scales = quantize_mx(x64)
    return codes, scales.reshape(rows, H, d // 32)


def quantize_mx_along_rows(x, offsets):
    """V layout: blocks of 32 consecutive rows of one sequence (counted from the
    sequence's first row; the last block of a sequence is zero-padded), one
    scale per (block, head, column).

    Returns codes [rows, H, d] and scales [n_blocks_total, H, d] where sequence
    b's blocks start at sum_{b'<b} ceil(n(b') / 32)."""
    x64 = _f64(x)
    offsets = _i32(offsets)
    rows, H, d = x64.shape
    codes = np.zeros((rows, H, d), np.uint8)
    nblk = [(int(offsets[b + 1]) - int(offsets[b]) + 31) // 32 for b in range(len(offsets) - 1)]
    scales = np.zeros((sum(nblk), H, d), np.uint8)
    blk0 = 0
    for b in range(len(offsets) - 1):
        r0, r1 = int(offsets[b]), int(offsets[b + 1])
        for c in range(nblk[b]):
            lo, hi = r0 + 32 * c, min(r1, r0 + 32 * c + 32)
            block = np.zeros((32, H, d))
            block[: hi - lo] = x64[lo:hi]
            # one MX block per (head, column): 32 values along rows
            bt = np.ascontiguousarray(block.transpose(1, 2, 0))  # [H, d, 32]
            cb, sb = quantize_mx(bt)
            codes[lo:hi] = cb.transpose(2, 0, 1)[: hi - lo]
            scales[blk0 + c] = sb.reshape(H, d)
        blk0 += nblk[b]
    return codes, scales


_E4M3_TABLE = None


def _e4m3_table() -> np.ndarray:
    """e4m3_decode of every byte, so that whole tensors decode by indexing."""
    global _E4M3_TABLE
    if _E4M3_TABLE is None:
        _E4M3_TABLE = np.array([e4m3_decode(c) for c in range(256)], np.float64)
    return _E4M3_TABLE


def dequantize_along_rows(codes, scales, offsets):
    codes = np.asarray(codes, np.uint8)
    offsets = _i32(offsets)
    rows, H, d = codes.shape
    out = np.zeros((rows, H, d))
    blk0 = 0
    for b in range(len(offsets) - 1):
        r0, r1 = int(offsets[b]), int(offsets[b + 1])
        nb = (r1 - r0 + 31) // 32
        for c in range(nb):
            lo, hi = r0 + 32 * c, min(r1, r0 + 32 * c + 32)
            # E4M3 value of each code times the block's power-of-two scale
            out[lo:hi] = _e4m3_table()[codes[lo:hi]] * np.power(
                2.0, scales[blk0 + c].astype(np.float64) - 127.0)
        blk0 += nb
    return out


# ---------------------------------------------------------------------------
# Longest-first tile schedule (plain restatement, integer arithmetic).
#
# A forward work item is (sequence b, head h, query tile t) covering query rows
# [t*tile, min(n_q, (t+1)*tile)); a backward item is (b, h, key tile t).  Its
# cost is the number of (query, key) pairs it computes: the number of keys each
# of its rows may see (bottom-right causal: row i sees keys j <= i + n_kv - n_q),
# or for a key tile the number of queries that may see each key.  Forward
# items are ordered by cost descending, ties by (b, t, h) ascending; backward
# items are grouped by (sequence, head) -- sequences by their total cost
# descending, ties by b -- with the key tiles of a group in ascending order.
# ---------------------------------------------------------------------------

def _visible_keys(i, nq, nkv, causal, window=0):
    p = i + nkv - nq                      # bottom-right aligned position
    hi = min(nkv - 1, p) if causal else (min(nkv - 1, p + window - 1) if window else nkv - 1)
    lo = max(0, p - window + 1) if window else 0
    return max(0, hi - lo + 1)


def _seeing_queries(j, nq, nkv, causal, window=0):
    shift = nkv - nq                      # query i sits at position i + shift
    lo = max(0, j - shift) if causal else (max(0, j - window + 1 - shift) if window else 0)
    hi = min(nq - 1, j + window - 1 - shift) if window else nq - 1
    return max(0, hi - lo + 1)


def schedule(q_off, kv_off, H, tile, causal, backward=False, window=0):
    """Returns int32 [N, 4] rows (b, h, t, cost) in execution order."""
    q_off, kv_off = _i32(q_off), _i32(kv_off)
    pairs = []
    for b in range(len(q_off) - 1):
        nq = int(q_off[b + 1] - q_off[b])
        nkv = int(kv_off[b + 1] - kv_off[b])
        n_rows = nkv if backward else nq
        n_tiles = (n_rows + tile - 1) // tile
        for t in range(n_tiles):
            lo, hi = t * tile, min(n_rows, (t + 1) * tile)
            if backward:
                cost = sum(_seeing_queries(j, nq, nkv, causal, window) for j in range(lo, hi))
            else:
                cost = sum(_visible_keys(i, nq, nkv, causal, window) for i in range(lo, hi))
            pairs.append((cost, b, t))
    if not backward:
        pairs.sort(key=lambda p: (-p[0], p[1], p[2]))
        out = [(b, h, t, cost) for (cost, b, t) in pairs for h in range(H)]
    else:
        # key tiles grouped by (sequence, head): sequences by their total pair
        # count descending (ties by b), then heads, then tiles ascending
        seq_cost, by_seq = {}, {}
        for cost, b, t in pairs:
            seq_cost[b] = seq_cost.get(b, 0) + cost
            by_seq.setdefault(b, []).append((t, cost))
        order = sorted(by_seq, key=lambda b: (-seq_cost[b], b))
        out = [(b, h, t, cost) for b in order for h in range(H) for (t, cost) in sorted(by_seq[b])]
    return np.asarray(out, dtype=np.int32).reshape(-1, 4)


def valid_pairs(q_off, kv_off, causal, window=0):
    """Number of (query, key) pairs that attention computes, per head."""
    q_off, kv_off = _i32(q_off), _i32(kv_off)
    total = 0
    for b in range(len(q_off) - 1):
        nq = int(q_off[b + 1] - q_off[b])
        nkv = int(kv_off[b + 1] - kv_off[b])
        total += sum(_visible_keys(i, nq, nkv, causal, window) for i in range(nq))
    return total


# ---------------------------------------------------------------------------
# Data-parallel split of a global batch (plain restatement).
#
# "Meta GEM Training Efficiency: Why LLM-Scale Recommenders Need a Different
# Stack", "Bottleneck move 4: memory relief to load balance": jagged batches
# leave ranks unevenly loaded; base batch shuffling sorts small sub-batches by
# total sequence length and interleaves heavy and light ones, with no
# cross-rank communication.  Read here as: sub-batches of ``sub_batch``
# consecutive sequences, sorted by sum(n_q + n_kv) descending (ties by index),
# dealt in snake order.  The alternative rule is longest-processing-time-first
# on the visible-pair cost.  The cost of a sequence is its number of visible
# (query, key) pairs, counted row by row.
# ---------------------------------------------------------------------------

def sequence_pairs(nq, nkv, causal, window=0):
    return sum(_visible_keys(i, nq, nkv, causal, window) for i in range(nq))


def partition(q_lens, kv_lens, causal, ranks, method="lpt", sub_batch=1, window=0):
    """Returns (rank_of [B], rank_cost [ranks]) as int lists."""
    q_lens = [int(x) for x in q_lens]
    kv_lens = [int(x) for x in kv_lens]
    B = len(q_lens)
    cost = [sequence_pairs(q_lens[b], kv_lens[b], causal, window) for b in range(B)]
    rank_of = [0] * B
    if method == "lpt":
        load = [0] * ranks
        for b in sorted(range(B), key=lambda b: (-cost[b], b)):
            r = min(range(ranks), key=lambda r: (load[r], r))
            rank_of[b] = r
            load[r] += cost[b]
    else:
        groups = [list(range(g, min(B, g + sub_batch))) for g in range(0, B, sub_batch)]
        length = [sum(q_lens[b] + kv_lens[b] for b in grp) for grp in groups]
        order = sorted(range(len(groups)), key=lambda g: (-length[g], g))
        for pos, g in enumerate(order):
            rnd, c = divmod(pos, ranks)
            r = c if rnd % 2 == 0 else ranks - 1 - c
            for b in groups[g]:
                rank_of[b] = r
    rank_cost = [0] * ranks
    for b in range(B):
        rank_cost[rank_of[b]] += cost[b]
    return rank_of, rank_cost


# ---------------------------------------------------------------------------
# Normalisation ahead of MX quantisation (plain fp64 definitions).
#   RMSNorm  : y = x * gamma / sqrt(mean(x^2) + eps)
#   LayerNorm: y = (x - mean(x)) * gamma / sqrt(mean((x - mean)^2) + eps) + beta
# "Meta Enhances GEM Training Efficiency ...", "Implementing Ultra-Low-Precision
# Methods": the quantisation is fused into the normalisation that produces the
# low-precision operand; the result is then quantised like quantize_mx.
# ---------------------------------------------------------------------------

def norm(x, gamma=None, beta=None, eps=1e-6, layernorm=False) -> np.ndarray:
    """x [rows, D] -> y [rows, D] in fp64."""
    x64 = _f64(x)
    mean = x64.mean(axis=-1, keepdims=True) if layernorm else 0.0
    c = x64 - mean
    var = (c * c).mean(axis=-1, keepdims=True)
    y = c / np.sqrt(var + eps)
    if gamma is not None:
        y = y * _f64(gamma)
    if layernorm and beta is not None:
        y = y + _f64(beta)
    return y
