"""Python binding of libjfa (ctypes).

Argument marshalling only: every step of the computation runs in the CUDA
kernels of ``libjfa.so``.  The functions named like the C entry points
(``jfa_forward``, ``jfa_backward``, ...) take torch tensors (device memory)
or raw integer addresses and raise :class:`JfaError` on a non-OK status.
``attention_forward`` / ``attention_backward`` additionally allocate outputs
and the workspace with torch.

If ``libjfa.so`` is missing it is built with nvcc (the same sm_100a build as
``python -m jagged_attention_recommender_jfa_b200.build``); if that is not
possible the import of the library fails loudly -- there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_PKG, "libjfa.so")
_LOCK = threading.Lock()
_LIB = None

JFA_OK, JFA_ERR_INVALID_ARGUMENT, JFA_ERR_UNSUPPORTED, JFA_ERR_WORKSPACE = 0, 1, 2, 3
JFA_ERR_CUDA, JFA_ERR_TIMEOUT, JFA_ERR_BAD_OFFSETS = 4, 5, 6
JFA_F32, JFA_BF16, JFA_MXFP8 = 0, 1, 2
ACT = {"softmax": 0, "silu": 1, "gelu_tanh": 2}
BIAS = {"none": 0, "relpos": 1, "dense": 2}
DTYPE = {"f32": JFA_F32, "bf16": JFA_BF16, "mxfp8": JFA_MXFP8}
STATUS_NAMES = {0: "JFA_OK", 1: "JFA_ERR_INVALID_ARGUMENT", 2: "JFA_ERR_UNSUPPORTED",
                3: "JFA_ERR_WORKSPACE", 4: "JFA_ERR_CUDA", 5: "JFA_ERR_TIMEOUT",
                6: "JFA_ERR_BAD_OFFSETS"}

# Every symbol include/jfa.h declares.
EXPORTS = ("jfa_workspace_bytes", "jfa_forward", "jfa_backward", "jfa_quantize_mxfp8",
           "jfa_quantize_mxfp8_dequant",
           "jfa_schedule", "jfa_check_error", "jfa_last_error", "jfa_path",
           "jfa_profile_enable", "jfa_profile_read", "jfa_kernel_name",
           "jfa_forward_fixed_scratch", "jfa_partition", "jfa_backward_dbias",
           "jfa_block_offsets", "jfa_test_inject", "jfa_forward_mxfp8",
           "jfa_norm_quantize_mxfp8")
JFA_TEST_FWD_SKIP_LOAD = 1
PARTITION = {"lpt": 0, "bbs": 1}


class JfaError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


class jfa_problem(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("max_q_len", ctypes.c_int32),
                ("max_kv_len", ctypes.c_int32), ("total_q", ctypes.c_int64),
                ("total_kv", ctypes.c_int64), ("dtype", ctypes.c_int), ("scale", ctypes.c_float),
                ("bias_kind", ctypes.c_int), ("relpos_len", ctypes.c_int32),
                ("window", ctypes.c_int32)]


def lib_path() -> str:
    return _LIB_PATH


def load():
    """Loads libjfa.so (building it if absent) and declares the signatures."""
    global _LIB
    with _LOCK:
        if _LIB is not None:
            return _LIB
        if not os.path.exists(_LIB_PATH):
            from . import build as _build
            _build.build()
        lib = ctypes.CDLL(_LIB_PATH)
        P, i32, i64, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
        PP = ctypes.POINTER(jfa_problem)
        lib.jfa_workspace_bytes.argtypes = [PP, i32]
        lib.jfa_workspace_bytes.restype = sz
        lib.jfa_forward.argtypes = [PP, P, P, P, P, P, P, i32, i32, P, P, P, sz, P]
        lib.jfa_forward.restype = i32
        lib.jfa_backward.argtypes = [PP, P, P, P, P, P, P, P, P, P, i32, i32, P, P, P, P, sz, P]
        lib.jfa_backward.restype = i32
        lib.jfa_quantize_mxfp8.argtypes = [P, i64, i32, i32, P, i32, i32, i32, P, P, P]
        lib.jfa_quantize_mxfp8.restype = i32
        lib.jfa_quantize_mxfp8_dequant.argtypes = [P, i64, i32, i32, P, i32, i32, i32, P, P, P, P]
        lib.jfa_quantize_mxfp8_dequant.restype = i32
        lib.jfa_schedule.argtypes = [PP, P, P, i32, i32, i32, P, i64, P, P, sz, P]
        lib.jfa_schedule.restype = i32
        lib.jfa_check_error.argtypes = [P, P]
        lib.jfa_check_error.restype = i32
        lib.jfa_last_error.restype = ctypes.c_char_p
        lib.jfa_path.argtypes = [PP, i32, i32]
        lib.jfa_path.restype = i32
        lib.jfa_profile_enable.argtypes = [i32]
        lib.jfa_profile_enable.restype = i32
        lib.jfa_profile_read.argtypes = [P, P, i32]
        lib.jfa_profile_read.restype = i32
        lib.jfa_kernel_name.argtypes = [i32]
        lib.jfa_kernel_name.restype = ctypes.c_char_p
        lib.jfa_forward_fixed_scratch.argtypes = [PP, P, P, P, P, P, P, i32, i32, P, P, P]
        lib.jfa_forward_fixed_scratch.restype = i32
        lib.jfa_backward_dbias.argtypes = [PP, P, P, P, P, P, P, P, P, P, i32, i32, P, P, P, P, P,
                                           sz, P]
        lib.jfa_backward_dbias.restype = i32
        lib.jfa_forward_mxfp8.argtypes = [PP, P, P, P, P, P, P, P, P, P, i32, P, P, P, sz, P]
        lib.jfa_forward_mxfp8.restype = i32
        lib.jfa_norm_quantize_mxfp8.argtypes = [P, i64, i32, P, P, ctypes.c_float, i32, P, P, P]
        lib.jfa_norm_quantize_mxfp8.restype = i32
        lib.jfa_test_inject.argtypes = [i32]
        lib.jfa_test_inject.restype = i32
        lib.jfa_block_offsets.argtypes = [P, i32, i64, i32, P, P]
        lib.jfa_block_offsets.restype = i32
        lib.jfa_partition.argtypes = [i32, P, P, i32, i32, i32, i32, i32, P, P]
        lib.jfa_partition.restype = i32
        _LIB = lib
        return lib


def _addr(x) -> Optional[int]:
    if x is None:
        return None
    if isinstance(x, torch.Tensor):
        return x.data_ptr() if x.numel() > 0 else None
    return int(x)


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _check(status: int):
    if status != JFA_OK:
        raise JfaError(status, load().jfa_last_error().decode())


def make_problem(*, batch, heads, head_dim, max_q_len, max_kv_len, total_q, total_kv,
                 dtype="bf16", scale=0.0, bias_kind="none", relpos_len=0, window=0) -> jfa_problem:
    """``window`` > 0: sliding window of that width (0: none)."""
    return jfa_problem(int(batch), int(heads), int(head_dim), int(max_q_len), int(max_kv_len),
                       int(total_q), int(total_kv), DTYPE[dtype] if isinstance(dtype, str) else int(dtype),
                       float(scale), BIAS[bias_kind] if isinstance(bias_kind, str) else int(bias_kind),
                       int(relpos_len), int(window))


def problem_of(p, dtype: Optional[str] = None, window: int = 0) -> jfa_problem:
    """Descriptor of an ``inputs.Problem`` batch."""
    return make_problem(batch=p.B, heads=p.H, head_dim=p.d, max_q_len=p.max_q_len,
                        max_kv_len=p.max_kv_len, total_q=p.total_q, total_kv=p.total_kv,
                        dtype=dtype or p.dtype, bias_kind=p.bias_kind, relpos_len=p.relpos_len,
                        window=window)


# ---------------------------------------------------------------------------
# Entry points (same names as the C ABI)
# ---------------------------------------------------------------------------

def jfa_workspace_bytes(problem: jfa_problem, backward: int) -> int:
    return int(load().jfa_workspace_bytes(ctypes.byref(problem), int(backward)))


def jfa_path(problem: jfa_problem, act, backward: int) -> int:
    return int(load().jfa_path(ctypes.byref(problem), ACT.get(act, act), int(backward)))


def jfa_forward(problem, q, k, v, q_offsets, kv_offsets, bias, act, causal, out, lse, workspace,
                ws_bytes=None, stream=None):
    if ws_bytes is None:
        ws_bytes = workspace.numel() * workspace.element_size()
    _check(load().jfa_forward(ctypes.byref(problem), _addr(q), _addr(k), _addr(v),
                              _addr(q_offsets), _addr(kv_offsets), _addr(bias),
                              ACT.get(act, act), int(bool(causal)), _addr(out), _addr(lse),
                              _addr(workspace), int(ws_bytes), _stream(stream)))


def jfa_forward_mxfp8(problem, q8, q_scales, k8, k_scales, v8, v_scales, q_offsets, kv_offsets,
                      bias, causal, out, lse, workspace, ws_bytes=None, stream=None):
    if ws_bytes is None:
        ws_bytes = workspace.numel() * workspace.element_size()
    _check(load().jfa_forward_mxfp8(ctypes.byref(problem), _addr(q8), _addr(q_scales), _addr(k8),
                                    _addr(k_scales), _addr(v8), _addr(v_scales), _addr(q_offsets),
                                    _addr(kv_offsets), _addr(bias), int(bool(causal)), _addr(out),
                                    _addr(lse), _addr(workspace), int(ws_bytes), _stream(stream)))


def jfa_forward_fixed_scratch(problem, q, k, v, q_offsets, kv_offsets, bias, act, causal, out,
                              lse, stream=None):
    """Forward without a workspace: for callers that cannot allocate device
    memory (scratch is a fixed 8 MiB array inside the library; see jfa.h)."""
    _check(load().jfa_forward_fixed_scratch(ctypes.byref(problem), _addr(q), _addr(k), _addr(v),
                                            _addr(q_offsets), _addr(kv_offsets), _addr(bias),
                                            ACT.get(act, act), int(bool(causal)), _addr(out),
                                            _addr(lse), _stream(stream)))


def jfa_backward(problem, q, k, v, out, lse, dout, q_offsets, kv_offsets, bias, act, causal,
                 dq, dk, dv, workspace, ws_bytes=None, stream=None):
    if ws_bytes is None:
        ws_bytes = workspace.numel() * workspace.element_size()
    _check(load().jfa_backward(ctypes.byref(problem), _addr(q), _addr(k), _addr(v), _addr(out),
                               _addr(lse), _addr(dout), _addr(q_offsets), _addr(kv_offsets),
                               _addr(bias), ACT.get(act, act), int(bool(causal)), _addr(dq),
                               _addr(dk), _addr(dv), _addr(workspace), int(ws_bytes),
                               _stream(stream)))


def jfa_backward_dbias(problem, q, k, v, out, lse, dout, q_offsets, kv_offsets, bias, act,
                       causal, dq, dk, dv, dbias, workspace, ws_bytes=None, stream=None):
    if ws_bytes is None:
        ws_bytes = workspace.numel() * workspace.element_size()
    _check(load().jfa_backward_dbias(ctypes.byref(problem), _addr(q), _addr(k), _addr(v),
                                     _addr(out), _addr(lse), _addr(dout), _addr(q_offsets),
                                     _addr(kv_offsets), _addr(bias), ACT.get(act, act),
                                     int(bool(causal)), _addr(dq), _addr(dk), _addr(dv),
                                     _addr(dbias), _addr(workspace), int(ws_bytes),
                                     _stream(stream)))


def jfa_quantize_mxfp8(x, rows, heads, d, offsets, batch, max_len, along_rows, codes, scales,
                       stream=None):
    _check(load().jfa_quantize_mxfp8(_addr(x), int(rows), int(heads), int(d), _addr(offsets),
                                     int(batch), int(max_len), int(bool(along_rows)),
                                     _addr(codes), _addr(scales), _stream(stream)))


def jfa_quantize_mxfp8_dequant(x, rows, heads, d, offsets, batch, max_len, along_rows, codes,
                               scales, dequant, stream=None):
    _check(load().jfa_quantize_mxfp8_dequant(_addr(x), int(rows), int(heads), int(d), _addr(offsets),
                                             int(batch), int(max_len), int(bool(along_rows)),
                                             _addr(codes), _addr(scales), _addr(dequant),
                                             _stream(stream)))


def jfa_schedule(problem, q_offsets, kv_offsets, causal, backward, tile, items, capacity, count,
                 workspace, ws_bytes=None, stream=None):
    if ws_bytes is None:
        ws_bytes = workspace.numel() * workspace.element_size()
    _check(load().jfa_schedule(ctypes.byref(problem), _addr(q_offsets), _addr(kv_offsets),
                               int(bool(causal)), int(bool(backward)), int(tile), _addr(items),
                               int(capacity), _addr(count), _addr(workspace), int(ws_bytes),
                               _stream(stream)))


def jfa_block_offsets(offsets, batch, total, block, block_offsets, stream=None):
    _check(load().jfa_block_offsets(_addr(offsets), int(batch), int(total), int(block),
                                    _addr(block_offsets), _stream(stream)))


def block_attention(problem: jfa_problem, offsets, block: int, stream=None):
    """BlockAttention with block length ``block`` as a jagged problem over the
    blocks: returns (descriptor, block offsets) to pass to jfa_forward /
    jfa_backward as both q and kv offsets (self-attention)."""
    n_out = problem.batch + problem.total_q // block
    boff = torch.empty(n_out + 1, dtype=torch.int32, device=offsets.device)
    jfa_block_offsets(offsets, problem.batch, problem.total_q, block, boff, stream)
    p2 = jfa_problem.from_buffer_copy(problem)
    p2.batch = n_out
    p2.max_q_len = min(block, problem.max_q_len)
    p2.max_kv_len = min(block, problem.max_kv_len)
    return p2, boff


def jfa_partition(q_lens, kv_lens, causal, ranks, method="lpt", sub_batch=1, window=0):
    """Host-side split of a global batch across ``ranks``: returns (rank_of
    int32 [batch], rank_cost int64 [ranks]) as numpy arrays.  ``window`` > 0
    counts a sliding window's pairs."""
    import numpy as np
    ql = np.ascontiguousarray(np.asarray(q_lens, np.int32))
    kl = np.ascontiguousarray(np.asarray(kv_lens, np.int32))
    assert ql.shape == kl.shape and ql.ndim == 1
    rank_of = np.zeros(len(ql), np.int32)
    rank_cost = np.zeros(int(ranks), np.int64)
    c = lambda a: a.ctypes.data_as(ctypes.c_void_p)
    _check(load().jfa_partition(len(ql), c(ql), c(kl), int(bool(causal)), int(window), int(ranks),
                                PARTITION.get(method, method), int(sub_batch), c(rank_of),
                                c(rank_cost)))
    return rank_of, rank_cost


def jfa_norm_quantize_mxfp8(x, rows, D, gamma, beta, eps, layernorm, codes, scales, stream=None):
    _check(load().jfa_norm_quantize_mxfp8(_addr(x), int(rows), int(D), _addr(gamma), _addr(beta),
                                          float(eps), int(bool(layernorm)), _addr(codes),
                                          _addr(scales), _stream(stream)))


def jfa_test_inject(what: int):
    _check(load().jfa_test_inject(int(what)))


def jfa_profile_enable(enable: bool):
    _check(load().jfa_profile_enable(int(bool(enable))))


def jfa_profile_read():
    """[(kernel name, ms), ...] of the launches recorded since profiling was enabled."""
    lib = load()
    n = lib.jfa_profile_read(None, None, 0)
    if n < 0:
        raise JfaError(JFA_ERR_CUDA, "profile read failed")
    ms = (ctypes.c_float * max(n, 1))()
    ids = (ctypes.c_int32 * max(n, 1))()
    n2 = lib.jfa_profile_read(ms, ids, n)
    if n2 < 0:
        raise JfaError(JFA_ERR_CUDA, "profile read failed")
    return [(lib.jfa_kernel_name(ids[i]).decode(), float(ms[i])) for i in range(n)]


def jfa_kernel_name(kernel_id: int) -> str:
    return load().jfa_kernel_name(int(kernel_id)).decode()


def jfa_check_error(workspace, stream=None):
    _check(load().jfa_check_error(_addr(workspace), _stream(stream)))


# ---------------------------------------------------------------------------
# Allocating conveniences (torch owns the memory)
# ---------------------------------------------------------------------------

def workspace(problem: jfa_problem, backward: bool, device) -> torch.Tensor:
    n = jfa_workspace_bytes(problem, int(backward))
    if n == 0:
        raise JfaError(JFA_ERR_INVALID_ARGUMENT, load().jfa_last_error().decode())
    return torch.empty(n, dtype=torch.uint8, device=device)


def attention_forward(problem, q, k, v, q_offsets, kv_offsets, bias=None, act="softmax",
                      causal=False, ws=None, stream=None, check=True):
    """Allocates out / lse (and the workspace unless ``ws`` is given) and runs
    jfa_forward.  With ``check`` (the default) the stream is synchronised and
    the workspace's device error word is read, so that bad offsets or a timed
    out device wait raise :class:`JfaError` here; ``check=False`` leaves that
    to the caller (``jfa_check_error(ws)``) and keeps the call asynchronous."""
    out = torch.empty_like(q)
    lse = None
    if act == "softmax":
        lse = torch.empty(q.shape[0], q.shape[1], dtype=torch.float32, device=q.device)
    if ws is None:
        ws = workspace(problem, False, q.device)
    jfa_forward(problem, q, k, v, q_offsets, kv_offsets, bias, act, causal, out, lse, ws,
                stream=stream)
    if check:
        jfa_check_error(ws, stream)
    return out, lse


def attention_backward(problem, q, k, v, out, lse, dout, q_offsets, kv_offsets, bias=None,
                       act="softmax", causal=False, ws=None, stream=None, check=True,
                       want_dbias=False):
    """Allocates dq / dk / dv (and the workspace unless ``ws`` is given) and
    runs jfa_backward; ``check`` as in :func:`attention_forward`.  With
    ``want_dbias`` it runs jfa_backward_dbias and also returns the bias
    gradient (shaped like ``bias``)."""
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    if ws is None:
        ws = workspace(problem, True, q.device)
    if want_dbias:
        dbias = torch.empty_like(bias)
        jfa_backward_dbias(problem, q, k, v, out, lse, dout, q_offsets, kv_offsets, bias, act,
                           causal, dq, dk, dv, dbias, ws, stream=stream)
    else:
        jfa_backward(problem, q, k, v, out, lse, dout, q_offsets, kv_offsets, bias, act, causal,
                     dq, dk, dv, ws, stream=stream)
    if check:
        jfa_check_error(ws, stream)
    return (dq, dk, dv, dbias) if want_dbias else (dq, dk, dv)
