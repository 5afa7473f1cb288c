"""Seeded synthetic inputs for jagged attention.

This module only draws numbers: sequence lengths, offsets and normally
distributed tensors.  It holds none of the attention arithmetic, so that both
the CUDA path and the CPU oracle can take the same inputs from it.

Workloads (the source pages measure on unpublished production shapes; these
synthetic batches stand in for them, with the length mixes of a recommender's
user-history encoder, target-aware cross attention, the GDPA variant and the
MXFP8 run):

* ``tiny_f32``      B=4, n ~ U{1..64} (n_q = n_kv), H=2, d=32, fp32, relative-
                    position table of 129 entries ~ N(0, 0.5), causal softmax.
* ``self_bf16``     B=256, n = clip(rint(LogNormal(6.5, 1.0)), 16, 4096), H=8,
                    d=128, bf16, table of 8193 entries ~ N(0, 0.5), causal.
* ``cross_bf16``    B=1024, n_q ~ U{1..64}, n_kv = clip(rint(LogNormal(7.0, 0.8)),
                    32, 8192), H=4, d=128, bf16, dense jagged bias ~ N(0, 0.1),
                    no mask, softmax.
* ``gdpa_bf16``     as ``cross_bf16`` with SiLU (or tanh-GELU) instead of softmax.
* ``self_mxfp8``    as ``self_bf16`` with B=512, lengths clipped to [16, 8192],
                    table of 16385 entries; MXFP8 compute, bf16 in/out.

Draw order from ``numpy.random.default_rng(seed)`` (PCG64): query lengths,
key/value lengths (when separate), then one 63-bit seed each for Q, K, V, bias
and dO; each tensor is filled from PCG64 streams spawned from its seed, one
stream per 2^22 elements (parallel, thread-count independent).  Values are
drawn as float32 standard normals and rounded to the stored dtype with
round-to-nearest-even (torch's conversion); a relative-position table for a bf16 run is
rounded to bf16 and stored as fp32, so that every consumer sees the same
values.
"""
from __future__ import annotations

import dataclasses
import os
from typing import Optional

import numpy as np
import torch

WORKLOADS = {
    "tiny_f32": dict(B=4, H=2, d=32, dtype="f32", q_len=("uniform", 1, 64), kv_len=None,
                     bias="relpos", bias_std=0.5, causal=True, act="softmax"),
    "self_bf16": dict(B=256, H=8, d=128, dtype="bf16", q_len=("lognormal", 6.5, 1.0, 16, 4096),
                      kv_len=None, bias="relpos", bias_std=0.5, causal=True, act="softmax"),
    "cross_bf16": dict(B=1024, H=4, d=128, dtype="bf16", q_len=("uniform", 1, 64),
                       kv_len=("lognormal", 7.0, 0.8, 32, 8192), bias="dense", bias_std=0.1,
                       causal=False, act="softmax"),
    "gdpa_bf16": dict(B=1024, H=4, d=128, dtype="bf16", q_len=("uniform", 1, 64),
                      kv_len=("lognormal", 7.0, 0.8, 32, 8192), bias="dense", bias_std=0.1,
                      causal=False, act="silu"),
    "self_mxfp8": dict(B=512, H=8, d=128, dtype="mxfp8",
                       q_len=("lognormal", 6.5, 1.0, 16, 8192), kv_len=None, bias="relpos",
                       bias_std=0.5, causal=True, act="softmax"),
}


@dataclasses.dataclass
class Problem:
    name: str
    B: int
    H: int
    d: int
    dtype: str            # "f32", "bf16" or "mxfp8" (bf16 storage, MXFP8 compute)
    causal: bool
    act: str              # "softmax", "silu", "gelu_tanh"
    bias_kind: str        # "none", "relpos", "dense"
    relpos_len: int
    q_off: torch.Tensor   # int32 [B+1]
    kv_off: torch.Tensor  # int32 [B+1]
    q: torch.Tensor       # [total_q, H, d]
    k: torch.Tensor       # [total_kv, H, d]
    v: torch.Tensor       # [total_kv, H, d]
    bias: Optional[torch.Tensor]
    dout: torch.Tensor    # [total_q, H, d]
    seed: int

    @property
    def total_q(self) -> int:
        return int(self.q_off[-1])

    @property
    def total_kv(self) -> int:
        return int(self.kv_off[-1])

    @property
    def q_lens(self) -> np.ndarray:
        return np.diff(self.q_off.numpy())

    @property
    def kv_lens(self) -> np.ndarray:
        return np.diff(self.kv_off.numpy())

    @property
    def max_q_len(self) -> int:
        return int(self.q_lens.max()) if self.B else 0

    @property
    def max_kv_len(self) -> int:
        return int(self.kv_lens.max()) if self.B else 0


def _lengths(rng, spec, B, hi_override=None):
    kind = spec[0]
    if kind == "uniform":
        lo, hi = spec[1], spec[2]
        if hi_override is not None:
            hi = min(hi, hi_override)
        return rng.integers(lo, hi + 1, size=B).astype(np.int64)
    if kind == "lognormal":
        mu, sigma, lo, hi = spec[1:]
        if hi_override is not None:
            hi = hi_override
        return np.clip(np.rint(rng.lognormal(mu, sigma, size=B)), lo, hi).astype(np.int64)
    raise ValueError(kind)


def _offsets(lens) -> torch.Tensor:
    off = np.zeros(len(lens) + 1, np.int64)
    off[1:] = np.cumsum(lens)
    assert off[-1] < 2**31
    return torch.from_numpy(off.astype(np.int32))


_CHUNK = 1 << 22  # elements per independent stream chunk


def _fill_chunk(seed_seq, out, lo, hi, std):
    g = np.random.Generator(np.random.PCG64(seed_seq))
    g.standard_normal(size=hi - lo, dtype=np.float32, out=out[lo:hi])
    if std != 1.0:
        out[lo:hi] *= np.float32(std)


def _normal(rng, shape, std, dtype):
    """Standard normals (times std) in chunks of 2^22 elements, chunk c drawn
    from child c of a SeedSequence seeded by one draw of ``rng``, so large
    tensors fill in parallel and the values do not depend on the thread
    count."""
    n = int(np.prod(shape))
    root = np.random.SeedSequence(int(rng.integers(0, 2**63 - 1)))
    n_chunks = max(1, (n + _CHUNK - 1) // _CHUNK)
    children = root.spawn(n_chunks)
    flat = np.empty(n, np.float32)
    if n_chunks == 1:
        _fill_chunk(children[0], flat, 0, n, std)
    else:
        import concurrent.futures as cf
        with cf.ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 1)) as ex:
            list(ex.map(lambda c: _fill_chunk(children[c], flat, c * _CHUNK,
                                              min(n, (c + 1) * _CHUNK), std), range(n_chunks)))
    t = torch.from_numpy(flat.reshape(shape))
    if dtype == "f32":
        return t
    return t.to(torch.bfloat16)


def draw_lengths(workload: str, seed: int = 0, *, B: Optional[int] = None,
                 max_len: Optional[int] = None):
    """The (q_lens, kv_lens) that make_problem(workload, seed, B=B,
    max_len=max_len) draws (the lengths are its first draws), without the
    tensors: every rank of a data-parallel run can draw the global batch's
    lengths and split it without drawing the tensors of other ranks."""
    spec = dict(WORKLOADS[workload])
    B = spec["B"] if B is None else B
    rng = np.random.default_rng(seed)
    q_lens = _lengths(rng, spec["q_len"], B, max_len if spec["kv_len"] is None else None)
    if spec["kv_len"] is None:
        kv_lens = q_lens.copy()
    else:
        kv_lens = _lengths(rng, spec["kv_len"], B, max_len)
    return q_lens, kv_lens


def make_problem(workload: str, seed: int = 0, *, B: Optional[int] = None,
                 max_len: Optional[int] = None, q_lens=None, kv_lens=None,
                 act: Optional[str] = None, causal: Optional[bool] = None,
                 bias: Optional[str] = None, d: Optional[int] = None,
                 H: Optional[int] = None, dtype: Optional[str] = None) -> Problem:
    """Draw one batch.  ``B``/``max_len`` shrink a workload (the length
    distribution is kept, the clip is lowered); explicit ``q_lens``/``kv_lens``
    replace the length draws (edge-case tests)."""
    spec = dict(WORKLOADS[workload])
    B = spec["B"] if B is None else B
    H = spec["H"] if H is None else H
    d = spec["d"] if d is None else d
    dtype = spec["dtype"] if dtype is None else dtype
    act = spec["act"] if act is None else act
    causal = spec["causal"] if causal is None else causal
    bias_kind = spec["bias"] if bias is None else bias
    rng = np.random.default_rng(seed)
    if q_lens is None:
        q_lens = _lengths(rng, spec["q_len"], B, max_len if spec["kv_len"] is None else None)
    q_lens = np.asarray(q_lens, np.int64)
    B = len(q_lens)
    if kv_lens is None:
        if spec["kv_len"] is None:
            kv_lens = q_lens.copy()
        else:
            kv_lens = _lengths(rng, spec["kv_len"], B, max_len)
    kv_lens = np.asarray(kv_lens, np.int64)
    assert len(kv_lens) == B
    q_off, kv_off = _offsets(q_lens), _offsets(kv_lens)
    tq, tkv = int(q_off[-1]), int(kv_off[-1])
    store = "f32" if dtype == "f32" else "bf16"
    q = _normal(rng, (tq, H, d), 1.0, store)
    k = _normal(rng, (tkv, H, d), 1.0, store)
    v = _normal(rng, (tkv, H, d), 1.0, store)
    relpos_len = 0
    bias_t = None
    if bias_kind == "relpos":
        clip_hi = spec["q_len"][2] if spec["q_len"][0] == "uniform" else spec["q_len"][4]
        if max_len is not None:
            clip_hi = max_len
        longest = int(max(q_lens.max(initial=0), kv_lens.max(initial=0)))
        relpos_len = 2 * max(clip_hi, longest) + 1
        tab = _normal(rng, (H, relpos_len), spec["bias_std"], store)
        bias_t = tab.float().contiguous()
    elif bias_kind == "dense":
        n = int(np.sum(H * q_lens * kv_lens))
        bias_t = _normal(rng, (n,), spec["bias_std"], store)
    dout = _normal(rng, (tq, H, d), 1.0, store)
    return Problem(name=workload, B=B, H=H, d=d, dtype=dtype, causal=bool(causal), act=act,
                   bias_kind=bias_kind, relpos_len=relpos_len, q_off=q_off, kv_off=kv_off,
                   q=q, k=k, v=v, bias=bias_t, dout=dout, seed=seed)
