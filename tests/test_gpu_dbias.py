"""GPU parity of the bias gradient (jfa_backward_dbias) against the oracle.

The backward takes the forward's output O and LSE as inputs, and D =
rowsum(dO * O) comes from that O.  A bf16 O carries its final rounding (2^-9
relative), which moves D -- and with it every score gradient ds of the row --
by up to |dO| |O| 2^-9: harmless in dQ / dK (sums over many pairs) but of the
order of the bound in a single ds.  So both sides here get the same O and LSE:
the oracle's forward, rounded to the stored types, is passed to the GPU
backward and, as out_for_d, to the oracle's backward.

Bounds, written here:
  dense jagged bias (one ds per entry): max |err| <= 2e-2 + half a bf16 ulp of
      the reference and mean |err| <= 2e-3, the benchmark spec's bounds for bf16
      gradients (fp32 path: max 1e-4);
  relative-position table: entry c sums ds over the n_c valid pairs on its
      (clamped) diagonal, so the per-pair bounds are applied to the error
      divided by sqrt(n_c) (independent per-pair errors add in quadrature):
      max_c |err_c| / sqrt(n_c) <= 2e-2 and mean_c |err_c| / sqrt(n_c) <= 2e-3.
"""
import numpy as np
import pytest
import torch

import oracle
from jagged_attention_recommender_jfa_b200 import jfa
from jagged_attention_recommender_jfa_b200.inputs import make_problem

pytestmark = pytest.mark.gpu

BF16_MAX, BF16_MEAN, F32_MAX = 2e-2, 2e-3, 1e-4


def half_ulp_bf16(x):
    ax = np.maximum(np.abs(x), 2.0 ** -126)
    return np.exp2(np.floor(np.log2(ax)) - 8)


def _dev(p, dev):
    t = lambda x: None if x is None else x.to(dev).contiguous()
    return {n: t(getattr(p, n)) for n in ("q", "k", "v", "dout", "bias", "q_off", "kv_off")}


def oracle_forward_inputs(p, act, dev):
    """The oracle's O (rounded to the stored type) and LSE (fp32), as the
    backward's inputs on both sides."""
    ro, rl = oracle.forward(p.q_off, p.kv_off, p.q, p.k, p.v, bias=p.bias,
                            bias_kind=p.bias_kind, relpos_len=p.relpos_len, act=act,
                            causal=p.causal)
    out = torch.from_numpy(ro).to(p.q.dtype).to(dev)
    lse = torch.from_numpy(rl).float().to(dev) if rl is not None else None
    return out, lse


def run_gpu(p, dev, act=None):
    act = act or p.act
    d = _dev(p, dev)
    prob = jfa.problem_of(p)
    out, lse = oracle_forward_inputs(p, act, dev)
    dq, dk, dv, db = jfa.attention_backward(prob, d["q"], d["k"], d["v"], out, lse, d["dout"],
                                            d["q_off"], d["kv_off"], d["bias"], act, p.causal,
                                            want_dbias=True)
    dq0, dk0, dv0 = jfa.attention_backward(prob, d["q"], d["k"], d["v"], out, lse, d["dout"],
                                           d["q_off"], d["kv_off"], d["bias"], act, p.causal)
    torch.cuda.synchronize()
    # asking for the bias gradient leaves the other gradients as they were
    # (dK, dV are written once per key tile; dQ adds in a varying order)
    assert torch.equal(dk, dk0) and torch.equal(dv, dv0)
    assert torch.allclose(dq.float(), dq0.float(), atol=1e-2, rtol=0)
    return db


def pairs_per_entry(p):
    """n_c: valid (query, key) pairs per table entry, per head."""
    C = (p.relpos_len - 1) // 2
    n = np.zeros(p.relpos_len, np.int64)
    for nq, nk in zip(p.q_lens, p.kv_lens):
        nq, nk = int(nq), int(nk)
        if nq == 0 or nk == 0:
            continue
        i = np.arange(nq)[:, None]
        j = np.arange(nk)[None, :]
        ok = np.ones((nq, nk), bool) if not p.causal else (j <= i + nk - nq)
        np.add.at(n, (np.clip(i - j, -C, C) + C)[ok], 1)
    return n


def check_relpos(name, db, ref, n_c, max_tol, mean_tol):
    g = db.double().cpu().numpy()
    err = np.abs(g - ref)
    used = n_c > 0
    # entries no pair reads are exactly 0
    assert np.all(g[:, ~used] == 0.0), f"{name}: unused entries written"
    w = err[:, used] / np.sqrt(n_c[used])[None, :]
    assert w.max() <= max_tol, f"{name}: max |err|/sqrt(n) {w.max():.3e}"
    assert w.mean() <= mean_tol, f"{name}: mean |err|/sqrt(n) {w.mean():.3e}"


def dense_mask(p):
    """True at the valid (query, key) pairs of the dense bias layout."""
    parts = []
    for nq, nk in zip(p.q_lens, p.kv_lens):
        nq, nk = int(nq), int(nk)
        i = np.arange(nq)[:, None]
        j = np.arange(nk)[None, :]
        ok = np.ones((nq, nk), bool) if not p.causal else (j <= i + nk - nq)
        parts.append(np.broadcast_to(ok, (p.H, nq, nk)).reshape(-1))
    return np.concatenate(parts) if parts else np.zeros(0, bool)


def check_dense(name, db, ref, max_tol, mean_tol, rows_mask=None, valid=None):
    g = db.double().cpu().numpy()
    if valid is not None:
        # masked pairs are exactly zero
        assert np.all(g[~valid] == 0.0), f"{name}: masked pairs not zero"
    if rows_mask is not None:
        g, ref = g[rows_mask], ref[rows_mask]
    assert np.all(np.isfinite(ref))
    err = np.abs(g - ref)
    bf16 = db.dtype == torch.bfloat16
    bound = max_tol + (half_ulp_bf16(ref) if bf16 else 0.0)
    assert np.all(err <= bound), f"{name}: max |err| {err.max():.3e}"
    refm = torch.from_numpy(ref).to(torch.bfloat16).double().numpy() if bf16 else ref
    assert np.abs(g - refm).mean() <= mean_tol, f"{name}: mean |err|"


def oracle_dbias(p, act, seq_mask=None):
    out, _ = oracle_forward_inputs(p, act, "cpu")
    return oracle.backward(p.q_off, p.kv_off, p.q, p.k, p.v, p.dout, bias=p.bias,
                           bias_kind=p.bias_kind, relpos_len=p.relpos_len, act=act,
                           causal=p.causal, seq_mask=seq_mask, dbias=True,
                           out_for_d=out if act == "softmax" else None)[3]


CASES = [
    # (workload, seed, kwargs, act)
    ("self_bf16", 40, dict(B=6, max_len=300), None),                       # relpos, causal
    ("self_bf16", 41, dict(B=5, max_len=260, act="silu"), None),           # relpos, GDPA
    ("cross_bf16", 42, dict(B=12, max_len=700), None),                     # dense, no mask
    ("gdpa_bf16", 43, dict(B=12, max_len=700), "gelu_tanh"),               # dense, GDPA
    ("cross_bf16", 44, dict(q_lens=[90, 10, 130, 1, 0], kv_lens=[30, 10, 20, 5, 3],
                            causal=True), None),                            # dense, causal, n_q > n_kv
    ("self_bf16", 45, dict(q_lens=[1, 64, 65, 127, 128, 129, 0, 2], bias="dense"), None),
    ("self_bf16", 46, dict(B=4, max_len=200, relpos_len_override=41), None),  # clamped table
]


@pytest.mark.parametrize("workload,seed,kw,act", CASES)
def test_dbias_small(cuda_device, workload, seed, kw, act):
    kw = dict(kw)
    rl = kw.pop("relpos_len_override", None)
    p = make_problem(workload, seed, **kw)
    if rl is not None:   # a table shorter than 2 max_len + 1: the ends collect the far pairs
        p.relpos_len = rl
        p.bias = p.bias[:, :rl].contiguous()
    act = act or p.act
    db = run_gpu(p, cuda_device, act)
    ref = oracle_dbias(p, act)
    if p.bias_kind == "relpos":
        check_relpos("dtable", db, ref, pairs_per_entry(p), BF16_MAX, BF16_MEAN)
    else:
        check_dense("dbias", db, ref, BF16_MAX, BF16_MEAN, valid=dense_mask(p))


@pytest.mark.parametrize("d,bias", [(32, "relpos"), (64, "dense")])
def test_dbias_cuda_core_path(cuda_device, d, bias):
    p = make_problem("self_bf16", 47, B=5, max_len=150, d=d, H=3, dtype="f32", bias=bias)
    assert jfa.jfa_path(jfa.problem_of(p), p.act, 1) == 0
    db = run_gpu(p, cuda_device)
    ref = oracle_dbias(p, p.act)
    if bias == "relpos":
        check_relpos("dtable", db, ref, pairs_per_entry(p), F32_MAX, F32_MAX)
    else:
        check_dense("dbias", db, ref, F32_MAX, F32_MAX, valid=dense_mask(p))


def test_dbias_tiny_f32(cuda_device):
    for seed in range(3):
        p = make_problem("tiny_f32", seed)
        db = run_gpu(p, cuda_device)
        check_relpos("dtable", db, oracle_dbias(p, p.act), pairs_per_entry(p), F32_MAX, F32_MAX)


def test_dbias_rejected_without_bias(cuda_device):
    p = make_problem("self_bf16", 48, B=2, max_len=40, bias="none")
    d = _dev(p, cuda_device)
    prob = jfa.problem_of(p)
    ws = jfa.workspace(prob, True, cuda_device)
    x = torch.empty_like(d["q"])
    with pytest.raises(jfa.JfaError) as ei:
        jfa.jfa_backward_dbias(prob, d["q"], d["k"], d["v"], x, None, d["dout"], d["q_off"],
                               d["kv_off"], None, "silu", True, x, x, x, x, ws)
    assert ei.value.status == jfa.JFA_ERR_INVALID_ARGUMENT


def test_dbias_full_size_cross_sampled(cuda_device):
    # the cross-attention workload at full size, as the benchmark launches it;
    # dense-bias blocks of sampled (sequence, head) items checked entry by entry
    p = make_problem("cross_bf16", 1)
    db = run_gpu(p, cuda_device)
    lens = p.kv_lens
    order = np.argsort(lens, kind="stable")
    picks = list(order[:3]) + list(order[-2:])
    mask = np.zeros(p.B * p.H, np.int32)
    sel = np.zeros(db.numel(), bool)
    starts = np.concatenate([[0], np.cumsum(p.H * p.q_lens * p.kv_lens)])
    for b in picks:
        for h in (0, p.H - 1):
            mask[b * p.H + h] = 1
            blk = int(p.q_lens[b] * p.kv_lens[b])
            s0 = int(starts[b]) + h * blk
            sel[s0:s0 + blk] = True
    ref = oracle_dbias(p, p.act, seq_mask=mask)
    check_dense("dbias", db, ref, BF16_MAX, BF16_MEAN, rows_mask=sel)


def test_dbias_full_length_relpos(cuda_device):
    # the self-attention workload's longest sequences (4096 tokens: 32 key
    # tiles, the table clamped at neither end) with a few short ones, all heads
    full = make_problem("self_bf16", 1)
    order = np.argsort(full.q_lens, kind="stable")
    picks = sorted(list(order[:2]) + list(order[-2:]))
    lens = full.q_lens[picks]
    p = make_problem("self_bf16", 2, q_lens=lens)
    assert p.relpos_len == full.relpos_len and int(lens.max()) == 4096
    db = run_gpu(p, cuda_device)
    ref = oracle_dbias(p, p.act)
    check_relpos("dtable", db, ref, pairs_per_entry(p), BF16_MAX, BF16_MEAN)
