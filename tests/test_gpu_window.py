"""Sliding-window attention on the GPU against the oracle's window.

Query i (aligned position p = i + n_kv - n_q) sees key j only when p - j < w,
and without the causal rule also when j - p < w.  The kernels compute only the
key tiles inside the band (forward) and the query tiles that see a key tile
(backward); the schedules count the band's pairs (bit-exact against the
oracle's restatement).  Tolerances are those of the parity tests.

Pages: "Meta Enhances GEM Training Efficiency with Advanced LLM-Scale
Innovations", "Exploring the Customized Kernel Library" -> "BlockAttention"
(windows instead of full attention over long user histories).
"""
import numpy as np
import pytest
import torch

import oracle
from jagged_attention_recommender_jfa_b200 import jfa
from jagged_attention_recommender_jfa_b200.inputs import make_problem
from test_gpu_parity import (BF16_MAX, BF16_MEAN, F32_MAX, LSE_MAX, MX_MAX, _check_items,
                             _dev, _item_rows, compare, mx_dequantised_inputs)

pytestmark = pytest.mark.gpu


def run_window(p, dev, w, act=None, dbias=False):
    act = act or p.act
    d = _dev(p, dev)
    prob = jfa.problem_of(p, window=w)
    out, lse = jfa.attention_forward(prob, d["q"], d["k"], d["v"], d["q_off"], d["kv_off"],
                                     d["bias"], act, p.causal)
    grads = jfa.attention_backward(prob, d["q"], d["k"], d["v"], out, lse, d["dout"],
                                   d["q_off"], d["kv_off"], d["bias"], act, p.causal,
                                   want_dbias=dbias)
    torch.cuda.synchronize()
    return out, lse, grads


def check_window(p, dev, w, act=None, strict_f32=False, inputs=None, quant_p=False, mx=False):
    act = act or p.act
    out, lse, (dq, dk, dv) = run_window(p, dev, w, act)
    q, k, v = inputs if inputs is not None else (p.q, p.k, p.v)
    kw = dict(bias=p.bias, bias_kind=p.bias_kind, relpos_len=p.relpos_len, act=act,
              causal=p.causal, window=w)
    ro, rl = oracle.forward(p.q_off, p.kv_off, q, k, v, quant_p=quant_p, **kw)
    rdq, rdk, rdv = oracle.backward(p.q_off, p.kv_off, q, k, v, p.dout,
                                    out_for_d=ro if mx else None, **kw)
    mxt = MX_MAX if mx else (F32_MAX if strict_f32 else BF16_MAX)
    mean = None if mx else BF16_MEAN
    rows = slice(None)
    compare("O", out, ro, rows, mxt, mean)
    if act == "softmax":
        compare("LSE", lse, rl, rows, F32_MAX if strict_f32 else LSE_MAX)
    compare("dQ", dq, rdq, rows, mxt, mean)
    compare("dK", dk, rdk, rows, mxt, mean)
    compare("dV", dv, rdv, rows, mxt, mean)


@pytest.mark.parametrize("tile", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("backward", [False, True])
@pytest.mark.parametrize("w", [1, 37, 200])
def test_window_schedule_bit_exact(cuda_device, tile, causal, backward, w):
    q_lens = [0, 1, tile - 1, tile, tile + 1, 3 * tile + 5, 7, 200, 1]
    kv_lens = [5, 1, tile, tile, tile + 3, 3 * tile + 5, 0, 150, 300]
    p = make_problem("cross_bf16", 0, q_lens=q_lens, kv_lens=kv_lens, H=3)
    prob = jfa.problem_of(p, window=w)
    d = _dev(p, cuda_device)
    cap = 4096
    items = torch.full((cap, 4), -7, dtype=torch.int32, device=cuda_device)
    count = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    ws = jfa.workspace(prob, True, cuda_device)
    jfa.jfa_schedule(prob, d["q_off"], d["kv_off"], causal, backward, tile, items, cap, count, ws)
    jfa.jfa_check_error(ws)
    n = int(count.item())
    ref = oracle.schedule(p.q_off, p.kv_off, 3, tile, causal, backward, window=w)
    assert n == len(ref)
    assert np.array_equal(items[:n].cpu().numpy(), ref)


# windows below, at and across the 128-key tile, and wider than most sequences
@pytest.mark.parametrize("w,act", [(1, "softmax"), (100, "softmax"), (128, "softmax"),
                                   (129, "softmax"), (300, "softmax"), (1000, "softmax"),
                                   (150, "silu"), (260, "gelu_tanh")])
def test_window_self_small(cuda_device, w, act):
    p = make_problem("self_bf16", 60, B=6, max_len=700, act=act)
    assert jfa.jfa_path(jfa.problem_of(p, window=w), act, 1) == 1
    check_window(p, cuda_device, w)


@pytest.mark.parametrize("w", [1, 90, 300])
def test_window_self_non_causal_band(cuda_device, w):
    p = make_problem("self_bf16", 61, B=5, max_len=600, causal=False)
    check_window(p, cuda_device, w)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("act", ["softmax", "silu"])
def test_window_cross_dense_bias(cuda_device, causal, act):
    # short queries against long histories: the window runs on the general
    # kernels (the short-query kernels take no window)
    p = make_problem("cross_bf16", 62, B=10, max_len=900, causal=causal, act=act)
    check_window(p, cuda_device, 170)


@pytest.mark.parametrize("q_lens,kv_lens,causal", [
    ([1, 64, 65, 127, 128, 129, 0, 2, 300], [1, 64, 65, 127, 128, 129, 3, 0, 300], True),
    ([90, 10, 130, 1, 0], [30, 10, 20, 5, 3], True),          # n_q > n_kv: rows with p < 0
    ([5, 40, 200], [300, 41, 180], False),
])
@pytest.mark.parametrize("w", [1, 64, 129])
def test_window_edge_lengths(cuda_device, q_lens, kv_lens, causal, w):
    p = make_problem("self_bf16", 63, q_lens=q_lens, kv_lens=kv_lens, causal=causal)
    check_window(p, cuda_device, w)


@pytest.mark.parametrize("d,dtype", [(32, "f32"), (64, "bf16"), (128, "f32")])
def test_window_cuda_core_path(cuda_device, d, dtype):
    p = make_problem("self_bf16", 64, B=5, max_len=300, d=d, dtype=dtype)
    assert jfa.jfa_path(jfa.problem_of(p, window=45), "softmax", 1) == 0
    check_window(p, cuda_device, 45, strict_f32=(dtype == "f32"))


def test_window_tiny_f32(cuda_device):
    p = make_problem("tiny_f32", 65)
    check_window(p, cuda_device, 5, strict_f32=True)


@pytest.mark.parametrize("w", [40, 200])
def test_window_mxfp8(cuda_device, w):
    p = make_problem("self_mxfp8", 66, B=6, max_len=500)
    check_window(p, cuda_device, w, inputs=mx_dequantised_inputs(p), quant_p=True, mx=True)


@pytest.mark.parametrize("workload,w", [("self_bf16", 150), ("cross_bf16", 200)])
def test_window_bias_gradient(cuda_device, workload, w):
    # both sides take the oracle's O (rounded to bf16) and LSE as the
    # backward's inputs, as in the bias-gradient parity tests
    from test_gpu_dbias import check_dense, check_relpos
    p = make_problem(workload, 67, B=5, max_len=500, causal=True)
    kw = dict(bias=p.bias, bias_kind=p.bias_kind, relpos_len=p.relpos_len, causal=True,
              window=w)
    ro, rl = oracle.forward(p.q_off, p.kv_off, p.q, p.k, p.v, **kw)
    out = torch.from_numpy(ro).to(p.q.dtype)
    ref = oracle.backward(p.q_off, p.kv_off, p.q, p.k, p.v, p.dout, dbias=True, out_for_d=out,
                          **kw)[3]
    d = _dev(p, cuda_device)
    prob = jfa.problem_of(p, window=w)
    *_, db = jfa.attention_backward(prob, d["q"], d["k"], d["v"], out.to(cuda_device),
                                    torch.from_numpy(rl).float().to(cuda_device), d["dout"],
                                    d["q_off"], d["kv_off"], d["bias"], "softmax", True,
                                    want_dbias=True)
    torch.cuda.synchronize()
    if p.bias_kind == "relpos":
        C = (p.relpos_len - 1) // 2
        n_c = np.zeros(p.relpos_len, np.int64)
        for n in p.q_lens:
            i = np.arange(n)[:, None]
            j = np.arange(n)[None, :]
            ok = (j <= i) & (i - j < w)
            np.add.at(n_c, (np.clip(i - j, -C, C) + C)[ok], 1)
        check_relpos("dtable", db, ref, n_c, BF16_MAX, BF16_MEAN)
    else:
        valid = []
        for nq, nk in zip(p.q_lens, p.kv_lens):
            pos = np.arange(nq)[:, None] + (nk - nq)
            j = np.arange(nk)[None, :]
            ok = (j <= pos) & (pos - j < w)
            valid.append(np.broadcast_to(ok, (p.H, nq, nk)).reshape(-1))
        check_dense("dbias", db, ref, BF16_MAX, BF16_MEAN, valid=np.concatenate(valid))


def test_window_full_size_sampled(cuda_device):
    # the self-attention workload at full size with a 512-key window, checked
    # on the shortest and the longest sequences (all heads)
    w = 512
    p = make_problem("self_bf16", 1)
    out, lse, (dq, dk, dv) = run_window(p, cuda_device, w)
    order = np.argsort(p.q_lens, kind="stable")
    mask = np.zeros(p.B * p.H, np.int32)
    for b in list(order[:2]) + list(order[-2:]):
        mask[b * p.H:(b + 1) * p.H] = 1
    kw = dict(bias=p.bias, bias_kind="relpos", relpos_len=p.relpos_len, causal=True, window=w,
              seq_mask=mask)
    ro, rl = oracle.forward(p.q_off, p.kv_off, p.q, p.k, p.v, **kw)
    rdq, rdk, rdv = oracle.backward(p.q_off, p.kv_off, p.q, p.k, p.v, p.dout, **kw)
    rows, heads = _item_rows(p.q_off, p.H, mask)
    _check_items("O", out, ro, rows, heads, BF16_MAX, BF16_MEAN)
    assert np.all(np.abs(lse.cpu().numpy()[rows, heads] - rl[rows, heads]) <= LSE_MAX)
    _check_items("dQ", dq, rdq, rows, heads, BF16_MAX, BF16_MEAN)
    _check_items("dK", dk, rdk, rows, heads, BF16_MAX, BF16_MEAN)
    _check_items("dV", dv, rdv, rows, heads, BF16_MAX, BF16_MEAN)
    assert torch.isfinite(out).all() and torch.isfinite(dq).all()
