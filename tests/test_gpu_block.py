"""BlockAttention on the GPU: jfa_block_offsets rewrites the offsets (bit
exact against a plain construction), and jagged attention over the blocks
matches the oracle's BlockAttention (each query sees only its own block of W
keys) within the bf16 bounds of the parity tests.

Pages: "Meta Enhances GEM Training Efficiency with Advanced LLM-Scale
Innovations", "Exploring the Customized Kernel Library" -> "BlockAttention";
"Meta GEM Training Efficiency: Why LLM-Scale Recommenders Need a Different
Stack", "Bottleneck move 1" (independent fixed-size blocks).
"""
import numpy as np
import pytest
import torch

import oracle
from jagged_attention_recommender_jfa_b200 import jfa
from jagged_attention_recommender_jfa_b200.inputs import make_problem
from test_gpu_parity import BF16_MAX, BF16_MEAN, LSE_MAX, compare, _check_items, _item_rows

pytestmark = pytest.mark.gpu


def expected_block_offsets(lens, W):
    cut = [min(W, n - c) for n in lens for c in range(0, n, W)]
    total = int(sum(lens))
    n_out = len(lens) + total // W
    off = np.full(n_out + 1, total, np.int64)
    off[:len(cut) + 1] = np.concatenate([[0], np.cumsum(cut)])
    return off


def run_block(p, dev, W, act=None, dbias=False):
    act = act or p.act
    t = {n: getattr(p, n).to(dev).contiguous() for n in ("q", "k", "v", "dout", "q_off")}
    bias = p.bias.to(dev).contiguous() if p.bias is not None else None
    prob, boff = jfa.block_attention(jfa.problem_of(p), t["q_off"], W)
    assert np.array_equal(boff.cpu().numpy(), expected_block_offsets(p.q_lens, W))
    out, lse = jfa.attention_forward(prob, t["q"], t["k"], t["v"], boff, boff, bias, act, p.causal)
    grads = jfa.attention_backward(prob, t["q"], t["k"], t["v"], out, lse, t["dout"], boff, boff,
                                   bias, act, p.causal, want_dbias=dbias)
    torch.cuda.synchronize()
    return out, lse, grads


@pytest.mark.parametrize("W,act", [(64, "softmax"), (128, "softmax"), (200, "softmax"),
                                   (1000, "softmax"), (96, "silu"), (256, "gelu_tanh")])
def test_block_attention_small(cuda_device, W, act):
    p = make_problem("self_bf16", 50, B=6, max_len=600, act=act)
    out, lse, (dq, dk, dv) = run_block(p, cuda_device, W)
    kw = dict(bias=p.bias, bias_kind="relpos", relpos_len=p.relpos_len, act=act,
              causal=p.causal, block=W)
    ro, rl = oracle.forward(p.q_off, p.kv_off, p.q, p.k, p.v, **kw)
    rdq, rdk, rdv = oracle.backward(p.q_off, p.kv_off, p.q, p.k, p.v, p.dout, **kw)
    rows = slice(None)
    compare("O", out, ro, rows, BF16_MAX, BF16_MEAN)
    if act == "softmax":
        compare("LSE", lse, rl, rows, LSE_MAX)
    compare("dQ", dq, rdq, rows, BF16_MAX, BF16_MEAN)
    compare("dK", dk, rdk, rows, BF16_MAX, BF16_MEAN)
    compare("dV", dv, rdv, rows, BF16_MAX, BF16_MEAN)


def test_block_attention_bias_gradient(cuda_device):
    from test_gpu_dbias import check_relpos
    p = make_problem("self_bf16", 51, B=5, max_len=500)
    W = 160
    *_, (dq, dk, dv, db) = run_block(p, cuda_device, W, dbias=True)
    ref = oracle.backward(p.q_off, p.kv_off, p.q, p.k, p.v, p.dout, bias=p.bias,
                          bias_kind="relpos", relpos_len=p.relpos_len, causal=True, block=W,
                          dbias=True)[3]
    C = (p.relpos_len - 1) // 2
    n_c = np.zeros(p.relpos_len, np.int64)
    for n in p.q_lens:
        i = np.arange(n)[:, None]
        j = np.arange(n)[None, :]
        ok = (j <= i) & (i // W == j // W)
        np.add.at(n_c, (np.clip(i - j, -C, C) + C)[ok], 1)
    check_relpos("dtable", db, ref, n_c, BF16_MAX, BF16_MEAN)


def test_block_offsets_bad_input_reported(cuda_device):
    off = torch.tensor([0, 5, 3, 9], dtype=torch.int32, device=cuda_device)
    boff = torch.zeros(3 + 9 // 4 + 1, dtype=torch.int32, device=cuda_device)
    jfa.jfa_block_offsets(off, 3, 9, 4, boff)
    torch.cuda.synchronize()
    assert int(boff[0]) == -1
    with pytest.raises(jfa.JfaError):
        jfa.jfa_block_offsets(off, 3, 9, 0, boff)


def test_block_attention_full_size_sampled(cuda_device):
    # the self-attention workload at full size with 256-row blocks, checked on
    # the shortest and the longest sequences (all heads)
    W = 256
    p = make_problem("self_bf16", 1)
    out, lse, (dq, dk, dv) = run_block(p, cuda_device, W)
    order = np.argsort(p.q_lens, kind="stable")
    mask = np.zeros(p.B * p.H, np.int32)
    for b in list(order[:2]) + list(order[-2:]):
        mask[b * p.H:(b + 1) * p.H] = 1
    kw = dict(bias=p.bias, bias_kind="relpos", relpos_len=p.relpos_len, causal=True, block=W,
              seq_mask=mask)
    ro, rl = oracle.forward(p.q_off, p.kv_off, p.q, p.k, p.v, **kw)
    rdq, rdk, rdv = oracle.backward(p.q_off, p.kv_off, p.q, p.k, p.v, p.dout, **kw)
    rows, heads = _item_rows(p.q_off, p.H, mask)
    _check_items("O", out, ro, rows, heads, BF16_MAX, BF16_MEAN)
    assert np.all(np.abs(lse.cpu().numpy()[rows, heads] - rl[rows, heads]) <= LSE_MAX)
    _check_items("dQ", dq, rdq, rows, heads, BF16_MAX, BF16_MEAN)
    _check_items("dK", dk, rdk, rows, heads, BF16_MAX, BF16_MEAN)
    _check_items("dV", dv, rdv, rows, heads, BF16_MAX, BF16_MEAN)
