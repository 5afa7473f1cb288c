"""Pins of the fp64 oracle against things other than itself.

Each test ties the oracle to a library routine, a closed form, an invariant or
finite differences, so that a dropped term, a wrong sign/index or a transposed
operand in ``oracle/jfa_oracle.c`` fails at least one of them:

* softmax forward/LSE/gradients  == padded ``scaled_dot_product_attention`` and
  ``logsumexp`` in float64 with ``torch.autograd`` (bottom-right causal from
  ``torch.nn.attention.bias.causal_lower_right``);
* GDPA forward/gradients         == padded einsum with ``F.silu`` /
  ``F.gelu(approximate="tanh")`` and autograd;
* all gradients                  == central finite differences of <dO, O>;
* closed forms (Q = 0), V = 1 normalisation, single key, permutation of
  sequences, neighbours not leaking in, empty rows.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F
from torch.nn.attention.bias import causal_lower_right

import oracle


def _jagged(seed, q_lens, kv_lens, H=2, d=8, bias_kind="relpos", relpos_len=None, dtype=torch.float64):
    g = torch.Generator().manual_seed(seed)
    q_lens = list(q_lens)
    kv_lens = list(kv_lens)
    q_off = torch.tensor([0] + list(np.cumsum(q_lens)), dtype=torch.int32)
    kv_off = torch.tensor([0] + list(np.cumsum(kv_lens)), dtype=torch.int32)
    tq, tk = int(q_off[-1]), int(kv_off[-1])
    q = torch.randn(tq, H, d, generator=g, dtype=dtype)
    k = torch.randn(tk, H, d, generator=g, dtype=dtype)
    v = torch.randn(tk, H, d, generator=g, dtype=dtype)
    do = torch.randn(tq, H, d, generator=g, dtype=dtype)
    bias = None
    if bias_kind == "relpos":
        relpos_len = relpos_len or 2 * max(q_lens + kv_lens) + 1
        bias = 0.5 * torch.randn(H, relpos_len, generator=g, dtype=dtype)
    elif bias_kind == "dense":
        n = sum(H * a * b for a, b in zip(q_lens, kv_lens))
        bias = 0.3 * torch.randn(n, generator=g, dtype=dtype)
        relpos_len = 0
    else:
        relpos_len = 0
    return dict(q_off=q_off, kv_off=kv_off, q=q, k=k, v=v, do=do, bias=bias,
                bias_kind=bias_kind, relpos_len=relpos_len or 0, H=H, d=d,
                q_lens=q_lens, kv_lens=kv_lens)


def _pad(x, off, L):
    B = len(off) - 1
    out = torch.zeros(B, L, *x.shape[1:], dtype=x.dtype)
    for b in range(B):
        n = int(off[b + 1] - off[b])
        out[b, :n] = x[int(off[b]):int(off[b + 1])]
    return out


def _padded_bias(P, Lq, Lk):
    """Dense [B, H, Lq, Lk] bias built from the storage formats by plain
    indexing: relative-position table entry of (i - j), or the jagged block."""
    B, H = len(P["q_lens"]), P["H"]
    out = torch.zeros(B, H, Lq, Lk, dtype=torch.float64)
    if P["bias_kind"] == "relpos":
        T = P["relpos_len"]
        C = (T - 1) // 2
        i = torch.arange(Lq)[:, None]
        j = torch.arange(Lk)[None, :]
        idx = (i - j).clamp(-C, C) + C
        for h in range(H):
            out[:, h] = P["bias"][h][idx]
    elif P["bias_kind"] == "dense":
        pos = 0
        for b in range(B):
            nq, nk = P["q_lens"][b], P["kv_lens"][b]
            blk = P["bias"][pos:pos + H * nq * nk].reshape(H, nq, nk)
            out[b, :, :nq, :nk] = blk
            pos += H * nq * nk
    return out


def _valid_mask(P, Lq, Lk, causal):
    B = len(P["q_lens"])
    m = torch.zeros(B, 1, Lq, Lk, dtype=torch.bool)
    for b in range(B):
        nq, nk = P["q_lens"][b], P["kv_lens"][b]
        if nq == 0 or nk == 0:
            continue
        blk = torch.ones(nq, nk, dtype=torch.bool)
        if causal:
            blk = causal_lower_right(nq, nk)._materialize()
        m[b, 0, :nq, :nk] = blk
    return m


def _padded_sdpa(P, causal, q=None, k=None, v=None):
    Lq, Lk = max(P["q_lens"]), max(P["kv_lens"])
    q = P["q"] if q is None else q
    k = P["k"] if k is None else k
    v = P["v"] if v is None else v
    qp = _pad(q, P["q_off"], Lq).transpose(1, 2)  # B, H, Lq, d
    kp = _pad(k, P["kv_off"], Lk).transpose(1, 2)
    vp = _pad(v, P["kv_off"], Lk).transpose(1, 2)
    valid = _valid_mask(P, Lq, Lk, causal)
    mask = _padded_bias(P, Lq, Lk).masked_fill(~valid, float("-inf"))
    return qp, kp, vp, mask, valid


def _unpad(xp, off):
    parts = []
    for b in range(len(off) - 1):
        n = int(off[b + 1] - off[b])
        parts.append(xp[b, :, :n].transpose(0, 1))
    return torch.cat(parts, 0)


CASES = [
    # (q_lens, kv_lens, causal, bias_kind)
    ([5, 1, 9, 4], [5, 1, 9, 4], True, "relpos"),
    ([7, 3, 12], [7, 3, 12], False, "relpos"),
    ([3, 8, 1], [11, 5, 6], False, "dense"),      # asymmetric, short q / long kv
    ([9, 6, 2], [4, 6, 7], True, "dense"),        # bottom-right causal, n_q != n_kv
    ([10, 2], [3, 9], True, "none"),
]


@pytest.mark.parametrize("q_lens,kv_lens,causal,bias_kind", CASES)
def test_softmax_forward_equals_padded_sdpa(q_lens, kv_lens, causal, bias_kind):
    P = _jagged(1, q_lens, kv_lens, bias_kind=bias_kind)
    out, lse = oracle.forward(P["q_off"], P["kv_off"], P["q"], P["k"], P["v"], bias=P["bias"],
                              bias_kind=bias_kind, relpos_len=P["relpos_len"], causal=causal)
    qp, kp, vp, mask, valid = _padded_sdpa(P, causal)
    ref = F.scaled_dot_product_attention(qp, kp, vp, attn_mask=mask)
    scores = qp @ kp.transpose(-1, -2) / math.sqrt(P["d"]) + mask
    ref_lse = torch.logsumexp(scores, dim=-1)  # B, H, Lq
    ref_o = _unpad(ref, P["q_off"]).numpy()
    ref_l = _unpad(ref_lse[..., None], P["q_off"])[..., 0].numpy()
    has_key = np.isfinite(ref_l)
    assert np.all(has_key.any(axis=1) | ~has_key.any(axis=1))
    np.testing.assert_allclose(out[has_key], ref_o[has_key], atol=1e-12, rtol=0)
    np.testing.assert_allclose(lse[has_key], ref_l[has_key], atol=1e-12, rtol=0)
    # rows that see no key: zero output, LSE = -inf
    assert np.all(out[~has_key] == 0.0)
    assert np.all(np.isneginf(lse[~has_key]))


@pytest.mark.parametrize("q_lens,kv_lens,causal,bias_kind", CASES)
def test_softmax_gradients_equal_autograd(q_lens, kv_lens, causal, bias_kind):
    P = _jagged(2, q_lens, kv_lens, bias_kind=bias_kind)
    dq, dk, dv = oracle.backward(P["q_off"], P["kv_off"], P["q"], P["k"], P["v"], P["do"],
                                 bias=P["bias"], bias_kind=bias_kind,
                                 relpos_len=P["relpos_len"], causal=causal)
    q = P["q"].clone().requires_grad_()
    k = P["k"].clone().requires_grad_()
    v = P["v"].clone().requires_grad_()
    qp, kp, vp, mask, valid = _padded_sdpa(P, causal, q, k, v)
    ref = F.scaled_dot_product_attention(qp, kp, vp, attn_mask=mask)
    row_ok = valid.any(-1, keepdim=True)  # rows that see at least one key
    ref = torch.where(row_ok, ref, torch.zeros_like(ref))
    o = _unpad(ref, P["q_off"])
    (o * P["do"]).sum().backward()
    np.testing.assert_allclose(dq, q.grad.numpy(), atol=1e-12, rtol=0)
    np.testing.assert_allclose(dk, k.grad.numpy(), atol=1e-12, rtol=0)
    np.testing.assert_allclose(dv, v.grad.numpy(), atol=1e-12, rtol=0)


def _padded_gdpa(P, causal, act, q, k, v):
    qp, kp, vp, mask, valid = _padded_sdpa(P, causal, q, k, v)
    bias = _padded_bias(P, qp.shape[2], kp.shape[2])
    s = torch.einsum("bhid,bhjd->bhij", qp, kp) / math.sqrt(P["d"]) + bias
    a = F.silu(s) if act == "silu" else F.gelu(s, approximate="tanh")
    nkv = torch.tensor(P["kv_lens"], dtype=torch.float64).view(-1, 1, 1, 1)
    a = torch.where(valid, a, torch.zeros_like(a)) / nkv
    return torch.einsum("bhij,bhjd->bhid", a, vp)


@pytest.mark.parametrize("act", ["silu", "gelu_tanh"])
@pytest.mark.parametrize("q_lens,kv_lens,causal,bias_kind", CASES)
def test_gdpa_equals_padded_einsum_and_autograd(act, q_lens, kv_lens, causal, bias_kind):
    P = _jagged(3, q_lens, kv_lens, bias_kind=bias_kind)
    out, lse = oracle.forward(P["q_off"], P["kv_off"], P["q"], P["k"], P["v"], bias=P["bias"],
                              bias_kind=bias_kind, relpos_len=P["relpos_len"], act=act,
                              causal=causal)
    assert lse is None
    q = P["q"].clone().requires_grad_()
    k = P["k"].clone().requires_grad_()
    v = P["v"].clone().requires_grad_()
    o = _unpad(_padded_gdpa(P, causal, act, q, k, v), P["q_off"])
    np.testing.assert_allclose(out, o.detach().numpy(), atol=1e-12, rtol=0)
    (o * P["do"]).sum().backward()
    dq, dk, dv = oracle.backward(P["q_off"], P["kv_off"], P["q"], P["k"], P["v"], P["do"],
                                 bias=P["bias"], bias_kind=bias_kind,
                                 relpos_len=P["relpos_len"], act=act, causal=causal)
    np.testing.assert_allclose(dq, q.grad.numpy(), atol=1e-12, rtol=0)
    np.testing.assert_allclose(dk, k.grad.numpy(), atol=1e-12, rtol=0)
    np.testing.assert_allclose(dv, v.grad.numpy(), atol=1e-12, rtol=0)


@pytest.mark.parametrize("act", ["softmax", "silu", "gelu_tanh"])
@pytest.mark.parametrize("causal", [False, True])
def test_gradients_match_central_differences(act, causal):
    P = _jagged(4, [4, 5], [5, 3], H=1, d=4, bias_kind="relpos")
    kw = dict(bias=P["bias"], bias_kind="relpos", relpos_len=P["relpos_len"], act=act,
              causal=causal)
    do = P["do"].numpy()

    def loss(q, k, v):
        o, _ = oracle.forward(P["q_off"], P["kv_off"], q, k, v, **kw)
        return float(np.sum(o * do))

    dq, dk, dv = oracle.backward(P["q_off"], P["kv_off"], P["q"], P["k"], P["v"], P["do"], **kw)
    h = 1e-6
    for name, grad in (("q", dq), ("k", dk), ("v", dv)):
        base = {n: P[n].numpy().copy() for n in ("q", "k", "v")}
        fd = np.zeros_like(grad)
        for idx in np.ndindex(*grad.shape):
            plus = {n: a.copy() for n, a in base.items()}
            minus = {n: a.copy() for n, a in base.items()}
            plus[name][idx] += h
            minus[name][idx] -= h
            fd[idx] = (loss(**plus) - loss(**minus)) / (2 * h)
        scale = max(1.0, np.abs(fd).max())
        assert np.abs(fd - grad).max() / scale < 1e-6, name


def test_closed_forms_zero_queries():
    q_lens, kv_lens = [6, 3, 7], [6, 3, 7]
    P = _jagged(5, q_lens, kv_lens, bias_kind="none")
    q0 = torch.zeros_like(P["q"])
    for causal in (False, True):
        out, lse = oracle.forward(P["q_off"], P["kv_off"], q0, P["k"], P["v"], causal=causal)
        for b in range(3):
            r0, n = int(P["q_off"][b]), q_lens[b]
            vb = P["v"][int(P["kv_off"][b]):int(P["kv_off"][b]) + kv_lens[b]].numpy()
            for i in range(n):
                nvis = i + 1 if causal else kv_lens[b]
                assert lse[r0 + i, 0] == pytest.approx(math.log(nvis), abs=1e-14)
                np.testing.assert_allclose(out[r0 + i], vb[:nvis].mean(0), atol=1e-14)
    # GDPA with Q = 0 and a constant bias c: o_i = act(c) * sum_valid v / n_kv
    c = 0.7
    T = 2 * 7 + 1
    tab = torch.full((2, T), c, dtype=torch.float64)
    for act, fn in (("silu", F.silu), ("gelu_tanh", lambda x: F.gelu(x, approximate="tanh"))):
        out, _ = oracle.forward(P["q_off"], P["kv_off"], q0, P["k"], P["v"], bias=tab,
                                bias_kind="relpos", relpos_len=T, act=act, causal=True)
        ac = float(fn(torch.tensor(c, dtype=torch.float64)))
        for b in range(3):
            r0 = int(P["q_off"][b])
            vb = P["v"][int(P["kv_off"][b]):int(P["kv_off"][b]) + kv_lens[b]].numpy()
            for i in range(q_lens[b]):
                np.testing.assert_allclose(out[r0 + i], ac * vb[:i + 1].sum(0) / kv_lens[b],
                                           atol=1e-14)
        # and act(0) = 0 for both activations
        out0, _ = oracle.forward(P["q_off"], P["kv_off"], q0, P["k"], P["v"], act=act)
        assert np.all(out0 == 0.0)


def test_rows_sum_to_one_and_single_key():
    P = _jagged(6, [5, 9, 1], [5, 9, 1], bias_kind="relpos")
    ones = torch.ones_like(P["v"])
    for causal in (False, True):
        out, _ = oracle.forward(P["q_off"], P["kv_off"], P["q"], P["k"], ones, bias=P["bias"],
                                bias_kind="relpos", relpos_len=P["relpos_len"], causal=causal)
        np.testing.assert_allclose(out, 1.0, atol=1e-14)
    # n_kv = 1: every query returns v_0 exactly (softmax weight 1)
    P1 = _jagged(7, [4, 3], [1, 1], bias_kind="dense")
    out, lse = oracle.forward(P1["q_off"], P1["kv_off"], P1["q"], P1["k"], P1["v"],
                              bias=P1["bias"], bias_kind="dense")
    for b in range(2):
        v0 = P1["v"][b].numpy()
        for i in range(int(P1["q_off"][b]), int(P1["q_off"][b + 1])):
            assert np.array_equal(out[i], v0)
    # causal self-attention row 0 sees only key 0
    out, _ = oracle.forward(P["q_off"], P["kv_off"], P["q"], P["k"], P["v"], bias=P["bias"],
                            bias_kind="relpos", relpos_len=P["relpos_len"], causal=True)
    for b in range(3):
        r0 = int(P["q_off"][b])
        assert np.array_equal(out[r0], P["v"][int(P["kv_off"][b])].numpy())


def test_permuting_sequences_permutes_outputs_and_neighbours_do_not_leak():
    q_lens, kv_lens = [4, 7, 2, 5], [6, 3, 8, 5]
    P = _jagged(8, q_lens, kv_lens, bias_kind="dense")
    kw = dict(bias_kind="dense", causal=True)
    out, lse = oracle.forward(P["q_off"], P["kv_off"], P["q"], P["k"], P["v"], bias=P["bias"], **kw)
    dq, dk, dv = oracle.backward(P["q_off"], P["kv_off"], P["q"], P["k"], P["v"], P["do"],
                                 bias=P["bias"], **kw)
    perm = [2, 0, 3, 1]

    def seg(x, off, b):
        return x[int(off[b]):int(off[b + 1])]

    def bias_seg(b):
        start = sum(2 * q_lens[c] * kv_lens[c] for c in range(b))
        return P["bias"][start:start + 2 * q_lens[b] * kv_lens[b]]

    Q = torch.cat([seg(P["q"], P["q_off"], b) for b in perm])
    K = torch.cat([seg(P["k"], P["kv_off"], b) for b in perm])
    V = torch.cat([seg(P["v"], P["kv_off"], b) for b in perm])
    DO = torch.cat([seg(P["do"], P["q_off"], b) for b in perm])
    Bb = torch.cat([bias_seg(b) for b in perm])
    qo = torch.tensor([0] + list(np.cumsum([q_lens[b] for b in perm])), dtype=torch.int32)
    ko = torch.tensor([0] + list(np.cumsum([kv_lens[b] for b in perm])), dtype=torch.int32)
    out2, lse2 = oracle.forward(qo, ko, Q, K, V, bias=Bb, **kw)
    dq2, dk2, dv2 = oracle.backward(qo, ko, Q, K, V, DO, bias=Bb, **kw)
    for pos, b in enumerate(perm):
        assert np.array_equal(seg(out2, qo, pos), seg(out, P["q_off"], b))
        assert np.array_equal(seg(lse2, qo, pos), seg(lse, P["q_off"], b))
        assert np.array_equal(seg(dq2, qo, pos), seg(dq, P["q_off"], b))
        assert np.array_equal(seg(dk2, ko, pos), seg(dk, P["kv_off"], b))
        assert np.array_equal(seg(dv2, ko, pos), seg(dv, P["kv_off"], b))
    # poison sequence 1 (huge values): the others are unchanged, bit for bit
    Qp, Kp, Vp = P["q"].clone(), P["k"].clone(), P["v"].clone()
    Qp[int(P["q_off"][1]):int(P["q_off"][2])] = 1e4
    Kp[int(P["kv_off"][1]):int(P["kv_off"][2])] = -1e4
    Vp[int(P["kv_off"][1]):int(P["kv_off"][2])] = float("nan")
    out3, _ = oracle.forward(P["q_off"], P["kv_off"], Qp, Kp, Vp, bias=P["bias"], **kw)
    for b in (0, 2, 3):
        assert np.array_equal(seg(out3, P["q_off"], b), seg(out, P["q_off"], b))


def test_empty_sequences_and_seq_mask():
    P = _jagged(9, [3, 0, 4, 2], [3, 2, 0, 2], bias_kind="dense")
    out, lse = oracle.forward(P["q_off"], P["kv_off"], P["q"], P["k"], P["v"], bias=P["bias"],
                              bias_kind="dense")
    # sequence 2 has queries but no keys: zero output, LSE -inf
    s2 = slice(int(P["q_off"][2]), int(P["q_off"][3]))
    assert np.all(out[s2] == 0.0) and np.all(np.isneginf(lse[s2]))
    dq, dk, dv = oracle.backward(P["q_off"], P["kv_off"], P["q"], P["k"], P["v"], P["do"],
                                 bias=P["bias"], bias_kind="dense")
    assert np.all(dq[s2] == 0.0)
    # sequence 1 has keys but no queries: zero dK, dV
    k1 = slice(int(P["kv_off"][1]), int(P["kv_off"][2]))
    assert np.all(dk[k1] == 0.0) and np.all(dv[k1] == 0.0)
    # a mask computes exactly the selected sequences
    outm, _ = oracle.forward(P["q_off"], P["kv_off"], P["q"], P["k"], P["v"], bias=P["bias"],
                             bias_kind="dense", seq_mask=[0, 0, 0, 1])
    s3 = slice(int(P["q_off"][3]), int(P["q_off"][4]))
    assert np.array_equal(outm[s3], out[s3])
    assert np.all(np.isnan(outm[: int(P["q_off"][3])]))


def test_schedule_covers_every_tile_once_longest_first():
    q_lens, kv_lens = [1, 16, 17, 40, 0, 33], [1, 16, 17, 40, 5, 70]
    q_off = np.array([0] + list(np.cumsum(q_lens)), np.int32)
    kv_off = np.array([0] + list(np.cumsum(kv_lens)), np.int32)
    H, tile = 3, 16
    for causal in (False, True):
        for backward in (False, True):
            items = oracle.schedule(q_off, kv_off, H, tile, causal, backward)
            rows = kv_lens if backward else q_lens
            expect = {(b, h, t) for b in range(len(rows)) for h in range(H)
                      for t in range((rows[b] + tile - 1) // tile)}
            got = [tuple(x[:3]) for x in items]
            assert len(got) == len(expect) and set(got) == expect
            costs = items[:, 3]
            if not backward:
                assert np.all(costs[:-1] >= costs[1:])
            else:
                # (sequence, head) groups are contiguous, their tiles ascending,
                # and sequences come by total cost descending
                keys = [(int(b), int(h)) for b, h, _, _ in items]
                starts = [i for i in range(len(keys)) if i == 0 or keys[i] != keys[i - 1]]
                assert len(starts) == len(set(keys))
                for i0, i1 in zip(starts, starts[1:] + [len(keys)]):
                    assert list(items[i0:i1, 2]) == list(range(i1 - i0))
                seq_tot = [int(costs[items[:, 0] == b].sum()) for b in range(len(rows))]
                seq_order = list(dict.fromkeys(int(b) for b in items[:, 0]))
                assert all(seq_tot[x] >= seq_tot[y] for x, y in zip(seq_order, seq_order[1:]))
            # per-item cost equals the number of pairs of the library's
            # bottom-right causal mask restricted to the tile
            total = 0
            for b, h, t, c in items:
                nq, nk = q_lens[b], kv_lens[b]
                m = (causal_lower_right(nq, nk)._materialize() if causal and nq and nk
                     else torch.ones(nq, nk, dtype=torch.bool))
                sub = m[:, t * tile:(t + 1) * tile] if backward else m[t * tile:(t + 1) * tile]
                assert int(sub.sum()) == c
                total += c
            assert total == H * oracle.valid_pairs(q_off, kv_off, causal)


def test_backward_d_from_saved_output():
    """D taken from a saved output equals the recomputed one when that output
    is the oracle's own forward; a perturbed output changes only the softmax
    score-gradient terms (dQ, dK), never dV."""
    P = _jagged(10, [6, 9], [6, 9], bias_kind="relpos")
    kw = dict(bias=P["bias"], bias_kind="relpos", relpos_len=P["relpos_len"], causal=True)
    out, _ = oracle.forward(P["q_off"], P["kv_off"], P["q"], P["k"], P["v"], **kw)
    ref = oracle.backward(P["q_off"], P["kv_off"], P["q"], P["k"], P["v"], P["do"], **kw)
    same = oracle.backward(P["q_off"], P["kv_off"], P["q"], P["k"], P["v"], P["do"],
                           out_for_d=out, **kw)
    for a, b in zip(ref, same):
        assert np.array_equal(a, b)
    bumped = oracle.backward(P["q_off"], P["kv_off"], P["q"], P["k"], P["v"], P["do"],
                             out_for_d=out * 1.01, **kw)
    assert np.array_equal(bumped[2], ref[2])
    assert not np.allclose(bumped[0], ref[0])


# ---------------------------------------------------------------------------
# Bias gradient ("custom biases": s = scale q.k + beta, so d loss / d beta is
# the score gradient summed over the pairs that read each bias entry)
# ---------------------------------------------------------------------------
BIAS_CASES = [c for c in CASES if c[3] != "none"]


@pytest.mark.parametrize("act", ["softmax", "silu", "gelu_tanh"])
@pytest.mark.parametrize("q_lens,kv_lens,causal,bias_kind", BIAS_CASES)
def test_bias_gradient_equals_autograd(act, q_lens, kv_lens, causal, bias_kind):
    P = _jagged(12, q_lens, kv_lens, bias_kind=bias_kind)
    got = oracle.backward(P["q_off"], P["kv_off"], P["q"], P["k"], P["v"], P["do"],
                          bias=P["bias"], bias_kind=bias_kind, relpos_len=P["relpos_len"],
                          act=act, causal=causal, dbias=True)
    P = dict(P)
    P["bias"] = P["bias"].clone().requires_grad_()
    if act == "softmax":
        qp, kp, vp, mask, valid = _padded_sdpa(P, causal)
        row_ok = valid.any(-1, keepdim=True)
        # rows that see no key take a zero mask (their output is discarded
        # below), so that no NaN of an all -inf row enters the backward
        mask = torch.where(row_ok, mask, torch.zeros_like(mask))
        ref = F.scaled_dot_product_attention(qp, kp, vp, attn_mask=mask)
        ref = torch.where(row_ok, ref, torch.zeros_like(ref))
    else:
        ref = _padded_gdpa(P, causal, act, P["q"], P["k"], P["v"])
    o = _unpad(ref, P["q_off"])
    (o * P["do"]).sum().backward()
    np.testing.assert_allclose(got[3], P["bias"].grad.numpy(), atol=1e-12, rtol=0)
    # and the other gradients are unchanged by asking for it
    base = oracle.backward(P["q_off"], P["kv_off"], P["q"], P["k"], P["v"], P["do"],
                           bias=P["bias"].detach(), bias_kind=bias_kind,
                           relpos_len=P["relpos_len"], act=act, causal=causal)
    for a, b in zip(base, got[:3]):
        assert np.array_equal(a, b)


@pytest.mark.parametrize("act", ["softmax", "gelu_tanh"])
@pytest.mark.parametrize("bias_kind", ["relpos", "dense"])
def test_bias_gradient_matches_central_differences(act, bias_kind):
    # relpos_len 5 < 2 * max_len + 1: the clamped end entries collect every
    # pair beyond the table
    P = _jagged(13, [4, 5], [5, 3], H=1, d=4, bias_kind=bias_kind, relpos_len=5)
    kw = dict(bias_kind=bias_kind, relpos_len=P["relpos_len"], act=act, causal=True)
    do = P["do"].numpy()
    base = P["bias"].numpy().copy()

    def loss(bias):
        o, _ = oracle.forward(P["q_off"], P["kv_off"], P["q"], P["k"], P["v"], bias=bias, **kw)
        return float(np.sum(o * do))

    _, _, _, db = oracle.backward(P["q_off"], P["kv_off"], P["q"], P["k"], P["v"], P["do"],
                                  bias=P["bias"], dbias=True, **kw)
    h = 1e-6
    fd = np.zeros_like(base)
    for idx in np.ndindex(*base.shape):
        plus, minus = base.copy(), base.copy()
        plus[idx] += h
        minus[idx] -= h
        fd[idx] = (loss(plus) - loss(minus)) / (2 * h)
    assert np.abs(fd - db).max() / max(1.0, np.abs(fd).max()) < 1e-6
    if bias_kind == "relpos":
        # bottom-right causal: i - j >= -1 in sequence 0 (n_kv = n_q + 1) and
        # >= 2 in sequence 1, so the clamped upper end collects pairs and the
        # lower end (i - j <= -2) is read by none
        assert db[0, -1] != 0.0 and db[0, 0] == 0.0


def test_bias_gradient_closed_form_uniform_scores():
    # Q = 0, zero bias, softmax: p_ij = 1 / n_vis(i) and, with V = 0,
    # dp = 0 and D = 0, so ds = 0; with dO = 1 and V = e_j-th basis-like
    # values ds_ij = p_ij (v_j . 1 - mean_vis(v . 1)).  Summed over a row the
    # bias gradient vanishes (softmax is shift-invariant): sum_j ds_ij = 0.
    P = _jagged(14, [6, 3], [6, 3], H=2, d=4, bias_kind="dense")
    q0 = torch.zeros_like(P["q"])
    b0 = torch.zeros_like(P["bias"])
    _, _, _, db = oracle.backward(P["q_off"], P["kv_off"], q0, P["k"], P["v"], P["do"],
                                  bias=b0, bias_kind="dense", causal=True, dbias=True)
    pos = 0
    for b, n in enumerate([6, 3]):
        blk = db[pos:pos + 2 * n * n].reshape(2, n, n)
        vb = P["v"][int(P["kv_off"][b]):int(P["kv_off"][b]) + n].numpy()
        dob = P["do"][int(P["q_off"][b]):int(P["q_off"][b]) + n].numpy()
        for h in range(2):
            np.testing.assert_allclose(blk[h].sum(1), 0.0, atol=1e-14)
            for i in range(n):
                dpv = vb[:i + 1, h] @ dob[i, h]            # dp_ij, j <= i
                want = (dpv - dpv.mean()) / (i + 1)
                np.testing.assert_allclose(blk[h, i, :i + 1], want, atol=1e-14)
                assert np.all(blk[h, i, i + 1:] == 0.0)    # masked pairs
        pos += 2 * n * n


# ---------------------------------------------------------------------------
# BlockAttention: each query sees only the keys of its own block of W
# consecutive positions (causal on top)
# ---------------------------------------------------------------------------
def _block_mask(P, Lq, Lk, causal, W):
    valid = _valid_mask(P, Lq, Lk, causal)
    i = torch.arange(Lq)[:, None]
    j = torch.arange(Lk)[None, :]
    return valid & ((i // W) == (j // W))[None, None]


@pytest.mark.parametrize("W", [1, 3, 4, 16])
@pytest.mark.parametrize("causal", [False, True])
def test_block_attention_equals_block_masked_sdpa(W, causal):
    lens = [5, 1, 9, 12]
    P = _jagged(15, lens, lens, bias_kind="relpos")
    kw = dict(bias=P["bias"], bias_kind="relpos", relpos_len=P["relpos_len"], causal=causal,
              block=W)
    out, lse = oracle.forward(P["q_off"], P["kv_off"], P["q"], P["k"], P["v"], **kw)
    dq, dk, dv, db = oracle.backward(P["q_off"], P["kv_off"], P["q"], P["k"], P["v"], P["do"],
                                     dbias=True, **kw)
    L = max(lens)
    q = P["q"].clone().requires_grad_()
    k = P["k"].clone().requires_grad_()
    v = P["v"].clone().requires_grad_()
    Pb = dict(P)
    Pb["bias"] = P["bias"].clone().requires_grad_()
    qp = _pad(q, P["q_off"], L).transpose(1, 2)
    kp = _pad(k, P["kv_off"], L).transpose(1, 2)
    vp = _pad(v, P["kv_off"], L).transpose(1, 2)
    valid = _block_mask(P, L, L, causal, W)
    row_ok = valid.any(-1, keepdim=True)
    mask = _padded_bias(Pb, L, L).masked_fill(~valid, float("-inf"))
    mask = torch.where(row_ok, mask, torch.zeros_like(mask))
    ref = F.scaled_dot_product_attention(qp, kp, vp, attn_mask=mask)
    ref = torch.where(row_ok, ref, torch.zeros_like(ref))
    scores = (qp @ kp.transpose(-1, -2) / math.sqrt(P["d"]) + mask).masked_fill(~valid, float("-inf"))
    ref_lse = _unpad(torch.logsumexp(scores, -1)[..., None], P["q_off"])[..., 0]
    o = _unpad(ref, P["q_off"])
    np.testing.assert_allclose(out, o.detach().numpy(), atol=1e-12, rtol=0)
    np.testing.assert_allclose(lse, ref_lse.detach().numpy(), atol=1e-12, rtol=0)
    (o * P["do"]).sum().backward()
    np.testing.assert_allclose(dq, q.grad.numpy(), atol=1e-12, rtol=0)
    np.testing.assert_allclose(dk, k.grad.numpy(), atol=1e-12, rtol=0)
    np.testing.assert_allclose(dv, v.grad.numpy(), atol=1e-12, rtol=0)
    np.testing.assert_allclose(db, Pb["bias"].grad.numpy(), atol=1e-12, rtol=0)


@pytest.mark.parametrize("act", ["softmax", "silu", "gelu_tanh"])
def test_block_attention_is_attention_on_the_blocks(act):
    # independent fixed-size blocks: the same as plain jagged attention over
    # the sequences cut into blocks of W (the last one shorter), bit for bit;
    # GDPA divides by the block's key count
    lens, W = [7, 1, 16, 10], 4
    P = _jagged(16, lens, lens, bias_kind="relpos")
    kw = dict(bias=P["bias"], bias_kind="relpos", relpos_len=P["relpos_len"], act=act,
              causal=True)
    out, lse = oracle.forward(P["q_off"], P["kv_off"], P["q"], P["k"], P["v"], block=W, **kw)
    grads = oracle.backward(P["q_off"], P["kv_off"], P["q"], P["k"], P["v"], P["do"], block=W,
                            **kw)
    cut = [min(W, n - c) for n in lens for c in range(0, n, W)]
    off = torch.tensor([0] + list(np.cumsum(cut)), dtype=torch.int32)
    out2, lse2 = oracle.forward(off, off, P["q"], P["k"], P["v"], **kw)
    grads2 = oracle.backward(off, off, P["q"], P["k"], P["v"], P["do"], **kw)
    assert np.array_equal(out, out2)
    if act == "softmax":
        assert np.array_equal(lse, lse2)
    for a, b in zip(grads, grads2):
        assert np.array_equal(a, b)
    # and it differs from full attention whenever a sequence spans blocks
    full, _ = oracle.forward(P["q_off"], P["kv_off"], P["q"], P["k"], P["v"], **kw)
    assert not np.allclose(full, out)


# ---------------------------------------------------------------------------
# Sliding-window attention: query i (aligned position p = i + n_kv - n_q)
# sees key j only when p - j < w, and without the causal rule also when
# j - p < w
# ---------------------------------------------------------------------------
def _window_mask(P, Lq, Lk, causal, w):
    B = len(P["q_lens"])
    m = torch.zeros(B, 1, Lq, Lk, dtype=torch.bool)
    for b in range(B):
        nq, nk = P["q_lens"][b], P["kv_lens"][b]
        if nq == 0 or nk == 0:
            continue
        p = torch.arange(nq)[:, None] + (nk - nq)
        j = torch.arange(nk)[None, :]
        blk = (p - j) < w
        blk &= (j <= p) if causal else ((j - p) < w)
        m[b, 0, :nq, :nk] = blk
    return m


WINDOW_CASES = [
    # (q_lens, kv_lens, causal, bias_kind, w)
    ([5, 1, 9, 12], [5, 1, 9, 12], True, "relpos", 3),
    ([5, 1, 9, 12], [5, 1, 9, 12], True, "relpos", 1),
    ([7, 3, 12], [7, 3, 12], False, "relpos", 4),
    ([3, 8, 1], [11, 5, 6], False, "dense", 2),     # short q / long kv, band around p
    ([9, 6, 2], [4, 6, 7], True, "dense", 3),       # n_q > n_kv: rows with p < 0 see nothing
]


@pytest.mark.parametrize("act", ["softmax", "silu", "gelu_tanh"])
@pytest.mark.parametrize("q_lens,kv_lens,causal,bias_kind,w", WINDOW_CASES)
def test_window_equals_band_masked_attention_and_autograd(act, q_lens, kv_lens, causal, bias_kind, w):
    P = _jagged(21, q_lens, kv_lens, bias_kind=bias_kind)
    kw = dict(bias=P["bias"], bias_kind=bias_kind, relpos_len=P["relpos_len"], causal=causal,
              act=act, window=w)
    out, lse = oracle.forward(P["q_off"], P["kv_off"], P["q"], P["k"], P["v"], **kw)
    dq, dk, dv, db = oracle.backward(P["q_off"], P["kv_off"], P["q"], P["k"], P["v"], P["do"],
                                     dbias=True, **kw)
    Lq, Lk = max(q_lens), max(kv_lens)
    q = P["q"].clone().requires_grad_()
    k = P["k"].clone().requires_grad_()
    v = P["v"].clone().requires_grad_()
    Pb = dict(P)
    Pb["bias"] = P["bias"].clone().requires_grad_()
    qp = _pad(q, P["q_off"], Lq).transpose(1, 2)
    kp = _pad(k, P["kv_off"], Lk).transpose(1, 2)
    vp = _pad(v, P["kv_off"], Lk).transpose(1, 2)
    valid = _window_mask(P, Lq, Lk, causal, w)
    row_ok = valid.any(-1, keepdim=True)
    bias = _padded_bias(Pb, Lq, Lk)
    s = qp @ kp.transpose(-1, -2) / math.sqrt(P["d"]) + bias
    if act == "softmax":
        mask = torch.where(valid, torch.zeros_like(s), torch.full_like(s, float("-inf")))
        mask = torch.where(row_ok, mask, torch.zeros_like(mask))
        ref = F.scaled_dot_product_attention(qp, kp, vp, attn_mask=bias + mask)
        ref = torch.where(row_ok, ref, torch.zeros_like(ref))
        ref_lse = _unpad(torch.logsumexp(s.masked_fill(~valid, float("-inf")), -1)[..., None],
                         P["q_off"])[..., 0]
        keep = np.isfinite(ref_lse.detach().numpy())
        np.testing.assert_allclose(lse[keep], ref_lse.detach().numpy()[keep], atol=1e-12, rtol=0)
        assert np.all(np.isneginf(lse[~keep]))
    else:
        a = F.silu(s) if act == "silu" else F.gelu(s, approximate="tanh")
        nkv = torch.tensor(P["kv_lens"], dtype=torch.float64)[:, None, None, None]
        ref = (a * valid / nkv) @ vp          # GDPA divides by n_kv, window or not
        assert lse is None
    o = _unpad(ref, P["q_off"])
    np.testing.assert_allclose(out, o.detach().numpy(), atol=1e-12, rtol=0)
    (o * P["do"]).sum().backward()
    np.testing.assert_allclose(dq, q.grad.numpy(), atol=1e-12, rtol=0)
    np.testing.assert_allclose(dk, k.grad.numpy(), atol=1e-12, rtol=0)
    np.testing.assert_allclose(dv, v.grad.numpy(), atol=1e-12, rtol=0)
    # masked pairs get 0 in the dense gradient, as in autograd
    np.testing.assert_allclose(db, Pb["bias"].grad.numpy(), atol=1e-12, rtol=0)


def test_window_special_cases():
    lens = [6, 1, 11]
    P = _jagged(22, lens, lens, bias_kind="relpos")
    kw = dict(bias=P["bias"], bias_kind="relpos", relpos_len=P["relpos_len"], causal=True)
    # w = 1 under the causal rule: each query sees only its own position, so
    # the softmax output is that row of V and LSE its score
    out, lse = oracle.forward(P["q_off"], P["kv_off"], P["q"], P["k"], P["v"], window=1, **kw)
    np.testing.assert_allclose(out, P["v"].numpy(), atol=1e-15, rtol=0)
    C = (P["relpos_len"] - 1) // 2
    s_ii = (P["q"] * P["k"]).sum(-1).numpy() / math.sqrt(P["d"]) + P["bias"][:, C].numpy()[None, :]
    np.testing.assert_allclose(lse, s_ii, atol=1e-12, rtol=0)
    # a window that covers every sequence is no window at all (bit for bit);
    # one less changes the longest sequence's last row only
    full, lse_f = oracle.forward(P["q_off"], P["kv_off"], P["q"], P["k"], P["v"], **kw)
    cov, lse_c = oracle.forward(P["q_off"], P["kv_off"], P["q"], P["k"], P["v"], window=11, **kw)
    assert np.array_equal(full, cov) and np.array_equal(lse_f, lse_c)
    short, _ = oracle.forward(P["q_off"], P["kv_off"], P["q"], P["k"], P["v"], window=10, **kw)
    diff = np.abs(short - full).max(axis=(1, 2)) > 0
    assert list(np.nonzero(diff)[0]) == [int(P["q_off"][3]) - 1]
    # the schedule costs count exactly the window's pairs
    for causal in (False, True):
        for w in (1, 3, 7):
            mask = _window_mask(P, 11, 11, causal, w)
            assert oracle.valid_pairs(P["q_off"], P["kv_off"], causal, w) == int(mask.sum())
