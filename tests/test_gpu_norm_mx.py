"""The fused normalisation + MX quantisation kernel (jfa_norm_quantize_mxfp8)
against the oracle's fp64 normalisation quantised by the oracle's MX
quantiser, and that producer feeding the MXFP8 attention forward
(jfa_forward_mxfp8) end to end.

The kernel normalises in fp32 and the oracle in fp64; a quantised code is an
integer decision on that value, so it is compared where the decision is
unique: the scale byte wherever the block maximum is not within fp32 rounding
of a power of two, and each code to within one E4M3 step (identical for all
but a handful of elements that sit on a rounding midpoint), with the decoded
value within the format's error of the fp64 result.
"""
import numpy as np
import pytest
import torch

import oracle
from jagged_attention_recommender_jfa_b200 import jfa
from jagged_attention_recommender_jfa_b200.inputs import make_problem

pytestmark = pytest.mark.gpu


def _e4m3_rank(codes):
    """Order of E4M3 codes by value (sign-magnitude -> signed integer)."""
    c = codes.astype(np.int32)
    mag = c & 0x7F
    return np.where(c & 0x80, -mag, mag)


def run_norm(x, gamma, beta, eps, layernorm, dev):
    rows, D = x.shape
    xd = x.to(dev).contiguous()
    codes = torch.empty(rows, D, dtype=torch.uint8, device=dev)
    scales = torch.empty(rows, D // 32, dtype=torch.uint8, device=dev)
    g = None if gamma is None else gamma.to(dev)
    b = None if beta is None else beta.to(dev)
    jfa.jfa_norm_quantize_mxfp8(xd, rows, D, g, b, eps, layernorm, codes, scales)
    torch.cuda.synchronize()
    return codes.cpu().numpy(), scales.cpu().numpy()


@pytest.mark.parametrize("D,layernorm", [(128, False), (128, True), (64, False), (1024, True),
                                         (1536, False), (4096, True)])
def test_norm_quantize_matches_oracle(cuda_device, D, layernorm):
    g = torch.Generator().manual_seed(D + layernorm)
    rows = 3001
    x = (torch.randn(rows, D, generator=g) * 2 + 0.3).to(torch.bfloat16)
    gamma = torch.randn(D, generator=g).abs() + 0.5
    beta = torch.randn(D, generator=g) * 0.1 if layernorm else None
    codes, scales = run_norm(x, gamma, beta, 1e-5, layernorm, cuda_device)
    y = oracle.norm(x, gamma, beta, 1e-5, layernorm)
    rc, rs = oracle.quantize_mx(y)
    rs = rs.reshape(rows, D // 32)
    # scale bytes: equal unless the block maximum sits within fp32 rounding of a power of two
    amax = np.abs(y).reshape(rows, D // 32, 32).max(-1)
    frac = np.log2(amax) - np.floor(np.log2(amax))
    safe = (frac > 1e-5) & (frac < 1 - 1e-5)
    assert np.array_equal(scales[safe], rs[safe])
    same = np.repeat(scales == rs, 32, axis=1)
    # codes: at most one E4M3 step apart, and nearly all identical
    step = np.abs(_e4m3_rank(codes) - _e4m3_rank(rc))
    assert step[same].max() <= 1
    assert (step[same] == 0).mean() >= 0.999
    # decoded values within the element format's error of the fp64 result;
    # a block maximum scaled into [448, 512) saturates to 448 2^X (the OCP
    # rule), so those elements are checked against that value instead
    deq = oracle.dequantize_mx(codes.reshape(-1), scales.reshape(-1)).reshape(rows, D)
    X = np.repeat(scales.astype(np.int64) - 127, 32, axis=1).astype(np.float64)
    sat = np.abs(y) * 2.0 ** -X > 448 * (1 - 1e-5)
    assert np.all(np.abs(np.abs(deq[sat]) - 448 * 2.0 ** X[sat]) == 0.0)
    bound = np.abs(y) * 2.0 ** -4 + 2.0 ** (X - 9.0) + 1e-5 * np.abs(y)
    assert np.all(np.abs(deq - y)[~sat] <= bound[~sat])


def test_norm_quantize_rejects_bad_sizes(cuda_device):
    x = torch.zeros(4, 48, dtype=torch.bfloat16, device=cuda_device)
    c = torch.empty(4, 48, dtype=torch.uint8, device=cuda_device)
    s = torch.empty(4, 2, dtype=torch.uint8, device=cuda_device)
    with pytest.raises(jfa.JfaError):
        jfa.jfa_norm_quantize_mxfp8(x, 4, 48, None, None, 1e-5, False, c, s)
    with pytest.raises(jfa.JfaError):
        jfa.jfa_norm_quantize_mxfp8(x, 4, 32, None, None, 0.0, False, c, s)


def test_norm_quantize_feeds_mxfp8_attention(cuda_device):
    # per-head RMSNorm of Q and K written straight to MX by the producer,
    # V quantised along keys, then the block-scaled forward on them; checked
    # against the oracle's MXFP8 attention on the decoded operands
    p = make_problem("self_mxfp8", 34, B=5, max_len=300)
    dev = cuda_device
    rows_q, H, d = p.q.shape
    rows_k = p.k.shape[0]
    g = torch.Generator().manual_seed(7)
    gq = (torch.randn(d, generator=g).abs() + 0.5)
    gk = (torch.randn(d, generator=g).abs() + 0.5)
    q8, qs = run_norm(p.q.reshape(rows_q * H, d), gq, None, 1e-6, False, dev)
    k8, ks = run_norm(p.k.reshape(rows_k * H, d), gk, None, 1e-6, False, dev)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    v8 = torch.empty(rows_k, H, d, dtype=torch.uint8, device=dev)
    vs = torch.zeros(rows_k // 32 + p.B, H, d, dtype=torch.uint8, device=dev)
    kv_off = p.kv_off.to(dev)
    jfa.jfa_quantize_mxfp8(p.v.to(dev), rows_k, H, d, kv_off, p.B, p.max_kv_len, True, v8, vs)
    prob = jfa.problem_of(p)
    ws = jfa.workspace(prob, False, dev)
    out = torch.empty(rows_q, H, d, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(rows_q, H, device=dev)
    jfa.jfa_forward_mxfp8(prob, t(q8.reshape(rows_q, H, d)), t(qs.reshape(rows_q, H, d // 32)),
                          t(k8.reshape(rows_k, H, d)), t(ks.reshape(rows_k, H, d // 32)), v8, vs,
                          p.q_off.to(dev), kv_off, p.bias.to(dev), True, out, lse, ws)
    jfa.jfa_check_error(ws)
    qd = oracle.dequantize_mx(q8.reshape(-1), qs.reshape(-1)).reshape(rows_q, H, d)
    kd = oracle.dequantize_mx(k8.reshape(-1), ks.reshape(-1)).reshape(rows_k, H, d)
    nb = int(sum((int(n) + 31) // 32 for n in p.kv_lens))
    vd = oracle.dequantize_along_rows(v8.cpu().numpy(), vs[:nb].cpu().numpy(), p.kv_off)
    ro, rl = oracle.forward(p.q_off, p.kv_off, qd, kd, vd, bias=p.bias, bias_kind="relpos",
                            relpos_len=p.relpos_len, causal=True, quant_p=True)
    g_out = out.float().cpu().numpy()
    half_ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(ro), 2.0 ** -126))) - 8)
    assert np.all(np.abs(g_out - ro) <= 6e-2 + half_ulp)
    assert np.all(np.abs(lse.cpu().numpy() - rl) <= 1e-3)
