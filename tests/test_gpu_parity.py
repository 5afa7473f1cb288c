"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the
same seeded inputs.

Tolerances (written here, applied element by element on every valid row):
  bf16 and MXFP8-backward : max |err| <= 2e-2 and mean |err| <= 2e-3 on O, dQ, dK, dV
  LSE (fp32 accumulation) : max |err| <= 1e-3
  fp32 CUDA-core path     : max |err| <= 1e-4 (stricter internal target) and the bf16 gate
  schedules / offsets     : bit-exact
A result stored as bf16 carries, on top of the computation's error, the final
rounding to bf16 (half an ulp of the value: 2^-9 relative, e.g. 0.031 for a
gradient entry of 10).  For a bf16 tensor the max bound is therefore
2e-2 + half_ulp_bf16(|reference|) per element, and the mean bound 2e-3 is
taken against the reference rounded to bf16 (the best any bf16 output can do).
"""
import numpy as np
import pytest
import torch

import oracle
from jagged_attention_recommender_jfa_b200 import jfa
from jagged_attention_recommender_jfa_b200.inputs import make_problem

pytestmark = pytest.mark.gpu

BF16_MAX, BF16_MEAN, LSE_MAX, F32_MAX = 2e-2, 2e-3, 1e-3, 1e-4


def _dev(p, dev):
    t = lambda x: None if x is None else x.to(dev).contiguous()
    return dict(q=t(p.q), k=t(p.k), v=t(p.v), dout=t(p.dout), bias=t(p.bias),
                q_off=t(p.q_off), kv_off=t(p.kv_off))


def run_gpu(p, dev, act=None, backward=True):
    act = act or p.act
    d = _dev(p, dev)
    prob = jfa.problem_of(p)
    out, lse = jfa.attention_forward(prob, d["q"], d["k"], d["v"], d["q_off"], d["kv_off"],
                                     d["bias"], act, p.causal)
    grads = None
    if backward:
        grads = jfa.attention_backward(prob, d["q"], d["k"], d["v"], out, lse, d["dout"],
                                       d["q_off"], d["kv_off"], d["bias"], act, p.causal)
    torch.cuda.synchronize()
    return out, lse, grads


def run_oracle(p, act=None, seq_mask=None, backward=True):
    act = act or p.act
    kw = dict(bias=p.bias, bias_kind=p.bias_kind, relpos_len=p.relpos_len, act=act,
              causal=p.causal, seq_mask=seq_mask)
    out, lse = oracle.forward(p.q_off, p.kv_off, p.q, p.k, p.v, **kw)
    grads = oracle.backward(p.q_off, p.kv_off, p.q, p.k, p.v, p.dout, **kw) if backward else None
    return out, lse, grads


def _rows(off, seq_mask):
    if seq_mask is None:
        return slice(None)
    idx = [np.arange(int(off[b]), int(off[b + 1])) for b in range(len(off) - 1) if seq_mask[b]]
    return np.concatenate(idx) if idx else np.zeros(0, np.int64)


def half_ulp_bf16(x):
    """Half a unit in the last place of bf16 (8 significant bits) at |x|."""
    ax = np.maximum(np.abs(x), 2.0 ** -126)
    return np.exp2(np.floor(np.log2(ax)) - 8)


def compare(name, gpu, ref, rows, max_tol, mean_tol=None, rms_scaled=False):
    bf16_out = gpu.dtype == torch.bfloat16
    g = gpu.float().cpu().numpy()[rows].astype(np.float64)
    r = ref[rows]
    if g.size == 0:
        return 0.0
    if rms_scaled:
        scale = max(1.0, float(np.sqrt(np.mean(r[np.isfinite(r)] ** 2))))
        max_tol *= scale
        mean_tol = None if mean_tol is None else mean_tol * scale
    finite = np.isfinite(r)
    assert np.array_equal(np.isfinite(g), finite), f"{name}: non-finite pattern differs"
    err = np.abs(g[finite] - r[finite])
    bound = max_tol + (half_ulp_bf16(r[finite]) if bf16_out else 0.0)
    mx = float(err.max()) if err.size else 0.0
    if bf16_out:
        r_bf16 = torch.from_numpy(r[finite]).to(torch.bfloat16).double().numpy()
        mn = float(np.abs(g[finite] - r_bf16).mean()) if err.size else 0.0
    else:
        mn = float(err.mean()) if err.size else 0.0
    worst = float((err - bound).max()) if err.size else -1.0
    assert worst <= 0.0, f"{name}: max abs err {mx:.3e} exceeds {max_tol} (+ bf16 half-ulp)"
    if mean_tol is not None:
        assert mn <= mean_tol, f"{name}: mean abs err {mn:.3e} > {mean_tol}"
    # -inf LSE rows must match exactly
    if not finite.all():
        assert np.array_equal(g[~finite], r[~finite]), f"{name}: -inf rows differ"
    return mx


def check_problem(p, dev, act=None, seq_mask=None, strict_f32=False, rms_scaled=False):
    act = act or p.act
    out, lse, (dq, dk, dv) = run_gpu(p, dev, act)
    ro, rl, (rdq, rdk, rdv) = run_oracle(p, act, seq_mask)
    qr, kr = _rows(p.q_off, seq_mask), _rows(p.kv_off, seq_mask)
    mx = BF16_MAX if not strict_f32 else F32_MAX
    mean = BF16_MEAN
    errs = {}
    errs["o"] = compare("O", out, ro, qr, mx, mean)
    if act == "softmax":
        errs["lse"] = compare("LSE", lse, rl, qr, LSE_MAX if not strict_f32 else F32_MAX)
    errs["dq"] = compare("dQ", dq, rdq, qr, mx, mean, rms_scaled)
    errs["dk"] = compare("dK", dk, rdk, kr, mx, mean, rms_scaled)
    errs["dv"] = compare("dV", dv, rdv, kr, mx, mean, rms_scaled)
    return errs


# ---------------------------------------------------------------------------
# schedule: bit-exact against the oracle's restatement
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("tile", [16, 64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("backward", [False, True])
def test_schedule_bit_exact(cuda_device, tile, causal, backward):
    q_lens = [0, 1, tile - 1, tile, tile + 1, 3 * tile + 5, 7, 200, 1]
    kv_lens = [5, 1, tile, tile, tile + 3, 3 * tile + 5, 0, 150, 300]
    p = make_problem("cross_bf16", 0, q_lens=q_lens, kv_lens=kv_lens, H=3)
    prob = jfa.problem_of(p)
    d = _dev(p, cuda_device)
    cap = 4096
    items = torch.full((cap, 4), -7, dtype=torch.int32, device=cuda_device)
    count = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    ws = jfa.workspace(prob, True, cuda_device)
    jfa.jfa_schedule(prob, d["q_off"], d["kv_off"], causal, backward, tile, items, cap, count, ws)
    jfa.jfa_check_error(ws)
    n = int(count.item())
    ref = oracle.schedule(p.q_off, p.kv_off, 3, tile, causal, backward)
    assert n == len(ref)
    assert np.array_equal(items[:n].cpu().numpy(), ref)
    assert np.all(items[n:].cpu().numpy() == -7)


# ---------------------------------------------------------------------------
# small full-parity cases
# ---------------------------------------------------------------------------
def test_tiny_f32_full(cuda_device):
    for seed in range(4):
        p = make_problem("tiny_f32", seed)
        check_problem(p, cuda_device, strict_f32=True)


@pytest.mark.parametrize("seed", [0, 1])
def test_self_bf16_small(cuda_device, seed):
    p = make_problem("self_bf16", seed, B=6, max_len=300)
    check_problem(p, cuda_device)


@pytest.mark.parametrize("seed", [0, 1])
def test_cross_bf16_small(cuda_device, seed):
    p = make_problem("cross_bf16", seed, B=12, max_len=700)
    check_problem(p, cuda_device)


@pytest.mark.parametrize("act", ["silu", "gelu_tanh"])
def test_gdpa_bf16_small(cuda_device, act):
    p = make_problem("gdpa_bf16", 3, B=12, max_len=700)
    check_problem(p, cuda_device, act=act)


@pytest.mark.parametrize("d", [32, 64])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_other_head_dims(cuda_device, d, dtype):
    p = make_problem("self_bf16", 5, B=5, max_len=150, d=d, H=3, dtype=dtype)
    check_problem(p, cuda_device)


EDGE_LENS = [
    # (q_lens, kv_lens, causal)
    ([1, 64, 65, 127, 128, 129, 0, 2], None, True),
    ([1, 64, 65, 127, 128, 129, 0, 2], None, False),
    ([5, 40, 200, 1], [1, 1, 1, 1], False),           # single key
    ([90, 10, 130], [30, 10, 20], True),              # n_q > n_kv: rows with no key
    ([3, 0, 0, 7], [0, 0, 9, 7], False),              # empty sequences on either side
]


@pytest.mark.parametrize("q_lens,kv_lens,causal", EDGE_LENS)
@pytest.mark.parametrize("act", ["softmax", "silu"])
def test_edge_lengths(cuda_device, q_lens, kv_lens, causal, act):
    kv_lens = kv_lens or q_lens
    p = make_problem("cross_bf16", 7, q_lens=q_lens, kv_lens=kv_lens, causal=causal,
                     bias="dense" if act == "silu" else "relpos")
    # GDPA over a single key does not divide the score gradient down
    # (dS = dP act'(s) / 1, |dS| ~ 11), so dK is a sum of large terms whose
    # bf16 MMA operands carry ~2^-9 relative error; the absolute bound, meant
    # for O(1) values, is applied relative to the tensor's RMS there.
    rms_scaled = act == "silu" and kv_lens == [1, 1, 1, 1]
    check_problem(p, cuda_device, act=act, rms_scaled=rms_scaled)


def test_no_bias(cuda_device):
    p = make_problem("self_bf16", 8, B=5, max_len=260, bias="none")
    check_problem(p, cuda_device)


# ---------------------------------------------------------------------------
# properties: neighbours do not leak, guards untouched, V = 1 gives O = 1
# ---------------------------------------------------------------------------
def test_poisoned_neighbours_and_guard_rows(cuda_device):
    p = make_problem("self_bf16", 9, B=5, max_len=300)
    out_ref, lse_ref, grads_ref = run_gpu(p, cuda_device)
    # poison sequence 2 with NaN / huge values
    s = slice(int(p.q_off[2]), int(p.q_off[3]))
    p.q[s] = float("nan")
    p.k[s] = 1e4
    p.v[s] = float("nan")
    p.dout[s] = float("nan")
    out, lse, grads = run_gpu(p, cuda_device)
    keep = np.ones(p.total_q, bool)
    keep[s] = False
    assert torch.equal(out[keep], out_ref[keep])
    assert torch.equal(lse[keep], lse_ref[keep])
    for g, gr in zip(grads, grads_ref):
        assert torch.equal(g[keep], gr[keep])
    # guard rows around every output stay untouched
    d = _dev(make_problem("self_bf16", 9, B=5, max_len=300), cuda_device)
    prob = jfa.problem_of(p)
    G = 16
    sentinel = 123.25

    def guarded(like):
        buf = torch.full((like.shape[0] + 2 * G, *like.shape[1:]), sentinel, dtype=like.dtype,
                         device=cuda_device)
        return buf, buf[G:G + like.shape[0]]

    ob, o = guarded(d["q"])
    lb = torch.full((p.total_q + 2 * G, p.H), sentinel, device=cuda_device)
    ls = lb[G:G + p.total_q]
    ws = jfa.workspace(prob, True, cuda_device)
    jfa.jfa_forward(prob, d["q"], d["k"], d["v"], d["q_off"], d["kv_off"], d["bias"], "softmax",
                    True, o, ls, ws)
    dqb, dq = guarded(d["q"])
    dkb, dk = guarded(d["k"])
    dvb, dv = guarded(d["v"])
    jfa.jfa_backward(prob, d["q"], d["k"], d["v"], o, ls, d["dout"], d["q_off"], d["kv_off"],
                     d["bias"], "softmax", True, dq, dk, dv, ws)
    jfa.jfa_check_error(ws)
    for buf in (ob, lb, dqb, dkb, dvb):
        assert torch.all(buf[:G] == sentinel) and torch.all(buf[-G:] == sentinel)


def test_unit_values_normalise(cuda_device):
    p = make_problem("self_bf16", 10, B=4, max_len=400)
    p.v[:] = 1.0
    out, _, _ = run_gpu(p, cuda_device, backward=False)
    assert torch.all((out.float() - 1.0).abs() <= 2 ** -8)


def test_bad_offsets_reported_and_nothing_written(cuda_device):
    p = make_problem("self_bf16", 11, B=4, max_len=100)
    d = _dev(p, cuda_device)
    prob = jfa.problem_of(p)
    bad = d["q_off"].clone()
    bad[2] = bad[1] - 1  # decreasing
    out = torch.full_like(d["q"], 7.0)
    lse = torch.full((p.total_q, p.H), 7.0, device=cuda_device)
    ws = jfa.workspace(prob, False, cuda_device)
    jfa.jfa_forward(prob, d["q"], d["k"], d["v"], bad, bad, d["bias"], "softmax", True, out,
                    lse, ws)
    with pytest.raises(jfa.JfaError) as ei:
        jfa.jfa_check_error(ws)
    assert ei.value.status == jfa.JFA_ERR_BAD_OFFSETS
    assert torch.all(out == 7.0) and torch.all(lse == 7.0)
    # lengths above max_q_len are rejected too
    prob2 = jfa.problem_of(p)
    prob2.max_q_len = 3
    prob2.max_kv_len = 3
    jfa.jfa_forward(prob2, d["q"], d["k"], d["v"], d["q_off"], d["kv_off"], d["bias"],
                    "softmax", True, out, lse, ws)
    with pytest.raises(jfa.JfaError):
        jfa.jfa_check_error(ws)
    # and the error word is cleared by the read: a good call reports OK
    jfa.jfa_forward(prob, d["q"], d["k"], d["v"], d["q_off"], d["kv_off"], d["bias"], "softmax",
                    True, out, lse, ws)
    jfa.jfa_check_error(ws)


# ---------------------------------------------------------------------------
# MXFP8 quantiser: bit-exact against the oracle
# ---------------------------------------------------------------------------
def test_quantize_mxfp8_bit_exact(cuda_device):
    p = make_problem("self_mxfp8", 12, B=6, max_len=200)
    x = p.k
    rows, H, d = x.shape
    xd = x.to(cuda_device)
    codes = torch.empty(rows, H, d, dtype=torch.uint8, device=cuda_device)
    scales = torch.empty(rows, H, d // 32, dtype=torch.uint8, device=cuda_device)
    jfa.jfa_quantize_mxfp8(xd, rows, H, d, None, 0, 0, False, codes, scales)
    rc, rs = oracle.quantize_mx_along_d(x)
    assert np.array_equal(codes.cpu().numpy(), rc)
    assert np.array_equal(scales.cpu().numpy(), rs)
    # along rows (per sequence), with special blocks: zeros, saturation, powers of two
    v = p.v.clone()
    v[int(p.kv_off[1]):int(p.kv_off[1]) + 32] = 0.0
    v[int(p.kv_off[2])] = 500.0
    nblk = rows // 32 + p.B
    codes = torch.empty(rows, H, d, dtype=torch.uint8, device=cuda_device)
    scales = torch.zeros(nblk, H, d, dtype=torch.uint8, device=cuda_device)
    jfa.jfa_quantize_mxfp8(v.to(cuda_device), rows, H, d, p.kv_off.to(cuda_device), p.B,
                           p.max_kv_len, True, codes, scales)
    rc, rs = oracle.quantize_mx_along_rows(v, p.kv_off)
    assert np.array_equal(codes.cpu().numpy(), rc)
    assert np.array_equal(scales[:rs.shape[0]].cpu().numpy(), rs)
