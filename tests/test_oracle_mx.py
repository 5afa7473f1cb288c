"""Pins of the oracle's MX (MXFP8) quantiser.

* fixed points of the E4M3 / E8M0 formats from the OCP MX v1.0 specification
  (``tests/golden/e4m3_e8m0_points.txt``);
* element rounding == torch's float8_e4m3fn conversion (round to nearest even)
  on every E4M3 value, every midpoint between neighbours and random values;
* the shared exponent == floor(log2(amax)) - 8 via math.log2;
* the dequantisation error bound of a 3-bit mantissa;
* the MXFP8 attention oracle: uniform scores quantise exactly, and quantising
  P moves the output by no more than the element format's error bound.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "e4m3_e8m0_points.txt")


def _golden():
    rows = []
    with open(GOLDEN) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            kind, val, code = line.split()
            rows.append((kind, float(val), int(code, 16)))
    return rows


def test_format_fixed_points():
    for kind, val, code in _golden():
        if kind == "e4m3":
            assert oracle.e4m3_encode(val) == code, (val, code)
            dec = oracle.e4m3_decode(code)
            assert dec == val and math.copysign(1, dec) == math.copysign(1, val)
        else:
            # a block whose amax is val * 2^8 gets shared exponent log2(val)
            x = np.zeros(32)
            x[3] = val * 256.0
            _, sc = oracle.quantize_mx(x)
            assert int(sc[0]) == code, (val, code)
    assert math.isnan(oracle.e4m3_decode(0x7F))


def _all_e4m3_values():
    vals = [oracle.e4m3_decode(c) for c in range(256) if (c & 0x7F) != 0x7F]
    return np.array(sorted(set(vals)), dtype=np.float64)


def _torch_e4m3_codes(x32):
    t = torch.from_numpy(np.clip(x32, -448, 448).astype(np.float32))
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_element_rounding_matches_torch_float8():
    vals = _all_e4m3_values()
    pos = vals[vals >= 0]
    mids = (pos[:-1] + pos[1:]) / 2  # exact ties -> even mantissa
    rng = np.random.default_rng(0)
    rand = np.concatenate([rng.uniform(-448, 448, 20000), rng.uniform(-0.02, 0.02, 20000),
                           rng.uniform(-1e-3, 1e-3, 5000)])
    x = np.concatenate([vals, mids, -mids, rand]).astype(np.float32)
    mine = np.array([oracle.e4m3_encode(float(v)) for v in x], np.uint8)
    ref = _torch_e4m3_codes(x)
    # torch keeps the sign of a value that rounds to zero; so does the oracle
    np.testing.assert_array_equal(mine, ref)
    # saturation: everything at or above 448 in magnitude becomes +-448
    for v in (448.0, 455.9, 464.0, 479.0, 511.9, 1e6):
        assert oracle.e4m3_encode(v) == 0x7E and oracle.e4m3_encode(-v) == 0xFE


def test_shared_exponent_and_error_bound():
    rng = np.random.default_rng(1)
    for trial in range(200):
        scale = 2.0 ** rng.integers(-20, 20)
        x = torch.from_numpy(rng.standard_normal(32) * scale).to(torch.bfloat16).double().numpy()
        codes, sc = oracle.quantize_mx(x)
        amax = np.abs(x).max()
        X = math.floor(math.log2(amax)) - 8
        assert int(sc[0]) == X + 127
        deq = oracle.dequantize_mx(codes, sc)
        # the floor rule puts amax * 2^-X in [256, 512): elements above 448 saturate
        sat = np.abs(x) * 2.0 ** -X > 448
        assert np.all(deq[sat] == np.sign(x[sat]) * 448 * 2.0 ** X)
        # normal E4M3 range: relative error <= 2^-4; subnormal: half a quantum 2^(X-10)
        err = np.abs(deq - x)
        bound = np.maximum(np.abs(x) * 2.0 ** -4, 2.0 ** (X - 10))
        assert np.all(err[~sat] <= bound[~sat])
    zero = np.zeros(32)
    codes, sc = oracle.quantize_mx(zero)
    assert sc[0] == 0 and np.all(codes == 0)
    # powers of two inside the block's range round-trip exactly
    x = np.array([2.0 ** -k for k in range(32)])
    codes, sc = oracle.quantize_mx(x)
    deq = oracle.dequantize_mx(codes, sc)
    X = int(sc[0]) - 127
    exact = x >= 2.0 ** (X - 9)
    assert np.array_equal(deq[exact], x[exact])
    # amax whose scaled value lands in [448, 512) saturates to 448 * 2^X
    x = np.zeros(32)
    x[0] = 500.0
    x[1] = -1.0
    codes, sc = oracle.quantize_mx(x)
    assert int(sc[0]) - 127 == 0 and codes[0] == 0x7E
    assert oracle.dequantize_mx(codes, sc)[0] == 448.0


def test_along_rows_layout():
    rng = np.random.default_rng(2)
    off = np.array([0, 5, 45, 45, 77], np.int32)
    x = torch.from_numpy(rng.standard_normal((77, 2, 64)).astype(np.float32)).to(torch.bfloat16)
    codes, scales = oracle.quantize_mx_along_rows(x, off)
    nblk = sum((off[b + 1] - off[b] + 31) // 32 for b in range(4))
    assert scales.shape == (nblk, 2, 64)
    # block 2 of the list = sequence 1, rows 5..36, column (h=1, c=7)
    col = x[5:37, 1, 7].double().numpy()
    c2, s2 = oracle.quantize_mx(col)
    assert np.array_equal(codes[5:37, 1, 7], c2) and scales[1, 1, 7] == s2[0]
    # last block of sequence 1 is rows 37..44 zero-padded to 32
    col = np.zeros(32)
    col[:8] = x[37:45, 0, 3].double().numpy()
    c3, s3 = oracle.quantize_mx(col)
    assert np.array_equal(codes[37:45, 0, 3], c3[:8]) and scales[2, 0, 3] == s3[0]


def test_mxfp8_attention_oracle():
    rng = np.random.default_rng(3)
    q_lens = [40, 7, 33]
    off = np.array([0] + list(np.cumsum(q_lens)), np.int32)
    H, d = 2, 32
    k = torch.from_numpy(rng.standard_normal((off[-1], H, d))).double()
    v = torch.from_numpy(rng.standard_normal((off[-1], H, d))).double()
    # uniform scores: exp(s - m) = 1 quantises exactly, so o is the mean of v
    q0 = torch.zeros_like(k)
    o_q, _ = oracle.forward(off, off, q0, k, v, causal=True, quant_p=True)
    o, _ = oracle.forward(off, off, q0, k, v, causal=True)
    np.testing.assert_allclose(o_q, o, atol=1e-14)
    # random scores: quantising P perturbs each weight by <= 2^-4 relative,
    # so |o_q - o| <= 2^-4 * sum_j p_ij |v_j| <= 2^-4 * max |v|
    q = torch.from_numpy(rng.standard_normal((off[-1], H, d))).double()
    o_q, _ = oracle.forward(off, off, q, k, v, causal=True, quant_p=True)
    o, _ = oracle.forward(off, off, q, k, v, causal=True)
    assert np.abs(o_q - o).max() <= 2.0 ** -4 * np.abs(v.numpy()).max()
    assert np.abs(o_q - o).max() > 0.0


# ---------------------------------------------------------------------------
# MXFP8 P quantisation, pinned on hand-built rows.
#
# With q = 0 the scores are the dense bias; a bias of (k_j + 1/2) ln 2 puts the
# log2-domain score of key j at x_j = k_j + 1/2 (k_j an integer).  The
# reference is R = ceil(max x) = k_max + 1, so the weights are
# w_j = 2^(e_j - 1/2), e_j = k_j - k_max.  In an MX block whose largest
# weight has exponent e_max the shared exponent is floor(log2 w_max) - 8 =
# e_max - 9, and the scaled element is sqrt(2) 2^p with p = 8 + e_j - e_max.
# E4M3 rounds sqrt(2) 2^p to 1.375 2^p in the normal range (p >= -6: 1.4142
# lies nearer 1.375 than 1.5) and to n 2^-9 below it, n = 6, 3, 1, 1, 0 for
# p = -7 .. -11.  The output is sum_j deq_j v_j / sum_j w_j (the unquantised
# sum).  Blocks hold 32 consecutive keys counted from the sequence's first
# key; the sequence below starts at packed row 5, so counting blocks from the
# packed row index instead would put key 31 (the row maximum) into the block
# of keys 32.. and flush those to zero.
# ---------------------------------------------------------------------------
_SUBNORMAL_N = {-7: 6, -8: 3, -9: 1, -10: 1}


def _e4m3_sqrt2_pow(p):
    """E4M3 value of sqrt(2) * 2^p (hand table above)."""
    if p >= -6:
        return 1.375 * 2.0 ** p
    return _SUBNORMAL_N.get(p, 0) * 2.0 ** -9


def test_e4m3_sqrt2_table_matches_torch_float8():
    for p in range(-14, 9):
        t = torch.tensor([math.sqrt(2.0) * 2.0 ** p], dtype=torch.float64)
        assert float(t.float().to(torch.float8_e4m3fn).double()) == _e4m3_sqrt2_pow(p), p
        assert oracle.e4m3_decode(oracle.e4m3_encode(math.sqrt(2.0) * 2.0 ** p)) == _e4m3_sqrt2_pow(p)


def _expected_row(e, vis, v, block_start):
    """Closed form of one output row: e[j] integer exponents (0 at the row
    maximum), vis[j] visibility, blocks of 32 keys starting at key
    -block_start (0 = the sequence's first key)."""
    n = len(e)
    w = np.array([2.0 ** (e[j] - 0.5) if vis[j] else 0.0 for j in range(n)])
    deq = np.zeros(n)
    for lo in range(-block_start, n, 32):
        js = [j for j in range(max(lo, 0), min(lo + 32, n)) if vis[j]]
        if not js:
            continue
        emax = max(e[j] for j in js)
        for j in js:
            deq[j] = _e4m3_sqrt2_pow(8 + e[j] - emax) * 2.0 ** (emax - 9)
    return (deq[:, None] * v).sum(0) / w.sum()


def _quant_p_case():
    rng = np.random.default_rng(11)
    n0, nq, nkv = 5, 3, 70            # sequence 0: 5 filler rows; sequence 1 under test
    H, d = 1, 8
    q_off = np.array([0, n0, n0 + nq], np.int32)
    kv_off = np.array([0, n0, n0 + nkv], np.int32)
    e = np.zeros((nq, nkv), np.int64)
    for i in range(nq):
        for j in range(nkv):
            if j < 31:
                e[i, j] = -((j + i) % 5)               # block 0: near the maximum
            elif j == 31:
                e[i, j] = 0                            # the row maximum, last key of block 0
            elif j < 64:
                e[i, j] = -20 - ((j + i) % 4)          # block 1: far below it
            else:
                e[i, j] = -3 - (j % 2)                 # block 2 (6 keys)
    e[2, 40] = -20 - 10                                # a subnormal inside block 1 (p = -2 - 10 + 2)
    x = e + 0.5                                        # k_max = 0 for every row
    dense = np.concatenate([rng.standard_normal(H * n0 * n0), (x * math.log(2.0)).reshape(-1)])
    k = rng.standard_normal((n0 + nkv, H, d))
    v = rng.standard_normal((n0 + nkv, H, d))
    q = np.zeros((n0 + nq, H, d))
    q[:n0] = rng.standard_normal((n0, H, d))
    return q_off, kv_off, q, k, v, dense, e


def test_mxfp8_p_quantisation_closed_form():
    q_off, kv_off, q, k, v, dense, e = _quant_p_case()
    nq, nkv = e.shape
    o, lse = oracle.forward(q_off, kv_off, q, k, v, bias=dense, bias_kind="dense",
                            quant_p=True)
    vs = v[5:5 + nkv, 0]
    for i in range(nq):
        want = _expected_row(e[i], np.ones(nkv, bool), vs, 0)
        np.testing.assert_allclose(o[5 + i, 0], want, rtol=0, atol=1e-12)
        # the pin separates the plausible mistakes by far more than its tolerance
        wrong_blocks = _expected_row(e[i], np.ones(nkv, bool), vs, 5)   # packed-row blocks
        assert np.abs(wrong_blocks - want).max() > 1e-9
        w = 2.0 ** (e[i] - 0.5)
        wrong_ref = (2.0 ** e[i])[:, None] * vs                      # R = max x, not ceil
        assert np.abs(wrong_ref.sum(0) / (2.0 ** e[i]).sum() - want).max() > 1e-3
        deq_sum = _expected_row(e[i], np.ones(nkv, bool), np.ones((nkv, 1)), 0)[0] * w.sum()
        assert abs(deq_sum / w.sum() - 1.0) > 1e-2                   # dividing by sum(deq)
        # LSE is that of the unquantised scores: ln sum_j e^{s_j}
        s = (e[i] + 0.5) * math.log(2.0)
        assert abs(lse[5 + i, 0] - np.log(np.exp(s).sum())) <= 1e-12


def test_mxfp8_p_quantisation_causal_blocks():
    # causal self-attention of one sequence of 40 starting at packed row 9:
    # row i sees keys 0..i; the block of keys 32..39 is quantised on its own
    rng = np.random.default_rng(12)
    n0, n = 9, 40
    off = np.array([0, n0, n0 + n], np.int32)
    H, d = 1, 4
    e = np.array([[-((i - j) % 3) if j != i else 0 for j in range(n)] for i in range(n)])
    e[:, 32:] -= 12
    for i in range(32, n):
        e[i, i] = 0
    x = (e + 0.5) * math.log(2.0)
    dense = np.concatenate([rng.standard_normal(n0 * n0), x.reshape(-1)])
    k = rng.standard_normal((n0 + n, H, d))
    v = rng.standard_normal((n0 + n, H, d))
    q = np.zeros((n0 + n, H, d))
    o, _ = oracle.forward(off, off, q, k, v, bias=dense, bias_kind="dense", causal=True,
                          quant_p=True)
    vs = v[n0:, 0]
    for i in range(n):
        vis = np.arange(n) <= i
        want = _expected_row(e[i], vis, vs, 0)
        np.testing.assert_allclose(o[n0 + i, 0], want, rtol=0, atol=1e-12)


def test_dequantize_along_rows_round_trip():
    # values exactly representable after MX quantisation along rows: per
    # (head, column) block of 32 rows, E4M3 mantissas in [1, 1.75] times
    # powers of two within 2^6 of the block maximum (a block maximum with
    # mantissa 1.875 would saturate to 1.75: 1.875 * 2^8 > 448)
    rng = np.random.default_rng(13)
    lens = [5, 70, 0, 33]
    off = np.array([0] + list(np.cumsum(lens)), np.int32)
    rows, H, d = int(off[-1]), 2, 32
    mant = 1.0 + rng.integers(0, 7, (rows, H, d)) / 8.0
    expo = rng.integers(-6, 1, (rows, H, d)).astype(np.float64)
    sign = rng.choice([-1.0, 1.0], (rows, H, d))
    x = sign * mant * 2.0 ** (expo + rng.integers(-3, 4, (1, H, d)))
    codes, scales = oracle.quantize_mx_along_rows(x, off)
    back = oracle.dequantize_along_rows(codes, scales, off)
    assert np.array_equal(back, x)
    # and row by row it is dequantize_mx of the same blocks: block c of
    # sequence b covers rows off[b] + 32 c .. + 31 (zero-padded at the end)
    blk0 = 0
    for b in range(len(lens)):
        nb = (lens[b] + 31) // 32
        for c in range(nb):
            lo, hi = int(off[b]) + 32 * c, min(int(off[b + 1]), int(off[b]) + 32 * c + 32)
            for h in range(H):
                for col in (0, 7, d - 1):
                    cb = np.zeros(32, np.uint8)
                    cb[:hi - lo] = codes[lo:hi, h, col]
                    ref = oracle.dequantize_mx(cb, np.array([scales[blk0 + c, h, col]], np.uint8))
                    assert np.array_equal(back[lo:hi, h, col], ref[:hi - lo])
        blk0 += nb
    assert blk0 == scales.shape[0]


# ---------------------------------------------------------------------------
# normalisation that feeds the MX quantiser: the oracle's plain definitions
# against torch's library routines in float64
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("layernorm", [False, True])
def test_norm_matches_torch(layernorm):
    rng = np.random.default_rng(20)
    x = rng.standard_normal((37, 256)) * 3 + 0.5
    g = rng.standard_normal(256)
    b = rng.standard_normal(256)
    y = oracle.norm(x, g, b, 1e-5, layernorm)
    xt = torch.from_numpy(x)
    if layernorm:
        ref = torch.nn.functional.layer_norm(xt, (256,), torch.from_numpy(g), torch.from_numpy(b), 1e-5)
    else:
        ref = torch.nn.functional.rms_norm(xt, (256,), torch.from_numpy(g), 1e-5)
    np.testing.assert_allclose(y, ref.numpy(), rtol=0, atol=1e-12)
    # without gamma / beta: unit RMS (RMSNorm) or zero mean, unit variance
    y0 = oracle.norm(x, None, None, 0.0 + 1e-300, layernorm)
    if layernorm:
        np.testing.assert_allclose(y0.mean(1), 0.0, atol=1e-12)
        np.testing.assert_allclose((y0 ** 2).mean(1), 1.0, atol=1e-12)
    else:
        np.testing.assert_allclose((y0 ** 2).mean(1), 1.0, atol=1e-12)
