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
