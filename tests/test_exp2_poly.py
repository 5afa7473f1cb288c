"""The exp2 that the tensor-core kernels evaluate on the FMA pipe for part of
the softmax weights: y = n + f with n = round(y) (taken from the low mantissa
bits of y + 1.5 * 2^23), 2^f by the cubic
    p(f) = 0.9999282 + f (0.69326097 + f (0.24260971 + f 0.05517098)),
fitted in this repository for minimax relative error on f in [-1/2, 1/2],
then 2^n added to the exponent field.  The same steps in float32 on the host
must stay within the stated bound of the exact 2^y over the range the kernels
use (scores minus the running maximum, at most 8 above it with the lazy
rescale), and far below bf16's relative step 2^-9, the precision P is kept in.
"""
import numpy as np

C = np.float32([0.9999282, 0.69326097, 0.24260971, 0.05517098])
MAGIC = np.float32(12582912.0)


def exp2_poly_f32(y):
    y = np.maximum(np.asarray(y, np.float32), np.float32(-126.0))
    t = (y + MAGIC).astype(np.float32)
    n = (t - MAGIC).astype(np.float32)
    f = (y - n).astype(np.float32)
    p = np.float32(C[3])
    for c in (C[2], C[1], C[0]):
        p = (p * f + c).astype(np.float32)
    bits = p.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.view(np.float32)


def test_relative_error_bound():
    y = np.linspace(-60.0, 8.0, 400001, dtype=np.float32)
    got = exp2_poly_f32(y).astype(np.float64)
    ref = np.exp2(y.astype(np.float64))
    rel = np.abs(got - ref) / ref
    assert rel.max() < 1.0e-4
    assert rel.max() < 2.0 ** -9 / 10


def test_integers_and_halves():
    # 2^f with f = 0 is p(0) = c0: the error at integers is |1 - c0|
    for n in (-20, -1, 0, 1, 7, 8):
        v = float(exp2_poly_f32(np.float32(n)))
        assert abs(v / 2.0 ** n - 1.0) < 1.0e-4
    # round-half cases land on either neighbour with the same accuracy
    for y in (-2.5, -0.5, 0.5, 3.5):
        v = float(exp2_poly_f32(np.float32(y)))
        assert abs(v / 2.0 ** y - 1.0) < 1.0e-4


def test_deep_negative_is_tiny_and_finite():
    v = exp2_poly_f32(np.float32([-126.0, -200.0, -1.0e30]))
    assert np.all(np.isfinite(v)) and np.all(v >= 0.0) and np.all(v < 1.2e-38)
