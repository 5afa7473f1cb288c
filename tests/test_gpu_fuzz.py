"""Randomised batches on the GPU against the oracle.

Each seed draws a workload (causal self-attention, short queries over long
keys, GDPA), an activation, the causal rule, a bias kind, a head count, a
sliding window or none, and sequence lengths mixed from tile edges (0, 1,
63..65, 127..129, 255..257) and uniform draws, so that the tile schedules,
the persistent backward's work queue, the forward's slot alternation and the
short-query kernels meet shapes no hand-picked case lists.  Two more draws
take the CUDA-core path (fp32 or bf16 storage, head_dim 32 / 64 / 128) and
the MXFP8 path (softmax, its own 6e-2 bound on the oracle's dequantised
operands), and one more the bias gradient (relative-position table or dense
jagged bias, against the oracle's, as the bias-gradient parity tests check
it); eight draws take a few sequences of 1,000 to 3,000 tokens.  Tolerances are
those of the parity tests; GDPA sequences keep at least 8 keys (a single
key leaves nothing to divide the score gradient, which the edge tests cover
with their own bound).

Pages: "Meta GEM Training Efficiency: Why LLM-Scale Recommenders Need a
Different Stack", "Bottleneck move 1: dense-sequence kernels to jagged
execution" (jagged tiles of uneven length, custom biases, GDPA).
"""
import numpy as np
import pytest

from jagged_attention_recommender_jfa_b200.inputs import make_problem
from test_gpu_parity import mx_dequantised_inputs
from test_gpu_window import check_window

pytestmark = pytest.mark.gpu

EDGES = [0, 1, 63, 64, 65, 127, 128, 129, 255, 256, 257]


def draw_case(seed):
    rng = np.random.default_rng(1000 + seed)
    workload = ["self_bf16", "cross_bf16", "gdpa_bf16"][rng.integers(0, 3)]
    if workload == "gdpa_bf16":
        act = ["silu", "gelu_tanh"][rng.integers(0, 2)]
    else:
        act = ["softmax", "softmax", "silu", "gelu_tanh"][rng.integers(0, 4)]
    causal = bool(rng.integers(0, 2))
    bias = ["none", "relpos", "dense"][rng.integers(0, 3)]
    H = int(rng.integers(1, 4))
    B = int(rng.integers(1, 7))

    def lengths(hi):
        return [int(EDGES[rng.integers(0, len(EDGES))]) if rng.random() < 0.5
                else int(rng.integers(1, hi)) for _ in range(B)]

    if workload == "self_bf16":
        q_lens = lengths(700)
        kv_lens = list(q_lens)
    else:
        short = rng.random() < 0.5
        q_lens = [min(x, 64) for x in lengths(65)] if short else lengths(400)
        kv_lens = lengths(900)
    if act != "softmax":
        kv_lens = [max(x, 8) for x in kv_lens]
    if sum(q_lens) == 0:
        q_lens[0] = 5
    if sum(kv_lens) == 0:
        kv_lens[0] = 9
    window = int([0, 0, 1, 17, 128, 300][rng.integers(0, 6)])
    return dict(workload=workload, act=act, causal=causal, bias=bias, H=H, q_lens=q_lens,
                kv_lens=kv_lens, window=window)


def test_draws_cover_the_kinds():
    cases = [draw_case(s) for s in range(16)]
    assert {c["workload"] for c in cases} == {"self_bf16", "cross_bf16", "gdpa_bf16"}
    assert {c["bias"] for c in cases} == {"none", "relpos", "dense"}
    assert any(c["window"] > 0 for c in cases) and any(c["window"] == 0 for c in cases)
    assert any(max(c["q_lens"]) <= 64 for c in cases) and any(max(c["q_lens"]) > 128 for c in cases)


@pytest.mark.parametrize("seed", range(64))
def test_random_batch(cuda_device, seed):
    c = draw_case(seed)
    p = make_problem(c["workload"], seed, q_lens=c["q_lens"], kv_lens=c["kv_lens"], act=c["act"],
                     causal=c["causal"], bias=c["bias"], H=c["H"])
    check_window(p, cuda_device, c["window"], act=c["act"])


@pytest.mark.parametrize("seed", range(16))
def test_random_batch_cuda_core(cuda_device, seed):
    c = draw_case(seed)
    rng = np.random.default_rng(2000 + seed)
    d = int([32, 64, 128][rng.integers(0, 3)])
    dtype = "f32" if (d == 128 or rng.random() < 0.5) else "bf16"
    p = make_problem(c["workload"], seed, q_lens=c["q_lens"], kv_lens=c["kv_lens"], act=c["act"],
                     causal=c["causal"], bias=c["bias"], H=c["H"], d=d, dtype=dtype)
    check_window(p, cuda_device, c["window"], act=c["act"], strict_f32=(dtype == "f32"))


@pytest.mark.parametrize("seed", range(16))
def test_random_batch_mxfp8(cuda_device, seed):
    c = draw_case(seed)
    p = make_problem("self_mxfp8", seed, q_lens=c["q_lens"], kv_lens=c["kv_lens"], act="softmax",
                     causal=c["causal"], bias=c["bias"], H=c["H"])
    check_window(p, cuda_device, c["window"], inputs=mx_dequantised_inputs(p), quant_p=True,
                 mx=True)


@pytest.mark.parametrize("seed", range(16))
def test_random_batch_bias_gradient(cuda_device, seed):
    from test_gpu_dbias import (BF16_MAX, BF16_MEAN, check_dense, check_relpos, dense_mask,
                                oracle_dbias, pairs_per_entry, run_gpu)
    c = draw_case(seed)
    bias = c["bias"] if c["bias"] != "none" else ["relpos", "dense"][seed % 2]
    p = make_problem(c["workload"], seed, q_lens=c["q_lens"], kv_lens=c["kv_lens"], act=c["act"],
                     causal=c["causal"], bias=bias, H=c["H"])
    db = run_gpu(p, cuda_device, c["act"])
    ref = oracle_dbias(p, c["act"])
    if bias == "relpos":
        check_relpos("dtable", db, ref, pairs_per_entry(p), BF16_MAX, BF16_MEAN)
    else:
        check_dense("dbias", db, ref, BF16_MAX, BF16_MEAN, valid=dense_mask(p))


@pytest.mark.parametrize("seed", range(8))
def test_random_long_sequences(cuda_device, seed):
    # a few sequences of 1,000 to 3,000 tokens: 8 to 24 key tiles per query
    # row, the lazy rescale firing again and again, long persistent items
    rng = np.random.default_rng(3000 + seed)
    B = int(rng.integers(1, 4))
    lens = [int(x) for x in rng.integers(1000, 3001, size=B)]
    causal = bool(rng.integers(0, 2))
    bias = ["none", "relpos"][rng.integers(0, 2)]
    window = int([0, 0, 700][rng.integers(0, 3)])
    act = ["softmax", "softmax", "silu"][rng.integers(0, 3)]
    p = make_problem("self_bf16", seed, q_lens=lens, kv_lens=lens, act=act, causal=causal,
                     bias=bias, H=2)
    check_window(p, cuda_device, window, act=act)
