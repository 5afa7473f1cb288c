"""jfa_forward_fixed_scratch: the forward for callers that cannot allocate.

Some callers cannot call cudaMalloc or get a workspace from anywhere (a plugin
whose host framework owns the whole device memory pool, a serving loop that
forbids allocation after start-up).  The fixed-scratch entry point gives them
the same forward with its scratch in an array inside the library.  This test
calls it through the C ABI and checks it against jfa_forward (caller
workspace) on two calls in a row with different problems, so that what the
first call leaves in the shared array cannot leak into the second.  Both
entry points run the same kernels on the same deterministic schedule and the
forward uses no atomics, so the outputs must be bitwise equal (NaN-aware):
any stale schedule or bias data would show up as a difference.  It lives in
its own file, collected last, and needs nothing from the other tests.
"""
import pytest
import torch

from jagged_attention_recommender_jfa_b200 import jfa
from jagged_attention_recommender_jfa_b200.inputs import make_problem

pytestmark = pytest.mark.gpu


def _run_both(p, dev):
    t = {n: getattr(p, n).to(dev).contiguous() for n in ("q", "k", "v", "q_off", "kv_off")}
    bias = p.bias.to(dev).contiguous() if p.bias is not None else None
    prob = jfa.problem_of(p)
    ref_out, ref_lse = jfa.attention_forward(prob, t["q"], t["k"], t["v"], t["q_off"],
                                             t["kv_off"], bias, p.act, p.causal)
    out = torch.full_like(t["q"], float("nan"))
    lse = torch.full((p.total_q, p.H), float("nan"), device=dev) if p.act == "softmax" else None
    jfa.jfa_forward_fixed_scratch(prob, t["q"], t["k"], t["v"], t["q_off"], t["kv_off"], bias,
                                  p.act, p.causal, out, lse)
    torch.cuda.synchronize(dev)
    return (out, lse), (ref_out, ref_lse)


def _same(a, b):
    """Bitwise equality; NaN (e.g. never-written) positions must coincide."""
    assert a.shape == b.shape and a.dtype == b.dtype
    assert torch.equal(torch.isnan(a), torch.isnan(b))
    keep = ~torch.isnan(a)
    assert torch.equal(a[keep], b[keep])


def test_fixed_scratch_forward_matches_workspace_forward(cuda_device):
    problems = [make_problem("self_bf16", 21, B=7, max_len=400),          # causal, relpos
                make_problem("gdpa_bf16", 22, B=9, max_len=500, act="silu")]  # dense bias, GDPA
    for p in problems:  # two calls in a row, different shapes
        (out, lse), (ref_out, ref_lse) = _run_both(p, cuda_device)
        _same(out, ref_out)
        if lse is not None:
            _same(lse, ref_lse)
    # and the first problem again after the second one used the array
    (out, lse), (ref_out, ref_lse) = _run_both(problems[0], cuda_device)
    _same(out, ref_out)
    _same(lse, ref_lse)


def test_fixed_scratch_bad_offsets_leave_sentinel(cuda_device):
    # the fixed-scratch call cannot report the on-device offset check; a
    # caller pre-fills the outputs with NaN and finds them unwritten
    p = make_problem("self_bf16", 23, B=4, max_len=100)
    t = {n: getattr(p, n).to(cuda_device).contiguous() for n in ("q", "k", "v", "q_off")}
    bias = p.bias.to(cuda_device)
    bad = t["q_off"].clone()
    bad[2] = bad[1] - 1  # decreasing
    prob = jfa.problem_of(p)
    out = torch.full_like(t["q"], float("nan"))
    lse = torch.full((p.total_q, p.H), float("nan"), device=cuda_device)
    jfa.jfa_forward_fixed_scratch(prob, t["q"], t["k"], t["v"], bad, bad, bias, "softmax", True,
                                  out, lse)
    torch.cuda.synchronize(cuda_device)
    assert torch.isnan(out).all() and torch.isnan(lse).all()
    # a good call right after it on the same array is complete and exact
    (out, lse), (ref_out, ref_lse) = _run_both(p, cuda_device)
    _same(out, ref_out)
    _same(lse, ref_lse)


def test_fixed_scratch_rejects_oversize_problem(cuda_device):
    # a descriptor whose schedule needs more than the fixed 8 MiB; rejected on
    # the host before anything is launched
    prob = jfa.make_problem(batch=4096, heads=16, head_dim=128, max_q_len=8192, max_kv_len=8192,
                            total_q=4096 * 2048, total_kv=4096 * 2048, dtype="bf16")
    assert jfa.jfa_workspace_bytes(prob, 0) > 8 << 20
    fake = 1 << 20
    with pytest.raises(jfa.JfaError) as ei:
        jfa.jfa_forward_fixed_scratch(prob, fake, fake, fake, fake, fake, None, "softmax", 1,
                                      fake, fake)
    assert ei.value.status == jfa.JFA_ERR_WORKSPACE
    assert "fixed array" in str(ei.value)
