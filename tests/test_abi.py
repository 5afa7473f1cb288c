"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every function include/jfa.h declares, sizes workspaces and rejects invalid
arguments on the host before touching the device."""
import ctypes
import os
import re

import pytest

from jagged_attention_recommender_jfa_b200 import jfa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if not fn.endswith(".h"):
            continue
        text = open(os.path.join(ROOT, "include", fn)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s+\*?(jfa_[a-z0-9_]+)\s*\(",
                             text, flags=re.M):
            names.add(m.group(1))
    return names


def test_library_exports_every_declared_symbol():
    lib = jfa.load()
    declared = _declared_functions()
    assert {"jfa_forward", "jfa_backward", "jfa_quantize_mxfp8", "jfa_workspace_bytes"} <= declared
    for name in declared:
        assert hasattr(lib, name), name
    assert set(jfa.EXPORTS) == declared
    # the built library is the in-tree one
    assert os.path.dirname(jfa.lib_path()) == os.path.join(ROOT, "jagged_attention_recommender_jfa_b200")


def _problem(**kw):
    base = dict(batch=4, heads=2, head_dim=32, max_q_len=64, max_kv_len=64, total_q=100,
                total_kv=100, dtype="f32", bias_kind="relpos", relpos_len=129)
    base.update(kw)
    return jfa.make_problem(**base)


def test_workspace_sizes():
    p = _problem()
    f = jfa.jfa_workspace_bytes(p, 0)
    b = jfa.jfa_workspace_bytes(p, 1)
    assert 256 < f < b
    # backward holds at least D = rowsum(dO*O): total_q * heads floats
    assert b - f >= 100 * 2 * 4
    assert jfa.jfa_workspace_bytes(_problem(head_dim=96), 0) == 0
    assert jfa.jfa_workspace_bytes(_problem(heads=0), 0) == 0


def test_invalid_arguments_rejected_on_host():
    p = _problem()
    ws_bytes = jfa.jfa_workspace_bytes(p, 0)
    fake = 1 << 20  # never dereferenced: every case fails host validation
    cases = [
        (_problem(head_dim=96), jfa.JFA_ERR_UNSUPPORTED),
        (_problem(relpos_len=128), jfa.JFA_ERR_INVALID_ARGUMENT),
        (_problem(dtype=7), jfa.JFA_ERR_INVALID_ARGUMENT),
        (_problem(total_q=-1), jfa.JFA_ERR_INVALID_ARGUMENT),
    ]
    for prob, status in cases:
        with pytest.raises(jfa.JfaError) as ei:
            jfa.jfa_forward(prob, fake, fake, fake, fake, fake, fake, "softmax", 1, fake, fake,
                            fake, ws_bytes, stream=0)
        assert ei.value.status == status
    # workspace too small
    with pytest.raises(jfa.JfaError) as ei:
        jfa.jfa_forward(p, fake, fake, fake, fake, fake, fake, "softmax", 1, fake, fake, fake,
                        ws_bytes - 1, stream=0)
    assert ei.value.status == jfa.JFA_ERR_WORKSPACE
    # misaligned tensor
    with pytest.raises(jfa.JfaError) as ei:
        jfa.jfa_forward(p, fake + 4, fake, fake, fake, fake, fake, "softmax", 1, fake, fake,
                        fake, ws_bytes, stream=0)
    assert ei.value.status == jfa.JFA_ERR_INVALID_ARGUMENT
    # missing bias for a bias kind, bad activation
    with pytest.raises(jfa.JfaError) as ei:
        jfa.jfa_forward(p, fake, fake, fake, fake, fake, None, "softmax", 1, fake, fake, fake,
                        ws_bytes, stream=0)
    assert ei.value.status == jfa.JFA_ERR_INVALID_ARGUMENT
    with pytest.raises(jfa.JfaError) as ei:
        jfa.jfa_forward(p, fake, fake, fake, fake, fake, fake, 9, 1, fake, fake, fake, ws_bytes,
                        stream=0)
    assert ei.value.status == jfa.JFA_ERR_INVALID_ARGUMENT
    # softmax backward without lse
    bws = jfa.jfa_workspace_bytes(p, 1)
    with pytest.raises(jfa.JfaError) as ei:
        jfa.jfa_backward(p, fake, fake, fake, fake, None, fake, fake, fake, fake, "softmax", 1,
                         fake, fake, fake, fake, bws, stream=0)
    assert ei.value.status == jfa.JFA_ERR_INVALID_ARGUMENT
    # schedule capacity / tile checks
    with pytest.raises(jfa.JfaError):
        jfa.jfa_schedule(p, fake, fake, 1, 0, 24, fake, 10**6, fake, fake, bws, stream=0)
    with pytest.raises(jfa.JfaError):
        jfa.jfa_schedule(p, fake, fake, 1, 0, 64, fake, 1, fake, fake, bws, stream=0)
    # quantiser sizes
    with pytest.raises(jfa.JfaError):
        jfa.jfa_quantize_mxfp8(fake, 10, 2, 48, None, 0, 0, 0, fake, fake, stream=0)
    assert "quantiser sizes" in jfa.load().jfa_last_error().decode()


def test_empty_batch_is_a_no_op():
    p = _problem(batch=0, total_q=0, total_kv=0, max_q_len=0, max_kv_len=0)
    ws = jfa.jfa_workspace_bytes(p, 0)
    fake = 1 << 20
    jfa.jfa_forward(p, None, None, None, fake, fake, fake, "softmax", 1, None, None, fake, ws,
                    stream=0)
