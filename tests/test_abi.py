"""The C-ABI library loads without a GPU, exports every entry point the header
declares, and rejects bad arguments on the host before touching the device."""
import ctypes
import os
import re

import pytest

import block_sparse_attention_dense_b200 as lf
from block_sparse_attention_dense_b200 import build as lfbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    inc = os.path.join(ROOT, "include")
    for f in os.listdir(inc):
        if f.endswith(".h"):
            src = open(os.path.join(inc, f)).read()
            names |= set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(lf_\w+)\s*\(", src, re.M))
    return names


@pytest.fixture(scope="module")
def L():
    lfbuild.build()
    return lf.lib()


def test_every_declared_symbol_is_exported(L):
    names = _declared()
    assert {"lf_attn_fwd", "lf_block_select", "lf_attn_bwd", "lf_workspace_size",
            "lf_status_string", "lf_check_device_error"} <= names
    for n in names:
        assert hasattr(L, n), n
    assert set(lf.EXPORTED) <= names


def test_status_strings(L):
    for code in range(6):
        assert lf.lf_status_string(code).startswith("LF_")


def _desc(**kw):
    base = dict(nseq=1, cu_seqlens=0x1000, max_seqlen=256, total_tokens=256, hq=4, hkv=2, d=128,
                softmax_scale=0.088, causal=1, block_q=128)
    base.update(kw)
    return lf.lf_attn_desc(**base)


@pytest.mark.parametrize("kw,code", [
    (dict(hq=6, hkv=4), lf.LF_ERR_INVALID_ARG),
    (dict(d=96), lf.LF_ERR_UNSUPPORTED),
    (dict(block_q=32), lf.LF_ERR_UNSUPPORTED),
    (dict(nseq=0), lf.LF_ERR_INVALID_ARG),
    (dict(cu_seqlens=0), lf.LF_ERR_INVALID_ARG),
    (dict(softmax_scale=-1.0), lf.LF_ERR_INVALID_ARG),
    (dict(causal=2), lf.LF_ERR_INVALID_ARG),
])
def test_bad_descriptors_rejected(L, kw, code):
    n = ctypes.c_size_t(0)
    assert L.lf_workspace_size(ctypes.byref(_desc(**kw)), lf.LF_WS_BWD, ctypes.byref(n)) == code


def test_workspace_size(L):
    n = ctypes.c_size_t(0)
    assert L.lf_workspace_size(ctypes.byref(_desc()), lf.LF_WS_BWD, ctypes.byref(n)) == 0
    assert n.value >= 256 * 4 * 128 * 4
    assert L.lf_workspace_size(ctypes.byref(_desc()), 7, ctypes.byref(n)) == lf.LF_ERR_INVALID_ARG


def test_null_and_misaligned_pointers_rejected_on_host(L):
    d = _desc()
    p = 0x10000
    assert L.lf_attn_fwd(ctypes.byref(d), None, p, p, p, p, None, 0, None) == lf.LF_ERR_INVALID_ARG
    assert L.lf_attn_fwd(ctypes.byref(d), p + 2, p, p, p, p, None, 0, None) == lf.LF_ERR_INVALID_ARG
    # delta outside [0, 1)
    args = [ctypes.byref(d), p, p, 1.0, 0, 0, 0] + [p] * 7 + [None, 0, None]
    assert L.lf_block_select(*args) == lf.LF_ERR_INVALID_ARG
    # unknown flag bits
    args = [ctypes.byref(d), p, p, 0.1, 0, 0, 0x80] + [p] * 7 + [None, 0, None]
    assert L.lf_block_select(*args) == lf.LF_ERR_INVALID_ARG
    # backward: workspace too small
    bargs = [ctypes.byref(d)] + [p] * 13 + [p, 16, None]
    assert L.lf_attn_bwd(*bargs) == lf.LF_ERR_WORKSPACE


def test_empty_problem_is_a_noop(L):
    d = _desc(total_tokens=0, max_seqlen=0)
    p = 0x10000
    assert L.lf_attn_fwd(ctypes.byref(d), p, p, p, p, p, None, 0, None) == 0
