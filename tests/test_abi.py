"""The C-ABI library: it loads, exports every symbol the header declares, and its
host-side argument checks answer without touching a GPU."""
import ctypes
import os
import re

import pytest

from block_sparse_gqa_nsa_b200 import nsa
from block_sparse_gqa_nsa_b200.build import build, LIB

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    src = open(os.path.join(ROOT, "include", "lsrm_nsa.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(lsrm_\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    build()
    return nsa.load_library()


def test_header_and_binding_agree():
    assert declared_symbols() == sorted(nsa.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    out = os.popen(f"nm -D --defined-only {LIB}").read()
    exported = set(re.findall(r" T (\w+)", out))
    for name in declared_symbols():
        assert name in exported, name
        assert hasattr(lib, name)
    # nothing else leaks out of the library (hidden visibility by default)
    assert {s for s in exported if s.startswith("lsrm_")} == set(declared_symbols())


def _desc(**kw):
    base = dict(n_tokens=1024, n_blocks=16, max_block_len=64, n_q_heads=32, n_kv_heads=2, head_dim=32, top_k=4,
                window=64, scale=0.0, pooled_q=False, n_gates=3)
    base.update(kw)
    return nsa.make_desc(**base)


def test_workspace_size_and_validation_on_host(lib):
    n = nsa.lsrm_nsa_workspace_size(_desc())
    assert n > 0 and n % 256 == 0
    for bad in (dict(head_dim=48), dict(top_k=17), dict(top_k=0), dict(n_q_heads=3), dict(window=3),
                dict(max_block_len=513), dict(n_gates=4), dict(scale=-1.0), dict(n_blocks=0),
                dict(pooled_q=True, n_gates=3)):
        assert nsa.lsrm_nsa_workspace_size(_desc(**bad)) == 0, bad


def test_calls_reject_bad_arguments_before_any_launch(lib):
    d = _desc()
    # a dummy 256-byte-aligned workspace address: the null tensors are rejected before it is touched
    rc = lib.lsrm_nsa_forward(ctypes.byref(d), None, None, None, None, None, None, 2, None, None, None, None, 256,
                              None)
    assert rc == 1  # invalid argument: null tensors
    d48 = _desc(head_dim=48)
    rc = lib.lsrm_nsa_compress(ctypes.byref(d48), None, None, None, None, None, None, None, None, None, None, None,
                               None)
    assert rc == 2  # unsupported head_dim
    rc = lib.lsrm_nsa_forward(ctypes.byref(d), 16, 16, 16, 16, 16, 16, 2, 16, None, None, None, None, None)
    assert rc == 6  # workspace missing
    # a saved-branch-output pointer off the 16-byte grid is an invalid argument
    rc = lib.lsrm_nsa_forward(ctypes.byref(d), 16, 16, 16, 16, 16, 16, 2, 16, None, None, 24, 256, None)
    assert rc == 1
    assert lib.lsrm_nsa_last_device_status(None, None) == 6
    assert nsa.lsrm_status_string(5) == "device bounds check failed"
