"""The C-ABI library loads and exports every symbol include/l3.h declares;
argument checks that run before any CUDA call (no GPU needed)."""
import ctypes
import os
import re

import pytest

import static_token_routed_b200 as l3
from static_token_routed_b200 import build as l3build

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "l3.h")


@pytest.fixture(scope="module")
def lib():
    l3build.build()
    return l3.library()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(l3_[a-z_]+)\s*\(", src)))


def test_header_lists_the_binding_symbols():
    assert declared_functions() == sorted(l3.EXPORTED)


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} missing from libl3.so"


def test_null_out_is_rejected(lib):
    dims = l3.make_dims(10, 20, 4, 16, 16, 16, 16)
    st = lib.l3_plan(None, 0, None, ctypes.byref(dims), None, None)
    assert st == 1 and "NULL" in l3.l3_last_error()


@pytest.mark.parametrize("field,value,status", [
    ("d_in", 24, 4),      # not a multiple of 16 for bf16
    ("k", 0, 1),
    ("v", 5, 1),          # v < vocab
    ("d_emb", 1024, 4),   # beyond the supported width
    ("dtype", 7, 1),
])
def test_bad_dims_are_rejected_before_any_launch(lib, field, value, status):
    dims = l3.make_dims(10, 20, 4, 16, 16, 16, 16)
    setattr(dims, field, value)
    out = ctypes.c_void_p(123)
    st = lib.l3_plan(None, 0, ctypes.c_void_p(16), ctypes.byref(dims), None, ctypes.byref(out))
    assert st == status, l3.l3_last_error()
    assert out.value is None


def test_forward_rejects_null_plan(lib):
    assert lib.l3_forward(None, None, None, None, None, None, None, None, None, None) == 1


def test_backward_rejects_null_plan(lib):
    assert lib.l3_backward(*([None] * 17)) == 1
    assert "plan" in l3.l3_last_error()
