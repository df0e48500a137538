"""The C-ABI library loads on a machine without a GPU and exports every
function include/tbik.h declares; host-only calls answer without a device."""
import ctypes

import pytest

from invariant_tree_ordered_b200 import _binding as B
from invariant_tree_ordered_b200 import build as libbuild


@pytest.fixture(scope="module")
def lib():
    libbuild.build_library()
    return B.load_library()


def test_every_declared_symbol_is_exported(lib):
    names = B.declared_functions()
    assert len(names) >= 11
    for n in names:
        assert hasattr(lib, n), n


def test_host_only_entry_points(lib):
    assert b"sm_100a" in lib.tbik_version()
    assert lib.tbik_status_string(B.TBIK_ERR_TIMEOUT) == b"device wait timed out"
    assert lib.tbik_status_string(B.TBIK_ERR_TARGET) == b"target index out of range"
    assert lib.tbik_debug_set(0, 0) == B.TBIK_OK


def test_rope_table_rejects_bad_arguments_before_touching_a_device(lib):
    assert lib.tbik_rope_table(None, 16, 128, 1e6, None) == B.TBIK_ERR_ARG
    buf = (ctypes.c_float * 4)()
    assert lib.tbik_rope_table(ctypes.cast(buf, ctypes.c_void_p), 16, 3, 1e6, None) == B.TBIK_ERR_ARG
    assert lib.tbik_rope_table(ctypes.cast(buf, ctypes.c_void_p), 16, 128, -1.0, None) == B.TBIK_ERR_ARG


def test_binding_refuses_to_run_without_the_library(tmp_path):
    with pytest.raises(OSError):
        B.load_library(str(tmp_path / "missing.so"))
