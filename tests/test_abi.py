"""The C-ABI library loads and exports every entry point include/mk.h
declares (no GPU needed: nothing here launches work)."""

import ctypes
import os
import re

from moe_persistent_cta_b200 import mk

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    src = open(os.path.join(ROOT, "include", "mk.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = set(re.findall(r"\b(mk_[a-z_]+)\s*\(", src))
    return names


def test_header_and_binding_agree():
    assert declared_symbols() == set(mk.EXPORTS)


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(mk._LIB_PATH)
    for name in declared_symbols():
        assert hasattr(lib, name), name


def test_strerror_and_argument_validation_without_gpu():
    assert mk.strerror(mk.MK_OK) == "ok"
    assert "deadline" in mk.strerror(mk.MK_ERR_TIMEOUT)
    # null arguments are rejected before any CUDA call
    assert mk.lib.mk_create(None, None, 0, None) == mk.MK_ERR_INVALID
    assert mk.lib.mk_check(None, None, None) == mk.MK_ERR_INVALID
    assert mk.lib.mk_decode_step(None, None, None, None, None, None, None) == mk.MK_ERR_INVALID
    assert mk.lib.mk_decode_step_static(None, None, None, None, None, None,
                                        None) == mk.MK_ERR_INVALID
    assert mk.lib.mk_selftest_timeout(None, 10, None, None) == mk.MK_ERR_INVALID
    mk.lib.mk_destroy(None)
