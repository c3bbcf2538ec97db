"""The C-ABI library loads and exports every entry point declared in
include/*.h; argument checks and status strings work without a GPU."""
import ctypes
import glob
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for path in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(path).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        names |= set(re.findall(r"^\s*(?:const\s+)?[\w\s\*]*?\b(sffn_\w+)\s*\(", src, flags=re.M))
    return names


@pytest.fixture(scope="module")
def pkg():
    from activation_sparse_gated_gemv_b200 import build
    build.build()
    import activation_sparse_gated_gemv_b200 as m
    return m


def test_every_declared_symbol_is_exported(pkg):
    declared = _declared()
    assert {"sffn_create", "sffn_set_weights", "sffn_forward", "sffn_forward_dense",
            "sffn_get_active", "sffn_destroy", "sffn_strerror"} <= declared
    lib = ctypes.CDLL(pkg.LIB_PATH)
    for name in sorted(declared):
        assert hasattr(lib, name), name
    assert declared == set(pkg.EXPORTED)


def test_status_strings(pkg):
    for code in range(0, 8):
        s = pkg.sffn_strerror(code)
        assert s and s.decode() != "unknown status"
    assert pkg.sffn_strerror(99).decode() == "unknown status"


@pytest.mark.parametrize("cfg", [
    (0, 64, 0, 1, 0, 0),        # d = 0
    (60, 64, 0, 1, 0, 0),       # d not a multiple of 8
    (64, 0, 0, 1, 0, 0),        # d_ff = 0
    (64, 64, 12, 1, 0, 0),      # rank not a multiple of 8
    (64, 64, 0, 0, 0, 0),       # max_tokens = 0
    (64, 64, 0, 2048, 0, 0),    # max_tokens too large
    (64, 64, 0, 1, 7, 0),       # unknown dtype
])
def test_create_rejects_bad_config_before_touching_cuda(pkg, cfg):
    h = ctypes.c_void_p()
    c = pkg.sffn_config(*cfg)
    assert pkg.sffn_create(ctypes.byref(h), ctypes.byref(c)) == pkg.SFFN_ERR_INVALID_ARG
    assert not h.value
    assert pkg.sffn_last_error().decode()


def test_null_handles_are_rejected(pkg):
    sel = pkg.make_select("threshold", 1.0)
    assert pkg.sffn_forward(None, None, 1, 0, ctypes.byref(sel), None, None) == pkg.SFFN_ERR_INVALID_ARG
    assert pkg.sffn_forward_dense(None, None, 1, 0, ctypes.byref(sel), None, None) == pkg.SFFN_ERR_INVALID_ARG
    assert pkg.sffn_forward_host(None, None, 1, 0, ctypes.byref(sel), None, None) == pkg.SFFN_ERR_INVALID_ARG
    assert pkg.sffn_set_weights(None, None, None, None, None, None, 0, None) == pkg.SFFN_ERR_INVALID_ARG
    assert pkg.sffn_get_active(None, None, None, None) == pkg.SFFN_ERR_INVALID_ARG
    assert pkg.sffn_check_status(None) == pkg.SFFN_ERR_INVALID_ARG
    assert pkg.sffn_last_launches(None, None) == pkg.SFFN_ERR_INVALID_ARG
    assert pkg.sffn_set_stage_events(None, None, 0) == pkg.SFFN_ERR_INVALID_ARG
    assert pkg.sffn_set_hot(None, None, 0) == pkg.SFFN_ERR_INVALID_ARG
    assert pkg.sffn_destroy(None) == pkg.SFFN_OK


def test_oracle_is_not_reachable_from_the_library():
    # The product path must not import the oracle: scan the package sources.
    pkg_dir = os.path.join(ROOT, "activation_sparse_gated_gemv_b200")
    for path in glob.glob(os.path.join(pkg_dir, "**", "*"), recursive=True):
        if path.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
            src = open(path).read()
            assert "import oracle" not in src and "from oracle" not in src, path
            assert "sffn_oracle" not in src and "liboracle" not in src, path
