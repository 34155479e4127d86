"""The C ABI: every function include/tsd.h declares is exported by
libtsd.so and bound by the Python layer (CPU only, nothing is launched)."""

import ctypes
import os
import re
import subprocess

import pytest

import tree_speculative_decoding_ancestor_b200 as tsd
from tree_speculative_decoding_ancestor_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            src = open(os.path.join(ROOT, "include", f)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(tsd_[a-z0-9_]+)\s*\(", src))
    return names


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(tsd.LIB_PATH):
        from tree_speculative_decoding_ancestor_b200 import build
        build.build()
    return tsd.load_library()


def test_header_declarations_exported(lib):
    names = _declared()
    assert {"tsd_tree_mask_build", "tsd_tree_attention", "tsd_tree_verify_greedy",
            "tsd_tree_verify_stochastic"} <= names
    out = subprocess.run(["nm", "-D", "--defined-only", tsd.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\b(tsd_[a-z0-9_]+)\b", out))
    assert names <= exported, names - exported
    for n in names:
        assert hasattr(lib, n)


def test_binding_covers_header():
    assert set(binding.exported_symbols()) == _declared()


def test_host_only_calls(lib):
    assert lib.tsd_version() >= 100
    assert lib.tsd_status_string(0) == b"ok"
    assert lib.tsd_status_string(-2).startswith(b"size")
    # shape errors are caught before any CUDA call
    assert lib.tsd_tree_mask_build(None, None, 1, 0, None, None, None, None, None, None) == -2
    assert lib.tsd_tree_mask_build(None, None, 1, 129, None, None, None, None, None, None) == -2
    assert lib.tsd_tree_mask_build(None, None, 0, 8, None, None, None, None, None, None) == 0
    assert lib.tsd_tree_mask_build(None, None, 1, 8, None, None, None, None, None, None) == -1
    assert lib.tsd_tree_verify_workspace_size(0, 8, 10) == 0
    assert lib.tsd_tree_verify_workspace_size(2, 8, 10) > 0
    assert lib.tsd_tree_verify_stochastic(None, 0.0, None, 1, None, None, None, None, None,
                                          None, None, 1, 4, 8, None, None, None, None, 0, None,
                                          None) == -2
