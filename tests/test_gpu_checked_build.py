"""The bounds-checked debug build (libtsd_checked.so, compiled with
-DTSD_CHECKS): on small cases of every kernel its results match the oracle
and no kernel computes an index outside its buffers (TSD_DEV_BOUNDS stays
clear).  It runs in a child process, since the library is chosen when the
binding first loads it."""

import os
import subprocess
import sys

import pytest

from tree_speculative_decoding_ancestor_b200 import build

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.mark.gpu
def test_checked_build_small_cases(cuda_device):
    lib = build.build(checked=True)
    env = dict(os.environ, TSD_LIBRARY=lib)
    r = subprocess.run([sys.executable, os.path.join(HERE, "checked_run.py")], env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0 and "checked ok" in r.stdout, r.stdout[-2000:] + r.stderr[-2000:]


def test_checked_build_exports_the_same_symbols():
    import re
    lib = build.build(checked=True)
    out = {}
    for path in (build.LIB, lib):
        if not os.path.exists(path):
            build.build()
        nm = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True,
                            text=True, check=True).stdout
        out[path] = set(re.findall(r"\b(tsd_[a-z0-9_]+)\b", nm))
    assert out[build.LIB] == out[lib] and "tsd_tree_attention" in out[lib]
