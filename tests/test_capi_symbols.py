"""The C ABI: every function include/tsd.h declares is exported by
libtsd.so and bound by the Python layer (CPU only, nothing is launched)."""

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


# Host-side argument checks of the other entry points: each call below is
# refused before any CUDA call, so fake (but aligned) addresses never reach a
# kernel.  Skipped where a GPU is present: if a check were ever missing, such
# a call would launch on addresses that are not device memory.
_A = 0x10000           # a 16-byte aligned stand-in address
_U = 0x10004           # a misaligned one


@pytest.mark.skipif(__import__("torch").cuda.is_available(),
                    reason="fake addresses must not reach a GPU")
def test_host_checks_of_every_entry_point(lib):
    ERR_NULL, ERR_SHAPE, ERR_DTYPE, ERR_ALIGN = -1, -2, -3, -6
    BF16, F32 = 1, 0

    def attn(q=_A, B=2, Tmax=8, Hq=8, Hkv=2, D=128, Lmax=64, dtype=BF16):
        return lib.tsd_tree_attention(q, _A, _A, _A, _A, _A, B, Tmax, Hq, Hkv, D, Lmax, 0.1,
                                      dtype, _A, _A, 1 << 20, _A, None)
    assert attn(B=0) == 0
    assert attn(q=None) == ERR_NULL
    assert attn(Hq=6, Hkv=4) == ERR_SHAPE          # heads not a multiple
    assert attn(Tmax=129) == ERR_SHAPE             # more tree slots than the mask holds
    assert attn(Lmax=4) == ERR_SHAPE               # cache shorter than the tree slots
    assert attn(D=96) == ERR_DTYPE
    assert attn(dtype=7) == ERR_DTYPE
    assert attn(q=_U) == ERR_ALIGN
    assert attn(B=40000, Hq=2, Hkv=2) == ERR_SHAPE   # (b, KV head) pairs beyond the grid's y
    assert lib.tsd_tree_attention_workspace_size(40000, 8, 2, 2, 128, 64, BF16) == 0
    assert lib.tsd_tree_verify_greedy(_A, _A, _A, _A, _A, _A, 70000, 8, 100, _A, _A, _A, _A,
                                      1 << 20, _A, None) == ERR_SHAPE

    def paged(table=_A, num_pages=4, page_size=64, max_blocks=4, B=2):
        return lib.tsd_tree_attention_paged(_A, _A, _A, table, num_pages, page_size, max_blocks,
                                            _A, _A, _A, B, 8, 8, 2, 128, 0.1, BF16, _A, _A,
                                            1 << 20, _A, None)
    for ps in (8, 24, 8192):                        # not a power of two in [16, 4096]
        assert paged(page_size=ps) == ERR_SHAPE
    assert paged(max_blocks=0) == ERR_SHAPE
    assert paged(num_pages=0) == ERR_SHAPE
    assert paged(table=None) == ERR_NULL
    assert paged(B=0) == 0

    def commit(k=_A, D=128, dtype=BF16, B=2, path=_A):
        return lib.tsd_kv_commit(k, _A, _A, path, _A, B, 8, 2, D, 64, dtype, _A, _A, None)
    assert commit(D=4) == ERR_SHAPE                 # 8-byte rows: not a 16-byte multiple
    assert commit(D=512) == ERR_SHAPE               # 1 KB rows: beyond the staging limit
    assert commit(dtype=7) == ERR_DTYPE
    assert commit(path=None) == ERR_NULL
    assert commit(k=_U) == ERR_ALIGN
    assert commit(B=0) == 0
    assert commit(B=70000) == ERR_SHAPE

    def expand(k=2, Tmax=8, q=_A, B=2):
        return lib.tsd_tree_expand(q, 9, 100, _A, k, _A, _A, _A, _A, _A, B, Tmax, _A, None)
    assert expand(k=0) == ERR_SHAPE
    assert expand(k=9) == ERR_SHAPE                 # k > Tmax
    assert expand(q=None) == ERR_NULL
    assert expand(B=0) == 0

    assert lib.tsd_tree_dfs_order(_A, _A, _A, _A, 2, 129, _A, _A, _A, _A, _A, None) == ERR_SHAPE
    assert lib.tsd_tree_dfs_order(_A, None, _A, _A, 2, 8, _A, _A, _A, _A, _A, None) == ERR_NULL

    def merge(M=3, L=4, Tmax=16, ct=_A):
        return lib.tsd_tree_merge_chains(ct, _A, _A, M, L, 2, Tmax, _A, _A, _A, _A, _A, None)
    assert merge(M=0) == ERR_SHAPE
    assert merge(L=0) == ERR_SHAPE
    assert merge(Tmax=200) == ERR_SHAPE
    assert merge(ct=None) == ERR_NULL

    probe = lib.tsd_debug_wait_probe
    assert probe(3, 50_000_000, _A, _A, None) == ERR_SHAPE       # unknown kind
    assert probe(0, 10, _A, _A, None) == ERR_SHAPE               # below 1 ms
    assert probe(1, 3_000_000_000, _A, _A, None) == ERR_SHAPE    # above 2 s
    assert probe(0, 50_000_000, None, _A, None) == ERR_NULL
    assert probe(0, 50_000_000, _U, _A, None) == ERR_ALIGN


def test_launching_entry_points_open_an_nvtx_range():
    # Every C-ABI call that launches work is a named range on a profiler's
    # timeline: its body starts with TSD_NVTX_RANGE().
    csrc = os.path.join(ROOT, "tree_speculative_decoding_ancestor_b200", "csrc")
    bodies = {}
    for f in ("capi.cu", "verify_noalloc.cu"):
        src = open(os.path.join(csrc, f)).read()
        for m in re.finditer(r"\n(?:extern \"C\" )?int (tsd_[a-z0-9_]+)\(([^{]*)\)\n\{\n(.*?)\n\}\n",
                             src, flags=re.S):
            bodies[m.group(1)] = m.group(3)
    launching = {n for n, body in bodies.items() if "launch" in body or "<<<" in body}
    assert {"tsd_tree_attention", "tsd_tree_verify_stochastic_noalloc",
            "tsd_kv_commit"} <= launching
    for n in launching:
        assert bodies[n].lstrip().startswith("TSD_NVTX_RANGE();"), n
