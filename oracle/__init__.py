"""CPU oracle for tree speculative decoding verification -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It never imports the CUDA package and
the CUDA package never imports it; both read their inputs from the seeded
generator in ``workloads``.

The arithmetic lives in ``tsd_oracle.c`` (plain C, fp64, one loop per step
of each definition); this module only marshals arguments through ctypes and
allocates outputs.  Every output array is pre-filled with a sentinel so that
callers can check which entries a function leaves untouched.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Dict, Optional, Sequence

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "tsd_oracle.c")
_LIB_DIR = os.path.join(_HERE, "_build")
_LIB = os.path.join(_LIB_DIR, "libtsd_oracle.so")
_lock = threading.Lock()
_lib: Optional[ctypes.CDLL] = None

SENTINEL = -7
BAD_TREE, BAD_TOKEN, BAD_QROW, BAD_PATH = 1, 2, 4, 32


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (IEEE semantics: no fast-math, no FMA
    contraction) into ``oracle/_build/libtsd_oracle.so``."""
    os.makedirs(_LIB_DIR, exist_ok=True)
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off",
                               "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load() -> ctypes.CDLL:
    global _lib
    with _lock:
        if _lib is None:
            _lib = ctypes.CDLL(build())
            _lib.oracle_num_threads.restype = ctypes.c_int
        return _lib


def num_threads() -> int:
    return int(_load().oracle_num_threads())


class use_library:
    """Context manager: route every oracle call to another build of the oracle
    source (the mutation tests plant mistakes in a copy and check that the
    pins catch them)."""

    def __init__(self, path: str):
        self.path = path
        self.saved: Optional[ctypes.CDLL] = None

    def __enter__(self):
        global _lib
        _load()
        with _lock:
            self.saved = _lib
            lib = ctypes.CDLL(self.path)
            lib.oracle_num_threads.restype = ctypes.c_int
            _lib = lib
        return self

    def __exit__(self, *exc):
        global _lib
        with _lock:
            _lib = self.saved
        return False


def build_variant(source: str, out_path: str) -> str:
    """Compile oracle C source text (same flags as build()) to out_path."""
    src = out_path + ".c"
    with open(src, "w") as f:
        f.write(source)
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fPIC",
                           "-shared", "-o", out_path, src, "-lm"])
    return out_path


def source() -> str:
    with open(_SRC) as f:
        return f.read()


def _np(t, dtype=None) -> np.ndarray:
    """Contiguous numpy view of a CPU tensor/array (bf16 as raw uint16 bits)."""
    if isinstance(t, torch.Tensor):
        t = t.detach().cpu().contiguous()
        if t.dtype == torch.bfloat16:
            return t.view(torch.int16).numpy().view(np.uint16)
        a = t.numpy()
    else:
        a = np.ascontiguousarray(t)
    if dtype is not None:
        a = np.ascontiguousarray(a, dtype=dtype)
    return a


def _p(a: np.ndarray) -> ctypes.c_void_p:
    return ctypes.c_void_p(a.ctypes.data)


def _dtype_code(t) -> int:
    if isinstance(t, torch.Tensor):
        if t.dtype == torch.float32:
            return 0
        if t.dtype == torch.bfloat16:
            return 1
    elif isinstance(t, np.ndarray) and t.dtype == np.float32:
        return 0
    raise TypeError("oracle attention inputs must be float32 or bfloat16")


def tree_mask(parent, n_nodes, Tmax: int) -> Dict[str, np.ndarray]:
    """Ancestor-or-self bitmask [B][Tmax][ceil(Tmax/32)] u32, depth (path
    length), first_child [B][Tmax+1] (slot 0 = root), next_sibling, status."""
    lib = _load()
    par = _np(parent, np.int32)
    nn = _np(n_nodes, np.int32)
    B = nn.shape[0]
    W = (Tmax + 31) // 32
    mask = np.zeros((B, Tmax, W), dtype=np.uint32)
    depth = np.zeros((B, Tmax), dtype=np.int32)
    fc = np.zeros((B, Tmax + 1), dtype=np.int32)
    ns = np.zeros((B, Tmax), dtype=np.int32)
    st = np.zeros(B, dtype=np.int32)
    lib.oracle_tree_mask(_p(par), _p(nn), B, Tmax, _p(mask), _p(depth), _p(fc), _p(ns), _p(st))
    return dict(mask=mask, depth=depth, first_child=fc, next_sibling=ns, status=st)


def tree_attention(q, k_cache, v_cache, prefix_len, n_nodes, parent, scale: float) -> np.ndarray:
    """All rows: float64 [B][Tmax][Hq][D]; padding rows are NaN."""
    lib = _load()
    dt = _dtype_code(q)
    qa, ka, va = _np(q), _np(k_cache), _np(v_cache)
    B, Tmax, Hq, D = qa.shape
    Hkv, Lmax = ka.shape[1], ka.shape[2]
    pl = _np(prefix_len, np.int32)
    nn = _np(n_nodes, np.int32)
    par = _np(parent, np.int32)
    out = np.full((B, Tmax, Hq, D), np.nan, dtype=np.float64)
    rc = lib.oracle_tree_attention(_p(qa), _p(ka), _p(va), dt, _p(pl), _p(nn), _p(par), B, Tmax,
                                   Hq, Hkv, D, Lmax, ctypes.c_double(scale), _p(out))
    if rc:
        raise ValueError(f"oracle_tree_attention: malformed input (status {rc})")
    return out


def tree_attention_rows(q, k_cache, v_cache, prefix_len, n_nodes, parent, scale: float,
                        rows: Sequence[Sequence[int]]) -> np.ndarray:
    """Selected rows (b, u, h) -> float64 [len(rows)][D]."""
    lib = _load()
    dt = _dtype_code(q)
    qa, ka, va = _np(q), _np(k_cache), _np(v_cache)
    B, Tmax, Hq, D = qa.shape
    Hkv, Lmax = ka.shape[1], ka.shape[2]
    pl, nn, par = _np(prefix_len, np.int32), _np(n_nodes, np.int32), _np(parent, np.int32)
    sel = np.ascontiguousarray(np.asarray(rows, dtype=np.int32).reshape(-1, 3))
    out = np.full((sel.shape[0], D), np.nan, dtype=np.float64)
    rc = lib.oracle_tree_attention_rows(_p(qa), _p(ka), _p(va), dt, _p(pl), _p(nn), _p(par),
                                        B, Tmax, Hq, Hkv, D, Lmax, ctypes.c_double(scale),
                                        sel.shape[0], _p(sel), _p(out))
    if rc:
        raise ValueError(f"oracle_tree_attention_rows: malformed input (status {rc})")
    return out


def verify_greedy(logits, tokens, parent, n_nodes) -> Dict[str, np.ndarray]:
    lib = _load()
    lg = _np(logits, np.float32)
    B, R, V = lg.shape
    Tmax = R - 1
    tk, par, nn = _np(tokens, np.int32), _np(parent, np.int32), _np(n_nodes, np.int32)
    out_tokens = np.full((B, Tmax + 1), SENTINEL, dtype=np.int32)
    out_path = np.full((B, Tmax), SENTINEL, dtype=np.int32)
    n_acc = np.full(B, SENTINEL, dtype=np.int32)
    st = np.zeros(B, dtype=np.int32)
    lib.oracle_verify_greedy(_p(lg), _p(tk), _p(par), _p(nn), B, Tmax, V, _p(out_tokens),
                             _p(out_path), _p(n_acc), _p(st))
    return dict(out_tokens=out_tokens, out_path=out_path, n_accepted=n_acc, status=st)


def verify_stochastic(logits, temperature: float, q_probs, q_row, tokens, parent, n_nodes,
                      u_accept, u_sample) -> Dict[str, np.ndarray]:
    lib = _load()
    lg = _np(logits, np.float32)
    B, R, V = lg.shape
    Tmax = R - 1
    qp = _np(q_probs, np.float32)
    Rq = qp.shape[1]
    qr, tk = _np(q_row, np.int32), _np(tokens, np.int32)
    par, nn = _np(parent, np.int32), _np(n_nodes, np.int32)
    ua, us = _np(u_accept, np.float64), _np(u_sample, np.float64)
    out_tokens = np.full((B, Tmax + 1), SENTINEL, dtype=np.int32)
    out_path = np.full((B, Tmax), SENTINEL, dtype=np.int32)
    n_acc = np.full(B, SENTINEL, dtype=np.int32)
    nflag = np.zeros(B, dtype=np.int32)
    ndec = np.zeros(B, dtype=np.int32)
    st = np.zeros(B, dtype=np.int32)
    lib.oracle_verify_stochastic(_p(lg), ctypes.c_double(temperature), _p(qp), _p(qr), Rq,
                                 _p(tk), _p(par), _p(nn), _p(ua), _p(us), B, Tmax, V,
                                 _p(out_tokens), _p(out_path), _p(n_acc), _p(nflag), _p(ndec),
                                 _p(st))
    return dict(out_tokens=out_tokens, out_path=out_path, n_accepted=n_acc, n_flagged=nflag,
                n_decisions=ndec, status=st)


def kv_commit(k_cache, v_cache, prefix_len, out_path, n_accepted) -> Dict[str, np.ndarray]:
    """Move the accepted nodes' K/V rows to the positions right after the
    prefix.  Works on copies: returns the new caches (same dtype/shape as
    the inputs, as numpy arrays; bf16 as raw uint16), new_prefix and status."""
    lib = _load()
    ka = _np(k_cache).copy()
    va = _np(v_cache).copy()
    B, Hkv, Lmax, D = ka.shape
    path = _np(out_path, np.int32)
    Tmax = path.shape[1]
    nacc = _np(n_accepted, np.int32)
    pl = _np(prefix_len, np.int32)
    newp = np.full(B, SENTINEL, dtype=np.int32)
    st = np.zeros(B, dtype=np.int32)
    lib.oracle_kv_commit(_p(ka), _p(va), _p(pl), _p(path), _p(nacc), B, Tmax, Hkv, Lmax,
                         D * ka.itemsize, _p(newp), _p(st))
    return dict(k_cache=ka, v_cache=va, new_prefix=newp, status=st)


def gather_pages(k_pages, v_pages, block_table, page_size: int, Lmax: int):
    """Paged K/V pools [num_pages][Hkv][page_size][D] + block table
    [B][max_blocks] -> contiguous caches [B][Hkv][Lmax][D] (logical position
    pos of sequence b lives in physical page block_table[b][pos // page_size]
    at row pos % page_size).  Logical pages beyond the table are zero."""
    kp, vp = _np(k_pages), _np(v_pages)
    bt = _np(block_table, np.int32)
    B, nblk = bt.shape
    _, Hkv, ps, D = kp.shape
    assert ps == page_size
    k = np.zeros((B, Hkv, Lmax, D), dtype=kp.dtype)
    v = np.zeros((B, Hkv, Lmax, D), dtype=vp.dtype)
    for b in range(B):
        for j in range(nblk):
            lo = j * page_size
            if lo >= Lmax:
                break
            hi = min(lo + page_size, Lmax)
            pg = int(bt[b, j])
            k[b, :, lo:hi] = kp[pg, :, :hi - lo]
            v[b, :, lo:hi] = vp[pg, :, :hi - lo]
    return k, v


def tree_attention_paged(q, k_pages, v_pages, block_table, page_size: int, prefix_len, n_nodes,
                         parent, scale: float) -> np.ndarray:
    """Tree attention over a paged KV cache: the same definition as
    tree_attention, on the cache the block table describes."""
    qa = _np(q)
    Tmax = qa.shape[1]
    Lmax = int(np.asarray(_np(block_table)).shape[1]) * page_size
    k, v = gather_pages(k_pages, v_pages, block_table, page_size, Lmax)
    if isinstance(q, torch.Tensor) and q.dtype == torch.bfloat16:
        k = torch.from_numpy(k.view(np.int16)).view(torch.bfloat16)
        v = torch.from_numpy(v.view(np.int16)).view(torch.bfloat16)
    return tree_attention(q, k, v, prefix_len, n_nodes, parent, scale)


def tree_expand(q_probs, frow, k: int, parent, tokens, q_row, n_nodes, lvl_begin):
    """One expansion level (on copies of the tree arrays): every frontier node
    gets the k best tokens of its q row as children.  Returns the new arrays
    and status."""
    lib = _load()
    qp = _np(q_probs, np.float32)
    B, Rq, V = qp.shape
    par = _np(parent, np.int32).copy()
    tok = _np(tokens, np.int32).copy()
    qr = _np(q_row, np.int32).copy()
    nn = _np(n_nodes, np.int32).copy()
    lb = _np(lvl_begin, np.int32).copy()
    fr = _np(frow, np.int32)
    Tmax = par.shape[1]
    st = np.zeros(B, dtype=np.int32)
    lib.oracle_tree_expand(_p(qp), Rq, V, _p(fr), int(k), _p(par), _p(tok), _p(qr), _p(nn),
                           _p(lb), B, Tmax, _p(st))
    return dict(parent=par, tokens=tok, q_row=qr, n_nodes=nn, lvl_begin=lb, status=st)


def tree_dfs_order(parent, tokens, q_row, n_nodes) -> Dict[str, np.ndarray]:
    """Depth-first pre-order renumbering (children in increasing index)."""
    lib = _load()
    par = _np(parent, np.int32)
    tok = _np(tokens, np.int32)
    qr = _np(q_row, np.int32)
    nn = _np(n_nodes, np.int32)
    B, Tmax = par.shape
    perm = np.full((B, Tmax), SENTINEL, dtype=np.int32)
    op = np.full((B, Tmax), SENTINEL, dtype=np.int32)
    ot = np.full((B, Tmax), SENTINEL, dtype=np.int32)
    oq = np.full((B, Tmax), SENTINEL, dtype=np.int32)
    st = np.zeros(B, dtype=np.int32)
    lib.oracle_tree_dfs_order(_p(par), _p(tok), _p(qr), _p(nn), B, Tmax, _p(perm), _p(op),
                              _p(ot), _p(oq), _p(st))
    return dict(perm=perm, parent=op, tokens=ot, q_row=oq, status=st)


def tree_merge_chains(chain_tokens, chain_q_row, chain_len, Tmax: int) -> Dict[str, np.ndarray]:
    """Merge M chains per sequence ([B][M][L] tokens and q rows, [B][M]
    lengths) into one token tree in depth-first pre-order."""
    lib = _load()
    ct = _np(chain_tokens, np.int32)
    cq = _np(chain_q_row, np.int32)
    cl = _np(chain_len, np.int32)
    B, M, L = ct.shape
    par = np.full((B, Tmax), SENTINEL, dtype=np.int32)
    tok = np.full((B, Tmax), SENTINEL, dtype=np.int32)
    qr = np.full((B, Tmax), SENTINEL, dtype=np.int32)
    nn = np.zeros(B, dtype=np.int32)
    st = np.zeros(B, dtype=np.int32)
    lib.oracle_tree_merge_chains(_p(ct), _p(cq), _p(cl), M, L, B, Tmax, _p(par), _p(tok),
                                 _p(qr), _p(nn), _p(st))
    return dict(parent=par, tokens=tok, q_row=qr, n_nodes=nn, status=st)


# Convenience wrappers over a workloads.Workload -----------------------------

def workload_attention(w) -> np.ndarray:
    return tree_attention(w.q, w.k_cache, w.v_cache, w.prefix_len, w.n_nodes, w.parent, w.scale)


def workload_greedy(w) -> Dict[str, np.ndarray]:
    return verify_greedy(w.logits, w.tokens, w.parent, w.n_nodes)


def workload_stochastic(w) -> Dict[str, np.ndarray]:
    return verify_stochastic(w.logits, w.temperature, w.q_probs, w.q_row, w.tokens, w.parent,
                             w.n_nodes, w.u_accept, w.u_sample)
