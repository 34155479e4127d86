"""ctypes binding of libtsd.so (the C ABI declared in include/tsd.h).

Argument marshalling only: shape/dtype/device checks, output and workspace
allocation through PyTorch's caching allocator, and the caller's current
CUDA stream.  Every step of the computation runs in the library's kernels;
there is no CPU or PyTorch fallback -- if the library is missing, every call
raises.
"""

from __future__ import annotations

import ctypes
import os
import threading
from typing import Dict, NamedTuple, Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# The library the binding loads: lib/libtsd.so, or the file TSD_LIBRARY names
# (for instance lib/libtsd_checked.so, the bounds-checked debug build).
LIB_PATH = os.environ.get("TSD_LIBRARY") or os.path.join(_HERE, "lib", "libtsd.so")

TSD_OK = 0
TSD_F32, TSD_BF16 = 0, 1
TSD_MAX_TREE = 128
TSD_TREE_INVALID = -2
DEV_BAD_TREE, DEV_BAD_TOKEN, DEV_BAD_QROW, DEV_BAD_PREFIX, DEV_TIMEOUT = 1, 2, 4, 8, 16
DEV_BAD_PATH, DEV_BAD_PAGE, DEV_BOUNDS = 32, 64, 128

_lock = threading.Lock()
_lib: Optional[ctypes.CDLL] = None

_P = ctypes.c_void_p
_I = ctypes.c_int
_SZ = ctypes.c_size_t

# name -> (restype, argtypes), mirroring include/tsd.h
_SIGNATURES: Dict[str, Tuple[object, list]] = {
    "tsd_status_string": (ctypes.c_char_p, [_I]),
    "tsd_version": (_I, []),
    "tsd_launch_count": (ctypes.c_ulonglong, []),
    "tsd_tree_mask_build": (_I, [_P, _P, _I, _I, _P, _P, _P, _P, _P, _P]),
    "tsd_tree_attention_workspace_size": (_SZ, [_I, _I, _I, _I, _I, _I, _I]),
    "tsd_tree_attention_plan": (_I, [_I, _I, _I, _I, _I, _I, _I, _I, _P]),
    "tsd_tree_attention": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, ctypes.c_float,
                                _I, _P, _P, _SZ, _P, _P]),
    "tsd_tree_verify_workspace_size": (_SZ, [_I, _I, _I]),
    "tsd_tree_verify_greedy": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _P, _P, _P, _P, _SZ, _P,
                                    _P]),
    "tsd_tree_verify_stochastic": (_I, [_P, ctypes.c_double, _P, _I, _P, _P, _P, _P, _P, _P, _P,
                                        _I, _I, _I, _P, _P, _P, _P, _SZ, _P, _P]),
    "tsd_tree_verify_stochastic_noalloc": (_I, [_P, ctypes.c_double, _P, _I, _P, _P, _P, _P, _P,
                                                _P, _P, _I, _I, _I, _P, _P, _P, _P, _P]),
    "tsd_tree_verify_stochastic_plan": (_I, [_I, _I, _I, _P]),
    "tsd_tree_verify_greedy_plan": (_I, [_I, _I, _I, _P]),
    "tsd_kv_commit": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _P]),
    "tsd_tree_attention_paged": (_I, [_P, _P, _P, _P, _I, _I, _I, _P, _P, _P, _I, _I, _I, _I,
                                      _I, ctypes.c_float, _I, _P, _P, _SZ, _P, _P]),
    "tsd_tree_expand": (_I, [_P, _I, _I, _P, _I, _P, _P, _P, _P, _P, _I, _I, _P, _P]),
    "tsd_tree_dfs_order": (_I, [_P, _P, _P, _P, _I, _I, _P, _P, _P, _P, _P, _P]),
    "tsd_tree_merge_chains": (_I, [_P, _P, _P, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P]),
    "tsd_debug_wait_probe": (_I, [_I, ctypes.c_ulonglong, _P, _P, _P]),
}


class TsdError(RuntimeError):
    pass


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libtsd.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(path):
                raise TsdError(f"{path} not found: build it with "
                               "`python -m tree_speculative_decoding_ancestor_b200.build`")
            lib = ctypes.CDLL(path)
            for name, (res, args) in _SIGNATURES.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _lib = lib
        return _lib


def exported_symbols() -> Tuple[str, ...]:
    return tuple(_SIGNATURES)


def launch_count() -> int:
    """Kernels libtsd has launched in this process."""
    return int(load_library().tsd_launch_count())


def _check(rc: int, what: str) -> None:
    if rc != TSD_OK:
        msg = load_library().tsd_status_string(rc).decode()
        raise TsdError(f"{what} failed: {msg} ({rc})")


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(device: torch.device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _cuda(device: torch.device) -> None:
    """The kernels read and write device memory only: refuse anything else
    before a host address can reach a launch."""
    if device.type != "cuda":
        raise ValueError(f"tensors must be on a CUDA device, got {device}")


def _need(t: torch.Tensor, name: str, dtype: torch.dtype, shape: Tuple[int, ...],
          device: torch.device) -> None:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device != device:
        raise ValueError(f"{name} must be on {device}, got {t.device}")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


# Per-device status word and workspace cache ---------------------------------
_status: Dict[int, torch.Tensor] = {}
# Workspaces the binding allocates when the caller passes none, one per
# (device, kind, stream): calls on one stream run one after another, so they
# can share a buffer; calls on different streams may overlap on the GPU, and
# a workspace must not be shared by calls that may overlap.
_workspace: Dict[Tuple[int, str, int], torch.Tensor] = {}


def device_status(device=None) -> torch.Tensor:
    """The int32 word that the kernels OR their TSD_DEV_* bits into."""
    device = torch.device(device or torch.cuda.current_device())
    idx = device.index if device.index is not None else torch.cuda.current_device()
    if idx not in _status:
        _status[idx] = torch.zeros(1, dtype=torch.int32, device=f"cuda:{idx}")
    return _status[idx]


def _get_workspace(device: torch.device, kind: str, nbytes: int) -> torch.Tensor:
    """The cached workspace of this kind for the caller's current stream on
    `device` (grown when too small; the caching allocator keeps a replaced
    buffer's memory for that stream's later work, so a kernel still running on
    it is not disturbed)."""
    with _lock:
        key = (device.index, kind, int(_stream(device)))
        ws = _workspace.get(key)
        if ws is None or ws.numel() < nbytes:
            ws = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)
            _workspace[key] = ws
        return ws


def _workspace_for(device: torch.device, kind: str, nbytes: int,
                   workspace: Optional[torch.Tensor]) -> torch.Tensor:
    """The caller's workspace (a contiguous uint8 tensor on the device: its
    element count is the byte count the library checks), or the cache's."""
    if workspace is None:
        return _get_workspace(device, kind, nbytes)
    _need(workspace, "workspace", torch.uint8, (workspace.numel(),), device)
    return workspace


def _status_for(device: torch.device, status: Optional[torch.Tensor]) -> torch.Tensor:
    """The caller's status word (an int32 tensor on the device), or the
    per-device one."""
    if status is None:
        return device_status(device)
    if not isinstance(status, torch.Tensor) or status.dtype != torch.int32 or \
            status.device != device or status.numel() < 1:
        raise ValueError(f"status must be an int32 tensor on {device}")
    return status


class TreeMask(NamedTuple):
    mask: torch.Tensor          # [B][Tmax][W] int32 (bit pattern of uint32)
    depth: torch.Tensor         # [B][Tmax] int32
    first_child: torch.Tensor   # [B][Tmax+1] int32
    next_sibling: torch.Tensor  # [B][Tmax] int32


class VerifyResult(NamedTuple):
    out_tokens: torch.Tensor    # [B][Tmax+1] int32
    out_path: torch.Tensor      # [B][Tmax] int32
    n_accepted: torch.Tensor    # [B] int32


def _need_tree(tree: TreeMask, B: int, Tmax: int, device: torch.device, fields) -> None:
    """Check the TreeMask fields a call reads or writes."""
    shapes = {"mask": (B, Tmax, (Tmax + 31) // 32), "depth": (B, Tmax),
              "first_child": (B, Tmax + 1), "next_sibling": (B, Tmax)}
    for f in fields:
        _need(getattr(tree, f), f, torch.int32, shapes[f], device)


def _need_result(out: VerifyResult, B: int, Tmax: int, device: torch.device) -> None:
    _need(out.out_tokens, "out_tokens", torch.int32, (B, Tmax + 1), device)
    _need(out.out_path, "out_path", torch.int32, (B, Tmax), device)
    _need(out.n_accepted, "n_accepted", torch.int32, (B,), device)


def tree_mask_build(parent: torch.Tensor, n_nodes: torch.Tensor,
                    out: Optional[TreeMask] = None, status: Optional[torch.Tensor] = None
                    ) -> TreeMask:
    """Ancestor mask, depth and child lists of each token tree."""
    lib = load_library()
    dev = parent.device
    _cuda(dev)
    B, Tmax = parent.shape
    W = (Tmax + 31) // 32
    _need(parent, "parent", torch.int32, (B, Tmax), dev)
    _need(n_nodes, "n_nodes", torch.int32, (B,), dev)
    if out is None:
        out = TreeMask(torch.empty((B, Tmax, W), dtype=torch.int32, device=dev),
                       torch.empty((B, Tmax), dtype=torch.int32, device=dev),
                       torch.empty((B, Tmax + 1), dtype=torch.int32, device=dev),
                       torch.empty((B, Tmax), dtype=torch.int32, device=dev))
    _need_tree(out, B, Tmax, dev, ("mask", "depth", "first_child", "next_sibling"))
    st = _status_for(dev, status)
    rc = lib.tsd_tree_mask_build(_ptr(parent), _ptr(n_nodes), B, Tmax, _ptr(out.mask),
                                 _ptr(out.depth), _ptr(out.first_child), _ptr(out.next_sibling),
                                 _ptr(st), _stream(dev))
    _check(rc, "tsd_tree_mask_build")
    return out


def attention_workspace_size(B: int, Tmax: int, Hq: int, Hkv: int, D: int, Lmax: int,
                             dtype: torch.dtype) -> int:
    code = TSD_BF16 if dtype == torch.bfloat16 else TSD_F32
    return int(load_library().tsd_tree_attention_workspace_size(B, Tmax, Hq, Hkv, D, Lmax, code))


PLAN_KERNELS = {0: "simt", 1: "rows128", 2: "rows64", 3: "keysplit", 4: "rows128x2"}


def attention_plan(B: int, Tmax: int, Hq: int, Hkv: int, D: int, Lmax: int,
                   dtype: torch.dtype, num_sms: int) -> Dict[str, object]:
    """The kernel and grid tree_attention would use for these sizes on a
    device with num_sms SMs (host only): kernel name, query-row blocks per
    (sequence, KV head), key-range splits, keys per split."""
    code = TSD_BF16 if dtype == torch.bfloat16 else TSD_F32
    plan = (ctypes.c_int32 * 4)()
    rc = load_library().tsd_tree_attention_plan(B, Tmax, Hq, Hkv, D, Lmax, code, num_sms,
                                                ctypes.addressof(plan))
    _check(rc, "tsd_tree_attention_plan")
    return {"kernel": PLAN_KERNELS[plan[0]], "row_blocks": plan[1], "splits": plan[2],
            "keys_per_split": plan[3]}


def tree_attention(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                   prefix_len: torch.Tensor, n_nodes: torch.Tensor, mask: torch.Tensor,
                   scale: Optional[float] = None, out: Optional[torch.Tensor] = None,
                   workspace: Optional[torch.Tensor] = None,
                   status: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Topology-aware tree attention over prefix KV + ancestors (out[B][Tmax][Hq][D])."""
    lib = load_library()
    dev = q.device
    _cuda(dev)
    B, Tmax, Hq, D = q.shape
    Hkv, Lmax = k_cache.shape[1], k_cache.shape[2]
    if q.dtype not in (torch.float32, torch.bfloat16):
        raise TypeError("q/k/v must be float32 or bfloat16")
    _need(q, "q", q.dtype, (B, Tmax, Hq, D), dev)
    _need(k_cache, "k_cache", q.dtype, (B, Hkv, Lmax, D), dev)
    _need(v_cache, "v_cache", q.dtype, (B, Hkv, Lmax, D), dev)
    _need(prefix_len, "prefix_len", torch.int32, (B,), dev)
    _need(n_nodes, "n_nodes", torch.int32, (B,), dev)
    _need(mask, "mask", torch.int32, (B, Tmax, (Tmax + 31) // 32), dev)
    if out is None:
        out = torch.empty_like(q)
    _need(out, "out", q.dtype, (B, Tmax, Hq, D), dev)
    if scale is None:
        scale = D ** -0.5
    code = TSD_BF16 if q.dtype == torch.bfloat16 else TSD_F32
    need = int(lib.tsd_tree_attention_workspace_size(B, Tmax, Hq, Hkv, D, Lmax, code))
    ws = _workspace_for(dev, "attn", need, workspace)
    st = _status_for(dev, status)
    rc = lib.tsd_tree_attention(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(prefix_len),
                                _ptr(n_nodes), _ptr(mask), B, Tmax, Hq, Hkv, D, Lmax,
                                float(scale), code, _ptr(out), _ptr(ws), ws.numel(), _ptr(st),
                                _stream(dev))
    _check(rc, "tsd_tree_attention")
    return out


def verify_workspace_size(B: int, Tmax: int, V: int) -> int:
    return int(load_library().tsd_tree_verify_workspace_size(B, Tmax, V))


def _verify_outputs(B, Tmax, dev, out):
    if out is None:
        out = VerifyResult(torch.empty((B, Tmax + 1), dtype=torch.int32, device=dev),
                           torch.empty((B, Tmax), dtype=torch.int32, device=dev),
                           torch.empty((B,), dtype=torch.int32, device=dev))
    return out


def tree_verify_greedy(logits: torch.Tensor, tokens: torch.Tensor, parent: torch.Tensor,
                       n_nodes: torch.Tensor, tree: TreeMask,
                       out: Optional[VerifyResult] = None,
                       workspace: Optional[torch.Tensor] = None,
                       status: Optional[torch.Tensor] = None) -> VerifyResult:
    """Longest root path matching the target argmax, plus one bonus token."""
    lib = load_library()
    dev = logits.device
    _cuda(dev)
    B, R, V = logits.shape
    Tmax = R - 1
    _need(logits, "logits", torch.float32, (B, Tmax + 1, V), dev)
    _need(tokens, "tokens", torch.int32, (B, Tmax), dev)
    _need(parent, "parent", torch.int32, (B, Tmax), dev)
    _need(n_nodes, "n_nodes", torch.int32, (B,), dev)
    _need_tree(tree, B, Tmax, dev, ("mask", "first_child"))
    out = _verify_outputs(B, Tmax, dev, out)
    _need_result(out, B, Tmax, dev)
    need = int(lib.tsd_tree_verify_workspace_size(B, Tmax, V))
    ws = _workspace_for(dev, "verify", need, workspace)
    st = _status_for(dev, status)
    rc = lib.tsd_tree_verify_greedy(_ptr(logits), _ptr(tokens), _ptr(parent), _ptr(n_nodes),
                                    _ptr(tree.mask), _ptr(tree.first_child), B, Tmax, V,
                                    _ptr(out.out_tokens), _ptr(out.out_path),
                                    _ptr(out.n_accepted), _ptr(ws), ws.numel(), _ptr(st),
                                    _stream(dev))
    _check(rc, "tsd_tree_verify_greedy")
    return out


def tree_verify_stochastic(logits: torch.Tensor, temperature: float, q_probs: torch.Tensor,
                           q_row: torch.Tensor, tokens: torch.Tensor, n_nodes: torch.Tensor,
                           tree: TreeMask, u_accept: torch.Tensor, u_sample: torch.Tensor,
                           out: Optional[VerifyResult] = None,
                           workspace: Optional[torch.Tensor] = None,
                           status: Optional[torch.Tensor] = None) -> VerifyResult:
    """Multi-step speculative sampling over the tree (exact target distribution)."""
    lib = load_library()
    dev = logits.device
    _cuda(dev)
    B, R, V = logits.shape
    Tmax = R - 1
    Rq = q_probs.shape[1]
    _need(logits, "logits", torch.float32, (B, Tmax + 1, V), dev)
    _need(q_probs, "q_probs", torch.float32, (B, Rq, V), dev)
    _need(q_row, "q_row", torch.int32, (B, Tmax), dev)
    _need(tokens, "tokens", torch.int32, (B, Tmax), dev)
    _need(n_nodes, "n_nodes", torch.int32, (B,), dev)
    _need(u_accept, "u_accept", torch.float64, (B, Tmax), dev)
    _need(u_sample, "u_sample", torch.float64, (B, Tmax + 1), dev)
    _need_tree(tree, B, Tmax, dev, ("first_child", "next_sibling"))
    out = _verify_outputs(B, Tmax, dev, out)
    _need_result(out, B, Tmax, dev)
    need = int(lib.tsd_tree_verify_workspace_size(B, Tmax, V))
    ws = _workspace_for(dev, "verify", need, workspace)
    st = _status_for(dev, status)
    rc = lib.tsd_tree_verify_stochastic(_ptr(logits), float(temperature), _ptr(q_probs), Rq,
                                        _ptr(q_row), _ptr(tokens), _ptr(n_nodes),
                                        _ptr(tree.first_child), _ptr(tree.next_sibling),
                                        _ptr(u_accept), _ptr(u_sample), B, Tmax, V,
                                        _ptr(out.out_tokens), _ptr(out.out_path),
                                        _ptr(out.n_accepted), _ptr(ws), ws.numel(), _ptr(st),
                                        _stream(dev))
    _check(rc, "tsd_tree_verify_stochastic")
    return out


def verify_stochastic_plan(B: int, Tmax: int, V: int) -> Dict[str, int]:
    """The grid tree_verify_stochastic launches for these sizes on the current
    device (host only): teams walking at once, CTAs per team, vocabulary
    entries per CTA, CTAs in the launch."""
    plan = (ctypes.c_int32 * 4)()
    rc = load_library().tsd_tree_verify_stochastic_plan(B, Tmax, V, ctypes.addressof(plan))
    _check(rc, "tsd_tree_verify_stochastic_plan")
    return {"teams": plan[0], "ctas_per_team": plan[1], "chunk": plan[2], "ctas": plan[3]}


GREEDY_FORMS = {0: "walk", 1: "rows"}


def verify_greedy_plan(B: int, Tmax: int, V: int) -> Dict[str, str]:
    """The form tree_verify_greedy takes for these sizes (host only): "walk"
    (one CTA per sequence over the matched nodes) or "rows" (the argmax of
    every row with children, then the path)."""
    form = ctypes.c_int32(-1)
    rc = load_library().tsd_tree_verify_greedy_plan(B, Tmax, V, ctypes.addressof(form))
    _check(rc, "tsd_tree_verify_greedy_plan")
    return {"form": GREEDY_FORMS[form.value]}


def tree_verify_stochastic_noalloc(logits: torch.Tensor, temperature: float,
                                   q_probs: torch.Tensor, q_row: torch.Tensor,
                                   tokens: torch.Tensor, n_nodes: torch.Tensor, tree: TreeMask,
                                   u_accept: torch.Tensor, u_sample: torch.Tensor,
                                   out: VerifyResult, status: Optional[torch.Tensor] = None
                                   ) -> VerifyResult:
    """tree_verify_stochastic for callers that cannot allocate device memory:
    the scratch lives in a fixed array inside the library, so the caller
    passes preallocated outputs and nothing is allocated here (see
    tsd_tree_verify_stochastic_noalloc in include/tsd.h for the fixed
    scratch, the first-call set-up and why overlapping calls race)."""
    lib = load_library()
    dev = logits.device
    _cuda(dev)
    B, R, V = logits.shape
    Tmax = R - 1
    Rq = q_probs.shape[1]
    _need(logits, "logits", torch.float32, (B, Tmax + 1, V), dev)
    _need(q_probs, "q_probs", torch.float32, (B, Rq, V), dev)
    _need(q_row, "q_row", torch.int32, (B, Tmax), dev)
    _need(tokens, "tokens", torch.int32, (B, Tmax), dev)
    _need(n_nodes, "n_nodes", torch.int32, (B,), dev)
    _need(u_accept, "u_accept", torch.float64, (B, Tmax), dev)
    _need(u_sample, "u_sample", torch.float64, (B, Tmax + 1), dev)
    _need_tree(tree, B, Tmax, dev, ("first_child", "next_sibling"))
    _need_result(out, B, Tmax, dev)
    st = _status_for(dev, status)
    rc = lib.tsd_tree_verify_stochastic_noalloc(
        _ptr(logits), float(temperature), _ptr(q_probs), Rq, _ptr(q_row), _ptr(tokens),
        _ptr(n_nodes), _ptr(tree.first_child), _ptr(tree.next_sibling), _ptr(u_accept),
        _ptr(u_sample), B, Tmax, V, _ptr(out.out_tokens), _ptr(out.out_path),
        _ptr(out.n_accepted), _ptr(st), _stream(dev))
    _check(rc, "tsd_tree_verify_stochastic_noalloc")
    return out


def kv_commit(k_cache: torch.Tensor, v_cache: torch.Tensor, prefix_len: torch.Tensor,
              result: VerifyResult, new_prefix_len: Optional[torch.Tensor] = None,
              status: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Move the accepted nodes' K/V rows (in place) to the positions right
    after each sequence's prefix; returns the new prefix lengths [B] int32."""
    lib = load_library()
    dev = k_cache.device
    _cuda(dev)
    B, Hkv, Lmax, D = k_cache.shape
    Tmax = result.out_path.shape[1]
    dt = {torch.float32: TSD_F32, torch.bfloat16: TSD_BF16}.get(k_cache.dtype)
    if dt is None:
        raise TypeError("k_cache must be float32 or bfloat16")
    _need(k_cache, "k_cache", k_cache.dtype, (B, Hkv, Lmax, D), dev)
    _need(v_cache, "v_cache", k_cache.dtype, (B, Hkv, Lmax, D), dev)
    _need(prefix_len, "prefix_len", torch.int32, (B,), dev)
    _need(result.out_path, "out_path", torch.int32, (B, Tmax), dev)
    _need(result.n_accepted, "n_accepted", torch.int32, (B,), dev)
    if new_prefix_len is None:
        new_prefix_len = torch.empty((B,), dtype=torch.int32, device=dev)
    _need(new_prefix_len, "new_prefix_len", torch.int32, (B,), dev)
    st = _status_for(dev, status)
    rc = lib.tsd_kv_commit(_ptr(k_cache), _ptr(v_cache), _ptr(prefix_len), _ptr(result.out_path),
                           _ptr(result.n_accepted), B, Tmax, Hkv, D, Lmax, dt,
                           _ptr(new_prefix_len), _ptr(st), _stream(dev))
    _check(rc, "tsd_kv_commit")
    return new_prefix_len


def tree_attention_paged(q: torch.Tensor, k_pages: torch.Tensor, v_pages: torch.Tensor,
                         block_table: torch.Tensor, prefix_len: torch.Tensor,
                         n_nodes: torch.Tensor, mask: torch.Tensor,
                         scale: Optional[float] = None, out: Optional[torch.Tensor] = None,
                         workspace: Optional[torch.Tensor] = None,
                         status: Optional[torch.Tensor] = None) -> torch.Tensor:
    """tree_attention over a paged KV cache: pools [num_pages][Hkv][page_size][D]
    and a block table [B][max_blocks] of physical page ids."""
    lib = load_library()
    dev = q.device
    _cuda(dev)
    B, Tmax, Hq, D = q.shape
    num_pages, Hkv, page_size, _ = k_pages.shape
    max_blocks = block_table.shape[1]
    dt = {torch.float32: TSD_F32, torch.bfloat16: TSD_BF16}.get(q.dtype)
    if dt is None:
        raise TypeError("q must be float32 or bfloat16")
    _need(q, "q", q.dtype, (B, Tmax, Hq, D), dev)
    _need(k_pages, "k_pages", q.dtype, (num_pages, Hkv, page_size, D), dev)
    _need(v_pages, "v_pages", q.dtype, (num_pages, Hkv, page_size, D), dev)
    _need(block_table, "block_table", torch.int32, (B, max_blocks), dev)
    _need(prefix_len, "prefix_len", torch.int32, (B,), dev)
    _need(n_nodes, "n_nodes", torch.int32, (B,), dev)
    _need(mask, "mask", torch.int32, (B, Tmax, (Tmax + 31) // 32), dev)
    if out is None:
        out = torch.empty_like(q)
    _need(out, "out", q.dtype, (B, Tmax, Hq, D), dev)
    Lmax = max_blocks * page_size
    need = int(lib.tsd_tree_attention_workspace_size(B, Tmax, Hq, Hkv, D, Lmax, dt))
    ws = _workspace_for(dev, "attn", need, workspace)
    st = _status_for(dev, status)
    sc = (1.0 / D ** 0.5) if scale is None else float(scale)
    rc = lib.tsd_tree_attention_paged(_ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(block_table),
                                      num_pages, page_size, max_blocks, _ptr(prefix_len),
                                      _ptr(n_nodes), _ptr(mask), B, Tmax, Hq, Hkv, D, sc, dt,
                                      _ptr(out), _ptr(ws), ws.numel(), _ptr(st), _stream(dev))
    _check(rc, "tsd_tree_attention_paged")
    return out


class Tree(NamedTuple):
    parent: torch.Tensor     # [B][Tmax] int32
    tokens: torch.Tensor     # [B][Tmax] int32
    q_row: torch.Tensor      # [B][Tmax] int32
    n_nodes: torch.Tensor    # [B] int32


def tree_expand(q_probs: torch.Tensor, frow: torch.Tensor, k: int, tree: Tree,
                lvl_begin: torch.Tensor, status: Optional[torch.Tensor] = None) -> Tree:
    """Add one expansion level in place (the k most probable tokens of each
    frontier node's SSM row become its children)."""
    lib = load_library()
    dev = q_probs.device
    _cuda(dev)
    B, Rq, V = q_probs.shape
    Tmax = tree.parent.shape[1]
    _need(q_probs, "q_probs", torch.float32, (B, Rq, V), dev)
    _need(frow, "frow", torch.int32, (B, Tmax), dev)
    for name in ("parent", "tokens", "q_row"):
        _need(getattr(tree, name), name, torch.int32, (B, Tmax), dev)
    _need(tree.n_nodes, "n_nodes", torch.int32, (B,), dev)
    _need(lvl_begin, "lvl_begin", torch.int32, (B,), dev)
    st = _status_for(dev, status)
    rc = lib.tsd_tree_expand(_ptr(q_probs), Rq, V, _ptr(frow), int(k), _ptr(tree.parent),
                             _ptr(tree.tokens), _ptr(tree.q_row), _ptr(tree.n_nodes),
                             _ptr(lvl_begin), B, Tmax, _ptr(st), _stream(dev))
    _check(rc, "tsd_tree_expand")
    return tree


def tree_dfs_order(tree: Tree, status: Optional[torch.Tensor] = None):
    """Depth-first renumbering: returns (perm [B][Tmax], renumbered Tree)."""
    lib = load_library()
    dev = tree.parent.device
    _cuda(dev)
    B, Tmax = tree.parent.shape
    for name in ("parent", "tokens", "q_row"):
        _need(getattr(tree, name), name, torch.int32, (B, Tmax), dev)
    _need(tree.n_nodes, "n_nodes", torch.int32, (B,), dev)
    perm = torch.full((B, Tmax), -1, dtype=torch.int32, device=dev)
    out = Tree(torch.full_like(tree.parent, -1), torch.zeros_like(tree.tokens),
               torch.zeros_like(tree.q_row), tree.n_nodes.clone())
    st = _status_for(dev, status)
    rc = lib.tsd_tree_dfs_order(_ptr(tree.parent), _ptr(tree.tokens), _ptr(tree.q_row),
                                _ptr(tree.n_nodes), B, Tmax, _ptr(perm), _ptr(out.parent),
                                _ptr(out.tokens), _ptr(out.q_row), _ptr(st), _stream(dev))
    _check(rc, "tsd_tree_dfs_order")
    return perm, out


def tree_merge_chains(chain_tokens: torch.Tensor, chain_q_row: torch.Tensor,
                      chain_len: torch.Tensor, Tmax: int,
                      status: Optional[torch.Tensor] = None) -> Tree:
    """Merge M draft chains per sequence into one token tree (depth-first)."""
    lib = load_library()
    dev = chain_tokens.device
    _cuda(dev)
    B, M, L = chain_tokens.shape
    _need(chain_tokens, "chain_tokens", torch.int32, (B, M, L), dev)
    _need(chain_q_row, "chain_q_row", torch.int32, (B, M, L), dev)
    _need(chain_len, "chain_len", torch.int32, (B, M), dev)
    out = Tree(torch.full((B, Tmax), -1, dtype=torch.int32, device=dev),
               torch.zeros((B, Tmax), dtype=torch.int32, device=dev),
               torch.zeros((B, Tmax), dtype=torch.int32, device=dev),
               torch.zeros((B,), dtype=torch.int32, device=dev))
    st = _status_for(dev, status)
    rc = lib.tsd_tree_merge_chains(_ptr(chain_tokens), _ptr(chain_q_row), _ptr(chain_len), M, L,
                                   B, Tmax, _ptr(out.parent), _ptr(out.tokens), _ptr(out.q_row),
                                   _ptr(out.n_nodes), _ptr(st), _stream(dev))
    _check(rc, "tsd_tree_merge_chains")
    return out


def debug_wait_probe(kind: int, limit_ns: int = 50_000_000, device=None,
                     status: Optional[torch.Tensor] = None) -> None:
    """Run the kernels' bounded wait routines on something that never completes
    (kind 0: mbarrier wait; kind 1: team barrier; kind 2: cluster exchange);
    they must end after about limit_ns with DEV_TIMEOUT set in the status
    word."""
    lib = load_library()
    dev = torch.device(device or torch.cuda.current_device())
    _cuda(dev)
    if dev.index is None:
        dev = torch.device("cuda", torch.cuda.current_device())
    scratch = torch.zeros(2, dtype=torch.int32, device=dev)
    st = _status_for(dev, status)
    rc = lib.tsd_debug_wait_probe(int(kind), int(limit_ns), _ptr(scratch), _ptr(st), _stream(dev))
    _check(rc, "tsd_debug_wait_probe")
