"""Synthetic workloads shaped like the settings on the SpecInfer explainer page.

Source: "論文解説: SpecInfer - 投機的推論とトークンツリー検証によるLLMサービング高速化"
(0h-n0.github.io/posts/paper-2305-09781), sections "トークンツリー構造の仕組み"
(token tree, S_u), "マルチドラフトモデルアプローチ" (expansion <k1..kn> and
merge-based trees, with the example <1,1,3,1,1,1,1,1> and the merge diagram)
and "ツリー検証アルゴリズム" (SSM / LLM distributions).

Conventions shared by every consumer:

* A tree has ``n_nodes[b] = T_b <= Tmax`` nodes.  Node ``u`` has parent
  ``parent[b][u]`` in ``[-1, u-1]``; ``-1`` means "child of the root".  The
  root is the last committed token: it lives in the prefix, it is not a
  tree node, and its target logits are row 0.  Node ``u`` owns logits row
  ``1 + u``.  Generated trees are numbered in depth-first pre-order (the
  KV-cache order described in "Tree Attention のカーネル融合", item 2).
* Query ``q[b][u][h][:]`` belongs to node ``u``; the KV cache is
  ``[B][Hkv][Lmax][D]`` with the committed prefix at positions
  ``0 .. P_b-1`` and tree node ``u`` at position ``P_b + u``.
* ``q_probs[b][r][:]`` is the distribution an SSM proposed from (one row per
  (parent, SSM) pair); ``q_row[b][u]`` names the row that proposed node u.
* Uniforms are fp64 in the open interval (0, 1), from SplitMix64:
  ``u_accept[b][u]`` for the acceptance test of child ``u``, ``u_sample[b][r]``
  for a draw at logits row ``r``.  The layout does not depend on the path
  taken, so every implementation consumes identical numbers.

Everything is seeded; the same (config, seed) always yields the same bytes.
"""

from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np
import torch

# ---------------------------------------------------------------------------
# SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom number
# generators", OOPSLA 2014; constants as published in Vigna's reference
# implementation).  Counter-based: output i is mix(key + (i + 1) * gamma).
# ---------------------------------------------------------------------------
_GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)


def _splitmix64(key: int, n: int) -> np.ndarray:
    i = np.arange(1, n + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = np.uint64(key & 0xFFFFFFFFFFFFFFFF) + i * _GAMMA
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
        z = z ^ (z >> np.uint64(31))
    return z


def splitmix64_uniforms(key: int, n: int) -> np.ndarray:
    """n doubles in (0, 1): ((z >> 11) + 0.5) * 2^-53 (never 0, never 1)."""
    z = _splitmix64(key, n) >> np.uint64(11)
    return (z.astype(np.float64) + 0.5) * (2.0 ** -53)


# ---------------------------------------------------------------------------
# Tree shapes.  Each builder returns (parent, ssm) in *creation* order, where
# parent[u] < u, and ssm[u] names the speculative model that proposed u.
# dfs_relabel() turns that into depth-first pre-order.
# ---------------------------------------------------------------------------

def tree_expansion(ks: Sequence[int]) -> Tuple[List[int], List[int]]:
    """Expansion-based tree <k1, ..., kn>: every node at depth i-1 gets k_i
    children (the root is depth 0).  <1,1,3,1,1,1,1,1> gives 20 nodes."""
    parent: List[int] = []
    frontier = [-1]
    for k in ks:
        nxt = []
        for p in frontier:
            for _ in range(k):
                parent.append(p)
                nxt.append(len(parent) - 1)
        frontier = nxt
    return parent, [0] * len(parent)


def tree_levels(level_sizes: Sequence[int], level_k: Sequence[int],
                rng: np.random.Generator) -> Tuple[List[int], List[int]]:
    """Expansion truncated per level: level i has level_sizes[i] nodes, made
    by expanding a seeded subset of level i-1 with level_k[i] children each."""
    parent: List[int] = []
    frontier = [-1]
    for size, k in zip(level_sizes, level_k):
        assert size % k == 0, "level size must be a multiple of its branching"
        n_par = size // k
        assert n_par <= len(frontier), "not enough parents on the previous level"
        chosen = sorted(rng.choice(len(frontier), size=n_par, replace=False).tolist())
        nxt = []
        for ci in chosen:
            for _ in range(k):
                parent.append(frontier[ci])
                nxt.append(len(parent) - 1)
        frontier = nxt
    return parent, [0] * len(parent)


def tree_random(n: int, max_depth: int, max_children: int,
                rng: np.random.Generator) -> Tuple[List[int], List[int]]:
    """n nodes added one at a time; each picks a uniform parent among the
    root and the nodes of depth < max_depth that have < max_children
    children."""
    parent: List[int] = []
    depth: List[int] = []
    nchild: Dict[int, int] = {-1: 0}
    for _ in range(n):
        cands = [-1] if nchild[-1] < max_children else []
        cands += [v for v in range(len(parent))
                  if depth[v] < max_depth and nchild[v] < max_children]
        if not cands:
            raise ValueError("tree_random: depth/branching limits admit fewer than n nodes")
        p = cands[int(rng.integers(len(cands)))]
        parent.append(p)
        depth.append(1 if p < 0 else depth[p] + 1)
        nchild[p] += 1
        nchild[len(parent) - 1] = 0
    return parent, [0] * len(parent)


def tree_merge_chains(n_chains: int, depth: int, max_shared: int,
                      rng: np.random.Generator) -> Tuple[List[int], List[int], List[int]]:
    """Merge-based tree: chain 0 is a full chain; every other chain shares a
    random prefix of 0..max_shared tokens with chain 0 and then branches off
    with its own nodes.  Returns (parent, ssm, shared) where shared[j] is the
    number of chain-0 nodes chain j re-uses."""
    parent: List[int] = []
    ssm: List[int] = []
    chain0: List[int] = []
    prev = -1
    for _ in range(depth):
        parent.append(prev)
        ssm.append(0)
        prev = len(parent) - 1
        chain0.append(prev)
    shared = [depth]
    for j in range(1, n_chains):
        s = int(rng.integers(0, max_shared + 1))
        shared.append(s)
        prev = -1 if s == 0 else chain0[s - 1]
        for _ in range(depth - s):
            parent.append(prev)
            ssm.append(j)
            prev = len(parent) - 1
    return parent, ssm, shared


def dfs_relabel(parent: Sequence[int]) -> List[int]:
    """Return perm with perm[new] = old, listing nodes in depth-first
    pre-order (children visited in creation order)."""
    n = len(parent)
    children: Dict[int, List[int]] = {-1: []}
    for u in range(n):
        children.setdefault(u, [])
        children[parent[u]].append(u)
    order: List[int] = []
    stack = list(reversed(children[-1]))
    while stack:
        u = stack.pop()
        order.append(u)
        stack.extend(reversed(children[u]))
    assert len(order) == n
    return order


def _apply_perm(parent: Sequence[int], extra: Sequence[Sequence[int]], perm: List[int]):
    inv = {old: new for new, old in enumerate(perm)}
    inv[-1] = -1
    new_parent = [inv[parent[old]] for old in perm]
    new_extra = [[e[old] for old in perm] for e in extra]
    return new_parent, new_extra


# ---------------------------------------------------------------------------
# Workload container
# ---------------------------------------------------------------------------

@dataclasses.dataclass
class Workload:
    name: str
    B: int
    Tmax: int
    Hq: int
    Hkv: int
    D: int
    Lmax: int
    V: int
    dtype: str                   # "f32" or "bf16" for Q / K / V
    scale: float
    temperature: float
    parent: torch.Tensor         # int32 [B][Tmax]
    n_nodes: torch.Tensor        # int32 [B]
    prefix_len: torch.Tensor     # int32 [B]
    tokens: torch.Tensor         # int32 [B][Tmax]
    q_row: torch.Tensor          # int32 [B][Tmax]
    Rq: int
    q: torch.Tensor              # [B][Tmax][Hq][D]
    k_cache: torch.Tensor        # [B][Hkv][Lmax][D]
    v_cache: torch.Tensor        # [B][Hkv][Lmax][D]
    logits: torch.Tensor         # float32 [B][Tmax+1][V]
    q_probs: torch.Tensor        # float32 [B][Rq][V]
    u_accept: torch.Tensor       # float64 [B][Tmax]
    u_sample: torch.Tensor       # float64 [B][Tmax+1]
    verify: Tuple[str, ...]
    seed: int

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    def total_nodes(self) -> int:
        return int(self.n_nodes.sum())

    def kv_bytes(self) -> int:
        """K+V bytes of the prefix and tree positions actually attended."""
        es = 4 if self.dtype == "f32" else 2
        pos = (self.prefix_len.to(torch.int64) + self.n_nodes.to(torch.int64)).sum().item()
        return int(2 * pos * self.Hkv * self.D * es)


_TORCH_DT = {"f32": torch.float32, "bf16": torch.bfloat16}


def _normal(rng: np.random.Generator, shape, sigma: float = 1.0) -> np.ndarray:
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if sigma != 1.0:
        x *= np.float32(sigma)
    return x


def _softmax64(x: np.ndarray) -> np.ndarray:
    # Input generation only: the SSM's proposal distribution.
    x = x.astype(np.float64)
    x = x - x.max(axis=-1, keepdims=True)
    e = np.exp(x)
    return e / e.sum(axis=-1, keepdims=True)


def _assemble(name: str, seed: int, B: int, Tmax: int, Hq: int, Hkv: int, D: int,
              prefix: np.ndarray, V: int, dtype: str,
              trees: List[Tuple[List[int], List[int]]],
              token_mode: str, q_sigma: float, verify: Tuple[str, ...],
              temperature: float = 1.0, logit_sigma: float = 2.0,
              with_attention: bool = True, lmax_pad: int = 0,
              merge_shared: Optional[List[List[int]]] = None) -> Workload:
    rng = np.random.default_rng(seed)
    parent = np.full((B, Tmax), -1, dtype=np.int32)
    n_nodes = np.zeros(B, dtype=np.int32)
    q_row = np.zeros((B, Tmax), dtype=np.int32)
    tokens = np.zeros((B, Tmax), dtype=np.int32)
    row_keys: List[Dict[Tuple[int, int], int]] = []
    for b, (par, ssm) in enumerate(trees):
        T = len(par)
        assert T <= Tmax
        n_nodes[b] = T
        parent[b, :T] = par
        keys: Dict[Tuple[int, int], int] = {}
        for u in range(T):
            key = (par[u], ssm[u])
            if key not in keys:
                keys[key] = len(keys)
            q_row[b, u] = keys[key]
        row_keys.append(keys)
    Rq = max(1, max(len(k) for k in row_keys))

    # Target logits ~ N(0, logit_sigma^2); rows beyond 1+T_b stay zero.
    logits = np.zeros((B, Tmax + 1, V), dtype=np.float32)
    for b in range(B):
        T = int(n_nodes[b])
        logits[b, :T + 1] = _normal(rng, (T + 1, V), logit_sigma)

    # SSM distributions: softmax(target logits of the parent row + noise).
    q_probs = np.zeros((B, Rq, V), dtype=np.float32)
    for b in range(B):
        for (p, _s), r in row_keys[b].items():
            noisy = logits[b, p + 1].astype(np.float64) + q_sigma * rng.standard_normal(V)
            q_probs[b, r] = _softmax64(noisy[None, :])[0].astype(np.float32)

    # Speculated tokens.
    for b in range(B):
        T = int(n_nodes[b])
        par = parent[b, :T]
        if token_mode == "topk":
            # Siblings proposed from one row take that row's top-k in order.
            used: Dict[int, int] = {}
            for u in range(T):
                r = int(q_row[b, u])
                if r not in used:
                    used[r] = 0
                    order = np.lexsort((np.arange(V), -q_probs[b, r].astype(np.float64)))
                    row_keys[b][("order", r)] = order  # type: ignore[index]
                order = row_keys[b][("order", r)]  # type: ignore[index]
                tokens[b, u] = int(order[used[r]])
                used[r] += 1
        elif token_mode == "sample":
            # Independent draws from the proposing row (duplicates allowed).
            for u in range(T):
                pr = q_probs[b, int(q_row[b, u])].astype(np.float64)
                pr = pr / pr.sum()
                tokens[b, u] = int(rng.choice(V, p=pr))
        elif token_mode in ("chains", "distinct"):
            # Merge trees: every chain samples its own tokens; a node where a
            # chain branches off must differ from its existing siblings.
            # Other trees ("distinct"): every child is drawn from its row,
            # again distinct from the siblings drawn before it.
            for u in range(T):
                pr = q_probs[b, int(q_row[b, u])].astype(np.float64)
                pr = pr / pr.sum()
                sib = {int(tokens[b, v]) for v in range(u) if par[v] == par[u]}
                while True:
                    t = int(rng.choice(V, p=pr))
                    if t not in sib:
                        break
                tokens[b, u] = t
        else:
            raise ValueError(token_mode)

    Lmax = int(prefix.max()) + Tmax + lmax_pad
    tdt = _TORCH_DT[dtype]
    if with_attention:
        q = torch.zeros((B, Tmax, Hq, D), dtype=tdt)
        k_cache = torch.zeros((B, Hkv, Lmax, D), dtype=tdt)
        v_cache = torch.zeros((B, Hkv, Lmax, D), dtype=tdt)
        for b in range(B):
            T = int(n_nodes[b])
            L = int(prefix[b]) + T
            q[b, :T] = torch.from_numpy(_normal(rng, (T, Hq, D))).to(tdt)
            k_cache[b, :, :L] = torch.from_numpy(_normal(rng, (Hkv, L, D))).to(tdt)
            v_cache[b, :, :L] = torch.from_numpy(_normal(rng, (Hkv, L, D))).to(tdt)
    else:
        q = torch.zeros((0,), dtype=tdt)
        k_cache = torch.zeros((0,), dtype=tdt)
        v_cache = torch.zeros((0,), dtype=tdt)

    u_accept = splitmix64_uniforms(2 * seed + 1, B * Tmax).reshape(B, Tmax)
    u_sample = splitmix64_uniforms(2 * seed + 2, B * (Tmax + 1)).reshape(B, Tmax + 1)

    return Workload(
        name=name, B=B, Tmax=Tmax, Hq=Hq, Hkv=Hkv, D=D, Lmax=Lmax, V=V, dtype=dtype,
        scale=1.0 / math.sqrt(D), temperature=temperature,
        parent=torch.from_numpy(parent), n_nodes=torch.from_numpy(n_nodes),
        prefix_len=torch.from_numpy(prefix.astype(np.int32)),
        tokens=torch.from_numpy(tokens), q_row=torch.from_numpy(q_row), Rq=Rq,
        q=q, k_cache=k_cache, v_cache=v_cache,
        logits=torch.from_numpy(logits), q_probs=torch.from_numpy(q_probs),
        u_accept=torch.from_numpy(u_accept), u_sample=torch.from_numpy(u_sample),
        verify=verify, seed=seed,
    )


# ---------------------------------------------------------------------------
# The five configurations (sizes of the target workloads).
# ---------------------------------------------------------------------------

CONFIGS: Dict[int, Dict] = {
    0: dict(name="tiny: B1 MHA4 D64 P64 fp32, tree <2,2>, V32",
            B=1, Hq=4, Hkv=4, D=64, P=64, dtype="f32", V=32, Tmax=6,
            verify=("greedy", "stochastic")),
    1: dict(name="llama7b-layer: B8 MHA32 D128 P1024 bf16, tree <1,1,3,1,1,1,1,1>, V32000",
            B=8, Hq=32, Hkv=32, D=128, P=1024, dtype="bf16", V=32000, Tmax=20,
            verify=("greedy",)),
    2: dict(name="merge-tree: B16 MHA32 D128 P2048 bf16, 3 chains depth 8 merged, V32000",
            B=16, Hq=32, Hkv=32, D=128, P=2048, dtype="bf16", V=32000, Tmax=24,
            verify=("stochastic",)),
    3: dict(name="70b-gqa: B32 Hq64/Hkv8 D128 P4096 bf16, random 64-node trees, V32000",
            B=32, Hq=64, Hkv=8, D=128, P=4096, dtype="bf16", V=32000, Tmax=64,
            verify=("greedy", "stochastic")),
    4: dict(name="long-context: B4 Hq32/Hkv8 D128 P32768 bf16, 128-node tree, V128256",
            B=4, Hq=32, Hkv=8, D=128, P=32768, dtype="bf16", V=128256, Tmax=128,
            verify=("stochastic",)),
}

SEED_BASE = 20261202

# Short names of the five workloads.
WORKLOAD_NAMES = {"tiny": 0, "llama7b": 1, "merge": 2, "gqa70b": 3, "long32k": 4}


# How the speculated tokens of the 70B-GQA and long-context workloads are
# proposed: "sampled" (the default) follows their stated recipe -- SSM rows
# softmax(target logits + N(0, 1)), each child's token drawn from its row,
# siblings distinct; "topk" is the alternative reading kept for comparison
# (the rows' top-k tokens at noise N(0, 0.3^2)), under which greedy
# acceptance is not near zero.
PROPOSALS = ("sampled", "topk")


def config_workload(index: int, seed: Optional[int] = None, B: Optional[int] = None,
                    with_attention: bool = True, proposal: str = "sampled") -> Workload:
    """Build configuration ``index`` (0..4).  ``B`` may shrink the batch (the
    per-sequence recipe is unchanged); ``proposal`` (one of PROPOSALS) picks
    how configurations 3 and 4 choose their tokens."""
    if proposal not in PROPOSALS:
        raise ValueError(proposal)
    c = CONFIGS[index]
    seed = SEED_BASE + index if seed is None else seed
    Bn = c["B"] if B is None else B
    rng = np.random.default_rng(seed ^ 0x5EED)
    trees: List[Tuple[List[int], List[int]]] = []
    # SSM perturbation and tokens, as each workload states them: the tiny
    # case N(0,1) with i.i.d. draws, the merge case N(0,0.5^2) with chain
    # draws, the 70B-GQA and long-context cases N(0,1) with draws (distinct
    # siblings).  The LLaMA-7B case says only "top-k tokens of a perturbed
    # target softmax": sigma = 0.3, so that greedy acceptance is not
    # trivially zero.
    token_mode, q_sigma = "topk", 0.3
    if index in (3, 4) and proposal == "sampled":
        token_mode, q_sigma = "distinct", 1.0
    for _b in range(Bn):
        if index == 0:
            # Kept in the breadth-first numbering the workload states:
            # parent = [-1, -1, 0, 0, 1, 1].
            par, ssm = tree_expansion((2, 2))
            token_mode, q_sigma = "sample", 1.0
            trees.append((par, ssm))
            continue
        elif index == 1:
            par, ssm = tree_expansion((1, 1, 3, 1, 1, 1, 1, 1))
        elif index == 2:
            par, ssm, _sh = tree_merge_chains(3, 8, 4, rng)
            token_mode, q_sigma = "chains", 0.5
        elif index == 3:
            par, ssm = tree_random(64, 8, 5, rng)
        elif index == 4:
            par, ssm = tree_levels((5, 25, 34, 32, 20, 12), (5, 5, 2, 2, 2, 2), rng)
        else:
            raise ValueError(index)
        perm = dfs_relabel(par)
        par, (ssm,) = _apply_perm(par, [ssm], perm)
        trees.append((par, ssm))
    prefix = np.full(Bn, c["P"], dtype=np.int64)
    return _assemble(c["name"], seed, Bn, c["Tmax"], c["Hq"], c["Hkv"], c["D"], prefix,
                     c["V"], c["dtype"], trees, token_mode, q_sigma, c["verify"],
                     with_attention=with_attention)


def random_workload(seed: int, B: int = 3, Tmax: int = 24, Hq: int = 4, Hkv: int = 2,
                    D: int = 64, P_max: int = 200, V: int = 64, dtype: str = "bf16",
                    ragged: bool = True, min_nodes: int = 1, max_children: int = 4,
                    max_depth: int = 8, token_mode: str = "sample", q_sigma: float = 1.0,
                    temperature: float = 1.0, P_min: int = 0, lmax_pad: int = 0,
                    dfs: bool = True, with_attention: bool = True) -> Workload:
    """Small random workload with ragged tree sizes and prefix lengths."""
    rng = np.random.default_rng(seed)
    trees = []
    for _b in range(B):
        T = int(rng.integers(min_nodes, Tmax + 1)) if ragged else Tmax
        par, ssm = tree_random(T, max_depth, max_children, rng)
        if dfs:
            perm = dfs_relabel(par)
            par, (ssm,) = _apply_perm(par, [ssm], perm)
        trees.append((par, ssm))
    if ragged:
        prefix = rng.integers(P_min, P_max + 1, size=B)
    else:
        prefix = np.full(B, P_max, dtype=np.int64)
    return _assemble(f"random-{seed}", seed, B, Tmax, Hq, Hkv, D, prefix, V, dtype, trees,
                     token_mode, q_sigma, ("greedy", "stochastic"), temperature=temperature,
                     with_attention=with_attention, lmax_pad=lmax_pad)
