"""Benchmark of the tree speculative decoding verification hot path.

One step = one pass of the whole path over one batch of synthetic input:
ancestor-mask build, tree attention (one attention layer), and tree
verification (greedy and/or stochastic, as the workload states).  The metric
is verified tree tokens/s = sum_b n_nodes[b] / step time, whole-job over all
ranks (each rank verifies its own batch: weak scaling, no collective on the
data path).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Workloads: tiny, llama7b, merge, gqa70b (default), long32k.

Prints ONE JSON line (rank 0).  `--impl reference` times the CPU oracle on a
bounded sample of the same workload instead.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from workloads import gen  # noqa: E402

METRIC = "verified tree tokens/s (attn+verify) and KV-cache GB/s as % of B200 HBM peak"
UNIT = "tokens/s"
DEFAULT_WORKLOAD = "gqa70b"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def rank_workload(cfg: int, rank: int, B=None):
    """Weak scaling: every rank verifies its own batch of independent
    sequences, drawn with a seed of its own (rank 0 = the single-GPU batch)."""
    return gen.config_workload(cfg, seed=gen.SEED_BASE + cfg + 1000 * rank, B=B)


def reduce_over_ranks(pg, device, tokens: int, ms: float):
    """Whole-job tokens (sum over ranks) and the slowest rank's time (max over
    ranks).  Every rank makes the same two collective calls, in this order."""
    if pg is None:
        return tokens, ms
    n = torch.tensor([float(tokens)], dtype=torch.float64, device=device)
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    pg.all_reduce(n, op=pg.ReduceOp.SUM)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return int(n.item()), float(t.item())


# ----------------------------------------------------------------- work
def attn_flops(w) -> int:
    """4*D flops per (query row, attended key): prefix + ancestors-or-self."""
    total = 0
    for b in range(w.B):
        T, P = int(w.n_nodes[b]), int(w.prefix_len[b])
        par = w.parent[b, :T].tolist()
        depth = []
        for u in range(T):
            depth.append(1 if par[u] < 0 else depth[par[u]] + 1)
        total += w.Hq * sum(P + d for d in depth) * 4 * w.D
    return total


def attn_bytes(w) -> int:
    """K+V of the attended positions, once per (b, KV head), + Q read + O write."""
    es = 4 if w.dtype == "f32" else 2
    qo = 2 * int(w.n_nodes.sum()) * w.Hq * w.D * es
    return w.kv_bytes() + qo


def verify_traffic(w, step) -> dict:
    """Algorithmic bytes of the verify calls of one step: every row a
    verifier must read, once.  Greedy: the logits rows of the root and of
    every node whose whole root path matched (each row's argmax decides which
    children match, the terminal's gives the bonus token; found level by
    level from the root on the host copy of the inputs) -- what the
    matched-node walk reads (the all-rows form, for small batches, reads every
    row with children).  Stochastic: the logits rows on the accepted path and
    the distinct q rows of the children tried there (the children before the
    accepted one, or all of them where the walk stops); read from the step's
    own results."""
    row = w.V * 4
    out = {}
    if "greedy" in w.verify:
        rows = 0
        for b in range(w.B):
            T = int(w.n_nodes[b])
            par = w.parent[b, :T].tolist()
            tok = w.tokens[b, :T].tolist()
            level = [-1]                   # -1 stands for the root
            while level:
                rows += len(level)
                nxt = []
                for f in level:
                    a = int(np.argmax(np.asarray(w.logits[b, f + 1])))
                    nxt += [c for c in range(T) if par[c] == f and tok[c] == a]
                level = nxt
        out["greedy"] = rows * row
    if "stochastic" in w.verify:
        n = step.s.n_accepted.cpu().tolist()
        path = step.s.out_path.cpu().tolist()
        qr = w.q_row.tolist()
        rows = 0
        for b in range(w.B):
            T = int(w.n_nodes[b])
            par = w.parent[b, :T].tolist()
            k = max(n[b], 0)
            nodes = [-1] + path[b][:k]
            for i, c in enumerate(nodes):
                rows += 1                  # the logits row of node c
                kids = [u for u in range(T) if par[u] == c]
                stop = path[b][i] if i < k else None
                tried = kids[:kids.index(stop) + 1] if stop is not None else kids
                rows += len({qr[b][u] for u in tried})
        out["stochastic"] = rows * row
    return out


def step_roofline(w, step, ms_per_step: float, peaks: dict) -> dict:
    """Roofline of the whole step: t_roof = max(bytes / HBM peak, FLOPs /
    tensor peak) with the bytes of the mask build, the attention layer and
    the verify calls, the FLOPs of the attention layer; frac = t_roof / the
    measured step time."""
    mask_bytes = w.B * w.Tmax * 4 * (1 + 1 + 1 + 1 + (w.Tmax + 31) // 32) + w.B * 8
    vb = verify_traffic(w, step)
    total = attn_bytes(w) + mask_bytes + sum(vb.values())
    flops = attn_flops(w)
    t_hbm = total / (peaks["hbm_gbs"] * 1e9)
    t_tc = flops / (peaks["bf16_tflops"] * 1e12)
    t_roof = max(t_hbm, t_tc)
    return {"bound": "tensor" if t_tc > t_hbm else "hbm", "t_roof_us": t_roof * 1e6,
            "step_us": ms_per_step * 1e3, "frac": t_roof / (ms_per_step * 1e-3),
            "bytes": total, "verify_bytes": vb, "flops": flops,
            "peaks": {"hbm_gbs": peaks["hbm_gbs"], "bf16_tflops": peaks["bf16_tflops"]}}


def kernel_roofline(w, att_s: float, peaks: dict) -> dict:
    """Roofline of the attention kernel alone (the dominant launch)."""
    flops, abytes = attn_flops(w), attn_bytes(w)
    t_hbm = abytes / (peaks["hbm_gbs"] * 1e9)
    t_tc = flops / (peaks["bf16_tflops"] * 1e12)
    if t_tc > t_hbm:
        roof = {"bound": "tensor", "achieved": flops / att_s / 1e12,
                "peak": peaks["bf16_tflops"], "unit": "TFLOP/s"}
    else:
        roof = {"bound": "hbm", "achieved": abytes / att_s / 1e9, "peak": peaks["hbm_gbs"],
                "unit": "GB/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    if roof["bound"] == "tensor" and peaks.get("bf16_tflops_sustained"):
        # The burst peak is the headline fraction; beside it the sustained
        # one (a GEMM loop held under the power cap), the regime this kernel
        # runs in inside the step loop: its SM clock, read from clock64
        # against %globaltimer in every CTA of a traced copy, is 1.5-1.8 GHz
        # there, not the 1965 MHz a lone burst gets.
        roof["peak_sustained"] = peaks["bf16_tflops_sustained"]
        roof["frac_sustained"] = roof["achieved"] / peaks["bf16_tflops_sustained"]
    roof["attn_us"] = att_s * 1e6
    roof["algorithmic_bytes"] = abytes
    roof["algorithmic_flops"] = flops
    return roof


INPUT_FIELDS = ("parent", "n_nodes", "prefix_len", "tokens", "q_row", "q", "k_cache", "v_cache",
                "logits", "q_probs", "u_accept", "u_sample")


def input_bytes(w) -> int:
    return sum(getattr(w, f).numel() * getattr(w, f).element_size() for f in INPUT_FIELDS)


def input_sets_for(w, max_bytes: float = 4e9) -> int:
    """How many device copies of the inputs the timed steps rotate over, so
    that no step finds its inputs in the L2: enough that the copies read since
    a copy's last use total more than twice the L2 (at least 2 copies; at most
    16 or max_bytes).  1 when that cannot be had (the steps then flush the L2
    by writing a buffer larger than it)."""
    nb = max(input_bytes(w), 1)
    n = max(2, -(-3 * L2_BYTES // nb))
    if n > 16 or n * nb > max_bytes:
        return 1
    return n


class Step:
    """Device buffers + one call sequence of the public API.  With n_sets > 1
    the inputs exist in n_sets device copies (the same values) and timed step
    i reads copy i % n_sets."""

    def __init__(self, w, dev, tsd, n_sets: int = 1):
        self.w, self.dev, self.tsd = w, dev, tsd
        self.sets = [{f: getattr(w, f).to(dev) for f in INPUT_FIELDS} for _ in range(n_sets)]
        self.d = self.sets[0]
        d = self.d
        self.tree = tsd.tree_mask_build(d["parent"], d["n_nodes"])
        self.out = torch.empty_like(d["q"])
        B, Tmax = w.B, w.Tmax
        self.g = tsd.VerifyResult(torch.empty((B, Tmax + 1), dtype=torch.int32, device=dev),
                                  torch.empty((B, Tmax), dtype=torch.int32, device=dev),
                                  torch.empty((B,), dtype=torch.int32, device=dev))
        self.s = tsd.VerifyResult(torch.empty((B, Tmax + 1), dtype=torch.int32, device=dev),
                                  torch.empty((B, Tmax), dtype=torch.int32, device=dev),
                                  torch.empty((B,), dtype=torch.int32, device=dev))
        self.ws_attn = torch.empty(max(256, tsd.attention_workspace_size(
            B, Tmax, w.Hq, w.Hkv, w.D, w.Lmax, d["q"].dtype)), dtype=torch.uint8, device=dev)
        self.ws_ver = torch.empty(max(256, tsd.verify_workspace_size(B, Tmax, w.V)),
                                  dtype=torch.uint8, device=dev)
        # the greedy call's own workspace and stream: with both verify modes
        # the two calls run side by side (they read the same inputs and
        # nothing of each other's)
        self.ws_ver_g = torch.empty_like(self.ws_ver)
        self.side = torch.cuda.Stream(device=dev)
        self.ev = None

    def run_mask(self):
        d = self.d
        self.tsd.tree_mask_build(d["parent"], d["n_nodes"], out=self.tree)

    def run_attention(self):
        d = self.d
        self.tsd.tree_attention(d["q"], d["k_cache"], d["v_cache"], d["prefix_len"],
                                d["n_nodes"], self.tree.mask, out=self.out,
                                workspace=self.ws_attn)

    def run(self, attn_events=None):
        self.run_mask()
        if attn_events is not None:
            attn_events[0].record()
        self.run_attention()
        if attn_events is not None:
            attn_events[1].record()
        self.run_verify()

    def capture_steps(self, steps: int, st_ev, att_ev, flush=None):
        """One CUDA graph of `steps` whole steps, step i on input copy
        i % n_sets: the mask build, the attention call and the verify
        call(s), between CUDA events recorded as graph nodes (external
        events: st_ev[i] around the step, att_ev[i] around the attention
        call, on the stream the kernels run on), with the L2 flush between
        steps outside the step's events when `flush` is given.  Replaying it
        times device work only: on the small workloads the Python and launch
        work in front of each call took longer than the kernels.  Returns the
        graph and the kernel launches it holds."""
        torch.cuda.synchronize(self.dev)
        n0 = self.tsd.launch_count()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for i in range(steps):
                self.d = self.sets[i % len(self.sets)]
                if flush is not None:
                    flush.fill_(float(i))
                st_ev[i][0].record()
                self.run_mask()
                att_ev[i][0].record()
                self.run_attention()
                att_ev[i][1].record()
                self.run_verify()
                st_ev[i][1].record()
        torch.cuda.synchronize(self.dev)
        self.d = self.sets[0]
        return graph, self.tsd.launch_count() - n0

    def run_verify(self):
        """The workload's verify calls.  With both modes, the greedy call runs
        on a second stream beside the stochastic one (forked after the mask
        build and the attention call, joined before the step ends): the
        stochastic walk is latency-bound on a few CTAs per SM and the greedy
        row scan bandwidth-bound, so they overlap."""
        w, d, tsd = self.w, self.d, self.tsd
        greedy = lambda ws: tsd.tree_verify_greedy(  # noqa: E731
            d["logits"], d["tokens"], d["parent"], d["n_nodes"], self.tree, out=self.g,
            workspace=ws)
        if "stochastic" not in w.verify:
            if "greedy" in w.verify:
                greedy(self.ws_ver)
            return
        main = torch.cuda.current_stream(self.dev)
        both = "greedy" in w.verify
        if both:
            self.side.wait_stream(main)
        tsd.tree_verify_stochastic(d["logits"], w.temperature, d["q_probs"], d["q_row"],
                                   d["tokens"], d["n_nodes"], self.tree, d["u_accept"],
                                   d["u_sample"], out=self.s, workspace=self.ws_ver)
        if both:
            with torch.cuda.stream(self.side):
                greedy(self.ws_ver_g)
            main.wait_stream(self.side)


def _clock_sampler(index):
    try:
        return subprocess.Popen(
            ["nvidia-smi", f"--id={index}",
             "--query-gpu=clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap",
             "--format=csv,noheader,nounits", "-lms", "20"],
            stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
    except OSError:
        return None


def _clock_summary(proc):
    if proc is None:
        return None
    proc.terminate()
    try:
        out, _ = proc.communicate(timeout=5)
    except subprocess.TimeoutExpired:
        proc.kill()
        out, _ = proc.communicate()
    sm, smax, reasons = [], None, set()
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    for line in out.strip().splitlines():
        parts = [p.strip() for p in line.split(",")]
        if len(parts) < 8:
            continue
        try:
            sm.append(float(parts[0]))
            smax = float(parts[1])
        except ValueError:
            continue
        for n, v in zip(names, parts[4:8]):
            if v.lower() == "active":
                reasons.add(n)
    if not sm:
        return None
    return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax, "reasons": sorted(reasons),
            "samples": len(sm)}


KERNEL_SECTION_END = "// ------------------------------------------------------------------ host"


def kernel_source_hash(text: str) -> str:
    """Hash of the kernels' source text in a CUDA file: from its first
    anonymous namespace to the host-section marker (the includes above and
    the host launch code below do not change what the kernels compute or
    move)."""
    i = text.index("namespace {\n")
    j = text.index(KERNEL_SECTION_END, i)
    return hashlib.sha256(text[i:j].encode()).hexdigest()[:16]


def _traffic_record(kernel_src: str, workload: str):
    """DRAM traffic of the dominant kernel from the committed ncu summary, if
    the summary was taken on the current source of the kernels."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    try:
        rec = json.load(open(p)).get(workload)
    except (ValueError, OSError):
        return None
    if not rec:
        return None
    try:
        h = kernel_source_hash(open(kernel_src).read())
    except (ValueError, OSError):
        return None
    return rec.get("bytes_per_launch") if rec.get("kernel_sha") == h else None


# ------------------------------------------------------------ CPU oracle
def cpu_baseline(w, budget_s: float = 15.0, keep=None):
    """Time the oracle (as it stands) on a bounded sample of the workload:
    whole sequences (attention over all heads + the verify call(s)), added
    one at a time until ~budget_s of CPU work.  With `keep` (a list), the
    oracle's outputs of each sequence are appended to it (outside the timed
    calls) for the parity record."""
    import oracle
    oracle.build()
    done_nodes, elapsed, seqs = 0, 0.0, 0
    for b in range(w.B):
        T = int(w.n_nodes[b])
        sub = _subset(w, b)
        out = {"b": b}
        t0 = time.perf_counter()
        if T:
            rows = [(0, u, h) for u in range(T) for h in range(w.Hq)]
            out["attn"] = oracle.tree_attention_rows(sub.q, sub.k_cache, sub.v_cache,
                                                     sub.prefix_len, sub.n_nodes, sub.parent,
                                                     sub.scale, rows)
        if "greedy" in w.verify:
            out["greedy"] = oracle.workload_greedy(sub)
        if "stochastic" in w.verify:
            out["stochastic"] = oracle.workload_stochastic(sub)
        elapsed += time.perf_counter() - t0
        if keep is not None:
            keep.append(out)
        done_nodes += T
        seqs += 1
        if elapsed >= budget_s:
            break
    return {"value": done_nodes / elapsed, "unit": UNIT, "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": f"{seqs} of {w.B} sequences ({done_nodes} nodes), full attention layer "
                      f"over all {w.Hq} heads + {'/'.join(w.verify)} verify, {elapsed:.1f} s"}


ATOL = {"bf16": 2e-2, "f32": 1e-4}   # attention max-abs tolerance against the fp64 oracle


def parity_record(w, step, ref_seqs) -> dict:
    """The GPU step's outputs against the oracle's on the sequences the oracle
    ran (every node and head of each): attention max-abs error, greedy paths
    and tokens bit-exact, stochastic ones bit-exact except on sequences whose
    oracle path has a decision within 1e-9 of its boundary (excused)."""
    rec = {"sequences": len(ref_seqs), "attn_tol": ATOL[w.dtype]}
    got = step.out.float().cpu().numpy().astype(np.float64)
    worst, rows = 0.0, 0
    for r in ref_seqs:
        if "attn" not in r:
            continue
        b, T = r["b"], int(w.n_nodes[r["b"]])
        g = got[b, :T].reshape(T * w.Hq, w.D)
        worst = max(worst, float(np.abs(g - r["attn"]).max()))
        rows += T * w.Hq
    rec.update(attn_max_abs=worst, attn_rows_compared=rows, attn_ok=worst <= ATOL[w.dtype])
    for mode, res in (("greedy", step.g), ("stochastic", step.s)):
        if mode not in w.verify:
            continue
        n = res.n_accepted.cpu().numpy()
        path, toks = res.out_path.cpu().numpy(), res.out_tokens.cpu().numpy()
        mism = excused = decisions = flagged = 0
        for r in ref_seqs:
            ref, b = r[mode], r["b"]
            k = int(ref["n_accepted"][0])
            same = int(n[b]) == k and (k < 0 or (
                (path[b, :k] == ref["out_path"][0, :k]).all() and
                (toks[b, :k + 1] == ref["out_tokens"][0, :k + 1]).all()))
            if mode == "stochastic":
                decisions += int(ref["n_decisions"].sum())
                flagged += int(ref["n_flagged"].sum())
                if not same and int(ref["n_flagged"][0]) > 0:
                    excused += 1
                    continue
            mism += 0 if same else 1
        if mode == "greedy":
            rec["greedy"] = {"mismatches": mism, "exact": mism == 0}
        else:
            rec["stochastic"] = {"mismatches": mism, "excused": excused,
                                 "flagged_decisions": flagged, "decisions": decisions,
                                 "exact": mism == 0 and excused <= 1e-4 * max(decisions, 1)}
    rec["ok"] = rec["attn_ok"] and all(rec[m]["exact"] for m in ("greedy", "stochastic")
                                       if m in rec)
    return rec


def oracle_single_thread(name: str, budget_s: float = 6.0):
    """The oracle on one host core (OMP_NUM_THREADS=1), on one sequence of
    the named workload, through this script's reference arm in a child
    process (the thread count is fixed when the oracle's OpenMP runtime
    starts)."""
    env = dict(os.environ, OMP_NUM_THREADS="1")
    try:
        r = subprocess.run([sys.executable, os.path.abspath(__file__), "--impl", "reference",
                            "--workload", name, "--steps", "1", "--warmup", "0", "--batch", "1",
                            "--oracle-budget", str(budget_s)],
                           env=env, capture_output=True, text=True, timeout=300)
        line = json.loads(r.stdout.strip().splitlines()[-1])
        cb = line["cpu_baseline"]
        return {"workload": name, "value": cb["value"], "unit": UNIT, "cores": cb["cores"],
                "kind": "oracle", "sample": cb["sample"]}
    except (subprocess.SubprocessError, ValueError, KeyError, IndexError, OSError) as e:
        return {"workload": name, "error": str(e)[:200]}


def _subset(w, b):
    import dataclasses
    sl = slice(b, b + 1)
    return dataclasses.replace(
        w, B=1, parent=w.parent[sl], n_nodes=w.n_nodes[sl], prefix_len=w.prefix_len[sl],
        tokens=w.tokens[sl], q_row=w.q_row[sl], q=w.q[sl], k_cache=w.k_cache[sl],
        v_cache=w.v_cache[sl], logits=w.logits[sl], q_probs=w.q_probs[sl],
        u_accept=w.u_accept[sl], u_sample=w.u_sample[sl])


# ------------------------------------------------------------------ main
def _workload_name(w):
    return w.name


def time_steps(step, w, dev, tsd, steps: int, warmup: int, pg=None, local: int = 0,
               clocks: bool = False) -> dict:
    """Warm-up (eager steps, then one replay of the timed graph), then the
    `steps` timed steps as one replay of a CUDA graph holding them back to
    back (Step.capture_steps), with a barrier and a synchronize on both
    sides; CUDA events per step and around the attention call, recorded by
    the graph on the launching stream.  The L2 is flushed between steps
    unless the steps rotate over enough input copies to exceed it."""
    for _ in range(max(3, warmup)):
        step.run()
    torch.cuda.synchronize(dev)
    if int(tsd.device_status(dev).item()) != 0:
        raise RuntimeError(f"device status set during warm-up ({w.name})")
    flush = None
    nsets = len(step.sets)
    working = input_bytes(w)
    if nsets == 1:
        flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
    ev = lambda: torch.cuda.Event(enable_timing=True, external=True)  # noqa: E731
    att_ev = [(ev(), ev()) for _ in range(steps)]
    st_ev = [(ev(), ev()) for _ in range(steps)]
    graph, launches = step.capture_steps(steps, st_ev, att_ev, flush)
    graph.replay()   # warm-up replay of the same work
    torch.cuda.synchronize(dev)
    sampler = _clock_sampler(local) if clocks else None
    if sampler is not None:
        time.sleep(0.3)
    if pg:
        pg.barrier()
    torch.cuda.synchronize(dev)
    graph.replay()
    torch.cuda.synchronize(dev)
    if pg:
        pg.barrier()
    clk = _clock_summary(sampler) if sampler is not None else None
    if int(tsd.device_status(dev).item()) != 0:
        raise RuntimeError(f"device status set during the timed steps ({w.name})")
    res = {"step_ms": [a.elapsed_time(b) for a, b in st_ev],
           "att_ms": [a.elapsed_time(b) for a, b in att_ev],
           "launches": launches, "clocks": clk,
           "l2": "flushed between steps (2x L2 write)" if flush is not None
           else f"inputs larger than L2: {nsets} device copies of the inputs "
                f"({working / 1e6:.0f} MB each), step i reads copy i mod {nsets}"}
    del graph
    return res


def workload_record(name, w, step, t, peaks, dev, tsd, parity_budget_s: float) -> dict:
    """One workload's figures for the `workloads` table of the line: tokens/s,
    step time, attention time and roofline, the step roofline, KV-cache
    bandwidth, acceptance, the attention plan, and parity against the oracle
    on a bounded sample of whole sequences."""
    ms = statistics.mean(t["step_ms"])
    att_s = statistics.mean(t["att_ms"]) / 1e3
    kv_gbs = w.kv_bytes() / att_s / 1e9
    ref = []
    cpu_baseline(w, budget_s=parity_budget_s, keep=ref)
    return {"workload": w.name, "value": int(w.n_nodes.sum()) / (ms / 1e3), "unit": UNIT,
            "ms_per_step": ms, "steps": len(t["step_ms"]), "dtype": w.dtype,
            "roofline": kernel_roofline(w, att_s, peaks),
            "roofline_step": step_roofline(w, step, ms, peaks),
            "kv_cache_gbs": kv_gbs, "kv_cache_frac_of_hbm": kv_gbs / peaks["hbm_gbs"],
            "acceptance": accepted_summary(w, step), "plan": _plan(w, dev, tsd),
            "verify_plan": _verify_plan(w, tsd),
            "parity": parity_record(w, step, ref), "l2": t["l2"]}


def _plan(w, dev, tsd):
    return tsd.attention_plan(
        w.B, w.Tmax, w.Hq, w.Hkv, w.D, int(w.k_cache.shape[2]),
        torch.bfloat16 if w.dtype == "bf16" else torch.float32,
        torch.cuda.get_device_properties(dev).multi_processor_count)


def _verify_plan(w, tsd) -> dict:
    """The form of each verify call the workload makes: the greedy one's
    (walk over matched nodes, or every row with children) and the stochastic
    walk's grid."""
    out = {}
    try:
        if "greedy" in w.verify:
            out["greedy"] = tsd.verify_greedy_plan(w.B, w.Tmax, w.V)["form"]
        if "stochastic" in w.verify:
            out["stochastic"] = tsd.verify_stochastic_plan(w.B, w.Tmax, w.V)
    except tsd.TsdError as e:   # informational: never fails the measurement
        out["error"] = str(e)
    return out


def acceptance_other_proposal(cfg, dev, tsd) -> dict:
    """Acceptance of the headline workload's trees under the other token
    proposal (top-k tokens of rows perturbed by N(0, 0.3^2) instead of draws
    from rows perturbed by N(0, 1)): the same trees and target logits, only
    the speculated tokens and SSM rows differ.  Verify calls only."""
    other = "topk" if cfg in (3, 4) else None
    if other is None:
        return None
    w = gen.config_workload(cfg, with_attention=False, proposal=other)
    d = {f: getattr(w, f).to(dev) for f in ("parent", "n_nodes", "tokens", "q_row", "logits",
                                            "q_probs", "u_accept", "u_sample")}
    tree = tsd.tree_mask_build(d["parent"], d["n_nodes"])
    out = {}
    if "greedy" in w.verify:
        r = tsd.tree_verify_greedy(d["logits"], d["tokens"], d["parent"], d["n_nodes"], tree)
        out["greedy"] = float(r.n_accepted.double().mean())
    if "stochastic" in w.verify:
        r = tsd.tree_verify_stochastic(d["logits"], w.temperature, d["q_probs"], d["q_row"],
                                       d["tokens"], d["n_nodes"], tree, d["u_accept"],
                                       d["u_sample"])
        out["stochastic"] = float(r.n_accepted.double().mean())
    torch.cuda.synchronize(dev)
    return {"proposal": "top-k tokens, SSM noise N(0, 0.3^2)",
            "mean_accepted_nodes": out}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(gen.WORKLOAD_NAMES))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--batch", type=int, default=None,
                    help="sequences per GPU (default: the workload's batch)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-side", action="store_true",
                    help="skip the side measurements (commit, paged attention, tree build)")
    ap.add_argument("--no-workloads", action="store_true",
                    help="time only the headline workload (no table of the other four)")
    ap.add_argument("--oracle-budget", type=float, default=None,
                    help="reference arm: seconds of oracle work per timed step")
    args = ap.parse_args()
    ws, rank, local = _dist()
    cfg = gen.WORKLOAD_NAMES[args.workload]

    if args.impl == "reference":
        if rank != 0:
            return
        w = gen.config_workload(cfg, B=args.batch)
        times = []
        cb = None
        budget = args.oracle_budget or 6.0
        for i in range(args.warmup + args.steps):
            cb = cpu_baseline(w, budget_s=min(2.0, budget) if i < args.warmup else budget)
            if i >= args.warmup:
                times.append(cb["value"])
        val = statistics.median(times)
        cb["value"] = val
        line = {"impl": "reference", "metric": METRIC, "value": val, "unit": UNIT,
                "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": None, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": {"workload": _workload_name(w)},
                "cpu_baseline": cb,
                "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    import tree_speculative_decoding_ancestor_b200 as tsd

    torch.cuda.set_device(local)
    dev = torch.device(f"cuda:{local}")
    pg = None
    if ws > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        pg = dist
    # weak scaling: every rank verifies its own batch (a different seed per rank)
    w = rank_workload(cfg, rank, args.batch)
    step = Step(w, dev, tsd, input_sets_for(w))
    tokens_per_step = int(w.n_nodes.sum())
    t = time_steps(step, w, dev, tsd, args.steps, args.warmup, pg, local, clocks=True)
    job_tokens, total_ms = reduce_over_ranks(pg, dev, tokens_per_step, float(sum(t["step_ms"])))
    ms_per_step = total_ms / args.steps
    value = job_tokens / (ms_per_step / 1e3)
    acceptance = accepted_summary(w, step)
    gathered = None
    if pg is not None:
        # the batch-sharded path's optional collective, outside the timed
        # steps: every rank's verify results on every rank (same call order
        # on every rank)
        res = step.s if "stochastic" in w.verify else step.g
        gathered = int(tsd.all_gather_accepted(res).n_accepted.shape[0])
    side = {}
    if not args.no_side:
        side["kv_commit"] = time_commit(step, dev, tsd)
        side["paged_attention"] = time_paged_attention(step, dev, tsd) \
            if w.dtype == "bf16" else None
        side["tree_build"] = time_tree_build(w, dev, tsd)

    peaks, peak_kind = _peaks()
    att_s = statistics.mean(t["att_ms"]) / 1e3
    roof = kernel_roofline(w, att_s, peaks)
    roof["peak_source"] = f"{peak_kind} (MEASURED_PEAKS.json burst)" if peak_kind == \
        "measured" else "fallback"
    kernel_src = os.path.join(ROOT, "tree_speculative_decoding_ancestor_b200", "csrc",
                              "attention_umma.cu")
    roof["traffic"] = _traffic_record(kernel_src, args.workload)
    roof["kernel"] = "tree attention (mask-aware split-KV), one layer"
    roof["plan"] = _plan(w, dev, tsd)
    kv_gbs = w.kv_bytes() / att_s / 1e9

    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
            "warmup": max(3, args.warmup), "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": w.dtype, "data": "synthetic",
            "config": {"workload": _workload_name(w), "batch_per_gpu": w.B,
                       "tree_nodes_per_step_per_gpu": tokens_per_step, "Hq": w.Hq,
                       "Hkv": w.Hkv, "head_dim": w.D, "prefix": int(w.prefix_len[0]),
                       "vocab": w.V, "verify": list(w.verify), "l2": t["l2"],
                       "parallelism": f"batch-sharded x{ws} (independent sequences)"},
            "kv_cache_gbs": kv_gbs, "kv_cache_frac_of_hbm": kv_gbs / peaks["hbm_gbs"],
            "roofline": roof,
            "roofline_step": step_roofline(w, step, statistics.mean(t["step_ms"]), peaks),
            "gpu_launches": t["launches"], "clocks": t["clocks"],
            "acceptance": acceptance, "verify_plan": _verify_plan(w, tsd)}
    if gathered is not None:
        line["gathered_sequences"] = gathered
    line.update(side)

    if not args.no_e2e:
        line["e2e"] = e2e(w, dev, tsd, args, pg, ws)
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        ref = []
        line["cpu_baseline"] = cpu_baseline(w, keep=ref)
        line["parity"] = parity_record(w, step, ref)
        line["cpu_baseline_1thread"] = oracle_single_thread("llama7b")
    if ws == 1 and not args.no_workloads:
        alt = acceptance_other_proposal(cfg, dev, tsd)
        if alt:
            line["acceptance_other_proposal"] = alt
        rec = {args.workload: workload_record(args.workload, w, step, t, peaks, dev, tsd,
                                              parity_budget_s=0.0)}
        rec[args.workload]["parity"] = line.get("parity", rec[args.workload]["parity"])
        del step
        torch.cuda.empty_cache()
        for name in sorted(gen.WORKLOAD_NAMES, key=gen.WORKLOAD_NAMES.get):
            if name == args.workload:
                continue
            wk = gen.config_workload(gen.WORKLOAD_NAMES[name])
            sk = Step(wk, dev, tsd, input_sets_for(wk))
            tk = time_steps(sk, wk, dev, tsd, min(args.steps, 20), 3)
            rec[name] = workload_record(name, wk, sk, tk, peaks, dev, tsd, parity_budget_s=3.0)
            del sk, wk
            torch.cuda.empty_cache()
        line["workloads"] = rec
    if rank == 0:
        print(json.dumps(line), flush=True)
    if pg:
        pg.destroy_process_group()


def accepted_summary(w, step) -> dict:
    """Mean tree nodes accepted per sequence by each verify mode of the
    workload, and the tokens one verification step emits per sequence (the
    accepted nodes plus the target's own token).  Read from the last timed
    step's results; malformed sequences (n_accepted = -1) are left out."""
    out = {}
    for mode, res in (("greedy", step.g), ("stochastic", step.s)):
        if mode not in w.verify:
            continue
        n = res.n_accepted.detach().to("cpu", torch.float64)
        ok = n >= 0
        if bool(ok.any()):
            m = float(n[ok].mean())
            out[mode] = {"mean_accepted_nodes": m, "mean_tokens_per_step": m + 1.0,
                         "sequences": int(ok.sum())}
    return out


def time_commit(step, dev, tsd, reps: int = 20):
    """The step after verification (outside the metric's step): move the
    accepted nodes' K/V rows after the prefix.  Timed alone with CUDA events
    on the verify result of the last step (repeating it moves the same rows
    again, which costs the same).  The kernel takes a few microseconds, less
    than the Python call around it, so the reps are captured in a CUDA graph
    and the replay is timed."""
    w, d = step.w, step.d
    res = step.s if "stochastic" in w.verify else step.g
    n = int(res.n_accepted.clamp(min=0).sum().item())
    row = w.D * d["k_cache"].element_size()
    newp = torch.empty_like(d["prefix_len"])
    tsd.kv_commit(d["k_cache"], d["v_cache"], d["prefix_len"], res, new_prefix_len=newp)
    torch.cuda.synchronize(dev)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for _ in range(reps):
            tsd.kv_commit(d["k_cache"], d["v_cache"], d["prefix_len"], res, new_prefix_len=newp)
    graph.replay()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    graph.replay()
    e1.record()
    torch.cuda.synchronize(dev)
    del graph
    if int(tsd.device_status(dev).item()) != 0:
        raise RuntimeError("device status set by the commit")
    us = e0.elapsed_time(e1) * 1e3 / reps
    moved = 4 * n * w.Hkv * row   # K and V rows, read once and written once
    return {"us": us, "accepted_nodes": n, "algorithmic_bytes": moved,
            "gbs": moved / (us * 1e-6) / 1e9 if us > 0 else None}


def time_tree_build(w, dev, tsd, reps: int = 10):
    """Token-tree construction on the GPU for the workload's batch and
    vocabulary: an expansion <4, 2, 2, ...> level by level (as many levels as
    the tree slots hold; the top-k of a random SSM row per frontier node),
    then the depth-first renumbering; the launches are captured in a CUDA
    graph and its replay is timed."""
    B, V = w.B, w.V
    ks, n, F = [4], 4, 4
    while n + 2 * F <= w.Tmax:
        ks.append(2)
        n, F = n + 2 * F, 2 * F
    n, F, start, frows = 0, 1, 0, []
    for k in ks:
        fr = torch.zeros((B, w.Tmax), dtype=torch.int32)   # root level: row 0
        if n > 0:   # frontier = the level added last, nodes start .. n-1; node u's row is u + 1
            fr[:, :F] = torch.arange(start, n, dtype=torch.int32) + 1
        frows.append(fr.to(dev))
        start = n
        n, F = n + F * k, F * k
    q = torch.rand((B, n + 1, V), device=dev, generator=None)
    z = lambda: torch.zeros((B, w.Tmax), dtype=torch.int32, device=dev)  # noqa: E731
    tree = tsd.Tree(z(), z(), z(), torch.zeros(B, dtype=torch.int32, device=dev))
    lvl = torch.zeros(B, dtype=torch.int32, device=dev)
    perm = z()
    out = tsd.Tree(z(), z(), z(), tree.n_nodes)
    lib = tsd.load_library()
    st = tsd.device_status(dev)
    stream = torch.cuda.current_stream(dev)

    def run():
        tree.n_nodes.zero_()
        lvl.zero_()
        for k, fr in zip(ks, frows):
            tsd.tree_expand(q, fr, k, tree, lvl)
        lib.tsd_tree_dfs_order(tree.parent.data_ptr(), tree.tokens.data_ptr(),
                               tree.q_row.data_ptr(), tree.n_nodes.data_ptr(), B, w.Tmax,
                               perm.data_ptr(), out.parent.data_ptr(), out.tokens.data_ptr(),
                               out.q_row.data_ptr(), st.data_ptr(), stream.cuda_stream)

    run()
    torch.cuda.synchronize(dev)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for _ in range(reps):
            run()
    graph.replay()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    graph.replay()
    e1.record()
    torch.cuda.synchronize(dev)
    del graph
    if int(st.item()) != 0 or int(tree.n_nodes[0].item()) != n:
        raise RuntimeError("tree construction failed in the benchmark")
    return {"expansion": list(ks), "nodes_per_sequence": n, "sequences": B, "vocab": V,
            "us": e0.elapsed_time(e1) * 1e3 / reps}


def time_paged_attention(step, dev, tsd, page_size: int = 128, reps: int = 10):
    """The same attention call through a paged KV cache (pools of page_size
    rows, physical pages in a shuffled order, a block table per sequence),
    replayed from a CUDA graph and timed with CUDA events; also reports the
    contiguous call's time measured the same way."""
    w, d = step.w, step.d
    B, Hkv, Lmax, D = d["k_cache"].shape
    nblk = (Lmax + page_size - 1) // page_size
    gen_ = torch.Generator().manual_seed(1234)
    perm = torch.randperm(B * nblk, generator=gen_).to(dev)

    def pool(cache):
        padded = torch.zeros((B, Hkv, nblk * page_size, D), dtype=cache.dtype, device=dev)
        padded[:, :, :Lmax] = cache
        logical = padded.view(B, Hkv, nblk, page_size, D).permute(0, 2, 1, 3, 4)
        out = torch.empty((B * nblk, Hkv, page_size, D), dtype=cache.dtype, device=dev)
        out[perm] = logical.reshape(B * nblk, Hkv, page_size, D)
        return out

    kp, vp = pool(d["k_cache"]), pool(d["v_cache"])
    table = perm.view(B, nblk).to(torch.int32)
    out = torch.empty_like(d["q"])

    def paged():
        tsd.tree_attention_paged(d["q"], kp, vp, table, d["prefix_len"], d["n_nodes"],
                                 step.tree.mask, out=out)

    def flat():
        tsd.tree_attention(d["q"], d["k_cache"], d["v_cache"], d["prefix_len"], d["n_nodes"],
                           step.tree.mask, out=out, workspace=step.ws_attn)

    res = {}
    for name, fn in (("us", paged), ("contiguous_us", flat)):
        # each call replayed from a CUDA graph of its own, so that the events
        # time the kernels and not the Python and tensor-map work in front
        fn()
        torch.cuda.synchronize(dev)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            fn()
        graph.replay()
        torch.cuda.synchronize(dev)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(reps)]
        for a, b in ev:
            a.record()
            graph.replay()
            b.record()
        torch.cuda.synchronize(dev)
        del graph
        res[name] = statistics.median(a.elapsed_time(b) * 1e3 for a, b in ev)
    if int(tsd.device_status(dev).item()) != 0:
        raise RuntimeError("device status set by the paged attention")
    res["page_size"] = page_size
    del kp, vp
    return res


def e2e(w, dev, tsd, args, pg, ws):
    """Same metric through the public API with the inputs in pinned host
    memory: every step copies its inputs host->device and the results back."""
    fields = ("parent", "n_nodes", "prefix_len", "tokens", "q_row", "q", "k_cache", "v_cache",
              "logits", "q_probs", "u_accept", "u_sample")
    host = {f: getattr(w, f).pin_memory() for f in fields}
    devb = {f: torch.empty_like(host[f], device=dev) for f in fields}
    step = Step(w, dev, tsd)
    step.d = devb
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    outs = [step.out, step.g.out_tokens, step.g.out_path, step.g.n_accepted,
            step.s.out_tokens, step.s.out_path, step.s.n_accepted]
    if "greedy" not in w.verify:
        outs = [o for o in outs if o is not step.g.out_tokens and o is not step.g.out_path
                and o is not step.g.n_accepted]
    if "stochastic" not in w.verify:
        outs = [o for o in outs if o is not step.s.out_tokens and o is not step.s.out_path
                and o is not step.s.n_accepted]
    host_out = [torch.empty_like(o, device="cpu").pin_memory() for o in outs]
    d2h = sum(o.numel() * o.element_size() for o in outs)
    steps = max(3, min(args.steps, 10))

    def one():
        for f in fields:
            devb[f].copy_(host[f], non_blocking=True)
        step.run()
        for o, h in zip(outs, host_out):
            h.copy_(o, non_blocking=True)

    for _ in range(2):
        one()
    torch.cuda.synchronize(dev)
    if pg:
        pg.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        one()
    e1.record()
    torch.cuda.synchronize(dev)
    job_tokens, ms = reduce_over_ranks(pg, dev, int(w.n_nodes.sum()),
                                       e0.elapsed_time(e1) / steps)
    return {"value": job_tokens / (ms / 1e3), "unit": UNIT,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "steps": steps,
            "ms_per_step": ms}


if __name__ == "__main__":
    main()
