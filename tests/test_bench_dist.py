"""The benchmark's multi-rank path on CPU: two `gloo` ranks (CPU only).

With N GPUs every rank verifies its own batch of independent sequences (weak
scaling, no collective on the data path); the only collectives are the
reduction of the whole job's tree tokens (sum over ranks) and of the timed
region (the slowest rank).  These tests run that reduction and the per-rank
workload choice in two spawned processes over `gloo`.
"""

import datetime
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import bench
from workloads import gen


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_q):
    import torch.distributed as dist
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        tokens = (100, 37, 5)[rank]
        ms = (2.5, 4.0, 3.0)[rank]
        got = bench.reduce_over_ranks(dist, torch.device("cpu"), tokens, ms)
        w = bench.rank_workload(3, rank, B=2)
        out_q.put((rank, got, int(w.n_nodes.sum()), np.asarray(w.tokens).tolist()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _run_ranks(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    try:
        for _ in range(world):
            rank, got, n, toks = q.get(timeout=120)
            res[rank] = (got, n, toks)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    return res


def test_two_ranks_sum_tokens_and_take_the_slowest_time():
    res = _run_ranks(2)
    for rank in (0, 1):
        (tokens, ms), _, _ = res[rank]
        assert tokens == 137          # 100 + 37
        assert ms == pytest.approx(4.0)   # max(2.5, 4.0)


def test_three_ranks_agree():
    res = _run_ranks(3)
    assert {res[r][0] for r in range(3)} == {(142, 4.0)}


def test_ranks_verify_different_sequences():
    res = _run_ranks(2)
    # rank 0 is the single-GPU batch; rank 1 draws its own trees and tokens
    w0 = gen.config_workload(3, B=2)
    assert res[0][2] == np.asarray(w0.tokens).tolist()
    assert res[1][2] != res[0][2]
    assert res[0][1] == int(w0.n_nodes.sum())


def _gather_main(rank, world, port, out_q):
    import torch.distributed as dist

    from tree_speculative_decoding_ancestor_b200 import VerifyResult, all_gather_accepted
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        B, Tmax = (2, 3, 1)[rank], 4
        base = 100 * rank
        res = VerifyResult(torch.arange(B * (Tmax + 1), dtype=torch.int32).view(B, Tmax + 1) + base,
                           torch.arange(B * Tmax, dtype=torch.int32).view(B, Tmax) + base,
                           torch.arange(B, dtype=torch.int32) + base)
        got = all_gather_accepted(res)
        out_q.put((rank, [t.tolist() for t in got]))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_all_gather_accepted_concatenates_in_rank_order(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_gather_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    try:
        for _ in range(world):
            rank, got = q.get(timeout=120)
            res[rank] = got
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    sizes, Tmax = (2, 3, 1)[:world], 4
    want_n = [100 * r + b for r in range(world) for b in range(sizes[r])]
    want_path = [[100 * r + b * Tmax + j for j in range(Tmax)]
                 for r in range(world) for b in range(sizes[r])]
    for r in range(world):
        assert res[r][2] == want_n
        assert res[r][1] == want_path
        assert len(res[r][0]) == sum(sizes) and len(res[r][0][0]) == Tmax + 1


def test_single_process_passthrough():
    assert bench.reduce_over_ranks(None, torch.device("cpu"), 11, 1.5) == (11, 1.5)


def test_accepted_summary_skips_malformed_sequences():
    from tree_speculative_decoding_ancestor_b200 import VerifyResult

    class _W:
        verify = ("greedy", "stochastic")

    class _Step:
        pass

    z = torch.zeros((4, 5), dtype=torch.int32)
    st = _Step()
    st.g = VerifyResult(z, z, torch.tensor([3, 0, -1, 1], dtype=torch.int32))
    st.s = VerifyResult(z, z, torch.tensor([2, 2, 2, 2], dtype=torch.int32))
    got = bench.accepted_summary(_W(), st)
    assert got["greedy"] == {"mean_accepted_nodes": 4 / 3, "mean_tokens_per_step": 4 / 3 + 1,
                             "sequences": 3}
    assert got["stochastic"]["mean_accepted_nodes"] == 2.0
    _W.verify = ("stochastic",)
    assert set(bench.accepted_summary(_W(), st)) == {"stochastic"}
    st.s = VerifyResult(z, z, torch.full((4,), -1, dtype=torch.int32))
    assert bench.accepted_summary(_W(), st) == {}


def test_traffic_record_is_keyed_by_the_kernel_section():
    src = ("#include <a>\nnamespace {\n__global__ void k() {}\n}\n"
           + bench.KERNEL_SECTION_END + "\nint launch() { return 0; }\n")
    h = bench.kernel_source_hash(src)
    # edits to the includes or the host launch code keep the key ...
    assert bench.kernel_source_hash("#include <b>\n" + src) == h
    assert bench.kernel_source_hash(src.replace("return 0", "return 1")) == h
    # ... an edit to a kernel does not
    assert bench.kernel_source_hash(src.replace("k() {}", "k() { }")) != h
