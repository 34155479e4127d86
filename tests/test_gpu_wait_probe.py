"""Bounded waits end with a status, not a hung GPU (tsd_debug_wait_probe).

Every wait in the kernels gives up after a time limit, sets TSD_DEV_TIMEOUT and
returns.  The probe runs the same wait routines -- the attention kernels'
mbarrier wait, the stochastic walk's team barrier and its cluster exchange --
on something nothing ever signals, with a 50 ms limit; the kernel must end on
its own with the status set, and the context must stay usable afterwards.
"""

import time

import numpy as np
import pytest
import torch

import oracle
import tree_speculative_decoding_ancestor_b200 as tsd
from workloads import gen

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("kind", [0, 1, 2])
def test_bounded_wait_ends_with_timeout_status(cuda_device, kind):
    st = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    torch.cuda.synchronize(cuda_device)
    t0 = time.perf_counter()
    tsd.binding.debug_wait_probe(kind, 50_000_000, device=cuda_device, status=st)
    torch.cuda.synchronize(cuda_device)
    dt = time.perf_counter() - t0
    assert int(st.item()) & tsd.binding.DEV_TIMEOUT
    assert 0.045 <= dt < 2.0, dt
    # the context still works: a small attention call matches the oracle
    w = gen.random_workload(81, B=2, Tmax=12, Hq=8, Hkv=2, D=128, P_max=200, V=8,
                            dtype="bf16", min_nodes=1)
    d = {k: getattr(w, k).to(cuda_device) for k in ("parent", "n_nodes", "prefix_len", "q",
                                                    "k_cache", "v_cache")}
    tsd.device_status(cuda_device).zero_()
    tree = tsd.tree_mask_build(d["parent"], d["n_nodes"])
    out = tsd.tree_attention(d["q"], d["k_cache"], d["v_cache"], d["prefix_len"], d["n_nodes"],
                             tree.mask)
    torch.cuda.synchronize(cuda_device)
    assert int(tsd.device_status(cuda_device).item()) == 0
    ref = oracle.workload_attention(w)
    got = out.float().cpu().numpy()
    for b in range(w.B):
        T = int(w.n_nodes[b])
        assert np.abs(got[b, :T] - ref[b, :T]).max() <= 2e-2


def test_probe_host_checks(cuda_device):
    lib = tsd.load_library()
    z = torch.zeros(2, dtype=torch.int32, device=cuda_device)
    s = torch.cuda.current_stream().cuda_stream
    assert lib.tsd_debug_wait_probe(3, 50_000_000, z.data_ptr(), z.data_ptr(), s) == -2
    assert lib.tsd_debug_wait_probe(0, 10, z.data_ptr(), z.data_ptr(), s) == -2      # < 1 ms
    assert lib.tsd_debug_wait_probe(0, 50_000_000, None, z.data_ptr(), s) == -1
