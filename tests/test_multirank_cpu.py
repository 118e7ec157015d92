"""The N > 1 host path of bench.py on CPU: two ranks over gloo (127.0.0.1).

Each rank draws its own seeded batch of the same shape; times are reduced
with MAX and units of work with SUM, so the reported throughput is the work of
all ranks over the slowest rank's time.  The reference arm runs on rank 0
only.  No GPU is touched."""
import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import torch.distributed as dist

    import bench
    import synth
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        t = bench.reduce_over_ranks(10.0 + rank, dist, dist.ReduceOp.MAX, "cpu")
        w = synth.WORKLOADS["ragged_prefill"]
        L = synth.uniform_lengths(w.B, *w.len_range, w.seed + bench.rank_seed_offset(rank))
        units = float(np.sum(L.astype(np.float64) * (L + 1) / 2))
        u = bench.reduce_over_ranks(units, dist, dist.ReduceOp.SUM, "cpu")
        q.put((rank, t, units, u, L.tolist()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_gloo_reductions_and_seeds():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = {}
    for _ in range(2):
        r = q.get(timeout=180)
        out[r[0]] = r
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (_, t0, u0, s0, l0), (_, t1, u1, s1, l1) = out[0], out[1]
    assert t0 == t1 == 11.0                      # max over ranks
    assert s0 == s1 == pytest.approx(u0 + u1)    # units of all ranks
    assert l0 != l1                              # each rank has its own batch ...
    assert len(l0) == len(l1)                    # ... of the same shape
    sys.path.insert(0, ROOT)
    import bench
    import synth
    w = synth.WORKLOADS["ragged_prefill"]
    assert l1 == synth.uniform_lengths(w.B, *w.len_range, w.seed + bench.rank_seed_offset(1)).tolist()


def test_single_process_reduction_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_over_ranks(3.5, None, None, "cpu") == 3.5


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    assert bench.run_reference(None) is None     # returns before touching args or the oracle
