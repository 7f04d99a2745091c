"""The multi-GPU bench path's host logic on two CPU ranks (gloo backend):
each rank gets its own batch of the same shape, and the whole-job totals are
the slowest rank's time and the sums of bytes and tokens."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        from paged_kv_cache_406_b200 import workloads as W
        w = bench.rank_workload(W.WORKLOADS["llama3_8b"], rank)
        lens = W.seq_lens(w)
        t, b, n = bench.combine_ranks(10.0 + 5 * rank, 1e9 * (rank + 1), 64.0, torch.device("cpu"))
        q.put((rank, t, b, n, w.seed, lens.tolist()))
    finally:
        dist.destroy_process_group()


def test_two_ranks_combine_and_own_batches():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    for _, t, b, n, _, _ in res:
        assert t == 15.0          # slowest rank
        assert b == 3e9           # bytes of both ranks
        assert n == 128.0         # tokens of both ranks
    (_, _, _, _, s0, l0), (_, _, _, _, s1, l1) = res
    assert s0 != s1 and l0 != l1  # independent batches
    assert len(l0) == len(l1) == 64


def test_single_process_combine_is_identity():
    import bench
    assert bench.combine_ranks(3.0, 7.0, 9.0, torch.device("cpu")) == (3.0, 7.0, 9.0)
