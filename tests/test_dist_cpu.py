"""Host logic of the N > 1 benchmark path, on CPU with world-size-2 gloo ranks:
each rank filters its own channels (own seed, same shape) and the timing is
the max over ranks."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import bench
    from kalman_linear_attention_b200 import workloads as wl
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = bench.rank_workload(wl.WORKLOADS["tiny"], rank)
        x = wl.generate(w.with_shape(T=8))
        m = bench.max_over_ranks(10.0 + rank, dist)
        q.put((rank, w.seed, (w.B, w.T, w.H, w.N), float(x["a"][0, 0, 0, 0]), m))
    finally:
        dist.destroy_process_group()


def test_two_rank_replicas_and_max_timing():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, s0, sh0, a0, m0), (r1, s1, sh1, a1, m1) = res
    assert sh0 == sh1                      # same shape per rank (weak scaling)
    assert s0 != s1 and a0 != a1           # independent channels per rank
    assert m0 == m1 == 11.0                # max over ranks


def test_max_over_ranks_without_group():
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    assert bench.max_over_ranks(3.5, None) == 3.5
    assert bench.max_over_ranks(3.5, dist) == 3.5  # not initialised: identity
