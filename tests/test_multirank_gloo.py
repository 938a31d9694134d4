"""Host logic of the multi-GPU benchmark path, on CPU with world size 2 (gloo).

Every rank runs an independent graph of the same size (weak scaling, no
collective on the data path); the timed region is reported as the max over
ranks and the edges as the sum."""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from workloads import SPECS, make_graph  # noqa: E402


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, queue):
    import datetime

    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        spec = bench.spec_for_rank("tiny", rank)
        g = make_graph(spec)
        times = [10.0 + rank, 3.0 * (rank + 1)]
        (t_max, f_max), edges = bench.reduce_over_ranks(times, g.num_edges, world)
        queue.put((rank, t_max, f_max, edges, g.num_edges, spec.graph_seed, spec.seed))
    finally:
        dist.destroy_process_group()


def test_two_rank_reduction_and_independent_graphs():
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, queue)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(queue.get(timeout=10) for _ in range(2))
    edges = [r[4] for r in res]
    for rank, t_max, f_max, total, _, gseed, seed in res:
        assert t_max == 11.0 and f_max == 6.0          # max over ranks
        assert total == sum(edges)                     # edges of all ranks
    assert res[0][5] != res[1][5] and res[0][6] != res[1][6]   # independent graphs and inputs
    assert edges[0] != edges[1] or res[0][5] != res[1][5]


def test_rank_zero_is_the_canonical_workload_and_single_rank_is_identity():
    for name in SPECS:
        assert bench.spec_for_rank(name, 0) == SPECS[name]
        assert bench.spec_for_rank(name, 3).graph_seed != SPECS[name].graph_seed
    (a, b), e = bench.reduce_over_ranks([1.5, 2.5], 123, 1)
    assert (a, b, e) == (1.5, 2.5, 123.0)
