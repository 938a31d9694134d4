"""Multi-rank path on CPU: receiver sharding of one graph over world-size-2 gloo
ranks (the host logic and the exchange step the GPU ranks run over NCCL).

* The row partition covers every receiver exactly once and balances edges
  + rows (e3conv_partition_rows).
* Each rank's sender table holds exactly the node rows its edges name: for the
  halo exchange the table IS the set of distinct senders of the rank's edges;
  for the all-gather every sender row is where the renumbered senders point.
* The oracle run on each rank's shard (its rows' edges, the received table,
  the renumbered senders) gives bitwise the rows of the oracle run on the
  whole graph, and the ranks' outputs concatenated are the whole output.
* Timings are reduced as the max over ranks, edges as the sum."""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import equivariant_graph_message_b200 as e3  # noqa: E402
from equivariant_graph_message_b200 import sharding  # noqa: E402

IRREPS = ("3x0e+3x1o", "1x0e+1x1o+1x2e", "3x0e+3x1o+3x1e+3x2e")


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _graph(seed, n, e, hub=None, empty_frac=0.2):
    rng = np.random.default_rng(seed)
    pool = np.nonzero(rng.random(n) >= empty_frac)[0]
    recv = pool[rng.integers(0, len(pool), e)]
    if hub is not None:
        recv[: e // 4] = hub
    send = rng.integers(0, n, e)
    o = np.lexsort((send, recv))
    rp = np.zeros(n + 1, np.int64)
    np.cumsum(np.bincount(recv, minlength=n), out=rp[1:])
    return send[o], recv[o], rp


def _inputs(seed, n, e):
    import oracle
    pl = oracle.plan(*IRREPS)
    rng = np.random.default_rng(seed + 1)
    return (rng.normal(size=(n, pl.nx, pl.C)), rng.normal(size=(e, pl.ny)),
            rng.normal(size=(e, len(pl.paths), pl.C)))


@pytest.mark.parametrize("parts", [1, 2, 3, 5, 8])
@pytest.mark.parametrize("kind", ["random", "hub", "no_edges", "one_node"])
def test_partition_covers_every_row_once_and_balances(kind, parts):
    n, e = {"random": (500, 9000), "hub": (400, 8000), "no_edges": (50, 0),
            "one_node": (1, 30)}[kind]
    if e:
        _, _, rp = _graph(7, n, e, hub=3 if kind == "hub" else None)
    else:
        rp = np.zeros(n + 1, np.int64)
    b = e3.partition_rows(rp.astype(np.int32), parts)
    assert len(b) == parts + 1 and b[0] == 0 and b[-1] == n
    assert np.all(np.diff(b) >= 0)
    owner = np.searchsorted(b, np.arange(n), side="right") - 1     # every row: exactly one range
    assert np.all((b[owner] <= np.arange(n)) & (np.arange(n) < b[owner + 1]))
    cost = rp - rp[0] + np.arange(n + 1)
    row_cost = np.diff(rp) + 1
    worst = row_cost.max() if n else 0
    for r in range(1, parts):                  # every boundary within one row of its share
        assert abs(cost[b[r]] - cost[-1] * r / parts) <= worst
    part = np.diff(cost[b])
    assert part.max() - cost[-1] / parts <= 2 * worst


def test_partition_rejects_bad_row_ptr():
    with pytest.raises(e3.E3ConvError):
        e3.partition_rows(np.array([0, 5, 3], np.int32), 2)
    with pytest.raises(e3.E3ConvError):
        e3.partition_rows(np.array([0, 1], np.int32), 0)


def _rank_main(rank, world, port, queue):
    import datetime

    import torch
    import torch.distributed as dist

    import oracle
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        results = []
        n, e, avg = 300, 5000, 17.0
        send, recv, rp = _graph(11, n, e, hub=5)
        x, Y, s = _inputs(11, n, e)            # the same seeded inputs on every rank
        whole = oracle.forward(*IRREPS, x, Y, s, send, recv, n, avg)
        for exchange in sharding.EXCHANGES:
            sh = sharding.shard_graph(rp, send, rank, world, exchange,
                                      requests=sharding.torch_requests())
            b0, b1 = int(sh.bounds[rank]), int(sh.bounds[rank + 1])
            own = x[b0:b1]                      # the node rows this rank owns
            if exchange == "allgather":
                block = np.zeros((sh.block_rows,) + x.shape[1:])
                block[:len(own)] = own
                table = torch.empty((world * sh.block_rows,) + x.shape[1:], dtype=torch.float64)
                sharding.exchange_rows(sh, torch.from_numpy(block), table)
            else:
                packed = own[sh.send_idx]       # what pack_halo gathers on the device
                table = torch.empty((sh.table_rows,) + x.shape[1:], dtype=torch.float64)
                sharding.exchange_rows(sh, torch.from_numpy(np.ascontiguousarray(packed)), table)
            table = table.numpy()
            snd_local = send[sh.edge_begin:sh.edge_end]
            named = np.unique(snd_local)
            if exchange == "halo":             # exactly the senders its edges name
                halo_exact = (sh.table_rows == len(named)
                              and np.array_equal(sh.needed, named)
                              and np.array_equal(table, x[named]))
            else:
                halo_exact = True
            rows_ok = np.array_equal(table[sh.senders], x[snd_local])
            # the oracle on the shard: local receivers 0..rows-1, the received table
            rows = sh.rows
            lrecv = np.repeat(np.arange(rows), np.diff(sh.row_ptr))
            t = np.zeros((max(rows, len(table)),) + x.shape[1:])
            t[:len(table)] = table
            out = oracle.forward(*IRREPS, t, Y[sh.edge_begin:sh.edge_end],
                                 s[sh.edge_begin:sh.edge_end], sh.senders, lrecv, len(t), avg)[:rows]
            same = np.array_equal(out, whole[b0:b1])
            # concatenation of all ranks' rows (padded all-gather of the outputs)
            pad = int(np.diff(sh.bounds).max())
            mine = np.zeros((pad,) + out.shape[1:])
            mine[:rows] = out
            got = [torch.empty(mine.shape, dtype=torch.float64) for _ in range(world)]
            dist.all_gather(got, torch.from_numpy(mine))
            cat = np.concatenate([got[q].numpy()[:int(sh.bounds[q + 1] - sh.bounds[q])]
                                  for q in range(world)])
            results.append((exchange, bool(halo_exact), bool(rows_ok), bool(same),
                            bool(np.array_equal(cat, whole)), rows, sh.edge_end - sh.edge_begin))
        (t_max,), edges = bench.reduce_over_ranks([10.0 + rank], 100 + rank, world)
        queue.put((rank, results, t_max, edges))
    finally:
        dist.destroy_process_group()


def test_two_rank_sharding_equals_the_whole_graph():
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, queue)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    res = sorted(queue.get(timeout=10) for _ in range(2))
    edges = {ex: 0 for ex in sharding.EXCHANGES}
    for rank, results, t_max, total in res:
        assert t_max == 11.0 and total == 201.0       # max of times, sum of edges over ranks
        assert len(results) == 2
        for exchange, halo_exact, rows_ok, same, cat_ok, rows, ne in results:
            assert halo_exact, (rank, exchange)
            assert rows_ok, (rank, exchange)
            assert same, (rank, exchange)
            assert cat_ok, (rank, exchange)
            assert rows > 0
            edges[exchange] += ne
    assert edges["allgather"] == edges["halo"] == 5000


def test_single_rank_reduction_is_identity():
    (a, b), e = bench.reduce_over_ranks([1.5, 2.5], 123, 1)
    assert (a, b, e) == (1.5, 2.5, 123.0)


def test_single_process_shards_cover_the_graph():
    # without any process group: every rank's all-gather shard, built alone, renumbers its
    # senders into the padded table consistently, and the ranks' edges tile the edge list
    send, recv, rp = _graph(4, 200, 3000, hub=7)
    world = 3
    bounds = e3.partition_rows(rp.astype(np.int32), world)
    e_seen = 0
    for r in range(world):
        sh = sharding.shard_graph(rp, send, r, world, "allgather", bounds=bounds)
        assert sh.edge_begin == e_seen
        e_seen = sh.edge_end
        owner = np.searchsorted(bounds, send[sh.edge_begin:sh.edge_end], side="right") - 1
        back = bounds[owner] + (sh.senders.astype(np.int64) - owner * sh.block_rows)
        assert np.array_equal(back, send[sh.edge_begin:sh.edge_end])
        assert sh.table_rows == world * sh.block_rows
        assert np.array_equal(sh.row_ptr, rp[sh.row_begin:sh.row_end + 1] - rp[sh.row_begin])
    assert e_seen == len(send)
    with pytest.raises(ValueError):
        sharding.shard_graph(rp, send, 0, world, "halo", bounds=bounds)    # no request exchange
