"""Receiver sharding of one graph over several ranks (one process per GPU).

The convolution shards along its receivers: every output row is one
receiver's sum over its incoming edges (page "e3j.core.Convolution",
"graph_ordering": with RECEIVER ordering each receiver's edges are one
contiguous segment), so ranks that own disjoint contiguous CSR row ranges
produce disjoint output rows and nothing is reduced afterwards.  A rank holds
its rows' edges (Y, s, senders) and, before each forward, needs the node
features of every sender its edges name.  That is the one exchange step:

* "allgather": every rank contributes the feature rows of the nodes it owns
  (the same row ranges), padded to the largest range, and receives all of
  them (one all-gather; NCCL runs it over NVLink / NVSwitch).  Senders are
  renumbered once into that padded table.
* "halo": every rank receives only the rows its edges name (one
  all-to-all of the requested rows; the requests are exchanged once per
  topology).  Senders are renumbered into that smaller table.

The partition is e3conv_partition_rows (ranges balanced on edges + rows); the
per-rank forward is e3conv_forward_rows over the rank's rebased row pointer.
Topology work (partition, renumbering, requests) runs once on the host; the
per-step work is the exchange plus one forward launch.  This module only
arranges indices and calls torch.distributed: the convolution's arithmetic
is in the library's kernels, and the halo rows are gathered by
e3conv_permute_rows.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

from . import partition_rows, permute_rows

EXCHANGES = ("allgather", "halo")


@dataclass
class RowShard:
    """What rank `rank` of `world` holds for one graph."""
    rank: int
    world: int
    exchange: str
    bounds: np.ndarray            # int64 [world+1]: rank q owns rows (and nodes) bounds[q]..bounds[q+1]-1
    row_begin: int
    row_end: int
    edge_begin: int               # the rank's edges are edge_begin..edge_end-1 of the graph's CSR order
    edge_end: int
    row_ptr: np.ndarray           # int32 [rows+1], the rank's rows, rebased to start at 0
    senders: np.ndarray           # int32 [local edges]: rows of the sender table this rank receives
    table_rows: int               # rows of that table
    block_rows: int               # allgather: rows of every rank's (padded) contribution
    # halo: rows (indices into this rank's own node block) sent to each rank, grouped by
    # destination, and the row counts exchanged with every rank
    send_idx: np.ndarray = field(default_factory=lambda: np.zeros(0, np.int32))
    send_counts: list = field(default_factory=list)
    recv_counts: list = field(default_factory=list)
    needed: np.ndarray = field(default_factory=lambda: np.zeros(0, np.int64))  # halo: global ids of the table rows

    @property
    def rows(self) -> int:
        return self.row_end - self.row_begin

    @property
    def own_rows(self) -> int:
        return int(self.bounds[self.rank + 1] - self.bounds[self.rank])


def _owner(bounds: np.ndarray, nodes: np.ndarray) -> np.ndarray:
    return np.searchsorted(bounds, nodes, side="right") - 1


def shard_graph(row_ptr: np.ndarray, senders: np.ndarray, rank: int, world: int,
                exchange: str = "allgather", bounds: np.ndarray | None = None,
                requests=None) -> RowShard:
    """The rank's shard of a receiver-sorted graph (host arrays: row_ptr [N+1], senders [E]).

    For "halo", `requests(counts, indices) -> (counts_in, indices_in)` performs the one-time
    exchange of requested row indices between ranks (see `torch_requests`); rank q's
    counts_in[r] rows of indices_in are the rows rank r asks q for, in q's local numbering."""
    if exchange not in EXCHANGES:
        raise ValueError(f"exchange must be one of {EXCHANGES}")
    row_ptr = np.asarray(row_ptr, dtype=np.int64)
    senders = np.asarray(senders, dtype=np.int64)
    N = len(row_ptr) - 1
    if bounds is None:
        bounds = partition_rows(row_ptr.astype(np.int32), world)
    bounds = np.asarray(bounds, dtype=np.int64)
    b0, b1 = int(bounds[rank]), int(bounds[rank + 1])
    e0, e1 = int(row_ptr[b0]), int(row_ptr[b1])
    local_rp = (row_ptr[b0:b1 + 1] - e0).astype(np.int32)
    snd = senders[e0:e1]
    if len(snd) and (snd.min() < 0 or snd.max() >= N):
        raise ValueError("sender outside [0, num_nodes)")
    block = int(np.diff(bounds).max()) if N else 0
    if exchange == "allgather":
        own = _owner(bounds, snd)
        local = own * block + (snd - bounds[own])
        return RowShard(rank, world, exchange, bounds, b0, b1, e0, e1, local_rp,
                        local.astype(np.int32), world * block, block)
    if requests is None:
        raise ValueError("the halo exchange needs `requests` (e.g. torch_requests()) to tell the "
                         "owners which rows each rank needs")
    needed = np.unique(snd)
    own = _owner(bounds, needed)
    recv_counts = np.bincount(own, minlength=world).astype(np.int64)
    want = (needed - bounds[own]).astype(np.int64)          # grouped by owner (needed is sorted)
    send_counts, send_idx = requests(recv_counts, want)
    local = np.searchsorted(needed, snd)
    return RowShard(rank, world, exchange, bounds, b0, b1, e0, e1, local_rp,
                    local.astype(np.int32), len(needed), block,
                    np.asarray(send_idx, dtype=np.int32), [int(c) for c in send_counts],
                    [int(c) for c in recv_counts], needed)


def torch_requests(group=None, device="cpu"):
    """The one-time request exchange of the halo shard, over torch.distributed."""
    import torch
    import torch.distributed as dist

    def exchange(counts, indices):
        c_out = torch.as_tensor(np.asarray(counts), dtype=torch.int64, device=device)
        c_in = torch.empty_like(c_out)
        dist.all_to_all_single(c_in, c_out, group=group)
        i_out = torch.as_tensor(np.asarray(indices), dtype=torch.int64, device=device)
        i_in = torch.empty(int(c_in.sum().item()), dtype=torch.int64, device=device)
        dist.all_to_all_single(i_in, i_out, output_split_sizes=c_in.tolist(),
                               input_split_sizes=c_out.tolist(), group=group)
        return c_in.cpu().numpy(), i_in.cpu().numpy()
    return exchange


# ---------------------------------------------------------------------------
# per-step exchange of node features

def pack_halo(x_own, send_idx_dev, out=None, stream=None):
    """The rows of this rank's own node block that the others asked for, grouped by
    destination (e3conv_permute_rows on the device)."""
    return permute_rows(x_own, send_idx_dev, dst=out, stream=stream)


def exchange_rows(shard: RowShard, send, table, group=None):
    """Fills the sender table: "allgather" sends `send` (this rank's padded node block,
    [block_rows][nx][C]) and receives every rank's block into `table`
    ([world * block_rows][nx][C]); "halo" sends the packed rows (pack_halo) and receives
    the rows this rank's edges name into `table` ([table_rows][nx][C], ascending node id)."""
    import torch.distributed as dist
    if shard.exchange == "allgather":
        if dist.get_backend(group) == "nccl":
            dist.all_gather_into_tensor(table, send, group=group)
        else:
            dist.all_gather(list(table.view(shard.world, *send.shape).unbind(0)), send, group=group)
        return table
    per_row = int(np.prod(table.shape[1:])) if table.dim() > 1 else 1
    dist.all_to_all_single(table.view(-1), send.reshape(-1),
                           output_split_sizes=[c * per_row for c in shard.recv_counts],
                           input_split_sizes=[c * per_row for c in shard.send_counts], group=group)
    return table
