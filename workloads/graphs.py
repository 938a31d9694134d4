"""Seeded point clouds and radius graphs (host, float64).

A directed edge a -> b (sender a, receiver b) exists iff a != b and the
distance |p_b - p_a| is strictly below the cutoff radius; periodic boxes use
the minimum-image convention.  Edges are returned sorted by (receiver,
sender), so the edge list is already in receiver-sorted (CSR) order.

The edge vector of a -> b is r_ab = p_b - p_a (from sender to receiver).
"""
from __future__ import annotations

import numpy as np

from .rng import uniform_np


def uniform_points(seed: int, tid: int, n: int, box: float) -> np.ndarray:
    """n points uniform in [0, box)^3; coordinate c of point i is draw 3i + c."""
    return uniform_np(seed, tid, np.arange(3 * n, dtype=np.uint64)).reshape(n, 3) * box


def _min_image(d: np.ndarray, box: float | None) -> np.ndarray:
    if box is None:
        return d
    return d - box * np.round(d / box)


def radius_graph_bruteforce(pos: np.ndarray, r: float, box: float | None = None,
                            batch: np.ndarray | None = None):
    """O(n^2) reference: returns (senders, receivers, vectors r_ab)."""
    n = len(pos)
    d = pos[None, :, :] - pos[:, None, :]          # d[b, a] = p_a - p_b
    d = _min_image(d, box)
    dist2 = np.einsum("bac,bac->ba", d, d)
    ok = dist2 < r * r
    np.fill_diagonal(ok, False)
    if batch is not None:
        ok &= batch[None, :] == batch[:, None]
    recv, send = np.nonzero(ok)                   # row-major: sorted by (b, a)
    vec = pos[recv] - pos[send]
    if box is not None:
        vec = _min_image(vec, box)
    return send.astype(np.int64), recv.astype(np.int64), vec


def radius_graph_cells(pos: np.ndarray, r: float, box: float | None = None):
    """Cell-list radius graph; same result as the brute force, O(n)."""
    n = len(pos)
    if n == 0:
        z = np.zeros(0, np.int64)
        return z, z, np.zeros((0, 3))
    if box is not None:
        m = int(np.floor(box / r))
        if m < 3:
            return radius_graph_bruteforce(pos, r, box)
        cell_size = box / m
        lo = np.zeros(3)
        dims = np.array([m, m, m])
        p = np.mod(pos, box)
    else:
        lo = pos.min(axis=0)
        span = pos.max(axis=0) - lo
        dims = np.maximum(1, np.floor(span / r).astype(np.int64) + 1)
        cell_size = r
        p = pos
    ci = np.floor((p - lo) / cell_size).astype(np.int64)
    ci = np.minimum(ci, dims - 1)
    cid = (ci[:, 0] * dims[1] + ci[:, 1]) * dims[2] + ci[:, 2]
    order = np.argsort(cid, kind="stable")
    ncell = int(dims.prod())
    counts = np.bincount(cid, minlength=ncell)
    start = np.zeros(ncell + 1, np.int64)
    np.cumsum(counts, out=start[1:])
    sends, recvs = [], []
    for dx in (-1, 0, 1):
        for dy in (-1, 0, 1):
            for dz in (-1, 0, 1):
                nb = ci + np.array([dx, dy, dz])
                if box is not None:
                    nb = np.mod(nb, dims)
                    valid = np.ones(n, bool)
                else:
                    valid = np.all((nb >= 0) & (nb < dims), axis=1)
                ncid = (nb[:, 0] * dims[1] + nb[:, 1]) * dims[2] + nb[:, 2]
                recv_idx = np.nonzero(valid)[0]
                nc = ncid[recv_idx]
                cnt = counts[nc]
                tot = int(cnt.sum())
                if tot == 0:
                    continue
                rr = np.repeat(recv_idx, cnt)
                base = np.repeat(start[nc], cnt)
                offs = np.arange(tot) - np.repeat(np.cumsum(cnt) - cnt, cnt)
                ss = order[base + offs]
                d = _min_image(pos[ss] - pos[rr], box)
                keep = (np.einsum("ec,ec->e", d, d) < r * r) & (ss != rr)
                sends.append(ss[keep])
                recvs.append(rr[keep])
    send = np.concatenate(sends) if sends else np.zeros(0, np.int64)
    recv = np.concatenate(recvs) if recvs else np.zeros(0, np.int64)
    # Periodic boxes with m == 3 visit the same neighbour cell from several
    # offsets; drop duplicate (receiver, sender) pairs.
    key = recv * n + send
    key = np.unique(key)
    recv, send = key // n, key % n
    vec = _min_image(pos[recv] - pos[send], box)
    return send.astype(np.int64), recv.astype(np.int64), vec


def batched_graphs(seed: int, tid: int, graphs: int, nodes: int, box: float, r: float):
    """`graphs` independent clouds of `nodes` points; node ids nodes*g .. nodes*g+nodes-1."""
    pos = uniform_points(seed, tid, graphs * nodes, box)
    p = pos.reshape(graphs, nodes, 3)
    d = p[:, None, :, :] - p[:, :, None, :]      # d[g, b, a] = p_a - p_b
    ok = np.einsum("gbac,gbac->gba", d, d) < r * r
    idx = np.arange(nodes)
    ok[:, idx, idx] = False
    g, b, a = np.nonzero(ok)                      # sorted by (g, b, a)
    recv = g * nodes + b
    send = g * nodes + a
    vec = pos[recv] - pos[send]
    return pos, send.astype(np.int64), recv.astype(np.int64), vec
