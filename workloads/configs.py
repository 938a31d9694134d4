"""The five synthetic workloads of the convolution, and their input tensors.

Inputs of workload w (all seeded, see rng.py for the generator):

* graph: points and radius graph from graphs.py, edges sorted by (receiver,
  sender); edge e is the e-th edge of that order.
* node features x[a, i, u] = normal(seed, TID_X, (a * nx + i) * C + u).
* edge vectors r_ab = p_b - p_a (float64 on the host; float32 [E][4] with a zero
  fourth component for the device, `edge_vectors_np`).
* edge scalars s[e, p, u] = normal(seed, TID_S, (e * P + p) * C + u), or, for
  the MACE-like layer (scalars="radial"), the radial MLP of |r_ab| with the
  seeded weights `radial_weights` (normal draws / sqrt(fan-in)).
* avg_num_neighbors = E / N, the measured mean degree.

The edge features Y (spherical harmonics of r_ab) and the radial scalars are
functions the method itself computes, so this module does not: each side
evaluates them with its own implementation (the oracle's, or the library's
kernels) from the edge vectors and weights drawn here.

Every drawn tensor is rounded once from float64 to the workload dtype
(float32 or float16); consumers that need float64 upcast the rounded values
exactly.  The layout is trailing channels: x [N][nx][C], Y [E][ny], s [E][P][C].
"""
from __future__ import annotations

from dataclasses import dataclass, field
from math import sqrt

import numpy as np

from . import graphs, rng

TID_POS = 0
TID_X = 1
TID_S = 2
TID_W = 10  # radial MLP weights use TID_W + layer


@dataclass(frozen=True)
class Spec:
    name: str
    irreps_node: str
    lmax: int
    irreps_out: str
    C: int
    nx: int          # sum of (2l+1) over node irreps
    num_paths: int   # P, number of uvu paths (scalars per edge and channel)
    dtype: str       # 'f32' or 'f16'
    graph: dict = field(default_factory=dict)
    graph_seed: int = 0
    seed: int = 0
    scalars: str = "normal"   # or 'radial' (the radial MLP of the edge lengths)
    description: str = ""

    @property
    def irreps_sh(self) -> str:
        return "+".join(f"1x{l}{'e' if l % 2 == 0 else 'o'}" for l in range(self.lmax + 1))

    @property
    def ny(self) -> int:
        return (self.lmax + 1) ** 2


SPECS = {
    "tiny": Spec(
        "tiny", "4x0e+4x1o", 2, "4x0e+4x1o+4x1e+4x2e", C=4, nx=4, num_paths=8, dtype="f32",
        graph=dict(kind="cube", n=24, box=2.0, r=1.0, periodic=False), graph_seed=1, seed=1,
        description="24 nodes in a cube of side 2, r=1.0; 4x0e+4x1o, Y l<=2, float32"),
    "gate_points": Spec(
        "gate_points", "5x0e+5x0o+5x1e+5x1o", 3, "5x0e+5x0o+5x1e+5x1o+5x2e+5x2o", C=5, nx=8,
        num_paths=20, dtype="f32",
        graph=dict(kind="batched", graphs=512, nodes=20, box=3.0, r=2.0), graph_seed=2, seed=2,
        description="512 graphs x 20 nodes, cube side 3, r=2.0; 5x(0e+0o+1e+1o), Y l<=3, float32"),
    "mace": Spec(
        "mace", "128x0e+128x1o", 3, "128x0e+128x1o+128x2e+128x3o", C=128, nx=4, num_paths=10,
        dtype="f32",
        graph=dict(kind="cube", n=5000, box=44.36, r=5.0, periodic=True), graph_seed=3, seed=3,
        scalars="radial",
        description="5000 nodes, periodic box 44.36, r=5.0 (~30 neighbours); 128x(0e+1o), Y l<=3, "
                    "s = 2-layer SiLU MLP(64) on 8 Bessel bases x cosine cutoff, float32"),
    "large_f32": Spec(
        "large_f32", "64x0e+64x1o+64x2e", 3, "64x0e+64x0o+64x1e+64x1o+64x2e+64x2o", C=64, nx=9,
        num_paths=18, dtype="f32",
        graph=dict(kind="cube", n=100000, box=21.878, r=1.0, periodic=True), graph_seed=4, seed=4,
        description="100000 nodes, periodic box 21.878, r=1.0 (~40 neighbours, ~4.0M edges); "
                    "64x(0e+1o+2e), Y l<=3, out l<=2, float32"),
    "large_f16": Spec(
        "large_f16", "128x0e+128x1o+128x2e+128x3o", 3,
        "128x0e+128x0o+128x1e+128x1o+128x2e+128x2o+128x3e+128x3o", C=128, nx=16, num_paths=34,
        dtype="f16",
        graph=dict(kind="cube", n=100000, box=21.878, r=1.0, periodic=True), graph_seed=4, seed=5,
        description="same graph as large_f32; 128x(0e+1o+2e+3o), Y l<=3, out l<=3, float16 "
                    "x/Y/s with float32 accumulation and output"),
}

ORDER = ["tiny", "gate_points", "mace", "large_f32", "large_f16"]


@dataclass
class Graph:
    num_nodes: int
    pos: np.ndarray
    senders: np.ndarray     # int64 [E], sorted by (receiver, sender)
    receivers: np.ndarray   # int64 [E]
    vec: np.ndarray         # float64 [E, 3], r_ab = p_b - p_a

    @property
    def num_edges(self) -> int:
        return len(self.senders)

    @property
    def avg_num_neighbors(self) -> float:
        return self.num_edges / self.num_nodes if self.num_nodes else 1.0


_graph_cache: dict = {}


def make_graph(spec: Spec, nodes: int | None = None) -> Graph:
    """The spec's graph; `nodes` overrides the node count at the same density."""
    g = dict(spec.graph)
    key = (spec.graph_seed, tuple(sorted(g.items())), nodes)
    if key in _graph_cache:
        return _graph_cache[key]
    if g["kind"] == "batched":
        graphs_n = g["graphs"] if nodes is None else max(1, nodes // g["nodes"])
        pos, s, r, v = graphs.batched_graphs(spec.graph_seed, TID_POS, graphs_n, g["nodes"],
                                             g["box"], g["r"])
        n = graphs_n * g["nodes"]
    else:
        n = g["n"] if nodes is None else nodes
        box = g["box"] * (n / g["n"]) ** (1.0 / 3.0)
        pos = graphs.uniform_points(spec.graph_seed, TID_POS, n, box)
        s, r, v = graphs.radius_graph_cells(pos, g["r"], box if g["periodic"] else None)
    out = Graph(n, pos, s, r, v)
    _graph_cache[key] = out
    return out


def np_dtype(spec: Spec):
    return np.float16 if spec.dtype == "f16" else np.float32


def torch_dtype(spec: Spec):
    import torch
    return torch.float16 if spec.dtype == "f16" else torch.float32


def edge_vectors_np(graph: Graph, e0: int = 0, e1: int | None = None) -> np.ndarray:
    """float32 [e1-e0][4]: (x, y, z, 0) of r_ab for edges e0..e1-1 (the device layout)."""
    e1 = graph.num_edges if e1 is None else e1
    v = np.zeros((e1 - e0, 4), np.float32)
    v[:, :3] = graph.vec[e0:e1]
    return v


def node_features_np(spec: Spec, num_nodes: int, rows: np.ndarray | None = None) -> np.ndarray:
    """Host x[rows] ([len(rows)][nx][C]); rows default to all nodes."""
    rows = np.arange(num_nodes) if rows is None else np.asarray(rows)
    k = (rows[:, None, None] * spec.nx + np.arange(spec.nx)[None, :, None]) * spec.C \
        + np.arange(spec.C)[None, None, :]
    return rng.normal_np(spec.seed, TID_X, k.astype(np.uint64)).astype(np_dtype(spec))


def node_features_torch(spec: Spec, num_nodes: int, device, first: int = 0):
    """x[first : first + num_nodes] on the device (the whole table by default)."""
    per = spec.nx * spec.C
    return rng.normal_torch(spec.seed, TID_X, num_nodes * per, torch_dtype(spec), device,
                            start=first * per).view(num_nodes, spec.nx, spec.C)


# --- edge scalars ------------------------------------------------------------

RADIAL_BASIS = 8      # bessel bases of the MACE-like layer's radial MLP
RADIAL_HIDDEN = 64    # neurons of each of its two hidden layers


def radial_weights(spec: Spec):
    """The seeded MLP weights [W_0 (8 x 64), W_1 (64 x 64), W_2 (64 x P*C)], float64."""
    sizes = [RADIAL_BASIS, RADIAL_HIDDEN, RADIAL_HIDDEN, spec.num_paths * spec.C]
    ws = []
    for layer, (fi, fo) in enumerate(zip(sizes[:-1], sizes[1:])):
        w = rng.normal_np(spec.seed, TID_W + layer, np.arange(fi * fo, dtype=np.uint64))
        ws.append(w.reshape(fi, fo) / sqrt(fi))
    return ws


def _drawn_scalars(spec: Spec):
    if spec.scalars != "normal":
        raise ValueError(f"{spec.name}: the edge scalars are the radial MLP of the edge lengths; "
                         "evaluate it from edge_vectors_np and radial_weights")


def scalars_np(spec: Spec, graph: Graph, edges: np.ndarray | None = None) -> np.ndarray:
    """Host s[edges] ([len(edges)][P][C]) in the spec dtype; edges default to all."""
    _drawn_scalars(spec)
    P, C = spec.num_paths, spec.C
    edges = np.arange(graph.num_edges) if edges is None else np.asarray(edges)
    k = (edges[:, None, None] * P + np.arange(P)[None, :, None]) * C + np.arange(C)[None, None, :]
    return rng.normal_np(spec.seed, TID_S, k.astype(np.uint64)).astype(np_dtype(spec))


def scalars_torch(spec: Spec, graph: Graph, device, edges: tuple | None = None):
    """s[e0:e1] on the device for edges = (e0, e1) (all edges by default)."""
    import torch
    _drawn_scalars(spec)
    e0, e1 = edges if edges is not None else (0, graph.num_edges)
    P, C = spec.num_paths, spec.C
    return rng.normal_torch(spec.seed, TID_S, (e1 - e0) * P * C, torch_dtype(spec), device,
                            start=e0 * P * C).view(e1 - e0, P, C)
