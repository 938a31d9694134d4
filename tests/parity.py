"""Shared helpers of the GPU parity tests: input generation, oracle calls and
the error metric.

Error metric: for every flattened output column c = (component, channel),
scale_c = max_b |ref[b, c]| (1 if the column is all zero), and
err = max_{b,c} |gpu - ref| / scale_c.  The bars are 1e-5 for float32 inputs
and 5e-3 for float16 inputs (both accumulate in float32; the oracle consumes
the same rounded inputs upcast exactly to float64)."""
from __future__ import annotations

import numpy as np
import torch

import equivariant_graph_message_b200 as e3
import oracle
from workloads import SPECS, make_graph, node_features_np, node_features_torch, radial_weights, \
    scalars_np, scalars_torch
from workloads.configs import np_dtype

TOL = {"f32": 1e-5, "f16": 5e-3}


def edge_sh(spec, graph, edges=None) -> np.ndarray:
    """Y [E][ny] in the workload dtype: the oracle's harmonics of the edge vectors."""
    v = graph.vec if edges is None else graph.vec[np.asarray(edges)]
    u = v / np.linalg.norm(v, axis=1, keepdims=True)
    return oracle.sh(spec.lmax, u).astype(np_dtype(spec))


def edge_scalars(spec, graph, edges=None) -> np.ndarray:
    """s [E][P][C] in the workload dtype: drawn, or the oracle's radial MLP of the edge
    lengths with the workload's seeded weights."""
    if spec.scalars == "normal":
        return scalars_np(spec, graph, edges)
    v = graph.vec if edges is None else graph.vec[np.asarray(edges)]
    s = oracle.radial_mlp(np.linalg.norm(v, axis=1), spec.graph["r"], radial_weights(spec))
    return s.reshape(len(v), spec.num_paths, spec.C).astype(np_dtype(spec))


def workload_inputs(spec, graph):
    """(x, Y, s) of a workload on the host, in its dtype."""
    return node_features_np(spec, graph.num_nodes), edge_sh(spec, graph), edge_scalars(spec, graph)


def column_scaled_error(gpu: np.ndarray, ref: np.ndarray) -> float:
    g = gpu.reshape(gpu.shape[0], -1).astype(np.float64)
    r = ref.reshape(ref.shape[0], -1)
    scale = np.abs(r).max(axis=0) if len(r) else np.ones(r.shape[1])
    scale = np.where(scale == 0, 1.0, scale)
    return float((np.abs(g - r) / scale).max()) if g.size else 0.0


def abs_bound(irreps, x, Y, s, senders, receivers, num_nodes, avg, norm="SQRT_DIM_OUT"):
    """Elementwise float32 error bound of the kernel's arithmetic.

    The kernel sums, for each output element, every product s*c*x*Y of every
    edge of its row in one float32 chain of length L (recursive summation,
    Higham's bound gamma_L = L u / (1 - L u), u = 2^-24), after rounding the
    CG constant, c*Y and s*x (or c*Y*x) once each (3u).  With
    A = (1/N) sum |s| |c| |x| |Y| (the same sum over absolute values):
        |gpu - exact| <= (gamma_L + 3u) A  (+ the float64 oracle's own error).
    L is bounded by (max row degree) x (max terms per edge of one element)."""
    pl = oracle.plan(*irreps)
    u = 2.0 ** -24
    A = np.zeros((num_nodes, pl.nout, pl.C))
    terms = np.zeros(pl.nout)
    for p, path in enumerate(pl.paths):
        W = np.abs(oracle.cg(path.l1, path.l2, path.l3, norm))
        terms[path.out_off:path.out_off + 2 * path.l3 + 1] += (W > 1e-12).sum(axis=(0, 1))
        xa = np.abs(np.asarray(x, np.float64)[senders][:, path.x_off:path.x_off + 2 * path.l1 + 1])
        ye = np.abs(np.asarray(Y, np.float64)[:, path.y_off:path.y_off + 2 * path.l2 + 1])
        msg = np.einsum("ijk,eiu,ej,eu->eku", W, xa, ye, np.abs(np.asarray(s, np.float64)[:, p]))
        np.add.at(A[:, path.out_off:path.out_off + 2 * path.l3 + 1, :], receivers, msg)
    deg = np.bincount(receivers, minlength=num_nodes).max() if len(receivers) else 0
    L = deg * terms.max() + 2
    gamma = L * u / (1 - L * u)
    return (gamma + 3 * u) * A / avg


def row_ptr_of(receivers: np.ndarray, num_nodes: int) -> np.ndarray:
    counts = np.bincount(receivers, minlength=num_nodes) if len(receivers) else \
        np.zeros(num_nodes, np.int64)
    rp = np.zeros(num_nodes + 1, np.int64)
    np.cumsum(counts, out=rp[1:])
    return rp


def to_dev(a, dtype=None, device="cuda"):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.to(dtype)
    return t.to(device)


def run_gpu(conv: e3.Conv, x, Y, s, senders, receivers, num_nodes, prefill=float("nan")):
    """Receiver-sorted host arrays -> GPU output (host, float32)."""
    tdt = torch.float16 if conv.dtype == "f16" else torch.float32
    rp = row_ptr_of(np.asarray(receivers), num_nodes)
    out = torch.full((num_nodes, conv.nout, conv.C), prefill, dtype=torch.float32, device="cuda")
    conv.forward(to_dev(x, tdt), to_dev(Y, tdt), to_dev(s, tdt),
                 to_dev(np.asarray(senders, np.int32)), to_dev(rp.astype(np.int32)), out=out)
    torch.cuda.synchronize()
    assert conv.check()
    return out.cpu().numpy()


def oracle_out(irreps, x, Y, s, senders, receivers, num_nodes, avg, norm="SQRT_DIM_OUT"):
    return oracle.forward(*irreps, np.asarray(x, np.float64), np.asarray(Y, np.float64),
                          np.asarray(s, np.float64), senders, receivers, num_nodes, avg, norm)


class DeviceWorkload:
    """A full-size workload generated on the device, as the benchmark times it."""

    def __init__(self, name: str, device="cuda", nodes: int | None = None):
        self.spec = spec = SPECS[name]
        self.graph = g = make_graph(spec, nodes)
        self.N, self.E = g.num_nodes, g.num_edges
        tdt = torch.float16 if spec.dtype == "f16" else torch.float32
        self.x = node_features_torch(spec, g.num_nodes, device)
        self.Y = torch.from_numpy(edge_sh(spec, g)).to(device)
        self.s = scalars_torch(spec, g, device) if spec.scalars == "normal" else \
            torch.from_numpy(edge_scalars(spec, g)).to(device)
        self.senders = torch.from_numpy(g.senders.astype(np.int32)).to(device)
        self.receivers = torch.from_numpy(g.receivers.astype(np.int32)).to(device)
        self.row_ptr = torch.from_numpy(row_ptr_of(g.receivers, g.num_nodes).astype(np.int32)).to(device)
        assert self.x.dtype == tdt and self.Y.dtype == tdt and self.s.dtype == tdt
        self.conv = e3.Conv(spec.irreps_node, spec.irreps_sh, spec.irreps_out,
                            g.avg_num_neighbors, dtype=spec.dtype)

    @property
    def irreps(self):
        return (self.spec.irreps_node, self.spec.irreps_sh, self.spec.irreps_out)

    def sample_reference(self, receivers: np.ndarray) -> np.ndarray:
        """Oracle output rows for the given receivers, from the device inputs."""
        g = self.graph
        rp = row_ptr_of(g.receivers, g.num_nodes)
        edges = np.concatenate([np.arange(rp[b], rp[b + 1]) for b in receivers]) \
            if len(receivers) else np.zeros(0, np.int64)
        senders = g.senders[edges]
        uniq, inv = np.unique(senders, return_inverse=True)
        x = self.x[torch.from_numpy(uniq).to(self.x.device)].cpu().numpy()
        eidx = torch.from_numpy(edges).to(self.s.device)
        Y = self.Y[eidx].cpu().numpy()
        s = self.s[eidx].cpu().numpy()
        local_recv = np.repeat(np.arange(len(receivers)), np.diff(rp)[receivers])
        # sample rows: receivers 0..len-1; senders remapped into the gathered x rows
        xr = np.zeros((max(len(receivers), len(uniq)),) + x.shape[1:], x.dtype)
        xr[:len(uniq)] = x
        out = oracle_out(self.irreps, xr, Y, s, inv, local_recv, len(xr), g.avg_num_neighbors)
        return out[:len(receivers)]
