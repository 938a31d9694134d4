"""GPU parity of the forward with edge vectors as input (E3CONV_OPT_EDGE_VECTORS):
the kernel evaluates the real spherical harmonics of r_ab / |r_ab| itself.
The reference is the oracle fed with the oracle's own harmonics (Rodrigues
polynomial, float64) of the same float32 vectors, so this checks the in-kernel
harmonics and the convolution together; all variants (direct, staged, path
split, tensor cores), a zero-length vector, and the full-size workloads."""
import numpy as np
import pytest
import torch

import equivariant_graph_message_b200 as e3
import oracle
from parity import TOL, DeviceWorkload, column_scaled_error, edge_scalars, oracle_out, row_ptr_of, \
    to_dev
from workloads import SPECS, make_graph, node_features_np

pytestmark = pytest.mark.gpu


def _vec4(vec):
    v = np.zeros((len(vec), 4), np.float32)
    v[:, :3] = vec
    return v


def _oracle_sh(lmax, vec4):
    v = vec4[:, :3].astype(np.float64)
    n = np.linalg.norm(v, axis=1, keepdims=True)
    Y = oracle.sh(lmax, np.where(n > 0, v / np.where(n > 0, n, 1), 0.0))
    Y[n[:, 0] == 0] = 0.0
    Y[n[:, 0] == 0, 0] = 1.0
    return Y


def _run(conv, x, vec4, s, senders, receivers, n):
    rp = row_ptr_of(np.asarray(receivers), n)
    tdt = torch.float16 if conv.dtype == "f16" else torch.float32
    out = conv.forward(to_dev(x, tdt), to_dev(vec4), to_dev(s, tdt),
                       to_dev(np.asarray(senders, np.int32)), to_dev(rp.astype(np.int32)))
    torch.cuda.synchronize()
    assert conv.check()
    return out.cpu().numpy()


@pytest.mark.parametrize("name", ["tiny", "gate_points", "mace"])
def test_edge_vectors_full_graphs(cuda_device, name):
    spec = SPECS[name]
    g = make_graph(spec)
    x = node_features_np(spec, g.num_nodes)
    s = edge_scalars(spec, g)
    v4 = _vec4(g.vec)
    irreps = (spec.irreps_node, spec.irreps_sh, spec.irreps_out)
    conv = e3.Conv(*irreps, g.avg_num_neighbors, dtype=spec.dtype)
    conv.set_edge_vectors(1)
    gpu = _run(conv, x, v4, s, g.senders, g.receivers, g.num_nodes)
    ref = oracle_out(irreps, x, _oracle_sh(spec.lmax, v4), s, g.senders, g.receivers,
                     g.num_nodes, g.avg_num_neighbors)
    assert column_scaled_error(gpu, ref) <= TOL[spec.dtype]


SH3 = "1x0e+1x1o+1x2e+1x3o"


@pytest.mark.parametrize("mode", ["direct", "staged", "staged_split", "tensor_cores", "lmax6"])
def test_edge_vectors_every_variant(cuda_device, mode):
    rng = np.random.default_rng(hash(mode) % 1000)
    irreps = {
        "direct": ("5x0e+5x1o", SH3, "5x0e+5x1o+5x2e"),
        "staged": ("64x0e+64x1o+64x2e", SH3, "64x0e+64x1o+64x2e"),
        "staged_split": ("128x0e+128x1o+128x2e+128x3o", SH3, "128x0e+128x1o+128x2e+128x3o"),
        "tensor_cores": ("128x0e+128x1o+128x2e+128x3o", SH3, "128x0e+128x1o+128x2e+128x3o"),
        "lmax6": ("32x0e+32x1o", "+".join(f"1x{l}{'eo'[l % 2]}" for l in range(7)),
                  "32x0e+32x1o+32x5o+32x6e"),
    }[mode]
    dt = "f16" if mode == "tensor_cores" else "f32"
    n, e = 500, 8000
    recv = rng.integers(0, n, e)
    send = rng.integers(0, n, e)
    o = np.lexsort((send, recv))
    send, recv = send[o], recv[o]
    conv = e3.Conv(*irreps, 16.0, dtype=dt)
    if mode == "staged_split":
        conv.set_path_split(2)
    if mode == "tensor_cores":
        conv.set_tensor_cores(1)
    conv.set_edge_vectors(1)
    info = conv.kernel_info()
    if mode == "direct":
        assert info["stages"] == 0
    if mode == "tensor_cores":
        assert info["tensor_cores"] == 1
    npdt = np.float16 if dt == "f16" else np.float32
    x = rng.normal(size=(n, conv.nx, conv.C)).astype(npdt)
    s = rng.normal(size=(e, conv.num_paths, conv.C)).astype(npdt)
    vec = rng.normal(size=(e, 3)) * rng.uniform(0.1, 3.0, size=(e, 1))
    vec[5] = 0.0                                    # a zero-length edge vector: Y = (1, 0, ...)
    v4 = _vec4(vec)
    gpu = _run(conv, x, v4, s, send, recv, n)
    lmax = int(round(np.sqrt(conv.ny))) - 1
    ref = oracle_out(irreps, x, _oracle_sh(lmax, v4), s, send, recv, n, 16.0)
    assert column_scaled_error(gpu, ref) <= 1e-5


@pytest.mark.parametrize("name", ["large_f32", "large_f16"])
def test_edge_vectors_full_size_sampled(cuda_device, name):
    w = DeviceWorkload(name)
    v4 = torch.from_numpy(_vec4(w.graph.vec)).cuda()
    w.conv.set_edge_vectors(1)
    out = w.conv.forward(w.x, v4, w.s, w.senders, w.row_ptr)
    torch.cuda.synchronize()
    assert w.conv.check()
    rng = np.random.default_rng(777)
    rows = np.unique(np.concatenate([[0, w.N - 1], rng.choice(w.N, 128, replace=False)]))
    # the sampled rows' oracle with the oracle's harmonics of the same float32 vectors
    g = w.graph
    rp = row_ptr_of(g.receivers, g.num_nodes)
    edges = np.concatenate([np.arange(rp[b], rp[b + 1]) for b in rows])
    uniq, inv = np.unique(g.senders[edges], return_inverse=True)
    x = w.x[torch.from_numpy(uniq).cuda()].cpu().numpy()
    s = w.s[torch.from_numpy(edges).cuda()].cpu().numpy()
    Y = _oracle_sh(w.spec.lmax, _vec4(g.vec[edges]))
    lrecv = np.repeat(np.arange(len(rows)), np.diff(rp)[rows])
    xr = np.zeros((max(len(rows), len(uniq)),) + x.shape[1:], x.dtype)
    xr[:len(uniq)] = x
    ref = oracle_out(w.irreps, xr, Y, s, inv, lrecv, len(xr), g.avg_num_neighbors)[:len(rows)]
    gpu = out[torch.from_numpy(rows).cuda()].cpu().numpy()
    assert column_scaled_error(gpu, ref) <= TOL[w.spec.dtype]
    del w, out, v4
    torch.cuda.empty_cache()


@pytest.mark.parametrize("dt", ["f32", "f16"])
@pytest.mark.parametrize("lmax", [0, 1, 2, 3, 6])
def test_standalone_harmonics_match_the_oracle(cuda_device, lmax, dt):
    # e3conv_edge_harmonics: the forward's edge_sh operand from edge vectors, against the
    # oracle's float64 harmonics of the same float32 vectors (a zero vector, widely varying
    # lengths, more edges than one grid pass covers); float32 evaluation within 1e-5 of the
    # largest component, float16 storage within half an ulp of float16 more
    irreps = ("8x0e", "+".join(f"1x{l}{'eo'[l % 2]}" for l in range(lmax + 1)), "8x0e")
    conv = e3.Conv(*irreps, 1.0, dtype=dt)
    rng = np.random.default_rng(10 * lmax + (dt == "f16"))
    e = 148 * 8 * 256 + 1234
    vec = rng.normal(size=(e, 3)) * rng.uniform(1e-3, 1e3, size=(e, 1))
    vec[7] = 0.0
    v4 = _vec4(vec)
    got = conv.edge_harmonics(to_dev(v4)).float().cpu().numpy()
    assert conv.check()
    ref = _oracle_sh(lmax, v4)
    scale = np.sqrt(2 * lmax + 1) * (2.0 if lmax else 1.0)
    tol = 1e-5 * scale + (2.0 ** -11 * np.abs(ref) if dt == "f16" else 0.0)
    assert np.all(np.abs(got - ref) <= tol)
    assert got.shape == (e, (lmax + 1) ** 2)
    assert conv.edge_harmonics(torch.zeros((0, 4), device="cuda")).shape == (0, (lmax + 1) ** 2)


def test_standalone_harmonics_feed_the_forward(cuda_device):
    # Y from the harmonics kernel fed to the forward, and the forward that evaluates the same
    # polynomials from the vectors itself: both within the float32 bar of the oracle
    spec = SPECS["mace"]
    g = make_graph(spec)
    x = node_features_np(spec, g.num_nodes)
    s = edge_scalars(spec, g)
    irreps = (spec.irreps_node, spec.irreps_sh, spec.irreps_out)
    v4 = to_dev(_vec4(g.vec))
    a = e3.Conv(*irreps, g.avg_num_neighbors, dtype="f32")
    Y = a.edge_harmonics(v4)
    rp = to_dev(row_ptr_of(g.receivers, g.num_nodes).astype(np.int32))
    snd = to_dev(g.senders.astype(np.int32))
    out_y = a.forward(to_dev(x), Y, to_dev(s), snd, rp)
    b = e3.Conv(*irreps, g.avg_num_neighbors, dtype="f32")
    b.set_edge_vectors(1)
    out_v = b.forward(to_dev(x), v4, to_dev(s), snd, rp)
    torch.cuda.synchronize()
    assert a.check() and b.check()
    ref = oracle_out(irreps, x, _oracle_sh(spec.lmax, _vec4(g.vec)), s, g.senders, g.receivers,
                     g.num_nodes, g.avg_num_neighbors)
    assert column_scaled_error(out_y.cpu().numpy(), ref) <= TOL["f32"]
    assert column_scaled_error(out_v.cpu().numpy(), ref) <= TOL["f32"]


def test_harmonics_worked_example_of_the_pages(cuda_device):
    # the pages' worked example (tests/golden/sh_worked_example.json): e3conv_edge_harmonics of
    # its two vectors against the closed forms of the unit-direction harmonics up to l = 2
    import json
    import pathlib
    fx = json.loads((pathlib.Path(__file__).parent / "golden" / "sh_worked_example.json").read_text())
    v = np.asarray(fx["vectors"], dtype=np.float32)
    conv = e3.Conv("8x0e", "1x0e+1x1o+1x2e", "8x0e", 1.0, dtype="f32")
    got = conv.edge_harmonics(to_dev(_vec4(v))).cpu().numpy().astype(np.float64)
    assert conv.check()
    u = v.astype(np.float64)
    u /= np.linalg.norm(u, axis=1, keepdims=True)
    x, y, z = u[:, 0], u[:, 1], u[:, 2]
    ref = np.concatenate([np.ones((2, 1)), np.sqrt(3) * np.stack([y, z, x], 1),
                          np.sqrt(15) * np.stack([x * y, y * z, (3 * z * z - 1) / (2 * np.sqrt(3)),
                                                  x * z, (x * x - y * y) / 2], 1)], 1)
    assert got.shape == (2, 9)
    # float32 evaluation: 1e-5 of the largest component (sqrt(5) * 2 for l = 2)
    assert np.abs(got - ref).max() <= 1e-5 * np.sqrt(5) * 2
