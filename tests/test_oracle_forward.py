"""Pins of the oracle's edgewise convolution loops (oracle/forward.c)."""
import numpy as np
import pytest

import oracle
from workloads import SPECS, make_graph, node_features_np, scalars_np
from workloads import graphs as wgraphs

RICH = ("2x0e+2x1o+2x2e+2x3o+2x1e", "1x0e+1x1o+1x2e+1x3o",
        "2x0e+2x0o+2x1e+2x1o+2x2e+2x2o+2x3e+2x3o")


def _random_case(g, irreps, n=7, e=30, pos=None):
    pl = oracle.plan(*irreps)
    send = g.integers(0, n, e)
    recv = (send + g.integers(1, n, e)) % n    # no self loops
    if pos is None:
        vec = g.normal(size=(e, 3))
    else:
        vec = pos[recv] - pos[send]
    lmax = int(np.sqrt(pl.ny)) - 1
    Y = oracle.sh(lmax, vec / np.linalg.norm(vec, axis=1, keepdims=True))
    x = g.normal(size=(n, pl.nx, pl.C))
    s = g.normal(size=(e, len(pl.paths), pl.C))
    return pl, x, Y, s, send, recv


def _einsum_reference(irreps, x, Y, s, send, recv, n, avg, norm="SQRT_DIM_OUT"):
    """Vectorised dense evaluation (independent of the loop code)."""
    pl = oracle.plan(*irreps)
    out = np.zeros((n, pl.nout, pl.C))
    for p, path in enumerate(pl.paths):
        W = oracle.cg(path.l1, path.l2, path.l3, norm)
        xa = x[send][:, path.x_off:path.x_off + 2 * path.l1 + 1, :]       # [E, d1, C]
        ye = Y[:, path.y_off:path.y_off + 2 * path.l2 + 1]                 # [E, d2]
        msg = np.einsum("ijk,eiu,ej,eu->eku", W, xa, ye, s[:, p, :])       # [E, d3, C]
        np.add.at(out[:, path.out_off:path.out_off + 2 * path.l3 + 1, :], recv, msg)
    return out / avg


def _run(irreps, x, Y, s, send, recv, n, avg=1.0, norm="SQRT_DIM_OUT"):
    return oracle.forward(*irreps, x, Y, s, send, recv, n, avg, norm)


def test_single_edge_scalar_path():
    irreps = ("1x0e", "1x0e", "1x0e")
    out = _run(irreps, [[[2.0]], [[3.0]]], [[1.0]], [[[0.5]]], [1], [0], 2, 4.0)
    np.testing.assert_allclose(out[:, 0, 0], [0.5 * 3.0 * 1.0 / 4.0, 0.0])


def test_single_edge_dot_and_cross_products():
    a = np.array([0.3, -1.2, 0.7])
    b = np.array([1.1, 0.4, -0.5])          # Y_1 = b (any edge feature vector)
    x = np.zeros((2, 3, 1))
    x[1, :, 0] = a[[1, 2, 0]]
    Y = np.concatenate([[1.0], b[[1, 2, 0]]])[None, :]
    s = np.array([[[2.0]]])
    dot = _run(("1x1o", "1x0e+1x1o", "1x0e"), x, Y, s, [1], [0], 2, 1.0)
    np.testing.assert_allclose(dot[0, 0, 0], 2.0 * a @ b / np.sqrt(3), rtol=1e-14)
    cross = _run(("1x1o", "1x0e+1x1o", "1x1e"), x, Y, s, [1], [0], 2, 1.0)
    np.testing.assert_allclose(cross[0, :, 0], 2.0 * np.cross(a, b)[[1, 2, 0]] / np.sqrt(2),
                               rtol=1e-13)
    assert np.all(dot[1] == 0) and np.all(cross[1] == 0)


def test_scalar_times_harmonic_is_scaling():
    # 0e x 2e -> 2e with SQRT_DIM_OUT: out = s * x0 * Y_2
    g = np.random.default_rng(1)
    Y = oracle.sh(2, np.array([[0.6, 0.0, 0.8]]))
    out = _run(("3x0e", "1x0e+1x1o+1x2e", "3x2e"), g.normal(size=(1, 1, 3)) * 0 + [[[1.5, -2, 3]]],
               Y, np.full((1, 1, 3), 0.25), [0], [0], 1, 1.0)
    np.testing.assert_allclose(out[0], 0.25 * Y[0, 4:9, None] * np.array([1.5, -2, 3])[None, :],
                               rtol=1e-14, atol=1e-14)


@pytest.mark.parametrize("irreps", [("4x0e+4x1o", "1x0e+1x1o+1x2e", "4x0e+4x1o+4x1e+4x2e"), RICH])
def test_brute_force_matches_loops(irreps):
    g = np.random.default_rng(2)
    pl, x, Y, s, send, recv = _random_case(g, irreps)
    ref = _einsum_reference(irreps, x, Y, s, send, recv, 7, 3.5)
    np.testing.assert_allclose(_run(irreps, x, Y, s, send, recv, 7, 3.5), ref, atol=1e-13)
    ref1 = _einsum_reference(irreps, x, Y, s, send, recv, 7, 1.0, "NONE")
    np.testing.assert_allclose(_run(irreps, x, Y, s, send, recv, 7, 1.0, "NONE"), ref1, atol=1e-13)


@pytest.mark.parametrize("improper", [False, True])
def test_o3_equivariance(improper):
    # Rotate (and invert) the geometry: Y' = D Y from the rotated edge vectors,
    # x' = p1^sigma D^{l1} x, s unchanged  =>  out' = p3^sigma D^{l3} out.
    irreps = RICH
    g = np.random.default_rng(3 + improper)
    n = 8
    pos = g.normal(size=(n, 3))
    for _ in range(10):
        pl, x, Y, s, send, recv = _random_case(g, irreps, n=n, e=40, pos=pos)
        keep = send != recv
        send, recv, Y, s = send[keep], recv[keep], Y[keep], s[keep]
        R = oracle.random_rotation(g)
        sigma = -1.0 if improper else 1.0
        pos2 = sigma * pos @ R.T
        vec2 = pos2[recv] - pos2[send]
        Y2 = oracle.sh(3, vec2 / np.linalg.norm(vec2, axis=1, keepdims=True))
        x2 = np.zeros_like(x)
        for ir_off, ir in zip(np.cumsum([0] + [i.dim for i in oracle.parse_irreps(irreps[0])]),
                              oracle.parse_irreps(irreps[0])):
            D = oracle.wigner_d(ir.l, R) * (ir.p if improper else 1)
            x2[:, ir_off:ir_off + ir.dim, :] = np.einsum("ij,njc->nic", D, x[:, ir_off:ir_off + ir.dim])
        out = _run(irreps, x, Y, s, send, recv, n, 5.0)
        out2 = _run(irreps, x2, Y2, s, send, recv, n, 5.0)
        expect = np.zeros_like(out)
        for l3, p3, off in pl.outputs:
            D = oracle.wigner_d(l3, R) * (p3 if improper else 1)
            expect[:, off:off + 2 * l3 + 1] = np.einsum("ij,njc->nic", D, out[:, off:off + 2 * l3 + 1])
        np.testing.assert_allclose(out2, expect, atol=1e-11)


def test_edge_order_invariance():
    g = np.random.default_rng(5)
    pl, x, Y, s, send, recv = _random_case(g, RICH)
    perm = g.permutation(len(send))
    a = _run(RICH, x, Y, s, send, recv, 7, 2.0)
    b = _run(RICH, x, Y[perm], s[perm], send[perm], recv[perm], 7, 2.0)
    np.testing.assert_allclose(a, b, atol=1e-12)


def test_zero_edges_and_isolated_nodes():
    pl = oracle.plan(*RICH)
    x = np.ones((5, pl.nx, pl.C))
    out = _run(RICH, x, np.zeros((0, pl.ny)), np.zeros((0, len(pl.paths), pl.C)), [], [], 5, 1.0)
    assert out.shape == (5, pl.nout, pl.C) and np.all(out == 0)
    g = np.random.default_rng(6)
    _, x, Y, s, send, recv = _random_case(g, RICH, n=9)
    recv = np.where(recv >= 5, 0, recv)      # nodes 5..8 receive nothing
    out = _run(RICH, x, Y, s, send, recv, 9, 1.0)
    assert np.all(out[5:] == 0)


def test_linearity_and_scaling():
    g = np.random.default_rng(7)
    pl, x, Y, s, send, recv = _random_case(g, RICH)
    base = _run(RICH, x, Y, s, send, recv, 7, 1.0)
    np.testing.assert_allclose(_run(RICH, 3 * x, Y, s, send, recv, 7, 1.0), 3 * base, atol=1e-12)
    s2 = g.normal(size=s.shape)
    np.testing.assert_allclose(_run(RICH, x, Y, s + s2, send, recv, 7, 1.0),
                               base + _run(RICH, x, Y, s2, send, recv, 7, 1.0), atol=1e-12)
    np.testing.assert_allclose(_run(RICH, x, Y, s, send, recv, 7, 4.0), base / 4, atol=1e-13)
    none = _run(RICH, x, Y, s, send, recv, 7, 1.0, "NONE")
    for l3, _, off in pl.outputs:
        sl = slice(off, off + 2 * l3 + 1)
        np.testing.assert_allclose(base[:, sl], np.sqrt(2 * l3 + 1) * none[:, sl], atol=1e-12)


def test_sum_over_edges_decomposes():
    g = np.random.default_rng(8)
    pl, x, Y, s, send, recv = _random_case(g, RICH, e=12)
    total = _run(RICH, x, Y, s, send, recv, 7, 1.0)
    parts = sum(_run(RICH, x, Y[e:e + 1], s[e:e + 1], send[e:e + 1], recv[e:e + 1], 7, 1.0)
                for e in range(12))
    np.testing.assert_allclose(total, parts, atol=1e-12)


def test_out_of_range_index_is_an_error():
    pl = oracle.plan("1x0e", "1x0e", "1x0e")
    with pytest.raises(ValueError):
        _run(("1x0e", "1x0e", "1x0e"), np.ones((2, 1, 1)), [[1.0]], [[[1.0]]], [2], [0], 2, 1.0)


def test_tiny_workload_against_brute_force():
    spec = SPECS["tiny"]
    gr = make_graph(spec)
    x = node_features_np(spec, gr.num_nodes)
    Y = oracle.sh(spec.lmax, gr.vec / np.linalg.norm(gr.vec, axis=1, keepdims=True))
    Y = Y.astype(np.float32)
    s = scalars_np(spec, gr)
    irreps = (spec.irreps_node, spec.irreps_sh, spec.irreps_out)
    ref = _einsum_reference(irreps, x.astype(np.float64), Y.astype(np.float64),
                            s.astype(np.float64), gr.senders, gr.receivers, gr.num_nodes,
                            gr.avg_num_neighbors)
    out = _run(irreps, x, Y, s, gr.senders, gr.receivers, gr.num_nodes, gr.avg_num_neighbors)
    np.testing.assert_allclose(out, ref, atol=1e-13)
    assert gr.num_edges > 0 and not np.all(out == 0)


def test_radius_graph_cell_list_matches_brute_force():
    pos = wgraphs.uniform_points(11, 0, 400, 6.0)
    for box in (None, 6.0):
        a = wgraphs.radius_graph_bruteforce(pos, 1.5, box)
        b = wgraphs.radius_graph_cells(pos, 1.5, box)
        for u, v in zip(a, b):
            np.testing.assert_array_equal(u, v)
        assert np.all(a[0] != a[1])
        assert np.all(np.diff(a[1]) >= 0)
