"""GPU parity of the backward (e3conv_backward: gradients of x, Y and s) against
the oracle's float64 backward, through the C ABI: the small workloads' full
graphs, the large workloads' irreps on smaller graphs, float16 inputs,
isolated nodes (no incoming or no outgoing edges), and out-of-range indices
flagged rather than faulted.  The sender CSR comes from e3conv_build_csr."""
import numpy as np
import pytest
import torch

import equivariant_graph_message_b200 as e3
import oracle
from parity import column_scaled_error, row_ptr_of, to_dev, workload_inputs
from workloads import SPECS, make_graph

pytestmark = pytest.mark.gpu


def _run(conv, x, Y, s, senders, receivers, n, g):
    tdt = torch.float16 if conv.dtype == "f16" else torch.float32
    rp = row_ptr_of(np.asarray(receivers), n)
    snd = to_dev(np.asarray(senders, np.int32))
    srp, sperm, _ = e3.build_csr(snd, n)
    gx, gY, gs = conv.backward(to_dev(x, tdt), to_dev(Y, tdt), to_dev(s, tdt), snd,
                               to_dev(rp.astype(np.int32)), to_dev(g.astype(np.float32)),
                               receivers=to_dev(np.asarray(receivers, np.int32)),
                               sender_row_ptr=srp, sender_perm=sperm)
    torch.cuda.synchronize()
    assert conv.check()
    return gx.cpu().numpy(), gY.cpu().numpy(), gs.cpu().numpy()


def _check(got, ref, tol):
    for a, b in zip(got, ref):
        assert a.shape == b.shape
        err = column_scaled_error(a.reshape(len(a), -1), b.reshape(len(b), -1))
        assert err <= tol, err


@pytest.mark.parametrize("name", ["tiny", "gate_points", "mace"])
def test_backward_full_graphs(cuda_device, name):
    spec = SPECS[name]
    g = make_graph(spec)
    x, Y, s = workload_inputs(spec, g)
    irreps = (spec.irreps_node, spec.irreps_sh, spec.irreps_out)
    conv = e3.Conv(*irreps, g.avg_num_neighbors, dtype=spec.dtype)
    pl = oracle.plan(*irreps)
    gout = np.random.default_rng(1).normal(size=(g.num_nodes, pl.nout, pl.C))
    got = _run(conv, x, Y, s, g.senders, g.receivers, g.num_nodes, gout)
    ref = oracle.backward(*irreps, x, Y, s, g.senders, g.receivers, g.num_nodes,
                          g.avg_num_neighbors, gout.astype(np.float32))
    _check(got, ref, 1e-5)


@pytest.mark.parametrize("name", ["large_f32", "large_f16"])
def test_backward_large_irreps(cuda_device, name):
    spec = SPECS[name]
    g = make_graph(spec, 1500)
    x, Y, s = workload_inputs(spec, g)
    irreps = (spec.irreps_node, spec.irreps_sh, spec.irreps_out)
    conv = e3.Conv(*irreps, g.avg_num_neighbors, dtype=spec.dtype)
    pl = oracle.plan(*irreps)
    gout = np.random.default_rng(2).normal(size=(g.num_nodes, pl.nout, pl.C))
    got = _run(conv, x, Y, s, g.senders, g.receivers, g.num_nodes, gout)
    ref = oracle.backward(*irreps, x, Y, s, g.senders, g.receivers, g.num_nodes,
                          g.avg_num_neighbors, gout.astype(np.float32))
    _check(got, ref, 1e-5)


def test_backward_isolated_nodes_and_bad_indices(cuda_device):
    irreps = ("32x0e+32x1o", "1x0e+1x1o+1x2e", "32x0e+32x1o+32x2e")
    pl = oracle.plan(*irreps)
    rng = np.random.default_rng(3)
    n = 9
    send = np.array([1, 2, 3, 8, 2])
    recv = np.array([0, 0, 4, 4, 6])                 # nodes 0, 5, 7 send nothing
    x = rng.normal(size=(n, pl.nx, pl.C)).astype(np.float32)
    Y = rng.normal(size=(5, pl.ny)).astype(np.float32)
    s = rng.normal(size=(5, len(pl.paths), pl.C)).astype(np.float32)
    gout = rng.normal(size=(n, pl.nout, pl.C))
    conv = e3.Conv(*irreps, 2.0)
    got = _run(conv, x, Y, s, send, recv, n, gout)
    ref = oracle.backward(*irreps, x, Y, s, send, recv, n, 2.0, gout.astype(np.float32))
    _check(got, ref, 1e-5)
    assert np.all(got[0][[0, 5, 7]] == 0)
    # an out-of-range sender: flagged, no fault
    bad = send.copy()
    bad[2] = n + 4
    rp = row_ptr_of(recv, n)
    snd = to_dev(bad.astype(np.int32))
    srp, sperm, _ = e3.build_csr(to_dev(send.astype(np.int32)), n)
    conv.backward(to_dev(x), to_dev(Y), to_dev(s), snd, to_dev(rp.astype(np.int32)),
                  to_dev(gout.astype(np.float32)), receivers=to_dev(recv.astype(np.int32)),
                  sender_row_ptr=srp, sender_perm=sperm)
    assert not conv.check()
    assert conv.check()


@pytest.mark.parametrize("parts", [1, 2, 3, 4])
@pytest.mark.parametrize("name", ["large_f16", "mace"])
def test_backward_split_over_output_irreps(cuda_device, name, parts):
    # one to four launches of each backward kernel, each over a share of the output irreps;
    # the later launches add to grad_Y and grad_x: every split meets the oracle
    spec = SPECS[name]
    g = make_graph(spec, 1200)
    x, Y, s = workload_inputs(spec, g)
    irreps = (spec.irreps_node, spec.irreps_sh, spec.irreps_out)
    conv = e3.Conv(*irreps, g.avg_num_neighbors, dtype=spec.dtype)
    conv.set_backward_parts(parts)
    want = min(parts, len(conv.outputs))
    assert f"// part 0 of {want}" in conv.backward_source(0)
    pl = oracle.plan(*irreps)
    gout = np.random.default_rng(parts).normal(size=(g.num_nodes, pl.nout, pl.C))
    got = _run(conv, x, Y, s, g.senders, g.receivers, g.num_nodes, gout)
    xs, Ys, ss = (np.asarray(a, np.float64) for a in (x, Y, s))
    ref = oracle.backward(*irreps, xs, Ys, ss, g.senders, g.receivers, g.num_nodes,
                          g.avg_num_neighbors, gout.astype(np.float32))
    _check(got, ref, 1e-5)
