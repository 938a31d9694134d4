"""GPU parity of e3conv_forward against the float64 oracle (through the C ABI)."""
import numpy as np
import pytest
import torch

import equivariant_graph_message_b200 as e3
import oracle
from parity import TOL, DeviceWorkload, abs_bound, column_scaled_error, oracle_out, row_ptr_of, \
    run_gpu, to_dev, workload_inputs
from workloads import SPECS, make_graph

pytestmark = pytest.mark.gpu


def _spec_inputs(name):
    spec = SPECS[name]
    g = make_graph(spec)
    return (spec, g) + workload_inputs(spec, g)


@pytest.mark.parametrize("name", ["tiny", "gate_points", "mace"])
def test_small_configs_full_graph(cuda_device, name):
    spec, g, x, Y, s = _spec_inputs(name)
    irreps = (spec.irreps_node, spec.irreps_sh, spec.irreps_out)
    conv = e3.Conv(*irreps, g.avg_num_neighbors, dtype=spec.dtype)
    gpu = run_gpu(conv, x, Y, s, g.senders, g.receivers, g.num_nodes)
    ref = oracle_out(irreps, x, Y, s, g.senders, g.receivers, g.num_nodes, g.avg_num_neighbors)
    err = column_scaled_error(gpu, ref)
    assert err <= TOL[spec.dtype], err
    assert not np.isnan(gpu).any()


@pytest.mark.parametrize("name", ["large_f32", "large_f16"])
def test_large_configs_sampled(cuda_device, name):
    # full-size inputs on the device, the launch configuration the benchmark times,
    # checked on 256 seeded receivers plus the first and last one
    w = DeviceWorkload(name)
    out = w.conv.forward(w.x, w.Y, w.s, w.senders, w.row_ptr)
    torch.cuda.synchronize()
    assert w.conv.check()
    rng = np.random.default_rng(12345)
    rows = np.unique(np.concatenate([[0, w.N - 1], rng.choice(w.N, 256, replace=False)]))
    ref = w.sample_reference(rows)
    gpu = out[torch.from_numpy(rows).cuda()].cpu().numpy()
    err = column_scaled_error(gpu, ref)
    assert err <= TOL[w.spec.dtype], err
    # properties at full size: finite everywhere, deterministic
    assert torch.isfinite(out).all()
    out2 = w.conv.forward(w.x, w.Y, w.s, w.senders, w.row_ptr)
    assert torch.equal(out, out2)
    del w, out, out2
    torch.cuda.empty_cache()


def _random_graph(rng, n, e, hub=None):
    recv = rng.integers(0, n, e)
    if hub is not None:
        recv[: e // 2] = hub
    send = rng.integers(0, n, e)
    order = np.lexsort((send, recv))
    return send[order], recv[order]


CASES = [
    # (irreps_node, lmax, irreps_out, n, e, dtype)
    ("40x0e+40x1o", 2, "40x0e+40x1o+40x1e+40x2e", 50, 600, "f32"),        # C=40: 10-lane teams
    ("3x0e+3x1o+3x2e", 3, "3x0e+3x1o+3x2e+3x3o", 70, 900, "f32"),          # C=3: V=1
    ("160x0e+160x1o", 1, "160x0e+160x1o+160x1e", 20, 300, "f32"),          # ragged 2nd tile
    ("1x0e+1x1o+1x2e+1x3o+1x4e", 4, "1x0e+1x1o+1x2e+1x3o+1x4e+1x1e+1x2o+1x3e+1x4o", 30, 200, "f32"),
    ("8x0e+8x1o+8x2e+8x3o", 3, "8x0e+8x0o+8x1e+8x1o+8x2e+8x2o+8x3e+8x3o", 40, 500, "f16"),
    ("24x0e+24x1o", 3, "24x0e+24x1o+24x2e+24x3o", 30, 400, "f16"),
    ("2x1o+2x0e+2x2e", 2, "2x1o+2x0e+2x2e+2x1e", 15, 90, "f32"),           # unsorted irreps
]


@pytest.mark.parametrize("case", CASES, ids=[f"C{c[0].split('x')[0]}-{c[5]}" for c in CASES])
@pytest.mark.parametrize("norm", ["SQRT_DIM_OUT", "NONE"])
def test_random_irreps(cuda_device, case, norm):
    node, lmax, outs, n, e, dt = case
    sh = "+".join(f"1x{l}{'eo'[l % 2]}" for l in range(lmax + 1))
    rng = np.random.default_rng(abs(hash((case, norm))) % 2 ** 32)
    send, recv = _random_graph(rng, n, e)
    pl = oracle.plan(node, sh, outs)
    npdt = np.float16 if dt == "f16" else np.float32
    x = rng.normal(size=(n, pl.nx, pl.C)).astype(npdt)
    Y = rng.normal(size=(e, pl.ny)).astype(npdt)
    s = rng.normal(size=(e, len(pl.paths), pl.C)).astype(npdt)
    conv = e3.Conv(node, sh, outs, 7.5, normalization=norm, dtype=dt)
    gpu = run_gpu(conv, x, Y, s, send, recv, n)
    ref = oracle_out((node, sh, outs), x, Y, s, send, recv, n, 7.5, norm)
    assert column_scaled_error(gpu, ref) <= TOL[dt]


@pytest.mark.parametrize("V,block", [(1, 32), (1, 256), (2, 64), (2, 128), (4, 512), (4, 1024)])
def test_launch_configs(cuda_device, V, block):
    spec, g, x, Y, s = _spec_inputs("mace")
    irreps = (spec.irreps_node, spec.irreps_sh, spec.irreps_out)
    conv = e3.Conv(*irreps, g.avg_num_neighbors)
    conv.set_launch_config(V, block)
    gpu = run_gpu(conv, x, Y, s, g.senders, g.receivers, g.num_nodes)
    ref = oracle_out(irreps, x, Y, s, g.senders, g.receivers, g.num_nodes, g.avg_num_neighbors)
    assert column_scaled_error(gpu, ref) <= 1e-5


def test_no_edges_and_isolated_nodes(cuda_device):
    irreps = ("16x0e+16x1o", "1x0e+1x1o+1x2e", "16x0e+16x1o+16x2e")
    conv = e3.Conv(*irreps, 2.0)
    pl = oracle.plan(*irreps)
    rng = np.random.default_rng(3)
    x = rng.normal(size=(9, pl.nx, pl.C)).astype(np.float32)
    gpu = run_gpu(conv, x, np.zeros((0, pl.ny), np.float32),
                  np.zeros((0, len(pl.paths), pl.C), np.float32), np.zeros(0, np.int64),
                  np.zeros(0, np.int64), 9)
    assert np.all(gpu == 0)
    send = np.array([1, 2, 3, 8])
    recv = np.array([0, 0, 4, 4])
    Y = rng.normal(size=(4, pl.ny)).astype(np.float32)
    s = rng.normal(size=(4, len(pl.paths), pl.C)).astype(np.float32)
    gpu = run_gpu(conv, x, Y, s, send, recv, 9)
    ref = oracle_out(irreps, x, Y, s, send, recv, 9, 2.0)
    assert np.all(gpu[[1, 2, 3, 5, 6, 7, 8]] == 0)
    assert column_scaled_error(gpu, ref) <= 1e-5


def test_single_node_and_hub(cuda_device):
    # Every row, the 6000-edge hub row included, meets the 1e-5 column-scaled bar: a row
    # is summed in chunks of 128 edges whose scaled sums are added in the output row.  The
    # elementwise recursive-summation bound of float32 arithmetic (parity.abs_bound) holds
    # as well.
    irreps = ("32x0e+32x1o+32x2e", "1x0e+1x1o+1x2e+1x3o", "32x0e+32x1o+32x2e+32x3o")
    pl = oracle.plan(*irreps)
    rng = np.random.default_rng(4)
    for n, e, hub in ((1, 37, None), (300, 12000, 17)):
        send, recv = _random_graph(rng, n, e, hub)
        x = rng.normal(size=(n, pl.nx, pl.C)).astype(np.float32)
        Y = rng.normal(size=(e, pl.ny)).astype(np.float32)
        s = rng.normal(size=(e, len(pl.paths), pl.C)).astype(np.float32)
        conv = e3.Conv(*irreps, 40.0)
        gpu = run_gpu(conv, x, Y, s, send, recv, n)
        ref = oracle_out(irreps, x, Y, s, send, recv, n, 40.0)
        bound = abs_bound(irreps, x, Y, s, send, recv, n, 40.0)
        assert np.all(np.abs(gpu - ref) <= bound + 1e-12)
        if hub is not None:
            assert column_scaled_error(gpu, ref) <= 1e-5
            # the other rows scaled by their own columns' maxima, without the hub
            rows = np.setdiff1d(np.arange(n), [hub])
            assert column_scaled_error(gpu[rows], ref[rows]) <= 1e-5


def test_bad_indices_are_flagged_not_faulted(cuda_device):
    irreps = ("8x0e+8x1o", "1x0e+1x1o", "8x0e+8x1o+8x1e")
    conv = e3.Conv(*irreps, 1.0)
    pl = oracle.plan(*irreps)
    rng = np.random.default_rng(5)
    n, e = 6, 12
    send, recv = _random_graph(rng, n, e)
    x = to_dev(rng.normal(size=(n, pl.nx, pl.C)).astype(np.float32))
    Y = to_dev(rng.normal(size=(e, pl.ny)).astype(np.float32))
    s = to_dev(rng.normal(size=(e, len(pl.paths), pl.C)).astype(np.float32))
    rp = to_dev(row_ptr_of(recv, n).astype(np.int32))
    bad_send = send.copy()
    bad_send[3] = n + 5          # in-kernel bounds check skips this edge
    bad_send[7] = -2
    out = conv.forward(x, Y, s, to_dev(bad_send.astype(np.int32)), rp)
    assert not conv.check()
    assert conv.check()          # cleared by the previous check
    keep = np.ones(e, bool)
    keep[[3, 7]] = False
    ref = oracle_out(irreps, x.cpu().numpy(), Y.cpu().numpy()[keep], s.cpu().numpy()[keep],
                     send[keep], recv[keep], n, 1.0)
    assert column_scaled_error(out.cpu().numpy(), ref) <= 1e-5
    # a row range beyond row_ptr[num_nodes] and a decreasing one are treated as empty
    bad_rp = row_ptr_of(recv, n).astype(np.int32)
    bad_rp[2] = e + 100
    conv.forward(x, Y, s, to_dev(send.astype(np.int32)), to_dev(bad_rp))
    assert not conv.check()


def test_unsorted_edges_through_csr_and_permute(cuda_device):
    # COO edges in random order -> e3conv_build_csr -> e3conv_permute_rows -> forward
    spec, g, x, Y, s = _spec_inputs("mace")
    irreps = (spec.irreps_node, spec.irreps_sh, spec.irreps_out)
    rng = np.random.default_rng(6)
    shuffle = rng.permutation(g.num_edges)
    send_u, recv_u = g.senders[shuffle], g.receivers[shuffle]
    Yd = to_dev(Y[shuffle])
    sd = to_dev(s[shuffle])
    recv_d = to_dev(recv_u.astype(np.int32))
    row_ptr, perm, ws = e3.build_csr(recv_d, g.num_nodes)
    assert e3.csr_check(ws)
    senders = e3.permute_rows(to_dev(send_u.astype(np.int32)), perm)
    Ys = e3.permute_rows(Yd, perm)
    ss = e3.permute_rows(sd, perm)
    conv = e3.Conv(*irreps, g.avg_num_neighbors)
    out = conv.forward(to_dev(x), Ys, ss, senders, row_ptr)
    ref = oracle_out(irreps, x, Y[shuffle], s[shuffle], send_u, recv_u, g.num_nodes,
                     g.avg_num_neighbors)
    assert column_scaled_error(out.cpu().numpy(), ref) <= 1e-5


def test_stream_ordering(cuda_device):
    spec, g, x, Y, s = _spec_inputs("gate_points")
    irreps = (spec.irreps_node, spec.irreps_sh, spec.irreps_out)
    conv = e3.Conv(*irreps, g.avg_num_neighbors)
    st = torch.cuda.Stream()
    with torch.cuda.stream(st):
        xd, Yd, sd = to_dev(x), to_dev(Y), to_dev(s)
        sd_ = to_dev(g.senders.astype(np.int32))
        rp = to_dev(row_ptr_of(g.receivers, g.num_nodes).astype(np.int32))
        out = conv.forward(xd, Yd, sd, sd_, rp, stream=st)
    st.synchronize()
    ref = oracle_out(irreps, x, Y, s, g.senders, g.receivers, g.num_nodes, g.avg_num_neighbors)
    assert column_scaled_error(out.cpu().numpy(), ref) <= 1e-5


@pytest.mark.parametrize("name", ["tiny", "gate_points"])
def test_direct_pipeline_is_bitwise_the_plain_walk(cuda_device, name):
    # the software-pipelined row walk of the direct variant loads edge e+1 while edge e is
    # computed; the arithmetic per output element is unchanged
    spec, g, x, Y, s = _spec_inputs(name)
    irreps = (spec.irreps_node, spec.irreps_sh, spec.irreps_out)
    a = e3.Conv(*irreps, g.avg_num_neighbors)
    a.set_direct_pipeline(0)
    b = e3.Conv(*irreps, g.avg_num_neighbors)
    b.set_direct_pipeline(1)
    assert a.kernel_info()["stages"] == 0 and b.kernel_info()["stages"] == 0
    assert "pipelined=1" in b.kernel_source() and "pipelined=0" in a.kernel_source()
    ga = run_gpu(a, x, Y, s, g.senders, g.receivers, g.num_nodes)
    gb = run_gpu(b, x, Y, s, g.senders, g.receivers, g.num_nodes)
    assert np.array_equal(ga, gb)
    # bad senders are skipped in the pipelined walk as well
    bad = g.senders.copy()
    bad[[0, len(bad) // 2, len(bad) - 1]] = g.num_nodes + 7
    rp = to_dev(row_ptr_of(g.receivers, g.num_nodes).astype(np.int32))
    out = b.forward(to_dev(x), to_dev(Y), to_dev(s), to_dev(bad.astype(np.int32)), rp)
    assert not b.check()
    keep = np.ones(len(bad), bool)
    keep[[0, len(bad) // 2, len(bad) - 1]] = False
    ref = oracle_out(irreps, x, Y[keep], s[keep], g.senders[keep], g.receivers[keep],
                     g.num_nodes, g.avg_num_neighbors)
    assert column_scaled_error(out.cpu().numpy(), ref) <= 1e-5
