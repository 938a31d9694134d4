"""GPU parity of the staged (persistent warps + shared-memory ring) forward variant."""
import numpy as np
import pytest
import torch

import equivariant_graph_message_b200 as e3
import oracle
from parity import TOL, column_scaled_error, oracle_out, row_ptr_of, run_gpu, to_dev

pytestmark = pytest.mark.gpu

SH3 = "1x0e+1x1o+1x2e+1x3o"
IRREPS = {
    32: ("32x0e+32x1o+32x2e", SH3, "32x0e+32x1o+32x2e+32x3o"),
    64: ("64x0e+64x1o", SH3, "64x0e+64x1o+64x2e+64x1e"),
    128: ("128x0e+128x1o+128x2e+128x3o", SH3, "128x0e+128x1o+128x2e+128x3o+128x1e"),
}


def _graph(rng, n, e, empty_frac=0.0):
    recv = rng.integers(0, n, e)
    if empty_frac:
        keep = rng.random(n) >= empty_frac
        pool = np.nonzero(keep)[0]
        recv = pool[rng.integers(0, len(pool), e)]
    send = rng.integers(0, n, e)
    o = np.lexsort((send, recv))
    return send[o], recv[o]


def _inputs(rng, irreps, n, e, dt):
    pl = oracle.plan(*irreps)
    npdt = np.float16 if dt == "f16" else np.float32
    return (pl, rng.normal(size=(n, pl.nx, pl.C)).astype(npdt),
            rng.normal(size=(e, pl.ny)).astype(npdt),
            rng.normal(size=(e, len(pl.paths), pl.C)).astype(npdt))


@pytest.mark.parametrize("C", [32, 64, 128])
@pytest.mark.parametrize("dt", ["f32", "f16"])
@pytest.mark.parametrize("contract_first", [0, 1])
def test_staged_parity_with_empty_rows(cuda_device, C, dt, contract_first):
    irreps = IRREPS[C]
    rng = np.random.default_rng(C + (dt == "f16"))
    n, e = 700, 9000
    send, recv = _graph(rng, n, e, empty_frac=0.2)
    pl, x, Y, s = _inputs(rng, irreps, n, e, dt)
    conv = e3.Conv(*irreps, 12.0, dtype=dt)
    conv.set_tensor_cores(0)          # the float32 staged path (tensor cores: test_gpu_tensor_cores)
    conv.set_contract_first(contract_first)
    info = conv.kernel_info()
    assert info["stages"] >= 2 and info["contract_first"] == contract_first
    gpu = run_gpu(conv, x, Y, s, send, recv, n)
    ref = oracle_out(irreps, x, Y, s, send, recv, n, 12.0)
    assert column_scaled_error(gpu, ref) <= TOL[dt]
    empty = np.setdiff1d(np.arange(n), recv)
    assert len(empty) > 50 and np.all(gpu[empty] == 0)


@pytest.mark.parametrize("stages,block", [(2, 32), (2, 128), (3, 64), (4, 96), (5, 32), (8, 32)])
@pytest.mark.parametrize("contract_first", [0, 1])
def test_staged_ring_depths(cuda_device, stages, block, contract_first):
    irreps = IRREPS[64]
    rng = np.random.default_rng(stages * 100 + block)
    n, e = 333, 5000
    send, recv = _graph(rng, n, e)
    pl, x, Y, s = _inputs(rng, irreps, n, e, "f32")
    conv = e3.Conv(*irreps, 9.0)
    conv.set_contract_first(contract_first)
    conv.set_launch_config(0, block, stages)
    info = conv.kernel_info()
    assert info["stages"] == stages and info["block_threads"] == block
    gpu = run_gpu(conv, x, Y, s, send, recv, n)
    ref = oracle_out(irreps, x, Y, s, send, recv, n, 9.0)
    assert column_scaled_error(gpu, ref) <= 1e-5


def test_staged_few_nodes_many_warps_and_no_edges(cuda_device):
    irreps = IRREPS[32]
    rng = np.random.default_rng(9)
    conv = e3.Conv(*irreps, 3.0)
    assert conv.kernel_info()["stages"] >= 2
    for n, e in ((1, 0), (3, 0), (1, 50), (5, 200)):
        send, recv = _graph(rng, n, e) if e else (np.zeros(0, np.int64), np.zeros(0, np.int64))
        pl, x, Y, s = _inputs(rng, irreps, n, e, "f32")
        gpu = run_gpu(conv, x, Y, s, send, recv, n)
        if e == 0:
            assert np.all(gpu == 0)
        else:
            ref = oracle_out(irreps, x, Y, s, send, recv, n, 3.0)
            assert np.all(np.abs(gpu - ref) <= 1e-5 * np.abs(ref).max())


def test_staged_long_rows(cuda_device):
    irreps = IRREPS[64]
    rng = np.random.default_rng(10)
    n, e = 40, 8000          # ~200 edges per row: several sender windows per row
    send, recv = _graph(rng, n, e)
    pl, x, Y, s = _inputs(rng, irreps, n, e, "f32")
    conv = e3.Conv(*irreps, 200.0)
    gpu = run_gpu(conv, x, Y, s, send, recv, n)
    ref = oracle_out(irreps, x, Y, s, send, recv, n, 200.0)
    assert column_scaled_error(gpu, ref) <= 1e-5


def test_staged_bad_indices_flagged(cuda_device):
    irreps = IRREPS[64]
    rng = np.random.default_rng(11)
    n, e = 50, 600
    send, recv = _graph(rng, n, e)
    pl, x, Y, s = _inputs(rng, irreps, n, e, "f32")
    conv = e3.Conv(*irreps, 1.0)
    assert conv.kernel_info()["stages"] >= 2
    xd, Yd, sd = to_dev(x), to_dev(Y), to_dev(s)
    rp = row_ptr_of(recv, n).astype(np.int32)
    bad = send.copy()
    bad[[5, 77, 300]] = [n, -1, 1 << 30]
    out = conv.forward(xd, Yd, sd, to_dev(bad.astype(np.int32)), to_dev(rp))
    assert not conv.check()
    keep = np.ones(e, bool)
    keep[[5, 77, 300]] = False
    ref = oracle_out(irreps, x, Y[keep], s[keep], send[keep], recv[keep], n, 1.0)
    assert column_scaled_error(out.cpu().numpy(), ref) <= 1e-5
    bad_rp = rp.copy()
    bad_rp[10] = e + 7
    out = conv.forward(xd, Yd, sd, to_dev(send.astype(np.int32)), to_dev(bad_rp))
    assert not conv.check()
    assert conv.check()
    assert torch.isfinite(out).all()


def test_staged_matches_direct_bitwise_order_free(cuda_device):
    # both variants sum a row's edges in row order with the same per-edge code
    irreps = IRREPS[128]
    rng = np.random.default_rng(12)
    n, e = 500, 15000
    send, recv = _graph(rng, n, e)
    pl, x, Y, s = _inputs(rng, irreps, n, e, "f16")
    a = e3.Conv(*irreps, 30.0, dtype="f16")
    b = e3.Conv(*irreps, 30.0, dtype="f16")
    b.set_launch_config(0, 0, 0)
    assert a.kernel_info()["stages"] >= 2 and b.kernel_info()["stages"] == 0
    ga = run_gpu(a, x, Y, s, send, recv, n)
    gb = run_gpu(b, x, Y, s, send, recv, n)
    ref = oracle_out(irreps, x, Y, s, send, recv, n, 30.0)
    assert column_scaled_error(ga, ref) <= 5e-3 and column_scaled_error(gb, ref) <= 5e-3
    np.testing.assert_allclose(ga, gb, rtol=1e-5, atol=1e-5 * np.abs(ref).max())


@pytest.mark.parametrize("V,block,stages", [(2, 64, 2), (2, 128, 3), (2, 192, 2), (2, 448, 2),
                                            (4, 32, 2), (4, 256, 2), (1, 128, 2)])
@pytest.mark.parametrize("contract_first", [0, 1])
def test_staged_team_shapes(cuda_device, V, block, stages, contract_first):
    # C = 128: V=2 -> teams of 2 warps sharing one ring; V=4 -> one warp; V=1 -> 4 warps
    irreps = IRREPS[128]
    rng = np.random.default_rng(V * 1000 + block + stages)
    n, e = 400, 7000
    send, recv = _graph(rng, n, e, empty_frac=0.1)
    pl, x, Y, s = _inputs(rng, irreps, n, e, "f16")
    conv = e3.Conv(*irreps, 17.0, dtype="f16")
    conv.set_contract_first(contract_first)
    conv.set_launch_config(V, block, stages)
    info = conv.kernel_info()
    assert info["stages"] == stages and info["block_threads"] == block
    assert info["channels_per_lane"] == V
    gpu = run_gpu(conv, x, Y, s, send, recv, n)
    ref = oracle_out(irreps, x, Y, s, send, recv, n, 17.0)
    assert column_scaled_error(gpu, ref) <= 5e-3
    assert np.all(gpu[np.setdiff1d(np.arange(n), recv)] == 0)


@pytest.mark.parametrize("split", [2, 3, 4])
@pytest.mark.parametrize("C,dt", [(128, "f16"), (128, "f32"), (64, "f32"), (32, "f32")])
def test_path_split_is_bitwise_the_unsplit_kernel(cuda_device, split, C, dt):
    # each warp of a path-split team forms and applies only its outputs' paths; every output
    # element is accumulated by the same FMA sequence as in the one-warp kernel, so the outputs
    # are bitwise equal (and match the oracle), with empty rows and a row of several chunks
    irreps = IRREPS[C]
    rng = np.random.default_rng(100 * split + C)
    n, e = 900, 16000
    send, recv = _graph(rng, n, e, empty_frac=0.1)
    recv[: 400] = 17                      # a row of more than three 128-edge chunks
    o = np.lexsort((send, recv))
    send, recv = send[o], recv[o]
    pl, x, Y, s = _inputs(rng, irreps, n, e, dt)
    base = e3.Conv(*irreps, 12.0, dtype=dt)
    base.set_path_split(0)
    sp = e3.Conv(*irreps, 12.0, dtype=dt)
    sp.set_path_split(split)
    src = sp.kernel_source()
    assert f"path_split={split}" in src, src[:400]
    assert sp.kernel_info()["local_bytes"] == 0
    a = run_gpu(base, x, Y, s, send, recv, n)
    b = run_gpu(sp, x, Y, s, send, recv, n)
    assert np.array_equal(a, b)
    ref = oracle_out(irreps, x, Y, s, send, recv, n, 12.0)
    assert column_scaled_error(b, ref) <= 1e-5


@pytest.mark.parametrize("group,stages", [(2, -1), (3, 6), (4, 4), (2, 8)])
@pytest.mark.parametrize("C,dt", [(128, "f16"), (64, "f32"), (32, "f32")])
def test_copy_groups_are_bitwise_the_single_edge_ring(cuda_device, group, stages, C, dt):
    # a ring group takes up to `group` consecutive edges of a row with one copy of their
    # scalars and one of their harmonics; rows shorter than a group, empty rows, a long row
    # and row ends inside a group leave the arithmetic unchanged
    irreps = IRREPS[C]
    rng = np.random.default_rng(10 * group + C + stages)
    n, e = 800, 12000
    send, recv = _graph(rng, n, e, empty_frac=0.1)
    recv[:300] = 5
    recv[300:303] = 6                      # a row of 3 edges
    o = np.lexsort((send, recv))
    send, recv = send[o], recv[o]
    pl, x, Y, s = _inputs(rng, irreps, n, e, dt)
    base = e3.Conv(*irreps, 9.0, dtype=dt)
    base.set_copy_group(1)
    grp = e3.Conv(*irreps, 9.0, dtype=dt)
    grp.set_copy_group(group)
    if stages != -1:
        grp.set_launch_config(0, 0, stages)
    assert f"copy_group={group}" in grp.kernel_source()
    a = run_gpu(base, x, Y, s, send, recv, n)
    b = run_gpu(grp, x, Y, s, send, recv, n)
    assert np.array_equal(a, b)
    ref = oracle_out(irreps, x, Y, s, send, recv, n, 9.0)
    assert column_scaled_error(b, ref) <= 1e-5


@pytest.mark.parametrize("layout", [1, 2, 3])
@pytest.mark.parametrize("C,dt", [(128, "f16"), (64, "f32")])
def test_a_layouts_are_bitwise_the_default(cuda_device, layout, C, dt):
    # the A entries' shared-memory layout changes where each entry is stored and how it is
    # loaded, not the products or their order: every layout gives the default's bits
    irreps = IRREPS[C]
    rng = np.random.default_rng(20 * layout + C)
    n, e = 700, 10000
    send, recv = _graph(rng, n, e, empty_frac=0.1)
    recv[:260] = 11                        # a row of more than two 128-edge chunks
    o = np.lexsort((send, recv))
    send, recv = send[o], recv[o]
    pl, x, Y, s = _inputs(rng, irreps, n, e, dt)
    base = e3.Conv(*irreps, 11.0, dtype=dt)
    base.set_a_layout(0)
    lay = e3.Conv(*irreps, 11.0, dtype=dt)
    lay.set_a_layout(layout)
    assert f"a_layout={layout}" in lay.kernel_source()
    a = run_gpu(base, x, Y, s, send, recv, n)
    b = run_gpu(lay, x, Y, s, send, recv, n)
    assert np.array_equal(a, b)
    ref = oracle_out(irreps, x, Y, s, send, recv, n, 11.0)
    assert column_scaled_error(b, ref) <= (5e-3 if dt == "f16" else 1e-5)
