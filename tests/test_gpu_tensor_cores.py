"""GPU parity of the tensor-core forward variant (float16 inputs, C = 128):
per edge T = x^T (A_hi + A_lo) on tcgen05 tensor cores, then s-scaling."""
import numpy as np
import pytest
import torch

import equivariant_graph_message_b200 as e3
import oracle
from parity import column_scaled_error, oracle_out, row_ptr_of, run_gpu, to_dev

pytestmark = pytest.mark.gpu

SH3 = "1x0e+1x1o+1x2e+1x3o"
CASES = {
    "full16": ("128x0e+128x1o+128x2e+128x3o", SH3,
               "128x0e+128x0o+128x1e+128x1o+128x2e+128x2o+128x3e+128x3o"),
    "nx9": ("128x0e+128x1o+128x2e", SH3, "128x0e+128x1o+128x2e+128x1e+128x2o"),   # K rows 9..15 zero
    "nx4": ("128x0e+128x1o", SH3, "128x0e+128x1o+128x2e+128x1e+128x3o"),
    "odd_in": ("128x1o+128x0e+128x2o", SH3, "128x0e+128x0o+128x1e+128x1o+128x2e+128x3e+128x3o"),
    # no scalar input irrep; every path starts from l1 = 1 or 2
    "l12_inputs": ("128x2e+128x1e+128x2o", SH3,
                  "128x0e+128x0o+128x1e+128x1o+128x2e+128x2o+128x3e+128x3o"),
}


def _graph(rng, n, e, empty_frac=0.0, hub=None):
    recv = rng.integers(0, n, e)
    if empty_frac:
        pool = np.nonzero(rng.random(n) >= empty_frac)[0]
        recv = pool[rng.integers(0, len(pool), e)]
    if hub is not None:
        recv[: e // 3] = hub
    send = rng.integers(0, n, e)
    o = np.lexsort((send, recv))
    return send[o], recv[o]


def _inputs(rng, irreps, n, e):
    pl = oracle.plan(*irreps)
    return (pl, rng.normal(size=(n, pl.nx, pl.C)).astype(np.float16),
            rng.normal(size=(e, pl.ny)).astype(np.float16),
            rng.normal(size=(e, len(pl.paths), pl.C)).astype(np.float16))


@pytest.mark.parametrize("case", list(CASES))
@pytest.mark.parametrize("stages", [-1, 2, 4])
def test_tensor_core_parity(cuda_device, case, stages):
    irreps = CASES[case]
    rng = np.random.default_rng(len(case) * 10 + stages)
    n, e = 600, 9000
    send, recv = _graph(rng, n, e, empty_frac=0.15)
    pl, x, Y, s = _inputs(rng, irreps, n, e)
    conv = e3.Conv(*irreps, 15.0, dtype="f16")
    conv.set_tensor_cores(1)
    if stages != -1:
        conv.set_launch_config(0, 0, stages)
        conv.set_tensor_cores(1)
    info = conv.kernel_info()
    assert info["tensor_cores"] == 1 and info["local_bytes"] == 0
    gpu = run_gpu(conv, x, Y, s, send, recv, n)
    ref = oracle_out(irreps, x, Y, s, send, recv, n, 15.0)
    # hi + lo float16 coefficients: float32-level accuracy, far inside the 5e-3 bar
    assert column_scaled_error(gpu, ref) <= 1e-5
    assert np.all(gpu[np.setdiff1d(np.arange(n), recv)] == 0)


def test_tensor_core_matches_fp32_path(cuda_device):
    irreps = CASES["full16"]
    rng = np.random.default_rng(77)
    n, e = 2000, 60000
    send, recv = _graph(rng, n, e, hub=5)
    pl, x, Y, s = _inputs(rng, irreps, n, e)
    a = e3.Conv(*irreps, 30.0, dtype="f16")
    b = e3.Conv(*irreps, 30.0, dtype="f16")
    a.set_tensor_cores(1)
    assert a.kernel_info()["tensor_cores"] == 1 and b.kernel_info()["tensor_cores"] == 0
    ga = run_gpu(a, x, Y, s, send, recv, n)
    gb = run_gpu(b, x, Y, s, send, recv, n)
    ref = oracle_out(irreps, x, Y, s, send, recv, n, 30.0)
    rows = np.setdiff1d(np.arange(n), [5])
    assert column_scaled_error(ga[rows], ref[rows]) <= 1e-5
    assert column_scaled_error(gb[rows], ref[rows]) <= 1e-5
    scale = np.abs(ref).max()
    assert np.abs(ga - gb).max() <= 1e-4 * scale


def test_tensor_cores_are_opt_in(cuda_device):
    conv = e3.Conv(*CASES["full16"], 2.0, dtype="f16")
    assert conv.kernel_info()["tensor_cores"] == 0


def test_ineligible_shapes_fall_back_to_the_fp32_path(cuda_device):
    # Y rows of 9 float16 (18 bytes) cannot be bulk-copied; float32 inputs; C != 128
    for irreps, dt in ((("128x0e+128x1o", "1x0e+1x1o+1x2e", "128x0e+128x1o"), "f16"),
                       (CASES["full16"], "f32"), (("64x0e+64x1o", SH3, "64x0e+64x1o"), "f16")):
        conv = e3.Conv(*irreps, 2.0, dtype=dt)
        conv.set_tensor_cores(1)
        assert conv.kernel_info()["tensor_cores"] == 0


def test_tensor_core_few_nodes_no_edges_bad_indices(cuda_device):
    irreps = CASES["full16"]
    rng = np.random.default_rng(78)
    conv = e3.Conv(*irreps, 2.0, dtype="f16")
    conv.set_tensor_cores(1)
    assert conv.kernel_info()["tensor_cores"] == 1
    for n, e in ((1, 0), (2, 0), (1, 30), (3, 100)):
        send, recv = _graph(rng, n, e) if e else (np.zeros(0, np.int64), np.zeros(0, np.int64))
        pl, x, Y, s = _inputs(rng, irreps, n, e)
        gpu = run_gpu(conv, x, Y, s, send, recv, n)
        if e == 0:
            assert np.all(gpu == 0)
        else:
            ref = oracle_out(irreps, x, Y, s, send, recv, n, 2.0)
            assert np.all(np.abs(gpu - ref) <= 1e-5 * np.abs(ref).max())
    n, e = 40, 500
    send, recv = _graph(rng, n, e)
    pl, x, Y, s = _inputs(rng, irreps, n, e)
    bad = send.copy()
    bad[[3, 100, 499]] = [n, -5, 1 << 29]
    out = conv.forward(to_dev(x), to_dev(Y), to_dev(s), to_dev(bad.astype(np.int32)),
                       to_dev(row_ptr_of(recv, n).astype(np.int32)))
    assert not conv.check()
    keep = np.ones(e, bool)
    keep[[3, 100, 499]] = False
    ref = oracle_out(irreps, x, Y[keep], s[keep], send[keep], recv[keep], n, 2.0)
    assert column_scaled_error(out.cpu().numpy(), ref) <= 1e-5
    bad_rp = row_ptr_of(recv, n).astype(np.int32)
    bad_rp[7] = e + 1
    out = conv.forward(to_dev(x), to_dev(Y), to_dev(s), to_dev(send.astype(np.int32)), to_dev(bad_rp))
    assert not conv.check()
    assert conv.check()
    assert torch.isfinite(out).all()


def test_tensor_cores_full_size_sampled(cuda_device):
    # the full large_f16 workload on the device through the tensor-core kernel, checked on 256
    # seeded receivers (plus the first and last) against the oracle, and everywhere against
    # the float32 staged path
    from parity import DeviceWorkload, TOL
    w = DeviceWorkload("large_f16")
    w.conv.set_tensor_cores(1)
    assert w.conv.kernel_info()["tensor_cores"] == 1
    out = w.conv.forward(w.x, w.Y, w.s, w.senders, w.row_ptr)
    torch.cuda.synchronize()
    assert w.conv.check()
    rng = np.random.default_rng(54321)
    rows = np.unique(np.concatenate([[0, w.N - 1], rng.choice(w.N, 256, replace=False)]))
    ref = w.sample_reference(rows)
    gpu = out[torch.from_numpy(rows).cuda()].cpu().numpy()
    err = column_scaled_error(gpu, ref)
    assert err <= TOL["f16"], err
    assert err <= 1e-5, err        # the hi/lo split keeps the product at float32 accuracy
    w.conv.set_tensor_cores(0)
    base = w.conv.forward(w.x, w.Y, w.s, w.senders, w.row_ptr)
    torch.cuda.synchronize()
    assert w.conv.check()
    assert ((out - base).abs().max() / base.abs().max()).item() <= 1e-5
    del w, out, base
    torch.cuda.empty_cache()
