"""GPU checks of e3conv_forward_rows, the forward over a contiguous range of
receiver rows (the rows one rank owns when receivers are partitioned into CSR
row ranges): a row's result does not depend on the range it is computed in,
so the ranges' outputs, concatenated, are bitwise the whole-graph output, for
the direct, staged and tensor-core variants; and the outputs match the
oracle."""
import numpy as np
import pytest
import torch

import equivariant_graph_message_b200 as e3
from parity import column_scaled_error, oracle_out, row_ptr_of, to_dev

pytestmark = pytest.mark.gpu

SH3 = "1x0e+1x1o+1x2e+1x3o"
CASES = {
    # (irreps, dtype, tensor cores)
    "direct_C5": (("5x0e+5x0o+5x1e+5x1o", SH3, "5x0e+5x0o+5x1e+5x1o+5x2e+5x2o"), "f32", 0),
    "staged_C128": (("128x0e+128x1o", SH3, "128x0e+128x1o+128x2e+128x3o"), "f32", 0),
    "staged_C64_f16": (("64x0e+64x1o+64x2e", SH3, "64x0e+64x1o+64x2e"), "f16", 0),
    "tensor_cores": (("128x0e+128x1o+128x2e+128x3o", SH3,
                      "128x0e+128x1o+128x2e+128x3o"), "f16", 1),
}


def _graph(rng, n, e):
    recv = rng.integers(0, n, e)
    recv[: e // 10] = n // 3          # a row longer than one 128-edge chunk
    send = rng.integers(0, n, e)
    o = np.lexsort((send, recv))
    return send[o], recv[o]


@pytest.mark.parametrize("case", list(CASES))
def test_row_ranges_concatenate_to_the_whole_graph(cuda_device, case):
    irreps, dt, tc = CASES[case]
    rng = np.random.default_rng(31 + len(case))
    n, e = 700, 14000
    send, recv = _graph(rng, n, e)
    conv = e3.Conv(*irreps, 20.0, dtype=dt)
    if tc:
        conv.set_tensor_cores(1)
        assert conv.kernel_info()["tensor_cores"] == 1
    npdt = np.float16 if dt == "f16" else np.float32
    x = rng.normal(size=(n, conv.nx, conv.C)).astype(npdt)
    Y = rng.normal(size=(e, conv.ny)).astype(npdt)
    s = rng.normal(size=(e, conv.num_paths, conv.C)).astype(npdt)
    rp = row_ptr_of(recv, n)
    xd, Yd, sd = to_dev(x), to_dev(Y), to_dev(s)
    snd = to_dev(send.astype(np.int32))
    rpd = to_dev(rp.astype(np.int32))
    whole = conv.forward(xd, Yd, sd, snd, rpd)
    bounds = [0, 1, 233, 234, 234, 512, n]          # includes an empty and a one-row range
    parts = []
    for b0, b1 in zip(bounds[:-1], bounds[1:]):
        e0, e1 = int(rp[b0]), int(rp[b1])
        parts.append(conv.forward_rows(xd, Yd[e0:e1].contiguous(), sd[e0:e1].contiguous(),
                                       snd[e0:e1].contiguous(), rpd, b0, b1))
    torch.cuda.synchronize()
    assert conv.check()
    assert torch.equal(torch.cat(parts), whole)
    ref = oracle_out(irreps, x, Y, s, send, recv, n, 20.0)
    tol = 5e-3 if dt == "f16" and not tc else 1e-5
    assert column_scaled_error(whole.cpu().numpy(), ref) <= tol


def test_rebased_row_ptr_and_a_separate_sender_table(cuda_device):
    # a rank's view: its rows' CSR rebased to start at 0, and a sender table whose rows are
    # not the receivers (here: the node rows permuted, senders renumbered to match)
    irreps, dt, _ = CASES["staged_C128"]
    rng = np.random.default_rng(5)
    n, e = 300, 6000
    send, recv = _graph(rng, n, e)
    conv = e3.Conv(*irreps, 20.0, dtype=dt)
    x = rng.normal(size=(n, conv.nx, conv.C)).astype(np.float32)
    Y = rng.normal(size=(e, conv.ny)).astype(np.float32)
    s = rng.normal(size=(e, conv.num_paths, conv.C)).astype(np.float32)
    rp = row_ptr_of(recv, n)
    whole = conv.forward(to_dev(x), to_dev(Y), to_dev(s), to_dev(send.astype(np.int32)),
                         to_dev(rp.astype(np.int32)))
    b0, b1 = 120, 250
    e0, e1 = int(rp[b0]), int(rp[b1])
    table_perm = rng.permutation(n + 17) % n          # a larger table with repeated rows
    pos = np.zeros(n, np.int64)
    pos[table_perm[::-1]] = np.arange(len(table_perm))[::-1]   # one table row per node
    table = x[table_perm]
    local_rp = (rp[b0:b1 + 1] - rp[b0]).astype(np.int32)
    out = conv.forward_rows(to_dev(table), to_dev(Y[e0:e1]), to_dev(s[e0:e1]),
                            to_dev(pos[send[e0:e1]].astype(np.int32)), to_dev(local_rp),
                            0, b1 - b0)
    torch.cuda.synchronize()
    assert conv.check()
    assert torch.equal(out, whole[b0:b1])
