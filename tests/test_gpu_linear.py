"""GPU parity of the irreps linear layer on the tensor cores (e3conv_linear_*)
against the oracle's float64 layer, for both kernels (tensor-map tiles and
row-per-thread): the convolution's output irreps mixed into other
multiplicities, unmatched output irreps, ragged row tiles, few nodes, and the
convolution's full-size output of the large mixed-precision workload."""
import numpy as np
import pytest
import torch

import equivariant_graph_message_b200 as e3
import oracle
from parity import to_dev

pytestmark = pytest.mark.gpu


# (irreps_in, irreps_out, whether the tensor-map kernel takes the shape)
SHAPES = [
    ("128x0e+128x1o+128x2e+128x3o", "64x0e+64x1o+64x2e+64x3o", True),
    ("64x0e+64x1o+64x2e", "128x0e+128x1e+128x1o+128x2e+128x3o", True),     # unmatched 1e, 3o
    ("32x0e+32x1o", "256x1o+256x0e", True),
    ("128x0e+128x1o+128x2e+128x3o", "16x3o+16x0e", False),                  # mul_out 16
    ("128x0e+128x1o", "256x0e+256x1o", False),                              # room for one stage
    ("64x0e+64x1o+64x2e+64x3o+64x4e+64x5o+64x6e", "96x6e+96x0e+96x4e+96x5o", True),  # 13 rows a node
]


@pytest.mark.parametrize("tma", [True, False])
@pytest.mark.parametrize("ins,outs,fits", SHAPES)
@pytest.mark.parametrize("nodes", [1, 5, 300, 2049])
def test_linear_matches_the_oracle(cuda_device, ins, outs, fits, nodes, tma):
    lin = e3.IrrepsLinear(ins, outs, 0.7)
    lin.set_tma(tma)
    assert lin.uses_tma == (tma and fits)
    rng = np.random.default_rng(nodes + len(ins))
    ws = [rng.normal(size=(lin.mul_in, lin.mul_out)).astype(np.float32)
          for _ in range(lin.num_weight_blocks)]
    lin.set_weights(ws)
    x = rng.normal(size=(nodes, lin.dim_in)).astype(np.float32)
    y = torch.full((nodes, lin.dim_out), float("nan"), device="cuda")
    lin(to_dev(x), out=y)
    torch.cuda.synchronize()
    assert lin.check()
    ref = oracle.irreps_linear(ins, outs, 0.7, x, ws)
    got = y.cpu().numpy()
    # elementwise against the float32 dot-product bound: each output is a sum of mul_in
    # products, whose rounding error is bounded by a multiple of the sum of their magnitudes
    # (the result itself may cancel); 1e-5 of that sum covers the split products' 2^-22 and
    # the float32 accumulation for mul_in <= 128
    mag = oracle.irreps_linear(ins, outs, 0.7, np.abs(x), [np.abs(w) for w in ws])
    assert np.all(np.abs(got - ref) <= 1e-5 * mag + 1e-30)
    unmatched = mag == 0
    assert np.all(got[unmatched] == 0)
    assert not np.isnan(got).any()


def test_linear_on_the_convolution_output_full_size(cuda_device):
    from parity import DeviceWorkload
    w = DeviceWorkload("large_f16")
    out = w.conv.forward(w.x, w.Y, w.s, w.senders, w.row_ptr)
    conv_irreps = "+".join(f"128x{l}{'e' if p > 0 else 'o'}" for l, p, _ in w.conv.outputs)
    lin = e3.IrrepsLinear(conv_irreps, conv_irreps, 1.0)
    rng = np.random.default_rng(5)
    ws = [rng.normal(size=(128, 128)).astype(np.float32) for _ in range(lin.num_weight_blocks)]
    lin.set_weights(ws)
    assert lin.uses_tma
    y = lin(out.view(w.N, -1))
    lin.set_tma(False)
    y_rows = lin(out.view(w.N, -1))       # the row-per-thread kernel on the same input
    torch.cuda.synchronize()
    assert lin.check()
    # both kernels form the same three float16 products per term and accumulate them in
    # float32 on the tensor cores in the same order: the same results
    assert torch.equal(y, y_rows)
    rows = np.unique(np.concatenate([[0, w.N - 1], rng.choice(w.N, 512, replace=False)]))
    xr = out.view(w.N, -1)[torch.from_numpy(rows).cuda()].cpu().numpy()
    ref = oracle.irreps_linear(conv_irreps, conv_irreps, 1.0, xr, ws)
    got = y[torch.from_numpy(rows).cuda()].cpu().numpy()
    assert np.abs(got - ref).max() <= 1e-5 * np.abs(ref).max()
    del w, out, y, y_rows
    torch.cuda.empty_cache()


def test_linear_repeated_and_changed_buffers(cuda_device):
    # the tensor-map kernel keeps the arguments of its last launch: repeated calls on the same
    # buffers (new contents), then other buffers and node counts, and new weights, all match
    ins = outs = "64x0e+64x1o+64x2e"
    lin = e3.IrrepsLinear(ins, outs, 1.0)
    assert lin.uses_tma
    rng = np.random.default_rng(11)

    def weights():
        ws = [rng.normal(size=(64, 64)).astype(np.float32) for _ in range(lin.num_weight_blocks)]
        lin.set_weights(ws)
        return ws

    def check(x, y, ws):
        torch.cuda.synchronize()
        assert lin.check()
        xs = x.cpu().numpy()
        ref = oracle.irreps_linear(ins, outs, 1.0, xs, ws)
        mag = oracle.irreps_linear(ins, outs, 1.0, np.abs(xs), [np.abs(w) for w in ws])
        assert np.all(np.abs(y.cpu().numpy() - ref) <= 1e-5 * mag + 1e-30)

    ws = weights()
    x1 = torch.from_numpy(rng.normal(size=(777, lin.dim_in)).astype(np.float32)).cuda()
    y1 = torch.empty((777, lin.dim_out), device="cuda")
    lin(x1, out=y1)
    check(x1, y1, ws)
    x1.copy_(torch.from_numpy(rng.normal(size=(777, lin.dim_in)).astype(np.float32)))
    lin(x1, out=y1)                                   # same buffers, new contents
    check(x1, y1, ws)
    lin(x1[:300], out=y1[:300])                       # same pointers, fewer nodes
    check(x1[:300], y1[:300], ws)
    x2 = torch.from_numpy(rng.normal(size=(1500, lin.dim_in)).astype(np.float32)).cuda()
    y2 = torch.empty((1500, lin.dim_out), device="cuda")
    lin(x2, out=y2)                                   # other buffers
    check(x2, y2, ws)
    ws = weights()                                    # new weights on the same buffers
    lin(x2, out=y2)
    check(x2, y2, ws)


@pytest.mark.parametrize("ins,outs", [
    ("64x0e+64x1o+64x2e", "64x0e+64x1o+64x2e"),                 # five 32 KB stages
    ("32x0e+32x1o", "256x1o+256x0e"),                           # six 16 KB stages, N = 256
    ("64x0e+64x1o+64x2e+64x3o", "96x3o+96x1e+96x0e"),           # unmatched 1e among them
])
def test_linear_many_tiles_per_cta(cuda_device, ins, outs):
    # 20,000 nodes: every CTA runs many tiles of several irreps, so the tensor-map kernel
    # wraps its ring of input stages, reuses both accumulators and changes weights mid-range
    lin = e3.IrrepsLinear(ins, outs, 0.9)
    assert lin.uses_tma
    rng = np.random.default_rng(21)
    ws = [rng.normal(size=(lin.mul_in, lin.mul_out)).astype(np.float32)
          for _ in range(lin.num_weight_blocks)]
    lin.set_weights(ws)
    n = 20000
    x = rng.normal(size=(n, lin.dim_in)).astype(np.float32)
    y = torch.full((n, lin.dim_out), float("nan"), device="cuda")
    lin(to_dev(x), out=y)
    torch.cuda.synchronize()
    assert lin.check()
    got = y.cpu().numpy()
    ref = oracle.irreps_linear(ins, outs, 0.9, x, ws)
    mag = oracle.irreps_linear(ins, outs, 0.9, np.abs(x), [np.abs(w) for w in ws])
    assert np.all(np.abs(got - ref) <= 1e-5 * mag + 1e-30)
    assert not np.isnan(got).any()
