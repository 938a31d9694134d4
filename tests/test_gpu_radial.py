"""GPU parity of the radial scalars on the tensor cores (e3conv_radial_scalars):
bessel basis x cosine cutoff of |r_ab|, SiLU hidden layers, output layer of
P*C scalars; against the oracle's float64 MLP of the same float32 vectors and
weights.  Ragged tiles, zero-length and out-of-radius edges, widths, depths,
float16 output, output counts that are not a multiple of the 128-column
chunk; then the convolution fed with these scalars against the oracle."""
import numpy as np
import pytest
import torch

import equivariant_graph_message_b200 as e3
import oracle
from parity import column_scaled_error, oracle_out, row_ptr_of, to_dev
from workloads import SPECS, configs, make_graph, node_features_np

pytestmark = pytest.mark.gpu

SH3 = "1x0e+1x1o+1x2e+1x3o"


def _vec4(vec):
    v = np.zeros((len(vec), 4), np.float32)
    v[:, :3] = vec
    return v


def _reference(v4, r_max, ws):
    d = np.linalg.norm(v4[:, :3].astype(np.float64), axis=1)
    return oracle.radial_mlp(d, r_max, [w.astype(np.float64) for w in ws])


def _weights(rng, nb, hidden, layers, nout):
    sizes = [nb] + [hidden] * layers + [nout]
    return [(rng.normal(size=(a, b)) / np.sqrt(a)).astype(np.float32)
            for a, b in zip(sizes[:-1], sizes[1:])]


@pytest.mark.parametrize("hidden,layers,nb", [(64, 2, 8), (32, 1, 5), (32, 3, 16), (64, 4, 8)])
@pytest.mark.parametrize("dtype", ["f32", "f16"])
def test_radial_scalars_match_the_oracle(cuda_device, hidden, layers, nb, dtype):
    irreps = ("32x0e+32x1o", SH3, "32x0e+32x1o+32x2e")       # P*C = 7 * 32 = 224: ragged chunk
    conv = e3.Conv(*irreps, 10.0, dtype=dtype)
    P, C = conv.num_paths, conv.C
    rng = np.random.default_rng(hidden + layers)
    r_max = 2.5
    ws = _weights(rng, nb, hidden, layers, P * C)
    conv.set_radial_mlp(r_max, ws)
    E = 1000                                                  # 7 full tiles + a ragged one
    vec = rng.normal(size=(E, 3))
    vec *= rng.uniform(0.05, 1.2 * r_max, size=(E, 1)) / np.linalg.norm(vec, axis=1, keepdims=True)
    vec[3] = 0.0                                              # zero length: the basis limit
    vec[4] = [r_max, 0, 0]                                    # on the cutoff radius: zeros
    vec[5] = [0, 0, 3 * r_max]                                # outside: zeros
    v4 = _vec4(vec)
    s = conv.radial_scalars(to_dev(v4))
    torch.cuda.synchronize()
    assert conv.check()
    got = s.float().cpu().numpy().reshape(E, P * C)
    ref = _reference(v4, r_max, ws)
    scale = np.abs(ref).max(axis=0)
    err = (np.abs(got - ref) / np.where(scale > 0, scale, 1)).max()
    # float32-level rounding compounds over the layers: 1e-5 for up to two hidden layers,
    # 1e-5 per hidden layer beyond (scalars rounded to float16 are checked at 2e-3)
    assert err <= (2e-3 if dtype == "f16" else 1e-5 * max(1, layers - 1)), err
    assert np.all(got[4] == 0) and np.all(got[5] == 0)


@pytest.mark.parametrize("hidden,layers,nb", [(64, 2, 8), (32, 1, 5), (32, 3, 16), (64, 4, 8)])
@pytest.mark.parametrize("dtype", ["f32", "f16"])
def test_radial_scalars_many_tiles_per_cta(cuda_device, hidden, layers, nb, dtype):
    # every CTA runs three or four tiles of four output chunks (the last ragged), so the
    # kernel reuses its activation buffers, its output-weight ring and its three output
    # accumulators across chunks and tiles; widths and depths cover one and two activation
    # buffers and rings of two to four weight chunks
    irreps = ("64x0e+64x1o", SH3, "64x0e+64x1o+64x2e")       # P*C = 7 * 64 = 448: 4 chunks
    conv = e3.Conv(*irreps, 10.0, dtype=dtype)
    P, C = conv.num_paths, conv.C
    rng = np.random.default_rng(7 * hidden + layers)
    r_max = 2.5
    ws = _weights(rng, nb, hidden, layers, P * C)
    conv.set_radial_mlp(r_max, ws)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    E = sms * 128 * 3 + 77                                    # 3 tiles per CTA, some 4
    vec = rng.normal(size=(E, 3))
    vec *= rng.uniform(0.05, 1.2 * r_max, size=(E, 1)) / np.linalg.norm(vec, axis=1, keepdims=True)
    v4 = _vec4(vec)
    s = conv.radial_scalars(to_dev(v4))
    torch.cuda.synchronize()
    assert conv.check()
    got = s.float().cpu().numpy().reshape(E, P * C)
    ref = _reference(v4, r_max, ws)
    scale = np.abs(ref).max(axis=0)
    err = (np.abs(got - ref) / np.where(scale > 0, scale, 1)).max()
    assert err <= (2e-3 if dtype == "f16" else 1e-5 * max(1, layers - 1)), err


def test_radial_scalars_few_edges_and_none(cuda_device):
    conv = e3.Conv("128x0e+128x1o", SH3, "128x0e+128x1o", 3.0)
    rng = np.random.default_rng(3)
    ws = _weights(rng, 8, 64, 2, conv.num_paths * conv.C)
    conv.set_radial_mlp(5.0, ws)
    for E in (1, 37, 128, 129):
        v4 = _vec4(rng.normal(size=(E, 3)))
        s = conv.radial_scalars(to_dev(v4)).cpu().numpy().reshape(E, -1)
        ref = _reference(v4, 5.0, ws)
        assert np.abs(s - ref).max() <= 1e-5 * np.abs(ref).max()
    empty = conv.radial_scalars(torch.zeros((0, 4), dtype=torch.float32, device="cuda"))
    assert empty.shape[0] == 0
    assert conv.check()


def test_mace_scalars_and_convolution(cuda_device):
    # the MACE-like workload: its seeded MLP on the tensor cores, then the convolution fed
    # with those scalars, against the oracle's MLP and convolution
    spec = SPECS["mace"]
    g = make_graph(spec)
    ws = [w.astype(np.float32) for w in configs.radial_weights(spec)]
    irreps = (spec.irreps_node, spec.irreps_sh, spec.irreps_out)
    conv = e3.Conv(*irreps, g.avg_num_neighbors)
    conv.set_radial_mlp(spec.graph["r"], ws)
    v4 = _vec4(g.vec)
    s = conv.radial_scalars(to_dev(v4))
    ref_s = _reference(v4, spec.graph["r"], ws).reshape(g.num_edges, spec.num_paths, spec.C)
    got_s = s.cpu().numpy()
    scale = np.abs(ref_s).max()
    assert np.abs(got_s - ref_s).max() <= 1e-5 * scale
    x = node_features_np(spec, g.num_nodes)
    conv.set_edge_vectors(1)
    out = conv.forward(to_dev(x), to_dev(v4), s, to_dev(g.senders.astype(np.int32)),
                       to_dev(row_ptr_of(g.receivers, g.num_nodes).astype(np.int32)))
    torch.cuda.synchronize()
    assert conv.check()
    d = np.linalg.norm(v4[:, :3].astype(np.float64), axis=1, keepdims=True)
    Y = oracle.sh(spec.lmax, v4[:, :3].astype(np.float64) / d)
    ref = oracle_out(irreps, x, Y, ref_s, g.senders, g.receivers, g.num_nodes, g.avg_num_neighbors)
    assert column_scaled_error(out.cpu().numpy(), ref) <= 1e-5


def test_radial_rejects_widths_beyond_shared_memory():
    conv = e3.Conv("32x0e+32x1o", SH3, "32x0e+32x1o", 3.0)
    rng = np.random.default_rng(0)
    with pytest.raises(e3.E3ConvError):
        conv.set_radial_mlp(2.0, _weights(rng, 8, 128, 2, conv.num_paths * conv.C))


@pytest.mark.parametrize("dtype", ["f32", "f16"])
def test_radial_scalars_rows_not_multiple_of_16_bytes(cuda_device, dtype):
    # P*C = 5 * 3 = 15 scalars per edge: rows of 60 (float32) or 30 (float16) bytes take the
    # element-by-element store path instead of the bulk row copies
    irreps = ("3x0e+3x1o", SH3, "3x0e+3x1o")
    conv = e3.Conv(*irreps, 10.0, dtype=dtype)
    nout = conv.num_paths * conv.C
    assert (nout * (2 if dtype == "f16" else 4)) % 16 != 0
    rng = np.random.default_rng(21)
    ws = _weights(rng, 8, 64, 2, nout)
    conv.set_radial_mlp(3.0, ws)
    E = 300
    v4 = _vec4(rng.normal(size=(E, 3)))
    s = conv.radial_scalars(to_dev(v4))
    torch.cuda.synchronize()
    assert conv.check()
    got = s.float().cpu().numpy().reshape(E, nout)
    ref = _reference(v4, 3.0, ws)
    scale = np.abs(ref).max(axis=0)
    err = (np.abs(got - ref) / np.where(scale > 0, scale, 1)).max()
    assert err <= (2e-3 if dtype == "f16" else 1e-5), err
