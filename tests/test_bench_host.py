"""Host-side checks of bench.py's accounting: the roofline's algorithmic bytes and FLOPs per
edge against independently enumerated per-config sizes, the peaks it divides by,
and the CPU-baseline sample sizing."""
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import equivariant_graph_message_b200 as e3  # noqa: E402
from workloads import configs  # noqa: E402

# (workload, bytes per edge of Y + s + sender index, sum of CG nonzeros, sum over paths of 2l3+1)
SIZES = [("gate_points", 468, 160, 68), ("mace", 5188, 86, 40),
         ("large_f32", 4676, 207, 64), ("large_f16", 8740, 611, 156)]


@pytest.mark.parametrize("name,edge_bytes,nnz,mix", SIZES)
def test_algorithmic_counts_match_enumerated_sizes(name, edge_bytes, nnz, mix):
    spec = configs.SPECS[name]
    conv = e3.Conv(spec.irreps_node, spec.irreps_sh, spec.irreps_out, 10.0, dtype=spec.dtype)
    b = 2 if spec.dtype == "f16" else 4
    E, N = 1000, 0
    nbytes, flops, got_nnz, got_mix = bench.algorithmic(conv, N, E, b)
    assert (got_nnz, got_mix) == (nnz, mix)
    assert nbytes == E * edge_bytes
    assert flops == 2 * E * conv.C * (nnz + mix)
    # per node: its features once, its outputs once, one row pointer
    nb1, _, _, _ = bench.algorithmic(conv, 1, 0, b)
    assert nb1 == conv.nx * conv.C * b + 4 * conv.nout * conv.C + 4


def test_peaks_are_positive_and_consistent():
    pk = bench.peaks()
    assert pk["hbm_gbs"] > 1000 and pk["f16_tflops"] > 100
    assert pk["fp32_tflops"] == pytest.approx(148 * 128 * 2 * pk["sm_max_mhz"] * 1e6 / 1e12)


def test_cpu_baseline_sample_is_seeded_and_bounded():
    spec = configs.SPECS["tiny"]
    g = configs.make_graph(spec)
    pl_x, yf, sf = bench.oracle_input_fns(spec, g)
    a = bench.calibrated_rows(spec, g, pl_x, yf, sf, 0.05)
    b = bench.calibrated_rows(spec, g, pl_x, yf, sf, 0.05)
    assert len(a) >= 1 and np.all(np.diff(a) > 0) and a[-1] < g.num_nodes
    # the same seed draws the same receivers, in the same order, up to the sample size
    n = min(len(a), len(b))
    order = np.random.default_rng(2024).permutation(g.num_nodes)
    assert set(a[:n]) <= set(order[:max(len(a), len(b))])


def test_traffic_is_reported_only_for_the_captured_configuration():
    # the committed DRAM counters belong to one (workload, node count, kernel source); any
    # other size or an edited kernel reports no traffic rather than a scaled guess
    import json
    d = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
    for key, rec in d.items():
        name, nodes = key.split("@")
        spec = configs.SPECS[name]
        c = e3.Conv(spec.irreps_node, spec.irreps_sh, spec.irreps_out, 40.0, dtype=spec.dtype)
        t, src = bench.traffic_for(name, c, int(nodes), rec["edges"])
        if rec["kernel_sha1"] == bench.kernel_hash(c):
            assert t == rec["dram_read_bytes"] + rec["dram_write_bytes"] and src
        else:
            assert t is None
        assert bench.traffic_for(name, c, int(nodes) * 10, rec["edges"] * 10) == (None, None)
        assert bench.traffic_for(name, c, int(nodes), rec["edges"], edge_vectors=True) == (None, None)


@pytest.mark.parametrize("name,flushed", [("tiny", True), ("gate_points", True), ("mace", False),
                                          ("large_f32", False), ("large_f16", False)])
def test_l2_flush_for_the_workloads_that_fit_in_l2(name, flushed):
    # a step's inputs smaller than twice the L2 are flushed before every timed step; the
    # workloads' full sizes decide which
    from workloads import make_graph
    spec = configs.SPECS[name]
    conv = e3.Conv(spec.irreps_node, spec.irreps_sh, spec.irreps_out, 10.0, dtype=spec.dtype)
    g = make_graph(spec)
    b = 2 if spec.dtype == "f16" else 4
    step_bytes = bench.algorithmic(conv, g.num_nodes, g.num_edges, b)[0]
    assert bench.needs_l2_flush(step_bytes) == flushed
