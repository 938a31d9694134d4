"""Host checks on what the library's kernels are made of: no bulk or tensor copy with cluster
multicast anywhere (hand-written sources or any generated kernel), and no batched memory-copy
call.  Runs without a GPU (the generated sources come from the planner on the host)."""
import pathlib
import re

import pytest

import equivariant_graph_message_b200 as e3
from workloads import ORDER, SPECS

ROOT = pathlib.Path(__file__).resolve().parents[1]
SOURCES = sorted((ROOT / "equivariant_graph_message_b200" / "csrc").glob("*")) + \
    sorted((ROOT / "include").glob("*.h"))
BATCHED_COPY = re.compile(r"Memcpy\w*Batch")
MULTICAST = re.compile(r"\.multicast")          # the PTX qualifier on a copy or commit


def test_library_sources_have_no_multicast_and_no_batched_copies():
    assert SOURCES
    for p in SOURCES:
        text = p.read_text()
        assert not MULTICAST.search(text), p
        assert not BATCHED_COPY.search(text), p


@pytest.mark.parametrize("name", ORDER)
def test_generated_kernels_have_no_multicast(name):
    s = SPECS[name]
    c = e3.Conv(s.irreps_node, s.irreps_sh, s.irreps_out, 10.0, dtype=s.dtype)
    srcs = [c.kernel_source(), c.backward_source(0), c.backward_source(1)]
    if s.dtype == "f16" and c.C == 128:            # the tensor-core variant's source too
        c.set_tensor_cores(1)
        srcs.append(c.kernel_source())
    for src in srcs:
        assert not MULTICAST.search(src)
        assert "cp.async.bulk" in src or "cp.async" in src or "ldg" in src
