"""GPU CSR indexing and row gather: bit-exact against a host stable counting sort."""
import numpy as np
import pytest
import torch

import equivariant_graph_message_b200 as e3
from parity import row_ptr_of, to_dev

pytestmark = pytest.mark.gpu


def _host_csr(recv: np.ndarray, n: int):
    valid = (recv >= 0) & (recv < n)
    key = np.where(valid, recv, n)
    perm = np.argsort(key, kind="stable")
    return row_ptr_of(recv[valid], n), perm


CASES = {
    "empty": (np.zeros(0, np.int64), 5),
    "one_node": (np.zeros(17, np.int64), 1),
    "no_nodes_no_edges": (np.zeros(0, np.int64), 0),
    "small": (np.array([3, 1, 3, 0, 1, 3, 2, 2, 0]), 4),
    "sorted": (np.sort(np.random.default_rng(1).integers(0, 1000, 50000)), 1000),
    "random_ragged": (np.random.default_rng(2).integers(0, 4099, 12345), 4099),
    "hub": (np.where(np.random.default_rng(3).random(70000) < 0.6, 7,
                     np.random.default_rng(4).integers(0, 257, 70000)), 257),
    "many_nodes": (np.random.default_rng(5).integers(0, 70000, 300000), 70001),
    # row counts scanned in one launch up to 32,768 entries (N + 1 = 32,768), in levels above
    "scan_one_launch_max": (np.random.default_rng(7).integers(0, 32767, 40000), 32767),
    "scan_levels_min": (np.random.default_rng(8).integers(0, 32768, 40000), 32768),
    "large": (np.random.default_rng(6).integers(0, 100000, 4_000_000), 100000),
}


@pytest.mark.parametrize("name", list(CASES))
def test_build_csr_bit_exact(cuda_device, name):
    recv, n = CASES[name]
    row_ptr, perm, ws = e3.build_csr(to_dev(recv.astype(np.int32)), n)
    assert e3.csr_check(ws)
    rp_ref, perm_ref = _host_csr(recv, n)
    np.testing.assert_array_equal(row_ptr.cpu().numpy(), rp_ref)
    np.testing.assert_array_equal(perm.cpu().numpy(), perm_ref)


def test_build_csr_repeatable_with_reused_workspace(cuda_device):
    rng = np.random.default_rng(7)
    recv = rng.integers(0, 3000, 90000).astype(np.int32)
    ws = torch.empty(e3.csr_workspace_size(len(recv), 3000), dtype=torch.uint8, device="cuda")
    a = e3.build_csr(to_dev(recv), 3000, workspace=ws)
    b = e3.build_csr(to_dev(recv), 3000, workspace=ws)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_invalid_receivers_sorted_last_and_flagged(cuda_device):
    recv = np.array([2, -1, 0, 7, 2, 1, 5, 0], np.int64)   # n = 5: -1, 7, 5 invalid
    row_ptr, perm, ws = e3.build_csr(to_dev(recv.astype(np.int32)), 5)
    assert not e3.csr_check(ws)
    rp_ref, perm_ref = _host_csr(recv, 5)
    np.testing.assert_array_equal(row_ptr.cpu().numpy(), rp_ref)
    np.testing.assert_array_equal(perm.cpu().numpy(), perm_ref)
    assert list(perm.cpu().numpy()[-3:]) == [1, 3, 6]


def test_small_workspace_rejected(cuda_device):
    recv = to_dev(np.zeros(100, np.int32))
    need = e3.csr_workspace_size(100, 10)
    ws = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(e3.E3ConvError) as ei:
        e3.build_csr(recv, 10, workspace=ws)
    assert ei.value.code == 9


@pytest.mark.parametrize("row_shape,dtype", [((5,), torch.float32), ((34, 128), torch.float16),
                                             ((16,), torch.float16), ((3,), torch.int32)])
def test_permute_rows_bit_exact(cuda_device, row_shape, dtype):
    rng = np.random.default_rng(8)
    rows = 5000
    src = torch.from_numpy(rng.normal(size=(rows,) + row_shape)).to(dtype).cuda()
    perm = rng.permutation(rows).astype(np.int32)
    dst = e3.permute_rows(src, to_dev(perm))
    assert torch.equal(dst, src[torch.from_numpy(perm).long().cuda()])


def test_permute_rows_out_of_range_zero_filled(cuda_device):
    src = torch.arange(40, dtype=torch.float32, device="cuda").view(10, 4)
    perm = to_dev(np.array([3, 10, -1, 0], np.int32))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    dst = e3.permute_rows(src, perm, status=status)
    assert status.item() != 0
    assert torch.equal(dst[0], src[3]) and torch.equal(dst[3], src[0])
    assert torch.all(dst[1:3] == 0)
