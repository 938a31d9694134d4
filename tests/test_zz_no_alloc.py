"""The allocation-free CSR build (e3conv_build_csr_noalloc), for callers that
cannot allocate device memory (a framework allocator owns it, a fixed memory
budget, or a latency-critical path that must not call cudaMalloc).

Called through the C ABI and compared bit for bit with e3conv_build_csr, the
entry point with a caller-provided workspace, on two calls in a row (the
second smaller than the first, so leftovers of the first in the shared
scratch would show).  This file sorts last so that a run stopping at the
first failure has run every other test first."""
import ctypes

import numpy as np
import pytest
import torch

import equivariant_graph_message_b200 as e3

pytestmark = pytest.mark.gpu


def _noalloc(recv_d, n):
    E = recv_d.shape[0]
    row_ptr = torch.full((n + 1,), -7, dtype=torch.int32, device=recv_d.device)
    perm = torch.full((max(E, 1),), -7, dtype=torch.int32, device=recv_d.device)[:E]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = e3._lib.e3conv_build_csr_noalloc(
        ctypes.c_void_p(recv_d.data_ptr()), ctypes.c_int64(E), ctypes.c_int64(n),
        ctypes.c_void_p(row_ptr.data_ptr()), ctypes.c_void_p(perm.data_ptr()), stream)
    return rc, row_ptr, perm


def test_noalloc_matches_workspace_entry_point_on_two_calls(cuda_device):
    rng = np.random.default_rng(2027)
    cases = [(1_500_000, 60_000), (40_000, 1_000)]
    for E, n in cases:
        recv = rng.integers(0, n, E).astype(np.int32)
        recv[rng.integers(0, E, 5)] = n + 3        # a few out-of-range receivers
        recv_d = torch.from_numpy(recv).cuda()
        rc, rp_b, perm_b = _noalloc(recv_d, n)
        assert rc == 0, e3._last_error().decode()
        rp_a, perm_a, ws = e3.build_csr(recv_d, n)
        torch.cuda.synchronize()
        assert torch.equal(rp_a, rp_b) and torch.equal(perm_a, perm_b)
        assert rp_b[-1].item() == E - 5            # out-of-range receivers are not counted
        valid = recv < n
        expect = np.argsort(np.where(valid, recv, n), kind="stable")
        assert np.array_equal(perm_b.cpu().numpy(), expect)


def test_noalloc_rejects_sizes_beyond_its_scratch(cuda_device):
    need = e3.csr_workspace_size(4_000_000, 100_000)
    assert need > (32 << 20)
    recv_d = torch.zeros(1, dtype=torch.int32, device="cuda")
    row_ptr = torch.zeros(2, dtype=torch.int32, device="cuda")
    # rejected on the host from the sizes alone, before any launch
    rc = e3._lib.e3conv_build_csr_noalloc(
        ctypes.c_void_p(recv_d.data_ptr()), ctypes.c_int64(4_000_000), ctypes.c_int64(100_000),
        ctypes.c_void_p(row_ptr.data_ptr()), ctypes.c_void_p(recv_d.data_ptr()), None)
    assert rc == 9
    assert "32" in e3._last_error().decode() or "scratch" in e3._last_error().decode()
