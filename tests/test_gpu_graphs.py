"""The step's library calls are safe to capture in CUDA graphs: e3conv_build_csr and
e3conv_forward launch on the given stream and neither allocate nor synchronise, so a
captured graph replayed over new inputs (written in place) gives bitwise the eager results,
and the status words stay clean."""
import numpy as np
import pytest
import torch

import equivariant_graph_message_b200 as e3
from parity import row_ptr_of, to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("irreps,dt", [
    (("128x0e+128x1o", "1x0e+1x1o+1x2e", "128x0e+128x1o+128x2e"), "f32"),
    (("5x0e+5x1o", "1x0e+1x1o+1x2e", "5x0e+5x1o+5x2e"), "f32"),
    (("128x0e+128x1o+128x2e+128x3o", "1x0e+1x1o+1x2e+1x3o", "128x0e+128x1o"), "f16"),
])
def test_captured_step_replays_bitwise(cuda_device, irreps, dt):
    rng = np.random.default_rng(5)
    n, e = 600, 9000
    conv = e3.Conv(*irreps, 15.0, dtype=dt)
    tdt = torch.float16 if dt == "f16" else torch.float32
    recv = to_dev(rng.integers(0, n, e).astype(np.int32))
    send = to_dev(rng.integers(0, n, e).astype(np.int32))
    x = torch.empty((n, conv.nx, conv.C), dtype=tdt, device="cuda")
    Y = torch.empty((e, conv.ny), dtype=tdt, device="cuda")
    s = torch.empty((e, conv.num_paths, conv.C), dtype=tdt, device="cuda")
    row_ptr = torch.empty(n + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(e, dtype=torch.int32, device="cuda")
    ws = torch.empty(e3.csr_workspace_size(e, n), dtype=torch.uint8, device="cuda")
    out = torch.empty((n, conv.nout, conv.C), dtype=torch.float32, device="cuda")
    send_sorted = torch.empty_like(send)

    def fill(seed):
        g = torch.Generator(device="cuda").manual_seed(seed)
        x.copy_(torch.randn(x.shape, generator=g, device="cuda"))
        Y.copy_(torch.randn(Y.shape, generator=g, device="cuda"))
        s.copy_(torch.randn(s.shape, generator=g, device="cuda"))

    def step(h):
        e3._ok(e3._build_csr(e3._ptr(recv), e, n, e3._ptr(row_ptr), e3._ptr(perm), e3._ptr(ws),
                             ws.numel(), h), "e3conv_build_csr")
        conv.forward_raw(e3._ptr(x), e3._ptr(Y), e3._ptr(s), e3._ptr(send_sorted),
                         e3._ptr(row_ptr), n, e3._ptr(out), h)

    # the edges are given in receiver order (senders permuted once, outside the step)
    order = np.argsort(recv.cpu().numpy(), kind="stable")
    send_sorted.copy_(send[torch.from_numpy(order).cuda()])
    recv.copy_(recv[torch.from_numpy(order).cuda()])
    fill(1)
    step(e3._stream_handle(torch.cuda.current_stream()))
    torch.cuda.synchronize()
    eager = out.clone()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step(e3._stream_handle(torch.cuda.current_stream()))
    out.fill_(float("nan"))
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, eager)
    fill(2)                                   # new inputs in place: the replay reads them
    step(e3._stream_handle(torch.cuda.current_stream()))
    torch.cuda.synchronize()
    eager2 = out.clone()
    out.fill_(float("nan"))
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, eager2) and not torch.equal(eager, eager2)
    assert np.array_equal(row_ptr.cpu().numpy(), row_ptr_of(recv.cpu().numpy(), n).astype(np.int32))
    assert e3.csr_check(ws) and conv.check()
