"""Pins of the oracle's backward (gradients of sum(g * out) with respect to x, Y
and s), each against the pinned forward oracle rather than the backward's own
loops:

* central finite differences of the forward along random directions in x, Y
  and s (the forward is linear in each, so the difference quotient is exact up
  to rounding);
* Euler's identity for a function linear in each argument:
  <g, f(x, Y, s)> = <grad_x, x> = <grad_Y, Y> = <grad_s, s>;
* per-edge locality: an edge's grad_Y and grad_s do not change when the other
  edges are removed, and grad_x of a node without outgoing edges is zero."""
import numpy as np
import pytest

import oracle

IRREPS = ("3x0e+3x1o+3x2e", "1x0e+1x1o+1x2e+1x3o", "3x0e+3x1o+3x1e+3x2e+3x3o")


def _case(seed, n=7, e=25):
    rng = np.random.default_rng(seed)
    pl = oracle.plan(*IRREPS)
    send, recv = rng.integers(0, n - 1, e), rng.integers(0, n, e)   # node n-1 sends nothing
    x = rng.normal(size=(n, pl.nx, pl.C))
    Y = rng.normal(size=(e, pl.ny))
    s = rng.normal(size=(e, len(pl.paths), pl.C))
    g = rng.normal(size=(n, pl.nout, pl.C))
    return rng, pl, send, recv, x, Y, s, g


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_directional_derivatives_match_finite_differences(seed):
    rng, pl, send, recv, x, Y, s, g = _case(seed)
    n, avg = len(x), 3.5
    gx, gY, gs = oracle.backward(*IRREPS, x, Y, s, send, recv, n, avg, g)

    def L(x_, Y_, s_):
        return float((g * oracle.forward(*IRREPS, x_, Y_, s_, send, recv, n, avg)).sum())

    h = 1e-3
    for arg, grad in ((0, gx), (1, gY), (2, gs)):
        base = [x, Y, s]
        d = rng.normal(size=base[arg].shape)
        plus = list(base)
        minus = list(base)
        plus[arg] = base[arg] + h * d
        minus[arg] = base[arg] - h * d
        fd = (L(*plus) - L(*minus)) / (2 * h)
        assert abs(fd - float((grad * d).sum())) <= 1e-9 * (1 + abs(fd))


def test_euler_identity_for_a_multilinear_function():
    rng, pl, send, recv, x, Y, s, g = _case(7, n=11, e=60)
    n, avg = len(x), 2.0
    gx, gY, gs = oracle.backward(*IRREPS, x, Y, s, send, recv, n, avg, g)
    total = float((g * oracle.forward(*IRREPS, x, Y, s, send, recv, n, avg)).sum())
    for grad, arg in ((gx, x), (gY, Y), (gs, s)):
        assert abs(float((grad * arg).sum()) - total) <= 1e-11 * (1 + abs(total))


def test_edge_locality_and_silent_senders():
    rng, pl, send, recv, x, Y, s, g = _case(3)
    n, avg = len(x), 1.7
    gx, gY, gs = oracle.backward(*IRREPS, x, Y, s, send, recv, n, avg, g)
    assert np.all(gx[n - 1] == 0)                        # node n-1 has no outgoing edge
    for e in (0, 5, 17):
        gx1, gY1, gs1 = oracle.backward(*IRREPS, x, Y[e:e + 1], s[e:e + 1], send[e:e + 1],
                                        recv[e:e + 1], n, avg, g)
        np.testing.assert_allclose(gY1[0], gY[e], rtol=1e-13, atol=1e-13)
        np.testing.assert_allclose(gs1[0], gs[e], rtol=1e-13, atol=1e-13)
