"""Pins of the oracle's irreps linear layer (channel mixing within matching irreps,
scale / sqrt(mul_in), unmatched outputs zero), each against something other
than its own einsum:

* identity weights give scale / sqrt(mul) times the matching blocks;
* outputs without a matching input irrep are exactly zero;
* explicit loops on a tiny case;
* equivariance: rotating every input block by its Wigner-D (acting on the
  2l+1 components) rotates the output the same way, and parity-odd blocks
  flip sign under inversion together with the input."""
from math import sqrt

import numpy as np

import oracle


def _blocks(irreps, x):
    out, off = [], 0
    for ir in oracle.parse_irreps(irreps):
        out.append((ir, x[:, off:off + ir.dim * ir.mul].reshape(len(x), ir.dim, ir.mul)))
        off += ir.dim * ir.mul
    return out


def test_identity_weights_and_unmatched_zeros():
    rng = np.random.default_rng(0)
    ins, outs = "4x0e+4x1o+4x2e", "4x0e+4x1e+4x1o+4x3o"
    x = rng.normal(size=(5, 4 + 12 + 20))
    y = oracle.irreps_linear(ins, outs, 0.7, x, [np.eye(4), np.eye(4)])
    bx = dict(((ir.l, ir.p), b) for ir, b in _blocks(ins, x))
    for ir, b in _blocks(outs, y):
        if (ir.l, ir.p) in bx:
            np.testing.assert_allclose(b, 0.7 / 2.0 * bx[(ir.l, ir.p)], rtol=1e-15)
        else:
            assert np.all(b == 0)


def test_explicit_loops():
    rng = np.random.default_rng(1)
    ins, outs = "3x0e+3x1o", "2x1o+2x0e"
    x = rng.normal(size=(2, 3 + 9))
    w1o, w0e = rng.normal(size=(3, 2)), rng.normal(size=(3, 2))
    y = oracle.irreps_linear(ins, outs, 1.3, x, [w1o, w0e])
    for n in range(2):
        for k in range(3):            # 1o block: output offset 0, input offset 3
            for v in range(2):
                ref = sum(x[n, 3 + 3 * k + u] * w1o[u, v] for u in range(3)) * 1.3 / sqrt(3)
                assert abs(y[n, 2 * k + v] - ref) < 1e-14
        for v in range(2):            # 0e block: output offset 6, input offset 0
            ref = sum(x[n, u] * w0e[u, v] for u in range(3)) * 1.3 / sqrt(3)
            assert abs(y[n, 6 + v] - ref) < 1e-14


def test_equivariance_under_rotations_and_inversion():
    rng = np.random.default_rng(2)
    ins, outs = "6x0e+6x1o+6x2e+6x3o", "5x0e+5x1o+5x2e+5x3o"
    x = rng.normal(size=(7, 6 * 16))
    ws = [rng.normal(size=(6, 5)) for _ in range(4)]

    def act(irreps, arr, R, inv):
        res = arr.copy()
        off = 0
        for ir in oracle.parse_irreps(irreps):
            b = arr[:, off:off + ir.dim * ir.mul].reshape(len(arr), ir.dim, ir.mul)
            D = oracle.wigner_d(ir.l, R) * (ir.p if inv else 1)
            res[:, off:off + ir.dim * ir.mul] = np.einsum("kj,nju->nku", D, b).reshape(len(arr), -1)
            off += ir.dim * ir.mul
        return res

    for trial in range(4):
        R = oracle.random_rotation(rng)
        inv = trial % 2 == 1
        y1 = oracle.irreps_linear(ins, outs, 1.0, act(ins, x, R, inv), ws)
        y2 = act(outs, oracle.irreps_linear(ins, outs, 1.0, x, ws), R, inv)
        np.testing.assert_allclose(y1, y2, atol=1e-11)
