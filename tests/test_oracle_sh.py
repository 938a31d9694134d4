"""Pins of the oracle's real spherical harmonics and fitted Wigner-D matrices.

None of these re-types the harmonics' formula: they check properties that any
correct real, component-normalised degree-l basis must have."""
import numpy as np
import pytest

import oracle

LMAX = 6


def _unit(g, n):
    v = g.normal(size=(n, 3))
    return v / np.linalg.norm(v, axis=1, keepdims=True)


@pytest.mark.parametrize("l", range(LMAX + 1))
def test_addition_theorem(l):
    # sum_m Y_lm(v)^2 = 2l+1 for every unit v (component normalisation)
    v = _unit(np.random.default_rng(l), 500)
    y = oracle.sh_l(l, v)
    np.testing.assert_allclose((y * y).sum(1), 2 * l + 1, rtol=1e-13)


@pytest.mark.parametrize("l", range(LMAX + 1))
def test_addition_theorem_two_points(l):
    # sum_m Y_lm(a) Y_lm(b) = (2l+1) P_l(a.b): the Legendre polynomial of the angle
    g = np.random.default_rng(10 + l)
    a, b = _unit(g, 200), _unit(g, 200)
    lhs = (oracle.sh_l(l, a) * oracle.sh_l(l, b)).sum(1)
    from numpy.polynomial import legendre
    rhs = (2 * l + 1) * legendre.legval((a * b).sum(1), [0] * l + [1])
    np.testing.assert_allclose(lhs, rhs, atol=1e-12)


def test_orthonormal_by_exact_quadrature():
    # Gauss-Legendre in z (n nodes) x uniform phi (M points) integrates the
    # products of degree <= 2*LMAX exactly; (1/4pi) int Y Y' = identity.
    n, M = LMAX + 2, 2 * LMAX + 3
    z, wz = np.polynomial.legendre.leggauss(n)
    phi = 2 * np.pi * np.arange(M) / M
    Z, PHI = np.meshgrid(z, phi, indexing="ij")
    rho = np.sqrt(1 - Z ** 2)
    v = np.stack([rho * np.cos(PHI), rho * np.sin(PHI), Z], -1).reshape(-1, 3)
    w = (wz[:, None] * np.full(M, 2 * np.pi / M)[None, :]).reshape(-1) / (4 * np.pi)
    Y = oracle.sh(LMAX, v)
    G = (Y * w[:, None]).T @ Y
    np.testing.assert_allclose(G, np.eye(len(G)), atol=1e-12)


@pytest.mark.parametrize("l", range(LMAX + 1))
def test_parity(l):
    v = _unit(np.random.default_rng(20 + l), 100)
    np.testing.assert_allclose(oracle.sh_l(l, -v), (-1) ** l * oracle.sh_l(l, v), atol=1e-13)


@pytest.mark.parametrize("l", range(LMAX + 1))
def test_span_is_rotation_invariant(l):
    # The fitted D^l reproduces Y_l(R v) on directions not used by the fit:
    # only a true degree-l harmonic basis spans a rotation-invariant space.
    g = np.random.default_rng(30 + l)
    for _ in range(3):
        R = oracle.random_rotation(g)
        D = oracle.wigner_d(l, R)
        v = _unit(g, 50)
        np.testing.assert_allclose(oracle.sh_l(l, v @ R.T), oracle.sh_l(l, v) @ D.T, atol=1e-12)


@pytest.mark.parametrize("l", range(LMAX + 1))
def test_wigner_d_is_orthogonal_representation(l):
    g = np.random.default_rng(40 + l)
    R1, R2 = oracle.random_rotation(g), oracle.random_rotation(g)
    D1, D2 = oracle.wigner_d(l, R1), oracle.wigner_d(l, R2)
    np.testing.assert_allclose(D1 @ D1.T, np.eye(2 * l + 1), atol=1e-12)
    np.testing.assert_allclose(oracle.wigner_d(l, R1 @ R2), D1 @ D2, atol=1e-12)
    np.testing.assert_allclose(oracle.wigner_d(l, np.eye(3)), np.eye(2 * l + 1), atol=1e-12)
    np.testing.assert_allclose(np.linalg.det(D1), 1.0, atol=1e-11)


def test_l1_is_scaled_direction_in_yzx_order():
    # basis convention (our choice, the pages print none): l=1 is sqrt(3)(y, z, x)
    v = _unit(np.random.default_rng(50), 20)
    np.testing.assert_allclose(oracle.sh_l(1, v), np.sqrt(3) * v[:, [1, 2, 0]], atol=1e-14)
    np.testing.assert_allclose(oracle.sh_l(0, v), 1.0)


def test_worked_example_of_the_pages():
    # the pages' worked example (tests/golden/sh_worked_example.json, with its citation): two
    # vectors, harmonics up to l = 2 as one (2l+1)-component block per l; the values are pinned
    # by closed forms of the unit-direction harmonics, not by stored oracle output
    import json
    import pathlib
    fx = json.loads((pathlib.Path(__file__).parent / "golden" / "sh_worked_example.json").read_text())
    v = np.asarray(fx["vectors"], dtype=np.float64)
    u = v / np.linalg.norm(v, axis=1, keepdims=True)
    Y = oracle.sh(fx["lmax"], u)
    blocks = {l: Y[:, l * l:(l + 1) ** 2].reshape(len(v), 1, 2 * l + 1) for l in range(fx["lmax"] + 1)}
    assert {str(l): list(b.shape) for l, b in blocks.items()} == fx["shapes"]
    x, y, z = u[:, 0], u[:, 1], u[:, 2]
    np.testing.assert_allclose(blocks[0][:, 0, 0], 1.0, rtol=0, atol=1e-15)
    np.testing.assert_allclose(blocks[1][:, 0], np.sqrt(3) * np.stack([y, z, x], 1), rtol=0, atol=1e-14)
    # l = 2, m = -2..2 (component normalisation, no Condon-Shortley phase, z polar axis)
    Y2 = np.sqrt(15) * np.stack([x * y, y * z, (3 * z * z - 1) / (2 * np.sqrt(3)), x * z,
                                 (x * x - y * y) / 2], 1)
    np.testing.assert_allclose(blocks[2][:, 0], Y2, rtol=0, atol=1e-13)
    for l, b in blocks.items():   # sum over m of Y_lm^2 = 2l+1 for unit directions
        np.testing.assert_allclose((b[:, 0] ** 2).sum(1), 2 * l + 1, rtol=1e-13)
