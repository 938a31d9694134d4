"""Pins of the oracle's real Wigner-3j / Clebsch-Gordan tensors."""
import itertools

import numpy as np
import pytest

import oracle

LMAX = 4
TRIPLES = [(a, b, c) for a in range(LMAX + 1) for b in range(LMAX + 1)
           for c in range(abs(a - b), min(a + b, LMAX) + 1)]


def _unit(g, n):
    v = g.normal(size=(n, 3))
    return v / np.linalg.norm(v, axis=1, keepdims=True)


def test_closed_form_000():
    np.testing.assert_allclose(oracle.wigner_3j(0, 0, 0), [[[1.0]]])


@pytest.mark.parametrize("l", range(LMAX + 1))
def test_closed_form_identity_paths(l):
    d = 2 * l + 1
    eye = np.eye(d) / np.sqrt(d)
    np.testing.assert_allclose(oracle.wigner_3j(0, l, l)[0], eye, atol=1e-13)   # 0 x l -> l
    np.testing.assert_allclose(oracle.wigner_3j(l, 0, l)[:, 0, :], eye, atol=1e-13)  # l x 0 -> l
    np.testing.assert_allclose(oracle.wigner_3j(l, l, 0)[:, :, 0], eye, atol=1e-13)  # dot product
    # with SQRT_DIM_OUT the 0 x l -> l path is exactly the identity (pure scaling)
    np.testing.assert_allclose(oracle.cg(0, l, l)[0], np.eye(d), atol=1e-13)


def test_closed_form_110_is_normalised_dot_product():
    np.testing.assert_allclose(oracle.cg(1, 1, 0)[:, :, 0], np.eye(3) / np.sqrt(3), atol=1e-14)


def test_closed_form_111_is_cross_product():
    # components ordered (y, z, x), a cyclic order of (x, y, z), so the
    # Levi-Civita symbol keeps its sign; first nonzero (0,1,2) is positive.
    eps = np.zeros((3, 3, 3))
    for (i, j, k), sgn in zip(itertools.permutations(range(3)), [1, -1, -1, 1, 1, -1]):
        eps[i, j, k] = sgn
    np.testing.assert_allclose(oracle.wigner_3j(1, 1, 1), eps / np.sqrt(6), atol=1e-14)
    a, b = np.array([0.3, -1.2, 0.7]), np.array([1.1, 0.4, -0.5])   # (x,y,z)
    out = np.einsum("ijk,i,j->k", oracle.cg(1, 1, 1), a[[1, 2, 0]], b[[1, 2, 0]])
    np.testing.assert_allclose(out, np.cross(a, b)[[1, 2, 0]] / np.sqrt(2), atol=1e-14)


def test_closed_form_112_symmetric_traceless():
    w = oracle.wigner_3j(1, 1, 2)
    np.testing.assert_allclose(w, w.transpose(1, 0, 2), atol=1e-14)
    np.testing.assert_allclose(np.einsum("iik->k", w), 0, atol=1e-14)


@pytest.mark.parametrize("l1,l2,l3", TRIPLES)
def test_unit_norm_and_sign_rule(l1, l2, l3):
    w = oracle.wigner_3j(l1, l2, l3)
    assert abs(np.linalg.norm(w) - 1) < 1e-13
    flat = w.ravel()
    assert flat[np.nonzero(np.abs(flat) > 1e-9)[0][0]] > 0


@pytest.mark.parametrize("l1,l2,l3", TRIPLES)
def test_equivariance_fresh_rotations(l1, l2, l3):
    g = np.random.default_rng(hash((l1, l2, l3)) % 2 ** 32)
    w = oracle.wigner_3j(l1, l2, l3)
    for _ in range(2):
        R = oracle.random_rotation(g)
        D1, D2, D3 = (oracle.wigner_d(l, R) for l in (l1, l2, l3))
        lhs = np.einsum("ijk,ia,jb->abk", w, D1, D2)
        rhs = np.einsum("kc,abc->abk", D3, w)
        np.testing.assert_allclose(lhs, rhs, atol=1e-12)


@pytest.mark.parametrize("l1,l2,l3", TRIPLES)
def test_swap_symmetry(l1, l2, l3):
    # W^{l2 l1 l3}_{jik} = (-1)^{l1+l2+l3} W^{l1 l2 l3}_{ijk} up to the sign rule;
    # for l1 == l2 the sign is fixed: W_jik = (-1)^{l3} W_ijk.
    w = oracle.wigner_3j(l1, l2, l3)
    v = oracle.wigner_3j(l2, l1, l3).transpose(1, 0, 2)
    assert np.allclose(v, w, atol=1e-13) or np.allclose(v, -w, atol=1e-13)
    if l1 == l2:
        np.testing.assert_allclose(v, (-1) ** l3 * w, atol=1e-13)


@pytest.mark.parametrize("l1,l2", [(a, b) for a in range(4) for b in range(4)])
def test_orthogonality_and_completeness(l1, l2):
    d1, d2 = 2 * l1 + 1, 2 * l2 + 1
    rows = []
    for l3 in range(abs(l1 - l2), l1 + l2 + 1):
        w = oracle.wigner_3j(l1, l2, l3)
        G = np.einsum("ijk,ijm->km", w, w)
        np.testing.assert_allclose(G, np.eye(2 * l3 + 1) / (2 * l3 + 1), atol=1e-13)
        for l3b in range(abs(l1 - l2), l3):
            wb = oracle.wigner_3j(l1, l2, l3b)
            np.testing.assert_allclose(np.einsum("ijk,ijm->km", w, wb), 0, atol=1e-13)
        rows.append(np.sqrt(2 * l3 + 1) * w.reshape(d1 * d2, -1))
    U = np.concatenate(rows, axis=1)     # (d1 d2) x (d1 d2): an orthogonal change of basis
    np.testing.assert_allclose(U @ U.T, np.eye(d1 * d2), atol=1e-12)


@pytest.mark.parametrize("l1,l2,l3", [t for t in TRIPLES if t[0] + t[1] <= LMAX])
def test_product_of_harmonics(l1, l2, l3):
    # sum_ij W_ijk Y^l1_i(v) Y^l2_j(v) = kappa Y^l3_k(v) with kappa independent of v,
    # nonzero iff l1 + l2 + l3 is even (parity of a product at one point).
    v = _unit(np.random.default_rng(7), 40)
    w = oracle.wigner_3j(l1, l2, l3)
    prod = np.einsum("ijk,vi,vj->vk", w, oracle.sh_l(l1, v), oracle.sh_l(l2, v))
    y3 = oracle.sh_l(l3, v)
    if (l1 + l2 + l3) % 2:
        np.testing.assert_allclose(prod, 0, atol=1e-12)
    else:
        kappa = (prod * y3).sum() / (y3 * y3).sum()
        assert abs(kappa) > 1e-3
        np.testing.assert_allclose(prod, kappa * y3, atol=1e-12)


def test_triangle_rule_rejected():
    with pytest.raises(ValueError):
        oracle.wigner_3j(1, 1, 3)
    with pytest.raises(ValueError):
        oracle.wigner_3j(0, 2, 1)


def test_normalizations():
    w = oracle.wigner_3j(2, 1, 3)
    np.testing.assert_allclose(oracle.cg(2, 1, 3, "NONE"), w)
    np.testing.assert_allclose(oracle.cg(2, 1, 3, "SQRT_DIM_OUT"), np.sqrt(7) * w)
    with pytest.raises(ValueError):
        oracle.cg(2, 1, 3, "NORM")
