"""Pins of the oracle's radial scalars (bessel basis x cosine cutoff -> SiLU MLP),
each against something other than the oracle's own formula:

* the cutoff's closed values (1 at d = 0, 1/2 at d = r/2, 0 at d = r) and the
  basis's zeros at d = r;
* the d -> 0 limit of sin(n pi d / r) / d, n pi / r (l'Hopital);
* orthonormality of the bessel functions under the weight d^2 on [0, r]
  (without the cutoff), by Gauss-Legendre quadrature;
* SiLU's identities: SiLU(0) = 0, SiLU(v) - SiLU(-v) = v, SiLU -> v for large v;
* the MLP against a brute-force evaluation with explicit loops on a tiny case;
* the scalars of the MACE-like workload (written by the input generator, a
  separate implementation) equal the oracle's to float32 rounding."""
from math import pi, sqrt

import numpy as np
import pytest

import oracle


@pytest.mark.parametrize("r", [1.0, 2.0, 5.0])
def test_cutoff_closed_values_and_zeros_at_the_radius(r):
    nb = 8
    b0 = oracle.bessel_cutoff([r * 1e-300], r, nb)[0]            # u(0) = 1: the bare limit
    np.testing.assert_allclose(b0, sqrt(2 / r) * np.arange(1, nb + 1) * pi / r, rtol=1e-12)
    half = oracle.bessel_cutoff([r / 2], r, nb)[0]
    bare = sqrt(2 / r) * np.sin(np.arange(1, nb + 1) * pi / 2) / (r / 2)
    np.testing.assert_allclose(half, 0.5 * bare, rtol=1e-13, atol=1e-15)   # u(r/2) = 1/2
    assert np.all(oracle.bessel_cutoff([r], r, nb) == 0)
    assert np.all(oracle.bessel_cutoff([1.5 * r], r, nb) == 0)
    near = oracle.bessel_cutoff([r * (1 - 1e-7)], r, nb)[0]
    assert np.abs(near).max() < 1e-12                                # B_n u -> 0 at the edge


def test_zero_length_takes_the_limit():
    r, nb = 5.0, 8
    at0 = oracle.bessel_cutoff([0.0], r, nb)[0]
    tiny = oracle.bessel_cutoff([1e-9], r, nb)[0]
    np.testing.assert_allclose(at0, sqrt(2 / r) * np.arange(1, nb + 1) * pi / r, rtol=1e-15)
    np.testing.assert_allclose(tiny, at0, rtol=1e-10)


def test_bessel_orthonormal_with_weight_d_squared():
    # int_0^r B_n(d) B_m(d) d^2 dd = (2/r) int_0^r sin(n pi d/r) sin(m pi d/r) dd = delta_nm;
    # the cutoff is divided out so only the basis is tested
    r, nb = 3.0, 8
    t, w = np.polynomial.legendre.leggauss(200)
    d = 0.5 * r * (t + 1)
    w = 0.5 * r * w
    u = 0.5 * (1 + np.cos(pi * d / r))
    B = oracle.bessel_cutoff(d, r, nb) / u[:, None]
    G = (B * (w * d * d)[:, None]).T @ B
    np.testing.assert_allclose(G, np.eye(nb), atol=1e-12)


def test_silu_identities():
    assert oracle.silu(0.0) == 0.0
    v = np.linspace(-20, 20, 81)
    np.testing.assert_allclose(oracle.silu(v) - oracle.silu(-v), v, atol=1e-13)
    assert abs(oracle.silu(40.0) - 40.0) < 1e-15
    assert abs(oracle.silu(-40.0)) < 1e-15
    np.testing.assert_allclose(oracle.silu(1.0), 1 / (1 + np.exp(-1.0)), rtol=1e-15)


def test_mlp_against_explicit_loops():
    rng = np.random.default_rng(9)
    r, sizes = 2.5, [3, 4, 5, 6]
    ws = [rng.normal(size=(a, b)) for a, b in zip(sizes[:-1], sizes[1:])]
    d = np.array([0.3, 1.1, 2.4])
    got = oracle.radial_mlp(d, r, ws)
    for q in range(len(d)):
        h = [sqrt(2 / r) * np.sin((n + 1) * pi * d[q] / r) / d[q] * 0.5 * (1 + np.cos(pi * d[q] / r))
             for n in range(sizes[0])]
        for layer, w in enumerate(ws):
            z = [sum(h[i] * w[i, j] for i in range(len(h))) for j in range(w.shape[1])]
            h = [zj / (1 + np.exp(-zj)) for zj in z] if layer < len(ws) - 1 else z
        np.testing.assert_allclose(got[q], h, rtol=1e-13, atol=1e-14)
