"""Real spherical harmonics of edge vectors, used to make edge features.

Basis (component normalisation, no Condon-Shortley phase, z polar axis,
components ordered m = -l..l):

    Y_{l,m}(v) = N_{l|m|} Q_l^{|m|}(z) * { Re (x+iy)^m   if m > 0
                                         { 1             if m = 0
                                         { Im (x+iy)^|m| if m < 0

for a unit vector v = (x, y, z), where Q_l^m = d^m P_l / dz^m and
N_{l0} = sqrt(2l+1), N_{lm} = sqrt(2 (2l+1) (l-m)! / (l+m)!), so that
sum_m Y_{l,m}(v)^2 = 2l+1.  Parity is (-1)^l.

This implementation uses the three-term Legendre recurrence; the oracle
evaluates the same basis independently from the Rodrigues polynomial.
A zero vector maps to Y^0 = 1 and Y^{l>0} = 0.
"""
from __future__ import annotations

from math import factorial, sqrt

import numpy as np


def sh_dim(lmax: int) -> int:
    return (lmax + 1) ** 2


def real_sh(vec: np.ndarray, lmax: int) -> np.ndarray:
    """vec: [E, 3] (any length; normalised here). Returns [E, (lmax+1)^2] float64."""
    vec = np.asarray(vec, dtype=np.float64)
    n = np.linalg.norm(vec, axis=1)
    zero = n == 0
    u = vec / np.where(zero, 1.0, n)[:, None]
    x, y, z = u[:, 0], u[:, 1], u[:, 2]
    E = len(vec)
    out = np.zeros((E, sh_dim(lmax)))
    # C_m + i S_m = (x + i y)^m
    C = [np.ones(E)]
    S = [np.zeros(E)]
    for m in range(lmax):
        C.append(x * C[m] - y * S[m])
        S.append(x * S[m] + y * C[m])
    # Q[l][m] = d^m P_l / dz^m via recurrences in l at fixed m
    Q = [[None] * (lmax + 1) for _ in range(lmax + 1)]
    for m in range(lmax + 1):
        dfact = 1.0
        for k in range(1, 2 * m, 2):
            dfact *= k
        Q[m][m] = np.full(E, dfact)
        if m + 1 <= lmax:
            Q[m + 1][m] = (2 * m + 1) * z * Q[m][m]
        for l in range(m + 2, lmax + 1):
            Q[l][m] = ((2 * l - 1) * z * Q[l - 1][m] - (l + m - 1) * Q[l - 2][m]) / (l - m)
    for l in range(lmax + 1):
        base = l * l + l
        out[:, base] = sqrt(2 * l + 1) * Q[l][0]
        for m in range(1, l + 1):
            nlm = sqrt(2.0 * (2 * l + 1) * factorial(l - m) / factorial(l + m))
            out[:, base + m] = nlm * Q[l][m] * C[m]
            out[:, base - m] = nlm * Q[l][m] * S[m]
    if zero.any():
        out[zero] = 0.0
        out[zero, 0] = 1.0
    return out
