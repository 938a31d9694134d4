"""Oracle for the equivariant message-passing convolution (float64, CPU).

TEST INFRASTRUCTURE ONLY.  Only the tests, the package's smoke check and the
benchmark's CPU-baseline / reference arm may import or run anything here.  It
shares no code with the CUDA path.

What it computes (page "e3j.core.Convolution", class docstring):

    m_b = (1/N) sum_{a -> b} (x_a (x)_CG Y_ab) . s_ab

* (x)_CG is the channelwise ("uvu") Clebsch-Gordan tensor product of the node
  irreps x_a with the real spherical harmonics Y_ab (cuEquivariance-JAX notes,
  "Dense polynomial" and "Split irrep polynomials on CPU": channelwise
  products, weights first).
* . s_ab multiplies every path and channel by its own edge scalar
  (e3j "__call__": edge_scalars has shape (num_edges, num_scalars, C)).
* Paths that produce the same output irrep are summed.
* N is avg_num_neighbors (e3j parameter list).
* CG normalisation SQRT_DIM_OUT (e3j default) = sqrt(2 l3 + 1) times the
  unit-Frobenius real Wigner-3j tensor; NONE = the unit-Frobenius tensor.

Independent pieces, each pinned by tests in tests/test_oracle_*.py:

* real spherical harmonics from the Rodrigues polynomial (sh_l);
* real Wigner-D matrices fitted from those harmonics by least squares
  (wigner_d);
* the real Wigner-3j tensor as the null space of the stacked intertwiner
  equations for two rotations (wigner_3j);
* path enumeration and output layout (plan);
* the explicit edgewise loops (forward.c, via forward()).

Readings where the pages are silent are listed in the design notes: sign of
the Wigner-3j tensor (first nonzero entry in row-major order is positive),
summing same-output paths, 1/N with N = avg_num_neighbors, the output filter
as an intersection, and the canonical path order (node irrep -> sh degree ->
output irrep in filter order).
"""
from __future__ import annotations

import ctypes
import os
import re
from dataclasses import dataclass
from functools import lru_cache
from math import factorial, sqrt

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liboracle.so")

# ---------------------------------------------------------------------------
# Irreps and paths


@dataclass(frozen=True)
class Irrep:
    mul: int
    l: int
    p: int  # +1 even, -1 odd

    @property
    def dim(self) -> int:
        return 2 * self.l + 1


def parse_irreps(text: str) -> list[Irrep]:
    """'4x0e+4x1o' -> [Irrep(4,0,+1), Irrep(4,1,-1)]; the multiplicity defaults to 1."""
    out = []
    for term in text.replace(" ", "").split("+"):
        if not term:
            continue
        m = re.fullmatch(r"(?:(\d+)x)?(\d+)([eo])", term)
        if not m:
            raise ValueError(f"bad irrep term {term!r}")
        out.append(Irrep(int(m.group(1) or 1), int(m.group(2)), 1 if m.group(3) == "e" else -1))
    return out


@dataclass(frozen=True)
class Path:
    n1: int      # index of the node irrep
    l1: int
    p1: int
    x_off: int   # first component of that irrep in a node feature row
    l2: int
    y_off: int   # l2 * l2
    o: int       # index of the output irrep among the produced ones
    l3: int
    p3: int
    out_off: int


@dataclass
class Plan:
    C: int
    nx: int
    ny: int
    nout: int
    paths: list
    outputs: list   # produced output irreps (l, p, offset)


def plan(irreps_node: str, irreps_sh: str, irreps_out: str) -> Plan:
    node = parse_irreps(irreps_node)
    sh = parse_irreps(irreps_sh)
    filt = parse_irreps(irreps_out)
    if not node:
        raise ValueError("no node irreps")
    C = node[0].mul
    if any(ir.mul != C for ir in node) or any(ir.mul != C for ir in filt):
        raise ValueError("all node and output multiplicities must equal C")
    for k, ir in enumerate(sh):
        if ir.mul != 1 or ir.l != k or ir.p != (-1) ** k:
            raise ValueError("edge irreps must be 1x0e+1x1o+1x2e+... (consecutive l, parity (-1)^l)")
    if len({(ir.l, ir.p) for ir in filt}) != len(filt):
        raise ValueError("duplicate output irrep")
    lmax = len(sh) - 1
    produced = set()
    raw = []
    x_off = 0
    for n1, ir in enumerate(node):
        for l2 in range(lmax + 1):
            for ir3 in filt:
                if abs(ir.l - l2) <= ir3.l <= ir.l + l2 and ir3.p == ir.p * (-1) ** l2:
                    raw.append((n1, ir.l, ir.p, x_off, l2, (ir3.l, ir3.p)))
                    produced.add((ir3.l, ir3.p))
        x_off += ir.dim
    outputs = []
    off = 0
    for ir3 in filt:
        if (ir3.l, ir3.p) in produced:
            outputs.append((ir3.l, ir3.p, off))
            off += 2 * ir3.l + 1
    where = {(l, p): (i, o) for i, (l, p, o) in enumerate(outputs)}
    paths = [Path(n1, l1, p1, xo, l2, l2 * l2, where[key][0], key[0], key[1], where[key][1])
             for (n1, l1, p1, xo, l2, key) in raw]
    return Plan(C, x_off, (lmax + 1) ** 2, off, paths, outputs)


# ---------------------------------------------------------------------------
# Real spherical harmonics (component normalisation, no Condon-Shortley
# phase, z polar, m = -l..l):
#   Y_{l,m}(v) = N_{l|m|} (d^{|m|} P_l / dz^{|m|})(z) * {Re (x+iy)^m, 1, Im (x+iy)^{|m|}}
# with N_{l0} = sqrt(2l+1), N_{lm} = sqrt(2 (2l+1) (l-m)!/(l+m)!).

def _legendre(l: int) -> np.polynomial.Polynomial:
    """P_l from the explicit sum 2^-l sum_k (-1)^k C(l,k) C(2l-2k,l) z^(l-2k)."""
    c = np.zeros(l + 1)
    for k in range(l // 2 + 1):
        c[l - 2 * k] = (-1) ** k * _binom(l, k) * _binom(2 * l - 2 * k, l) / 2.0 ** l
    return np.polynomial.Polynomial(c)


def _binom(n: int, k: int) -> float:
    return factorial(n) / (factorial(k) * factorial(n - k))


def sh_l(l: int, v: np.ndarray) -> np.ndarray:
    """Real SH of degree l of unit vectors v [K,3] -> [K, 2l+1]."""
    v = np.asarray(v, dtype=np.float64)
    x, y, z = v[:, 0], v[:, 1], v[:, 2]
    pl = _legendre(l)
    out = np.zeros((len(v), 2 * l + 1))
    w = (x + 1j * y)
    for m in range(l + 1):
        q = pl.deriv(m)(z) if m else pl(z)
        if m == 0:
            out[:, l] = sqrt(2 * l + 1) * q
        else:
            nlm = sqrt(2.0 * (2 * l + 1) * factorial(l - m) / factorial(l + m))
            wm = w ** m
            out[:, l + m] = nlm * q * wm.real
            out[:, l - m] = nlm * q * wm.imag
    return out


def sh(lmax: int, v: np.ndarray) -> np.ndarray:
    """[K,3] unit vectors -> [K, (lmax+1)^2], l-major."""
    return np.concatenate([sh_l(l, v) for l in range(lmax + 1)], axis=1)


# ---------------------------------------------------------------------------
# Real Wigner-D, fitted from the harmonics: Y_l(R v) = D^l(R) Y_l(v)

def _fit_points(l: int) -> np.ndarray:
    g = np.random.default_rng(1000 + l)
    v = g.normal(size=(8 * (2 * l + 1) + 8, 3))
    return v / np.linalg.norm(v, axis=1, keepdims=True)


def wigner_d(l: int, R: np.ndarray) -> np.ndarray:
    """Least-squares D with sh_l(V R^T) = sh_l(V) D^T for sample directions V."""
    V = _fit_points(l)
    A = sh_l(l, V)
    B = sh_l(l, V @ np.asarray(R).T)
    Dt, *_ = np.linalg.lstsq(A, B, rcond=None)
    return Dt.T


def random_rotation(g: np.random.Generator) -> np.ndarray:
    q, r = np.linalg.qr(g.normal(size=(3, 3)))
    q = q * np.sign(np.diag(r))
    if np.linalg.det(q) < 0:
        q[:, 0] = -q[:, 0]
    return q


# ---------------------------------------------------------------------------
# Real Wigner-3j: the unit vector spanning the null space of
#   sum_ij W_ijk D1_ii' D2_jj' - sum_k' D3_kk' W_i'j'k' = 0
# stacked for two fixed rotations; sign: first |W| > 1e-9 (row-major) positive.

@lru_cache(maxsize=None)
def wigner_3j(l1: int, l2: int, l3: int) -> np.ndarray:
    if not abs(l1 - l2) <= l3 <= l1 + l2:
        raise ValueError("triangle rule violated")
    d1, d2, d3 = 2 * l1 + 1, 2 * l2 + 1, 2 * l3 + 1
    g = np.random.default_rng(4242)
    blocks = []
    for _ in range(2):
        R = random_rotation(g)
        D1, D2, D3 = wigner_d(l1, R), wigner_d(l2, R), wigner_d(l3, R)
        blocks.append(np.kron(np.kron(D1.T, D2.T), np.eye(d3))
                      - np.kron(np.eye(d1 * d2), D3))
    M = np.concatenate(blocks, axis=0)
    _, sv, vt = np.linalg.svd(M)
    if not (sv[-1] < 1e-9 and (len(sv) < 2 or sv[-2] > 1e-3)):
        raise RuntimeError(f"intertwiner null space not one-dimensional for {(l1, l2, l3)}")
    w = vt[-1].reshape(d1, d2, d3)
    w = w / np.linalg.norm(w)
    flat = w.ravel()
    first = flat[np.nonzero(np.abs(flat) > 1e-9)[0][0]]
    return w * np.sign(first)


NORMALIZATIONS = {"SQRT_DIM_OUT": 0, "NONE": 1}


def cg(l1: int, l2: int, l3: int, normalization: str = "SQRT_DIM_OUT") -> np.ndarray:
    w = wigner_3j(l1, l2, l3)
    if normalization == "SQRT_DIM_OUT":
        return sqrt(2 * l3 + 1) * w
    if normalization == "NONE":
        return w.copy()
    raise ValueError(normalization)


# ---------------------------------------------------------------------------
# Radial scalars s_ab: an MLP of radial-basis encodings of the edge length
# (e3j.core.Convolution, class docstring: the edge scalars are an MLP of RBF
# encodings; gate_points_2102 page, "Scope": bessel radial bases and a cosine
# cutoff; its Network parameters number_of_basis, radial_layers and
# radial_neurons).  The pages print neither formula; the readings are
#   B_n(d) = sqrt(2 / r) sin(n pi d / r) / d,   n = 1 .. num_basis
#   u(d)   = (1 + cos(pi d / r)) / 2 for d < r, 0 otherwise (cosine cutoff)
#   h_0 = B(d) u(d);  h_{l+1} = SiLU(h_l W_l) for the hidden layers;
#   s = h_L W_L (no activation on the output layer, no biases),
# with SiLU(v) = v / (1 + exp(-v)).


def bessel_cutoff(d, r_max: float, num_basis: int) -> np.ndarray:
    """[K, num_basis]: B_n(d) u(d) for edge lengths d [K] (d = 0 takes the limit n pi / r)."""
    d = np.asarray(d, dtype=np.float64)
    n = np.arange(1, num_basis + 1, dtype=np.float64)
    out = np.empty((len(d), num_basis))
    for q in range(len(d)):
        if d[q] >= r_max:
            out[q] = 0.0
            continue
        u = 0.5 * (1.0 + np.cos(np.pi * d[q] / r_max))
        if d[q] == 0.0:
            out[q] = sqrt(2.0 / r_max) * n * np.pi / r_max * u
        else:
            out[q] = sqrt(2.0 / r_max) * np.sin(n * np.pi * d[q] / r_max) / d[q] * u
    return out


def silu(v):
    v = np.asarray(v, dtype=np.float64)
    return v / (1.0 + np.exp(-v))


def radial_mlp(d, r_max: float, weights) -> np.ndarray:
    """[K, out] edge scalars from edge lengths d [K]; weights = [W_0 (num_basis x h), ...,
    W_L (h x out)] in float64 (inputs are upcast exactly)."""
    ws = [np.asarray(w, dtype=np.float64) for w in weights]
    h = bessel_cutoff(d, r_max, ws[0].shape[0])
    for w in ws[:-1]:
        h = silu(h @ w)
    return h @ ws[-1]


# ---------------------------------------------------------------------------
# Irreps linear layer (cuEquivariance-JAX notes, "Flax NNX layers": channel
# mixing within matching irreps, scale / sqrt(mul_in), unmatched outputs zero),
# on the convolution's layout: per node, each irrep block is [2l+1][mul].


def irreps_linear(irreps_in: str, irreps_out: str, scale: float, x, weights) -> np.ndarray:
    """y [N][dim_out] (float64): for each output irrep matching an input irrep (same l and
    parity), y_o[n, k, v] = scale / sqrt(mul_in) * sum_u x_o[n, k, u] W[u, v], with the next
    weight block of `weights` (one per matched output irrep, in output order); others 0."""
    ins, outs = parse_irreps(irreps_in), parse_irreps(irreps_out)
    x = np.asarray(x, dtype=np.float64)
    n = x.shape[0]
    dim_out = sum(ir.dim * ir.mul for ir in outs)
    y = np.zeros((n, dim_out))
    w_iter = iter(weights)
    off_out = 0
    for ir in outs:
        off_in = 0
        match = None
        for jr in ins:
            if (jr.l, jr.p) == (ir.l, ir.p):
                match = (jr, off_in)
            off_in += jr.dim * jr.mul
        if match is not None:
            jr, oi = match
            W = np.asarray(next(w_iter), dtype=np.float64)
            xb = x[:, oi:oi + jr.dim * jr.mul].reshape(n, jr.dim, jr.mul)
            yb = scale / sqrt(jr.mul) * np.einsum("nku,uv->nkv", xb, W)
            y[:, off_out:off_out + ir.dim * ir.mul] = yb.reshape(n, -1)
        off_out += ir.dim * ir.mul
    return y


# ---------------------------------------------------------------------------
# Forward (explicit loops in forward.c)

_lib = None


def _load():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            from .build import build
            build()
        lib = ctypes.CDLL(LIB_PATH)
        i64p = np.ctypeslib.ndpointer(np.int64, flags="C")
        f64p = np.ctypeslib.ndpointer(np.float64, flags="C")
        i32p = np.ctypeslib.ndpointer(np.int32, flags="C")
        lib.oracle_forward.argtypes = [ctypes.c_int64, ctypes.c_int64] + [ctypes.c_int] * 5 + \
            [f64p, f64p, f64p, i64p, i64p] + [i32p] * 6 + [f64p, i64p, ctypes.c_double, f64p,
                                                          ctypes.c_int]
        lib.oracle_forward.restype = ctypes.c_int
        lib.oracle_backward.argtypes = [ctypes.c_int64, ctypes.c_int64] + [ctypes.c_int] * 5 + \
            [f64p, f64p, f64p, i64p, i64p] + [i32p] * 6 + [f64p, i64p, ctypes.c_double, f64p,
                                                          f64p, f64p, f64p]
        lib.oracle_backward.restype = ctypes.c_int
        lib.oracle_max_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def max_threads() -> int:
    return _load().oracle_max_threads()


def forward(irreps_node: str, irreps_sh: str, irreps_out: str, x, Y, s, senders, receivers,
            num_nodes: int, avg_num_neighbors: float, normalization: str = "SQRT_DIM_OUT",
            threads: int = 0) -> np.ndarray:
    """out[N][nout][C] (float64) of the convolution; inputs are upcast exactly to float64."""
    pl = plan(irreps_node, irreps_sh, irreps_out)
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
    Y = np.ascontiguousarray(np.asarray(Y, dtype=np.float64))
    s = np.ascontiguousarray(np.asarray(s, dtype=np.float64))
    senders = np.ascontiguousarray(np.asarray(senders, dtype=np.int64))
    receivers = np.ascontiguousarray(np.asarray(receivers, dtype=np.int64))
    E = len(senders)
    P = len(pl.paths)
    assert x.shape == (num_nodes, pl.nx, pl.C), (x.shape, (num_nodes, pl.nx, pl.C))
    assert Y.shape == (E, pl.ny), Y.shape
    assert s.shape == (E, P, pl.C), s.shape
    assert receivers.shape == (E,)
    cols = {k: np.array([getattr(p, k) for p in pl.paths] or [0], dtype=np.int32)
            for k in ("l1", "x_off", "l2", "y_off", "l3", "out_off")}
    cgs = [cg(p.l1, p.l2, p.l3, normalization).ravel() for p in pl.paths]
    offs = np.zeros(max(1, P), dtype=np.int64)
    if P:
        offs[1:P] = np.cumsum([c.size for c in cgs])[:-1]
    cgcat = np.concatenate(cgs) if cgs else np.zeros(1)
    out = np.zeros((num_nodes, pl.nout, pl.C))
    rc = _load().oracle_forward(num_nodes, E, pl.C, pl.nx, pl.ny, P, pl.nout, x, Y, s, senders,
                                receivers, cols["l1"], cols["x_off"], cols["l2"], cols["y_off"],
                                cols["l3"], cols["out_off"], cgcat, offs,
                                1.0 / avg_num_neighbors, out, int(threads))
    if rc != 0:
        raise ValueError("oracle_forward: index out of range" if rc == -1 else "oracle_forward failed")
    return out


def backward(irreps_node: str, irreps_sh: str, irreps_out: str, x, Y, s, senders, receivers,
             num_nodes: int, avg_num_neighbors: float, grad_out,
             normalization: str = "SQRT_DIM_OUT"):
    """(grad_x [N][nx][C], grad_Y [E][ny], grad_s [E][P][C]) in float64: the gradients of
    sum(grad_out * forward(...)) with respect to x, Y and s (explicit loops in backward.c)."""
    pl = plan(irreps_node, irreps_sh, irreps_out)
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
    Y = np.ascontiguousarray(np.asarray(Y, dtype=np.float64))
    s = np.ascontiguousarray(np.asarray(s, dtype=np.float64))
    g = np.ascontiguousarray(np.asarray(grad_out, dtype=np.float64))
    senders = np.ascontiguousarray(np.asarray(senders, dtype=np.int64))
    receivers = np.ascontiguousarray(np.asarray(receivers, dtype=np.int64))
    E = len(senders)
    P = len(pl.paths)
    assert x.shape == (num_nodes, pl.nx, pl.C) and Y.shape == (E, pl.ny)
    assert s.shape == (E, P, pl.C) and g.shape == (num_nodes, pl.nout, pl.C)
    cols = {k: np.array([getattr(p, k) for p in pl.paths] or [0], dtype=np.int32)
            for k in ("l1", "x_off", "l2", "y_off", "l3", "out_off")}
    cgs = [cg(p.l1, p.l2, p.l3, normalization).ravel() for p in pl.paths]
    offs = np.zeros(max(1, P), dtype=np.int64)
    if P:
        offs[1:P] = np.cumsum([c.size for c in cgs])[:-1]
    cgcat = np.concatenate(cgs) if cgs else np.zeros(1)
    gx = np.zeros_like(x)
    gY = np.zeros_like(Y) if E else np.zeros((1, pl.ny))
    gs = np.zeros_like(s) if E else np.zeros((1, P, pl.C))
    rc = _load().oracle_backward(num_nodes, E, pl.C, pl.nx, pl.ny, P, pl.nout, x,
                                 Y if E else np.zeros((1, pl.ny)), s if E else np.zeros((1, P, pl.C)),
                                 senders if E else np.zeros(1, np.int64),
                                 receivers if E else np.zeros(1, np.int64),
                                 cols["l1"], cols["x_off"], cols["l2"], cols["y_off"], cols["l3"],
                                 cols["out_off"], cgcat, offs, 1.0 / avg_num_neighbors, g, gx, gY, gs)
    if rc != 0:
        raise ValueError("oracle_backward: index out of range")
    return gx, gY[:E], gs[:E]
