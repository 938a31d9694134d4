"""Counter-based seeded random numbers for the synthetic workloads.

Every random tensor of a workload is a function of (seed, tensor id, element
index), so any single element can be regenerated on the host without
materialising the whole tensor.  This is what lets a test compare a sample of
a multi-gigabyte device tensor against a host recomputation.

Generator (both host and device follow the same published definitions):

* splitmix64 (S. Vigna, public-domain reference generator): the output for
  state z is mix(z + 0x9E3779B97F4A7C15) with
  mix(z) = z ^ (z >> 31) after z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9 and
  z = (z ^ (z >> 27)) * 0x94D049BB133111EB.
* The stream for (seed, tid) starts at key = splitmix64(seed * 2**16 + tid);
  draw k of that stream is splitmix64(key + k * 0x9E3779B97F4A7C15), i.e. the
  (k+1)-th output of a splitmix64 generator seeded with key.
* uniform(k) = (draw(k) >> 11) * 2**-53, in [0, 1).
* normal(k) uses the Box-Muller transform on draws 2k and 2k+1:
  sqrt(-2 ln(1 - u0)) * cos(2 pi u1).

This module holds no arithmetic of the convolution itself.
"""
from __future__ import annotations

import numpy as np

GAMMA = 0x9E3779B97F4A7C15
M1 = 0xBF58476D1CE4E5B9
M2 = 0x94D049BB133111EB
MASK64 = (1 << 64) - 1


def _mix_np(z: np.ndarray) -> np.ndarray:
    z = z.astype(np.uint64, copy=False)
    z = (z ^ (z >> np.uint64(30))) * np.uint64(M1)
    z = (z ^ (z >> np.uint64(27))) * np.uint64(M2)
    return z ^ (z >> np.uint64(31))


def splitmix64_next(state: int) -> tuple[int, int]:
    """One step of the reference splitmix64 generator: returns (new_state, output)."""
    state = (state + GAMMA) & MASK64
    z = state
    z = ((z ^ (z >> 30)) * M1) & MASK64
    z = ((z ^ (z >> 27)) * M2) & MASK64
    return state, z ^ (z >> 31)


def stream_key(seed: int, tid: int) -> int:
    _, out = splitmix64_next(((seed << 16) + tid) & MASK64)
    return out


def draws_np(seed: int, tid: int, idx: np.ndarray) -> np.ndarray:
    """Raw 64-bit draws k (idx) of stream (seed, tid), as uint64."""
    key = np.uint64(stream_key(seed, tid))
    idx = np.asarray(idx, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = key + (idx + np.uint64(1)) * np.uint64(GAMMA)
        return _mix_np(z)


def uniform_np(seed: int, tid: int, idx) -> np.ndarray:
    d = draws_np(seed, tid, np.asarray(idx, dtype=np.uint64))
    return (d >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)


def normal_np(seed: int, tid: int, idx) -> np.ndarray:
    idx = np.asarray(idx, dtype=np.uint64)
    u0 = uniform_np(seed, tid, idx * np.uint64(2))
    u1 = uniform_np(seed, tid, idx * np.uint64(2) + np.uint64(1))
    return np.sqrt(-2.0 * np.log1p(-u0)) * np.cos(2.0 * np.pi * u1)


# ---------------------------------------------------------------------------
# Device (torch) version of the same generator, for tensors too large to make
# on the host.  int64 arithmetic in torch wraps modulo 2**64; logical right
# shifts are arithmetic shifts followed by a mask.

def _to_i64(v: int) -> int:
    v &= MASK64
    return v - (1 << 64) if v >= (1 << 63) else v


def _lsr(z, k: int):
    return (z >> k) & ((1 << (64 - k)) - 1)


def _mix_torch(z):
    z = (z ^ _lsr(z, 30)) * _to_i64(M1)
    z = (z ^ _lsr(z, 27)) * _to_i64(M2)
    return z ^ _lsr(z, 31)


def _uniform_torch(key: int, k):
    z = _mix_torch(k.add(1).mul_(_to_i64(GAMMA)).add_(_to_i64(key)))
    return _lsr(z, 11).to(__import__("torch").float64).mul_(2.0 ** -53)


def normal_torch(seed: int, tid: int, n: int, dtype, device, start: int = 0,
                 chunk: int = 1 << 26):
    """normal(k) for k in [start, start + n), returned as a 1-D tensor of dtype."""
    import torch
    out = torch.empty(n, dtype=dtype, device=device)
    key = stream_key(seed, tid)
    for c0 in range(0, n, chunk):
        c1 = min(n, c0 + chunk)
        k = torch.arange(start + c0, start + c1, dtype=torch.int64, device=device)
        u0 = _uniform_torch(key, k * 2)
        u1 = _uniform_torch(key, k * 2 + 1)
        z = torch.sqrt(-2.0 * torch.log1p(-u0)) * torch.cos((2.0 * np.pi) * u1)
        out[c0:c1] = z.to(dtype)
        del k, u0, u1, z
    return out


def uniform_torch(seed: int, tid: int, n: int, device, start: int = 0):
    import torch
    k = torch.arange(start, start + n, dtype=torch.int64, device=device)
    return _uniform_torch(stream_key(seed, tid), k)
