"""Counter-based Gaussian stream for the QJL projection matrix (oracle).

The QJL correction of SpectralQuant (README, "Repository Structure":
``selective_qjl.py -- QJL correction on signal dims only``) projects a key's
residual with a random Gaussian matrix S. The pages fix no generator, so the
matrix is drawn from a published, counter-based definition that the CUDA
library implements separately:

* SplitMix64 (S. Vigna, public-domain reference ``splitmix64.c``): the state
  advances by 0x9E3779B97F4A7C15 and each output is the state passed through
  the mixing function
      z ^= z >> 30; z *= 0xBF58476D1CE4E5B9;
      z ^= z >> 27; z *= 0x94D049BB133111EB;
      z ^= z >> 31.
* A 53-bit uniform u = ((x >> 11) + 1) * 2**-53, which lies in (0, 1].
* Box-Muller: from (u1, u2), r = sqrt(-2 ln u1), theta = 2 pi u2, and the
  pair (r cos theta, r sin theta), taken in that order.

The stream of head ``h`` under ``seed`` starts from the state
``mix(seed ^ mix(h + 1))``, where ``mix`` is the mixing function above.
"""

from __future__ import annotations

import math

import numpy as np

_MASK = (1 << 64) - 1
GOLDEN = 0x9E3779B97F4A7C15


def mix64(z: int) -> int:
    """SplitMix64's output mixing function on a 64-bit integer."""
    z &= _MASK
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _MASK
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _MASK
    return z ^ (z >> 31)


def splitmix64(state: int, n: int) -> tuple[list[int], int]:
    """``n`` outputs of SplitMix64 from ``state``; returns (outputs, new state)."""
    out = []
    for _ in range(n):
        state = (state + GOLDEN) & _MASK
        out.append(mix64(state))
    return out, state


def stream_state(seed: int, head: int) -> int:
    """Initial state of head ``head``'s stream under ``seed``."""
    return mix64((seed & _MASK) ^ mix64(head + 1))


def gaussians(seed: int, head: int, n: int) -> np.ndarray:
    """The first ``n`` N(0,1) draws of head ``head``'s stream (float64)."""
    n_pairs = (n + 1) // 2
    raw, _ = splitmix64(stream_state(seed, head), 2 * n_pairs)
    out = np.empty(2 * n_pairs)
    for k in range(n_pairs):
        u1 = ((raw[2 * k] >> 11) + 1) * 2.0 ** -53
        u2 = ((raw[2 * k + 1] >> 11) + 1) * 2.0 ** -53
        r = math.sqrt(-2.0 * math.log(u1))
        theta = 2.0 * math.pi * u2
        out[2 * k] = r * math.cos(theta)
        out[2 * k + 1] = r * math.sin(theta)
    return out[:n]


def qjl_matrix(seed: int, head: int, m: int) -> np.ndarray:
    """The m x m QJL projection of a head: the stream's first m*m draws, row-major."""
    if m == 0:
        return np.zeros((0, 0))
    return gaussians(seed, head, m * m).reshape(m, m)
