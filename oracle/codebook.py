"""Lloyd–Max scalar quantiser for a Gaussian source (oracle, fp64).

[TQ-RQ] section "Lloyd-Max 最优量化": after rotation every coordinate follows one
known law, so the optimal b-bit scalar quantiser (minimum mean-squared error) is
computed once, offline, by Lloyd's iteration -- assign each value to the nearest
centre, move each centre to the mean of its cell, repeat until nothing moves --
and runtime quantisation is a table lookup.  Section "Beta 分布的魔力": for a
rotated unit vector in d dimensions the law tends to N(0, 1/d), so the codebook
used on the path is the N(0,1) codebook divided by sqrt(d).

The cell means and cell masses of N(0,1) have closed forms, so each Lloyd step
here is exact up to fp64 rounding (no sampling):
    mass  P(a < X <= b)        = Phi(b) - Phi(a)
    mean  E[X | a < X <= b]    = (phi(a) - phi(b)) / (Phi(b) - Phi(a))
    E[X^2 ; a < X <= b]        = (Phi(b) - Phi(a)) + a*phi(a) - b*phi(b)
"""

import math

import numpy as np

_SQRT2 = math.sqrt(2.0)
_INV_SQRT2PI = 1.0 / math.sqrt(2.0 * math.pi)


def _phi(x):
    if math.isinf(x):
        return 0.0
    return _INV_SQRT2PI * math.exp(-0.5 * x * x)


def _Phi(x):
    if x == -math.inf:
        return 0.0
    if x == math.inf:
        return 1.0
    return 0.5 * math.erfc(-x / _SQRT2)


def _cell_stats(a, b):
    """(mass, first moment, second moment) of N(0,1) restricted to (a, b]."""
    mass = _Phi(b) - _Phi(a)
    m1 = _phi(a) - _phi(b)
    m2 = mass + (a * _phi(a) if math.isfinite(a) else 0.0) - (b * _phi(b) if math.isfinite(b) else 0.0)
    return mass, m1, m2


def lloyd_max_gaussian(bits=3, tol=1e-15, max_iter=200000):
    """Optimal 2**bits-level quantiser of N(0,1) by Lloyd's iteration.

    Returns (centroids ascending, boundaries ascending, iterations).  Boundaries are
    the midpoints of neighbouring centroids (the nearest-centre rule of step 2 of
    Lloyd's method); centroids are the cell means (step 3).  Starts from the
    centres of 2**bits equal-probability cells.
    """
    n = 1 << bits
    # equal-probability start: cell edges at the N(0,1) quantiles, found by bisection
    edges = [-math.inf]
    for k in range(1, n):
        target = k / n
        lo, hi = -10.0, 10.0
        for _ in range(200):
            mid = 0.5 * (lo + hi)
            if _Phi(mid) < target:
                lo = mid
            else:
                hi = mid
        edges.append(0.5 * (lo + hi))
    edges.append(math.inf)
    c = []
    for k in range(n):
        mass, m1, _ = _cell_stats(edges[k], edges[k + 1])
        c.append(m1 / mass)
    it = 0
    for it in range(1, max_iter + 1):
        b = [0.5 * (c[k] + c[k + 1]) for k in range(n - 1)]
        e = [-math.inf] + b + [math.inf]
        new_c = []
        for k in range(n):
            mass, m1, _ = _cell_stats(e[k], e[k + 1])
            new_c.append(m1 / mass)
        # N(0,1) is symmetric, so the optimum is odd-symmetric; impose it exactly so the
        # middle boundary is exactly 0 rather than a rounding residue.
        new_c = [0.5 * (new_c[k] - new_c[n - 1 - k]) for k in range(n)]
        delta = max(abs(x - y) for x, y in zip(new_c, c))
        c = new_c
        if delta < tol:
            break
    b = [0.5 * (c[k] + c[k + 1]) for k in range(n - 1)]
    return np.array(c, dtype=np.float64), np.array(b, dtype=np.float64), it


def gaussian_mse(centroids, boundaries):
    """E[(X - Q(X))^2] for X ~ N(0,1) under the given cells and output levels."""
    e = [-math.inf] + list(boundaries) + [math.inf]
    total = 0.0
    for k, ck in enumerate(centroids):
        mass, m1, m2 = _cell_stats(e[k], e[k + 1])
        total += m2 - 2.0 * ck * m1 + ck * ck * mass
    return total


_CACHE = {}


def codebook(bits=3):
    """(centroids, boundaries) of the N(0,1) Lloyd–Max quantiser, cached."""
    if bits not in _CACHE:
        c, b, _ = lloyd_max_gaussian(bits)
        _CACHE[bits] = (c, b)
    return _CACHE[bits]


def codebook_for_dim(d=128, bits=3):
    """Centroids and boundaries for N(0, 1/d): the N(0,1) ones divided by sqrt(d)."""
    c, b = codebook(bits)
    s = math.sqrt(d)
    return c / s, b / s
