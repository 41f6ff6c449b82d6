"""Fixed scalar codebook: Lloyd-Max quantiser for a standard normal source.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

The method keeps one fixed codebook for every window and only moves the range
it is applied to (pchao.org, "方法概览": the codebook stays fixed while the
key range is min-max scaled per short window; TurboQuant, which it starts from,
uses a fixed codebook after a random Hadamard rotation, "关联工作"). The
2-bit codebook is the 4-level Lloyd-Max quantiser of N(0,1) (values
+-0.4528, +-1.5104); the 4-bit one is the 16-level quantiser of the same source.

Lloyd's conditions for a minimum-MSE scalar quantiser:
  * each threshold is the midpoint of its two neighbouring levels;
  * each level is the conditional mean of the source over its cell,
    E[X | a < X <= b] = (phi(a) - phi(b)) / (Phi(b) - Phi(a)) for X ~ N(0,1).
Iterating the two conditions from a symmetric start converges to the fixed
point. Everything is fp64 with math.erf / math.exp.
"""
from __future__ import annotations

import math


def _phi(x: float) -> float:
    if math.isinf(x):
        return 0.0
    return math.exp(-0.5 * x * x) / math.sqrt(2.0 * math.pi)


def _Phi(x: float) -> float:
    if x == math.inf:
        return 1.0
    if x == -math.inf:
        return 0.0
    return 0.5 * (1.0 + math.erf(x / math.sqrt(2.0)))


def cell_mean(a: float, b: float) -> float:
    """E[X | a < X <= b] for X ~ N(0,1)."""
    return (_phi(a) - _phi(b)) / (_Phi(b) - _Phi(a))


def lloyd_max_gaussian(levels: int, tol: float = 1e-15, max_iter: int = 200000):
    """Levels c_0 < ... < c_{L-1} of the L-level Lloyd-Max quantiser of N(0,1).

    The iteration runs on the positive half only and mirrors it, so the result
    is exactly symmetric (c_j == -c_{L-1-j}), as the source is.
    """
    if levels < 2 or levels % 2:
        raise ValueError("levels must be even and >= 2")
    half = levels // 2
    # start: uniform spacing of the positive half over (0, 3]
    pos = [3.0 * (i + 0.5) / half for i in range(half)]
    for _ in range(max_iter):
        full = [-p for p in reversed(pos)] + pos
        thr = [-math.inf] + [0.5 * (full[j] + full[j + 1]) for j in range(levels - 1)] + [math.inf]
        new_full = [cell_mean(thr[j], thr[j + 1]) for j in range(levels)]
        new_pos = new_full[half:]
        delta = max(abs(x - y) for x, y in zip(new_pos, pos))
        pos = new_pos
        if delta < tol:
            break
    return [-p for p in reversed(pos)] + pos


def distortion(levels_list) -> float:
    """Mean squared error E[(X - Q(X))^2] of the quantiser with the given levels
    and midpoint thresholds, for X ~ N(0,1), in closed form per cell:
    E[X^2; cell] - 2 c E[X; cell] + c^2 P(cell), with
    E[X^2; a<X<=b] = (Phi(b)-Phi(a)) + a phi(a) - b phi(b) (with x phi(x) -> 0 at +-inf).
    """
    c = list(levels_list)
    L = len(c)
    thr = [-math.inf] + [0.5 * (c[j] + c[j + 1]) for j in range(L - 1)] + [math.inf]
    total = 0.0
    for j in range(L):
        a, b = thr[j], thr[j + 1]
        p = _Phi(b) - _Phi(a)
        m1 = _phi(a) - _phi(b)
        xa = 0.0 if math.isinf(a) else a * _phi(a)
        xb = 0.0 if math.isinf(b) else b * _phi(b)
        m2 = p + xa - xb
        total += m2 - 2.0 * c[j] * m1 + c[j] * c[j] * p
    return total
