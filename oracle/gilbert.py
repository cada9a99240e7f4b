"""Locality-preserving token order: a generalised Hilbert ("Gilbert") curve.

Video-BLADE, section "Adaptive Block-Sparse Attention", paragraph "Preprocessing:
Locality-preserving token rearrangement": the flattened (T, H, W) video tokens are
reordered along a Gilbert space-filling curve before they are cut into blocks, so
that each block holds spatially contiguous tokens.  The pages name the curve but
do not define it, so this module restates a generalised Hilbert construction of
our own:

* A box is an origin ``o``, a signed major direction ``a`` of length ``P`` and two
  signed minor directions ``b`` (length ``Q``) and ``c`` (length ``R``).  The path
  over the box enters at ``o`` and leaves at ``o + (P-1) a``.
* ``Q == R == 1``: walk straight along ``a``.
* ``2P > 3 max(Q, R)`` ("long" box): cut ``a`` at ``P1 = P//2`` (moved up by one
  to an even value when ``P1`` is odd and ``Q`` or ``R`` is even) and walk both
  halves along ``a``.
* otherwise ("U" step, the Hilbert move): let ``b`` be the longer minor (``R > Q``
  swaps them), ``Q1 = P_even(Q//2)`` (``Q//2`` rounded up to even), ``P1 = P//2``;
  walk (1) ``[0,P1) x [0,Q1)`` up along ``b``, (2) ``[0,P) x [Q1,Q)`` across along
  ``a``, (3) ``[P1,P) x [0,Q1)`` back down along ``-b``.
* The top-level major axis is the longest even-length axis (ties: x=W, then
  y=H, then t=T); with no even axis it is the longest axis.

With that choice every sub-box admits a unit-step path (major even, or all three
sides odd), so consecutive cells are always grid neighbours (no diagonal steps),
and on 2^m x 2^m frames the order is the textbook Hilbert curve.

Raster index convention: ``(t * H + y) * W + x`` (x fastest), the order of a
flattened [T, H, W] latent.  ``gilbert_order(T, H, W)[i]`` is the raster index of
the token at curve position ``i``.
"""
from __future__ import annotations

import numpy as np


def _walk(o, a, P, b, Q, c, R, out):
    """Append the cells of one box to ``out`` in curve order (recursive)."""
    if Q == 1 and R == 1:
        for i in range(P):
            out.append((o[0] + i * a[0], o[1] + i * a[1], o[2] + i * a[2]))
        return
    if P < 2:
        raise AssertionError("major side of length 1 with a longer minor side")
    if 2 * P > 3 * max(Q, R):
        P1 = P // 2
        if P1 % 2 == 1 and (Q % 2 == 0 or R % 2 == 0):
            P1 += 1
        _walk(o, a, P1, b, Q, c, R, out)
        o2 = (o[0] + P1 * a[0], o[1] + P1 * a[1], o[2] + P1 * a[2])
        _walk(o2, a, P - P1, b, Q, c, R, out)
        return
    if R > Q:
        b, Q, c, R = c, R, b, Q
    Q1 = Q // 2
    if Q1 % 2 == 1:
        Q1 += 1
    P1 = P // 2
    neg_a = (-a[0], -a[1], -a[2])
    neg_b = (-b[0], -b[1], -b[2])
    # (1) up along b over the near half of a
    _walk(o, b, Q1, a, P1, c, R, out)
    # (2) across along a over the far rows of b
    if Q1 < Q:
        o2 = (o[0] + Q1 * b[0], o[1] + Q1 * b[1], o[2] + Q1 * b[2])
        _walk(o2, a, P, b, Q - Q1, c, R, out)
    # (3) back down along -b over the far half of a
    o3 = (o[0] + (P - 1) * a[0] + (Q1 - 1) * b[0],
          o[1] + (P - 1) * a[1] + (Q1 - 1) * b[1],
          o[2] + (P - 1) * a[2] + (Q1 - 1) * b[2])
    _walk(o3, neg_b, Q1, neg_a, P - P1, c, R, out)


def gilbert_cells(T: int, H: int, W: int) -> list[tuple[int, int, int]]:
    """Cells (x, y, t) of the T x H x W grid in curve order."""
    if T < 1 or H < 1 or W < 1:
        raise ValueError("grid sides must be >= 1")
    sides = [W, H, T]                      # axis 0 = x, 1 = y, 2 = t
    unit = [(1, 0, 0), (0, 1, 0), (0, 0, 1)]
    even = [i for i in range(3) if sides[i] % 2 == 0]
    pool = even if even else [0, 1, 2]
    major = pool[0]
    for i in pool:
        if sides[i] > sides[major]:
            major = i
    minors = [i for i in range(3) if i != major]
    out: list[tuple[int, int, int]] = []
    _walk((0, 0, 0), unit[major], sides[major], unit[minors[0]], sides[minors[0]],
          unit[minors[1]], sides[minors[1]], out)
    return out


def gilbert_order(T: int, H: int, W: int) -> np.ndarray:
    """perm[i] = raster index (x fastest) of the token at curve position i."""
    cells = gilbert_cells(T, H, W)
    perm = np.fromiter(((t * H + y) * W + x for (x, y, t) in cells),
                       dtype=np.int64, count=len(cells))
    return perm
