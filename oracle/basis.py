"""Minimal symmetric basis M_p and its weights (oracle; test infrastructure only).

[SATA-eng] section "对称张量分解的核心洞察": the order-p symmetric tensor built
from (q^T k)^p has d_K^p entries, but only the index tuples of the
upper-triangular region are distinct; those tuples form the fixed tables M_p.
Section "硬件优化路径与当前局限" states the order i_1 <= i_2 <= ... <= i_p.

Reading: tuples are 0-based and listed in lexicographic order within a degree,
degrees concatenated from p = 0 (one empty tuple) to p = P-1.
"""
from __future__ import annotations

import math

import numpy as np


def basis_rows(dK: int, p: int) -> np.ndarray:
    """M_p: every tuple i_1 <= ... <= i_p over range(dK), lexicographic, int32 [count, p].

    Enumerated by plain recursion (each next index starts at the previous one);
    the count is whatever the enumeration yields, never a formula.
    """
    if dK < 1 or p < 0:
        raise ValueError("dK >= 1 and p >= 0 required")
    rows: list[tuple[int, ...]] = []
    prefix: list[int] = []

    def extend(start: int) -> None:
        if len(prefix) == p:
            rows.append(tuple(prefix))
            return
        for i in range(start, dK):
            prefix.append(i)
            extend(i)
            prefix.pop()

    extend(0)
    return np.asarray(rows, dtype=np.int32).reshape(len(rows), p)


def multiplicity_factorial(row) -> int:
    """alpha! = product over distinct indices of (multiplicity)!  for one tuple."""
    out = 1
    counts: dict[int, int] = {}
    for i in row:
        counts[int(i)] = counts.get(int(i), 0) + 1
    for c in counts.values():
        out *= math.factorial(c)
    return out


def basis_weights(dK: int, p: int, rows: np.ndarray | None = None) -> np.ndarray:
    """fp64 weight of every row of M_p: w = 1 / sqrt(alpha! * dK^(p/2)).

    Derivation: (q.k)^p = sum over ordered tuples of prod q * prod k; grouping
    the ordered tuples by their sorted form gives p!/alpha! copies of each
    minimal-basis monomial (multinomial theorem).  The Taylor term is
    (q.k / sqrt(dK))^p / p!, so each sorted tuple carries
    (p!/alpha!) / (p! dK^(p/2)) = 1/(alpha! dK^(p/2)); the square root goes to
    each side.
    """
    if rows is None:
        rows = basis_rows(dK, p)
    w = np.empty(len(rows), dtype=np.float64)
    for r, row in enumerate(rows):
        w[r] = 1.0 / math.sqrt(multiplicity_factorial(row) * dK ** (p / 2.0))
    return w


def basis_all(dK: int, P: int):
    """Concatenated basis for degrees 0..P-1: list of (p, rows, weights)."""
    return [(p, basis_rows(dK, p), basis_weights(dK, p)) for p in range(P)]
