"""Full d_K^p expansion for tiny d_K (oracle; test infrastructure only).

[SATA-eng] section "对称张量分解的核心洞察" describes the plain expansion of
(q^T k)^p into d_K^p monomials that the minimal basis avoids.  This module
builds that plain expansion over ORDERED index tuples (no symmetry used), so it
shares nothing with ``basis``: each ordered tuple carries weight
1/sqrt(p! d_K^(p/2)), giving sum_tuples phi(q) phi(k) = (q.k/sqrt(d_K))^p / p!.
Pure Python loops; only for d_K <= 4, N <= 16.
"""
from __future__ import annotations

import itertools
import math

import numpy as np


def full_feature_map(x, P: int) -> np.ndarray:
    """x [dK] -> concatenation over p < P of all dK^p ordered products."""
    x = [float(t) for t in x]
    dK = len(x)
    feats = []
    for p in range(P):
        w = 1.0 / math.sqrt(math.factorial(p) * dK ** (p / 2.0))
        for tup in itertools.product(range(dK), repeat=p):
            prod = 1.0
            for i in tup:
                prod *= x[i]
            feats.append(w * prod)
    return np.asarray(feats, dtype=np.float64)


def brute_attention(q, k, v, P: int):
    """Causal attention through the full expansion, token by token, for one head.

    q, k [N, dK]; v [N, dV] -> (num [N, dV], den [N]).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    N, dV = v.shape
    num = np.zeros((N, dV))
    den = np.zeros(N)
    fk = [full_feature_map(k[j], P) for j in range(N)]
    for i in range(N):
        fq = full_feature_map(q[i], P)
        for j in range(i + 1):
            t = float(np.dot(fq, fk[j]))
            num[i] += t * v[j]
            den[i] += t
    return num, den
