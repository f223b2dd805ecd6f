"""Brute-force selection by enumeration (test infrastructure, tiny inputs only).

Independent of ``oracle.c``: instead of ranking, it enumerates every subset of
n channels out of an M-block (or k out of a whole token) and keeps the subset
with the largest exact score sum; among equal sums it keeps the subset whose
sorted index tuple is lexicographically smallest.  That is the same selection
as "top-n by score, equal scores to the lower index" (activation-sparsity
overview §2.1 / §2.2.1 for N:M; WiSparse §2.2 for a per-token keep count),
reached by a different route.  Scores are compared as exact rationals.
"""
from __future__ import annotations

from fractions import Fraction
from itertools import combinations

import numpy as np


def count_subsets(m: int, n: int) -> int:
    """Number of distinct n-of-m keep patterns, counted by enumeration."""
    return sum(1 for _ in combinations(range(m), n))


def best_subset(scores, n: int) -> tuple[int, ...]:
    exact = [Fraction(float(v)) for v in scores]
    best, best_sum = None, None
    for sub in combinations(range(len(exact)), n):  # lexicographic order
        s = sum((exact[i] for i in sub), Fraction(0))
        if best_sum is None or s > best_sum:
            best, best_sum = sub, s
    return best


def select_nm(s: np.ndarray, n: int, m: int) -> np.ndarray:
    s = np.asarray(s, np.float32)
    T, k = s.shape
    mask = np.zeros((T, k), np.uint8)
    for t in range(T):
        for b in range(0, k, m):
            for i in best_subset(s[t, b:b + m], n):
                mask[t, b + i] = 1
    return mask


def select_topk(s: np.ndarray, kk: int) -> np.ndarray:
    s = np.asarray(s, np.float32)
    T, k = s.shape
    mask = np.zeros((T, k), np.uint8)
    for t in range(T):
        for i in best_subset(s[t], kk):
            mask[t, i] = 1
    return mask
