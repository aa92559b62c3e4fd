"""The associative combine and three prefix algorithms over it, in numpy fp64.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).  This is a second,
independent route to the hidden states: the tests check that its prefixes
reproduce the sequential oracle's states, which pins the recurrence, its time
indexing and the initial state without reusing the oracle's loop.

Source: page "yongjin360.com/news/29389", the parallel-scan derivation:

* step 1 -- each time step is a pair T_t = (Abar_t, b_t) with the input term
  b_t = Bbar_t x_t formed up front;
* step 2 -- applying T_i and then T_j equals one pair,
  T_j (+) T_i = (Abar_j * Abar_i, Abar_j * b_i + b_j);
* step 3 -- (+) is associative;
* step 4 -- the inclusive prefix S_t = T_t (+) ... (+) T_0 maps h_{-1} to h_t,
  so with h_{-1} = 0 the state h_t is the second component of S_t; a
  work-efficient up-sweep / down-sweep computes every S_t.

Page "blog.csdn.net/qq_54407673/article/details/139121849" names the
Blelloch work-efficient scan for this step.  All products are element-wise
over the state dimension (A is diagonal).
"""
from __future__ import annotations

import numpy as np


def combine(Tj, Ti):
    """T_j (+) T_i: the pair equal to applying T_i first, then T_j."""
    aj, bj = Tj
    ai, bi = Ti
    return aj * ai, aj * bi + bj


IDENTITY_A = 1.0
IDENTITY_B = 0.0


def prefix_sequential(abar, b):
    """Left fold: S_t = T_t (+) S_{t-1}, S_0 = T_0.  abar, b: (L, N)."""
    L = abar.shape[0]
    SA = np.empty_like(abar)
    SB = np.empty_like(b)
    acc = (abar[0], b[0])
    SA[0], SB[0] = acc
    for t in range(1, L):
        acc = combine((abar[t], b[t]), acc)
        SA[t], SB[t] = acc
    return SA, SB


def prefix_hillis_steele(abar, b):
    """Inclusive prefix in ceil(log2 L) rounds; round k folds in T_{t - 2^k}."""
    SA = abar.copy()
    SB = b.copy()
    L = abar.shape[0]
    step = 1
    while step < L:
        newA = SA.copy()
        newB = SB.copy()
        # position t (>= step) absorbs the segment ending at t - step, which is older
        newA[step:], newB[step:] = combine((SA[step:], SB[step:]), (SA[:-step], SB[:-step]))
        SA, SB = newA, newB
        step *= 2
    return SA, SB


def prefix_blelloch(abar, b):
    """Work-efficient inclusive prefix: up-sweep, then down-sweep (exclusive), then fold in T_t.

    The array is padded to a power of two with identity pairs (1, 0).
    """
    L, N = abar.shape
    size = 1
    while size < L:
        size *= 2
    A = np.ones((size, N))
    B = np.zeros((size, N))
    A[:L], B[:L] = abar, b
    # up-sweep: node at the right end of each block holds the block's total
    d = 1
    while d < size:
        right = np.arange(2 * d - 1, size, 2 * d)
        left = right - d
        A[right], B[right] = combine((A[right], B[right]), (A[left], B[left]))
        d *= 2
    # down-sweep: turn the tree into exclusive prefixes (older segment on the right operand)
    A[size - 1], B[size - 1] = IDENTITY_A, IDENTITY_B
    d = size // 2
    while d >= 1:
        right = np.arange(2 * d - 1, size, 2 * d)
        left = right - d
        oldA, oldB = A[left].copy(), B[left].copy()
        A[left], B[left] = A[right], B[right]
        A[right], B[right] = combine((oldA, oldB), (A[right], B[right]))
        d //= 2
    exA, exB = A[:L], B[:L]
    return combine((abar, b), (exA, exB))


def prefix_split(abar, b, k):
    """Every S_t for t >= k as (segment k..t) (+) S_{k-1}: checks any split point."""
    SA_head, SB_head = prefix_sequential(abar[:k], b[:k])
    tailA, tailB = prefix_sequential(abar[k:], b[k:])
    outA, outB = combine((tailA, tailB), (SA_head[-1], SB_head[-1]))
    return np.concatenate([SA_head, outA]), np.concatenate([SB_head, outB])
