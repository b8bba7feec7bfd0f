"""Plain float64 CPU oracle of a first-order Taylor correction for skipped blocks (PISA reading).

TEST INFRASTRUCTURE ONLY. Only the test-suite, the package's smoke check and the benchmark's
CPU-baseline leg may import this module. The CUDA library never calls it and shares no code with it.

The review page of the Sol Video Inference Engine paper lists PISA among the sparse-attention
techniques ("five acceleration techniques"): the critical blocks are computed exactly, and the
others are compensated by a first-order Taylor approximation. The page prints no formula, so this
oracle takes the plainest reading: expand each skipped block's exponentials to first order
around the block's mean key.

For query row q and a skipped block j with keys k_t, values v_t (its n_j valid tokens), mean key
k_bar_j, mean value v_bar_j and s_j = q . k_bar_j / sqrt(d):

    exp(q . k_t / sqrt(d)) ~ exp(s_j) * (1 + q . (k_t - k_bar_j) / sqrt(d)).

Summed over the block, the first-order terms of the denominator cancel (the deviations from the
mean key sum to zero), and the numerator gains a term through the key-value cross moment
C_j = sum_t (k_t - k_bar_j) v_t^T (d x d):

    denominator  n_j exp(s_j)
    numerator    exp(s_j) * (n_j v_bar_j + q^T C_j / sqrt(d)).

Dropping the C_j term gives the zeroth-order correction of the Sol-Attn definition (mean key and
value with multiplicity n_j, sol_attn_oracle). Kept blocks are exact, routing is the threshold
routing of sol_attn_oracle, and every term enters one softmax per row (two-pass: the row max over
the exact logits and the s_j first).

Parity with an upstream PISA kernel is unpinned: the page gives no formula. The pins in
tests/test_oracle_taylor_pins.py tie this oracle to closed forms (identical keys, constant values,
a hand-derived one-dimensional block) and to its defining property: its error against dense
attention shrinks quadratically with the spread of the keys inside a block, the zeroth-order
correction's only linearly.

Every function takes and returns float64 arrays.
"""
from __future__ import annotations

import math

import numpy as np

from .sol_attn_oracle import block_counts, pool_blocks, proxy_scores, route


def cross_moments(K, V, block):
    """C_j = sum over the valid tokens t of block j of (k_t - k_bar_j) v_t^T, as [N_kb, d, d]."""
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    nb, n = block_counts(K.shape[0], block)
    kbar = pool_blocks(K, block)
    C = np.empty((nb, K.shape[1], V.shape[1]))
    for j in range(nb):
        t0, t1 = j * block, j * block + n[j]
        C[j] = (K[t0:t1] - kbar[j]).T @ V[t0:t1]
    return C


def unit_forward_taylor(q_rows, K, V, kbar, vbar, C, keep, block, order=1):
    """Output rows of one query block: exact kept blocks, skipped blocks by their Taylor terms of
    the given order (0: mean key and value with multiplicity n_j; 1: plus q^T C_j / sqrt(d))."""
    q_rows = np.asarray(q_rows, dtype=np.float64)
    L, d = K.shape
    _, n = block_counts(L, block)
    kept = np.flatnonzero(keep)
    skipped = np.flatnonzero(~keep)
    idx = np.concatenate([np.arange(j * block, j * block + n[j]) for j in kept]) if kept.size else \
        np.zeros(0, dtype=np.int64)
    exact = (q_rows @ K[idx].T) / math.sqrt(d)            # [m, keys of kept blocks]
    pooled = (q_rows @ kbar[skipped].T) / math.sqrt(d)    # [m, skipped blocks]
    top = np.max(np.concatenate([exact, pooled], axis=1), axis=1, keepdims=True)
    e_exact = np.exp(exact - top)
    e_pool = np.exp(pooled - top) * n[skipped][None, :]
    num = e_exact @ V[idx] + e_pool @ vbar[skipped]
    den = e_exact.sum(axis=1, keepdims=True) + e_pool.sum(axis=1, keepdims=True)
    if order >= 1 and skipped.size:
        # q^T C_j / sqrt(d) per row and skipped block, weighted by exp(s_j - top) (no multiplicity)
        qc = np.einsum("rc,jce->rje", q_rows, C[skipped]) / math.sqrt(d)
        num = num + np.einsum("rj,rje->re", np.exp(pooled - top), qc)
    return num / den


def forward_head_taylor(Q, K, V, tau, block, n_force=0, order=1, units=None):
    """One (batch, head): returns (O [L, d], keep [N_qb, N_kb]); rows outside `units` are NaN."""
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    L, d = Q.shape
    nqb, nq = block_counts(L, block)
    nkb, _ = block_counts(L, block)
    kbar = pool_blocks(K, block)
    vbar = pool_blocks(V, block)
    C = cross_moments(K, V, block)
    O = np.full((L, d), np.nan)
    keep_all = np.zeros((nqb, nkb), dtype=bool)
    for i in (range(nqb) if units is None else units):
        r0, r1 = i * block, i * block + nq[i]
        qbar = Q[r0:r1].sum(axis=0) / nq[i]
        keep, _ = route(proxy_scores(qbar, kbar, d), tau, n_force)
        keep_all[i] = keep
        O[r0:r1] = unit_forward_taylor(Q[r0:r1], K, V, kbar, vbar, C, keep, block, order)
    return O, keep_all
