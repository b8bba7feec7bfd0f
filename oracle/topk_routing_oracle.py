"""Plain float64 CPU oracle of fixed-sparsity (top-k) routing, the routing half of NEXT-4.

TEST INFRASTRUCTURE ONLY. Only the test-suite, the package's smoke check and the benchmark's
CPU-baseline leg may import this module. The CUDA library never calls it and shares no code with it.

The review page of the Sol Video Inference Engine paper names PISA among the sparse-attention
options ("five acceleration techniques", sparse attention). PISA computes the critical blocks
exactly and compensates the others. The page's code-analysis section runs it at a fixed
sparsity of 0.9 with blocks of 64 (the LTX-2.3 refinement stage). The page gives no formula for
the selection, so this oracle takes the plainest reading of fixed-sparsity routing:
* each query block keeps the k key blocks with the highest proxy scores s_bar_ij (the same
  scores as the threshold routing), k = max(1, ceil((1 - sparsity) * N_kb));
* equal scores are broken by the lower block index;
* the first n_force blocks are OR-ed in afterwards, as in the threshold routing;
* everything after routing (the exact kept tiles, the pooled correction of the skipped blocks,
  one softmax per row) is the bf16 definition of sol_attn_oracle, unchanged.

PISA's first-order Taylor compensation of the non-critical blocks is not restated: the page
gives no formula for it.

Parity with an upstream top-k kernel is unpinned: the pages give no formula. The pins in
tests/test_oracle_topk_pins.py tie this oracle to the definition above and to the threshold
routing.
"""
from __future__ import annotations

import math

import numpy as np

from .sol_attn_oracle import block_counts, pool_blocks, proxy_scores, unit_forward


def keep_count(nkb: int, sparsity: float) -> int:
    """Blocks kept per query block at a given sparsity (share of skipped blocks), at least one."""
    if not 0.0 <= sparsity < 1.0:
        raise ValueError("sparsity must lie in [0, 1)")
    return max(1, min(nkb, math.ceil((1.0 - sparsity) * nkb - 1e-12)))


def route_topk(sbar: np.ndarray, k: int, n_force: int = 0) -> np.ndarray:
    """Keep the k blocks with the largest s_bar (ties: lower index first), then OR the first n_force."""
    n = sbar.size
    if not 1 <= k <= n:
        raise ValueError("k must lie in [1, N_kb]")
    order = np.lexsort((np.arange(n), -sbar))  # descending score, then ascending index
    keep = np.zeros(n, dtype=bool)
    keep[order[:k]] = True
    keep[: min(n_force, n)] = True
    return keep


def forward_head_topk(Q, K, V, k, block, n_force=0, units=None):
    """One (batch, head) with top-k routing: returns (O [L, d], keep [N_qb, N_kb]); rows outside
    `units` are NaN."""
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    L, d = Q.shape
    nqb, nq = block_counts(L, block)
    nkb, _ = block_counts(L, block)
    kbar = pool_blocks(K, block)
    vbar = pool_blocks(V, block)
    O = np.full((L, d), np.nan)
    keep_all = np.zeros((nqb, nkb), dtype=bool)
    for i in (range(nqb) if units is None else units):
        rows = Q[i * block: i * block + nq[i]]
        keep = route_topk(proxy_scores(rows.sum(axis=0) / nq[i], kbar, d), k, n_force)
        keep_all[i] = keep
        O[i * block: i * block + nq[i]] = unit_forward(rows, K, V, kbar, vbar, keep, block)
    return O, keep_all
