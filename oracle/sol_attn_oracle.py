"""Plain float64 CPU oracle of the Sol-Attn block-sparse attention forward.

TEST INFRASTRUCTURE ONLY. Only the test-suite, the package's smoke check and the benchmark's
CPU-baseline leg may import this module. The CUDA library never calls it and shares no code with it.

What the method computes (Sol-Attn project page, "Sol-Attn: Accelerating Video Generation
Inference via On-the-Fly Attention Sparsification", Abstract): one softmax pass that combines
(i) a query-dependent threshold that routes each query block to key blocks, selected on chip
from a proxy score that is never written out, (ii) exact attention on the selected blocks only,
and (iii) an approximate correction that keeps the long-tail contribution of the skipped
blocks. The Sol-Engine README (section "Sol-Attention") restates it: only the most relevant
key blocks are computed, and a light compensating term stands in for the rest.

The pages print no formula. This oracle uses one definition, and the CUDA path uses the
same definition:

1. k_bar_j, v_bar_j: mean of the keys / values of key block j (its n_j valid tokens).
2. q_bar_i: mean of the valid query rows of query block i. s_bar_ij = q_bar_i . k_bar_j / sqrt(d).
   Block j is kept iff s_bar_ij >= max_j' s_bar_ij' - tau (ties kept), or j < n_force.
3. Kept block j: exact logits q_r . k_t / sqrt(d) for each valid key t of the block, value v_t.
4. Skipped block j: one logit q_r . k_bar_j / sqrt(d) with multiplicity n_j and value v_bar_j.
   All terms of 3 and 4 enter one softmax per query row.

Readings taken where the pages are silent:
* multiplicity of a skipped block = n_j, its number of valid keys. This equals the block
  size for every full block. For a ragged last block it keeps the result exact when every key
  of a block is identical.
* q_bar_i is the arithmetic mean of the valid query rows (the pages do not define it).
* bidirectional attention with no causal mask (video self-attention).
* tau = +inf keeps every block (M - inf = -inf), giving dense softmax attention.
  tau < 0 or NaN is invalid.
* forced blocks are OR-ed in after routing. The max M_i runs over all blocks, forced ones
  included. Forced blocks count toward density.

Parity with upstream Sol-Attn's own arithmetic is unpinned: the pages print no formula. The
pins in tests/test_oracle_pins.py tie this oracle to the definition above, through dense special
cases, invariants, brute force on tiny inputs and a hand-derived example.

The softmax is the two-pass form (the exact row max first, then the weighted sums). It is
deliberately not the online form used on the GPU. Every function takes float64 arrays.
"""
from __future__ import annotations

import math

import numpy as np

BAND = 1e-3  # |s_bar - (M - tau)| below this: fp32 and float64 routing may legitimately differ


def block_counts(L: int, block: int):
    """Number of blocks ceil(L/block) and the valid-token count n_j of each block."""
    if L < 1 or block < 1:
        raise ValueError("L and block must be positive")
    nb = -(-L // block)
    n = np.array([min(block, L - j * block) for j in range(nb)], dtype=np.int64)
    return nb, n


def pool_blocks(X: np.ndarray, block: int) -> np.ndarray:
    """Definition 1: the mean over each block of `block` consecutive tokens (valid tokens only).

    X is [L, d]; returns [ceil(L/block), d].
    """
    L = X.shape[0]
    nb, n = block_counts(L, block)
    out = np.empty((nb, X.shape[1]), dtype=np.float64)
    for j in range(nb):
        out[j] = X[j * block: j * block + n[j]].sum(axis=0) / n[j]
    return out


def proxy_scores(qbar_i: np.ndarray, kbar: np.ndarray, d: int) -> np.ndarray:
    """Definition 2: s_bar_ij = q_bar_i . k_bar_j / sqrt(d) for every key block j."""
    return (kbar @ qbar_i) / math.sqrt(d)


def route(sbar: np.ndarray, tau: float, n_force: int = 0):
    """Definition 2: keep block j iff s_bar_j >= max(s_bar) - tau, or j < n_force.

    Returns (keep bool [N_kb], M). tau = +inf keeps everything.
    """
    if math.isnan(tau) or tau < 0:
        raise ValueError("tau must be >= 0 (and not NaN)")
    M = float(np.max(sbar))
    thr = M - tau
    keep = sbar >= thr
    keep[: min(n_force, keep.size)] = True
    return keep, M


def unit_terms(q_rows: np.ndarray, K: np.ndarray, V: np.ndarray, kbar: np.ndarray,
               vbar: np.ndarray, keep: np.ndarray, block: int):
    """Definitions 3 and 4: the (weight, logit, value) terms one query row sees.

    Returns weights [T], logits [m, T], values [T, d]. The columns are the exact keys of the kept
    blocks followed by one pooled column per skipped block.
    """
    L, d = K.shape
    _, n = block_counts(L, block)
    kept = np.flatnonzero(keep)
    skipped = np.flatnonzero(~keep)
    key_idx = np.concatenate([np.arange(j * block, j * block + n[j]) for j in kept]) if kept.size else \
        np.zeros(0, dtype=np.int64)
    keys = np.concatenate([K[key_idx], kbar[skipped]])
    vals = np.concatenate([V[key_idx], vbar[skipped]])
    w = np.concatenate([np.ones(key_idx.size), n[skipped].astype(np.float64)])
    logits = (q_rows @ keys.T) / math.sqrt(d)
    return w, logits, vals


def unit_forward(q_rows, K, V, kbar, vbar, keep, block):
    """Output rows of one query block: O_r = sum w e^{l-m} u / sum w e^{l-m} (two-pass softmax)."""
    w, logits, vals = unit_terms(q_rows, K, V, kbar, vbar, keep, block)
    m = logits.max(axis=1, keepdims=True)
    e = w[None, :] * np.exp(logits - m)
    return (e @ vals) / e.sum(axis=1, keepdims=True)


def forward_head(Q, K, V, tau, block_q, block_k, n_force=0, units=None, keep_override=None):
    """All of one (batch, head): returns O [L, d] (rows outside `units` are NaN), keep
    [N_qb, N_kb], s_bar [N_qb, N_kb] (only for the computed units) and M [N_qb].

    `keep_override` ([N_qb, N_kb] bool) replaces the routing decision only where the
    entry lies in the near-threshold band |s_bar - (M - tau)| < BAND. Float32 and
    float64 routing may both be right there.
    """
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    L, d = Q.shape
    nqb, nq = block_counts(L, block_q)
    nkb, _ = block_counts(L, block_k)
    kbar = pool_blocks(K, block_k)
    vbar = pool_blocks(V, block_k)
    units = range(nqb) if units is None else units
    O = np.full((L, d), np.nan)
    keep = np.zeros((nqb, nkb), dtype=bool)
    sbar_all = np.full((nqb, nkb), np.nan)
    M_all = np.full(nqb, np.nan)
    for i in units:
        rows = Q[i * block_q: i * block_q + nq[i]]
        qbar = rows.sum(axis=0) / nq[i]
        sbar = proxy_scores(qbar, kbar, d)
        kp, M = route(sbar, tau, n_force)
        if keep_override is not None:
            band = band_mask(sbar[None, :], np.array([M]), tau, n_force)[0]
            kp = adopt_in_band(kp, band, keep_override[i])
        keep[i] = kp
        sbar_all[i] = sbar
        M_all[i] = M
        O[i * block_q: i * block_q + nq[i]] = unit_forward(rows, K, V, kbar, vbar, kp, block_k)
    return O, keep, sbar_all, M_all


def forward(Q, K, V, tau, block_q, block_k, n_force=0):
    """Whole problem: Q, K, V [B, H, L, d]; tau [H]. Returns O, keep [B,H,N_qb,N_kb], density [B,H]."""
    B, H, L, d = Q.shape
    tau = np.broadcast_to(np.asarray(tau, dtype=np.float64), (H,))
    nqb, _ = block_counts(L, block_q)
    nkb, _ = block_counts(L, block_k)
    O = np.empty((B, H, L, d))
    keep = np.zeros((B, H, nqb, nkb), dtype=bool)
    for b in range(B):
        for h in range(H):
            O[b, h], keep[b, h], _, _ = forward_head(Q[b, h], K[b, h], V[b, h], float(tau[h]),
                                                     block_q, block_k, n_force)
    density = keep.sum(axis=(2, 3)) / float(nqb * nkb)
    return O, keep, density


def band_mask(sbar, M, tau, n_force=0):
    """Entries whose routing decision lies within BAND of the threshold (never forced ones).

    sbar is [units, N_kb] and M [units]. At tau = +inf the threshold is -inf and no entry is
    near it.
    """
    if math.isinf(tau):
        return np.zeros_like(sbar, dtype=bool)
    band = np.abs(sbar - (np.asarray(M, dtype=np.float64)[:, None] - tau)) < BAND
    band[:, : n_force] = False
    return band


def adopt_in_band(keep, band, override):
    """The oracle's routing decisions with `override` taken where `band` is set, and only there."""
    return np.where(band, np.asarray(override, dtype=bool), keep)


# ---------------------------------------------------------------------------------------------
# Which kept sets a float32 evaluation of definition 2 may produce
# ---------------------------------------------------------------------------------------------

U32 = 2.0 ** -24  # unit roundoff of float32 (round to nearest)


def _gamma(n: int) -> float:
    """gamma_n = n u / (1 - n u): the relative bound of an n-operation float32 sum (Higham, 3.1)."""
    return n * U32 / (1.0 - n * U32)


def proxy_error_bound(Q, K, block_q, block_k, units=None):
    """Upper bound on |s_fp32 - s_bar| for a float32 evaluation of definition 2 in ANY order.

    The float32 pipeline: q_bar and k_bar are float32 sums of the m (n) valid rows of a block,
    then one division or multiplication by the count; s is a float32 dot product of d terms,
    then one multiplication by a rounded 1/sqrt(d). With A_c = mean_r |q_rc| over the query
    block and B_jc = mean_t |k_tc| over key block j, the standard summation bound gives
        |s_fp32 - s_bar| <= [(1 + g_{m+1})(1 + g_{n+1})(1 + g_d)(1 + 3u) - 1] * sum_c A_c B_jc / sqrt(d),
    g_k = gamma_k: each float32 level is exact up to a relative factor of its absolute-value
    sum, and those sums are bounded by A and B. Inputs are assumed exactly representable in
    float32 (bf16 or float32 tensors). Returns [N_qb, N_kb] (rows outside `units` are NaN).
    """
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    L, d = Q.shape
    nqb, nq = block_counts(L, block_q)
    nkb, nk = block_counts(K.shape[0], block_k)
    B = pool_blocks(np.abs(K), block_k)  # [N_kb, d]
    units = range(nqb) if units is None else units
    eps = np.full((nqb, nkb), np.nan)
    g_k = np.array([_gamma(int(n) + 1) for n in nk])
    for i in units:
        A = np.abs(Q[i * block_q: i * block_q + nq[i]]).sum(axis=0) / nq[i]
        rel = (1 + _gamma(int(nq[i]) + 1)) * (1 + g_k) * (1 + _gamma(d)) * (1 + 3 * U32) - 1
        eps[i] = rel * (B @ A) / math.sqrt(d)
    return eps


def routing_violations(sbar, M, tau, mask, eps, n_force=0):
    """Check that `mask` is a kept set a float32 evaluation of definition 2 could produce.

    sbar, eps, mask: [units, N_kb] (float64 scores, their float32 error bounds, the kept set under
    test); M: [units]. For a float32 evaluation s~ with |s~ - s_bar| <= eps, the threshold
    routing keeps j iff s~_j >= fl(M~ - tau) (or j is forced). Whatever the rounding, that gives:
      forced      : every j < n_force is kept;
      outside_band: outside the band |s_bar - (M - tau)| < BAND the decision equals the oracle's;
      max_kept    : the float32 argmax is kept (fl(M~ - tau) <= M~ for tau >= 0), so some kept j
                    has s_bar_j + eps_j >= M - eps_{argmax};
      threshold   : a kept set of a threshold is upward closed in s~, so every non-forced kept j
                    and skipped k satisfy s_bar_j + eps_j >= s_bar_k - eps_k.
    Returns the number of rows (entries for the first two) that break each condition.
    """
    sbar = np.asarray(sbar, dtype=np.float64)
    eps = np.asarray(eps, dtype=np.float64)
    mask = np.asarray(mask, dtype=bool)
    M = np.asarray(M, dtype=np.float64)
    nf = min(n_force, sbar.shape[1])
    keep_ref = sbar >= (M[:, None] - tau)
    keep_ref[:, :nf] = True
    band = band_mask(sbar, M, tau, n_force)
    out = {"forced": int((~mask[:, :nf]).sum()),
           "outside_band": int((mask[~band] != keep_ref[~band]).sum()),
           "max_kept": 0, "threshold": 0}
    for r in range(sbar.shape[0]):
        s, e, m = sbar[r], eps[r], mask[r]
        jstar = int(np.argmax(s))
        if not m.any() or np.max(np.where(m, s + e, -np.inf)) < M[r] - e[jstar]:
            out["max_kept"] += 1
        free = np.arange(s.size) >= nf
        kept, skipped = m & free, ~m
        if kept.any() and skipped.any():
            if np.min((s + e)[kept]) < np.max((s - e)[skipped]):
                out["threshold"] += 1
    return out
