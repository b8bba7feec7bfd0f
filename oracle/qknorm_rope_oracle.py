"""Plain float64 CPU oracle of the fused QK-norm + RoPE + block pooling step.

TEST INFRASTRUCTURE ONLY. Only the test-suite, the package's smoke check and the benchmark's
CPU-baseline leg may import this module. The CUDA library never calls it and shares no code with it.

The step is the one before the sparse attention. The Sol-Engine README ("The five acceleration
methods", method 3, kernel fusion) names the QK-norm + RoPE glue of a DiT block as memory-bound
work to fuse, and its news list names "fused QK+RoPE". The pages print no formula for either, so
this oracle takes the textbook forms:

* RMS norm of one head's query or key vector x (length d) with a learned gain g:
      y = x / sqrt(mean(x^2) + eps) * g
* rotary embedding on interleaved pairs: pair i = (y_{2i}, y_{2i+1}) of token t is rotated by the
  angle phi_{t,i}, given by the caller as cos / sin tables [L, d/2]:
      y'_{2i}   = y_{2i} cos(phi) - y_{2i+1} sin(phi)
      y'_{2i+1} = y_{2i} sin(phi) + y_{2i+1} cos(phi)
  How the angles come from a (t, y, x) video grid is the caller's business (the tables); the
  seeded generator builds 3-D tables for the tests and the benchmark.
* the pooled keys and values of the sparse attention (block means, the same definition as
  ``sol_attn_oracle.pool_blocks``), taken from the rotated keys after their rounding to the
  output dtype, so they equal what pooling the stored keys would give.

Parity with upstream's fused kernel is unpinned: the pages give no formula. The pins in
tests/test_oracle_rope_pins.py tie this oracle to the textbook forms above.

Every function takes and returns float64 arrays.
"""
from __future__ import annotations

import numpy as np

from .sol_attn_oracle import pool_blocks


def rms_norm(X: np.ndarray, gain: np.ndarray, eps: float) -> np.ndarray:
    """Rows of X [L, d] divided by their root mean square (plus eps under the root), times gain [d]."""
    X = np.asarray(X, dtype=np.float64)
    ms = np.mean(X * X, axis=-1, keepdims=True)
    return X / np.sqrt(ms + eps) * np.asarray(gain, dtype=np.float64)


def rope(Y: np.ndarray, cos: np.ndarray, sin: np.ndarray) -> np.ndarray:
    """Rotate the interleaved pairs of each row of Y [L, d] by the angles of cos / sin [L, d/2]."""
    Y = np.asarray(Y, dtype=np.float64)
    a, b = Y[:, 0::2], Y[:, 1::2]
    c, s = np.asarray(cos, dtype=np.float64), np.asarray(sin, dtype=np.float64)
    out = np.empty_like(Y)
    out[:, 0::2] = a * c - b * s
    out[:, 1::2] = a * s + b * c
    return out


def qknorm_rope_pool_head(Qraw, Kraw, V, gain_q, gain_k, cos, sin, eps, block_k, round_out):
    """One (batch, head): returns (Q', K', kbar, vbar).

    Q' and K' are the float64 normed and rotated rows. ``round_out`` maps them to the values the
    output dtype stores (e.g. bf16 rounding); kbar is the block mean of round_out(K'), vbar the
    block mean of V.
    """
    Qn = rope(rms_norm(Qraw, gain_q, eps), cos, sin)
    Kn = rope(rms_norm(Kraw, gain_k, eps), cos, sin)
    kbar = pool_blocks(round_out(Kn), block_k)
    vbar = pool_blocks(np.asarray(V, dtype=np.float64), block_k)
    return Qn, Kn, kbar, vbar
