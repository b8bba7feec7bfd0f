"""Plain float64 CPU oracle of the low-precision (8-bit) variant of the Sol-Attn forward.

TEST INFRASTRUCTURE ONLY. Only the test-suite, the package's smoke check and the benchmark's
CPU-baseline leg may import this module. The CUDA library never calls it and shares no code with it.

The variant the pages point to: the review page of the Sol Video Inference Engine paper lists
SageAttention under quantization ("five acceleration techniques"): 8-bit to 4-bit attention with
outlier smoothing. A Sol-Engine README news item reports "fused MXFP8 compute" for a B300
deployment. Neither prints a formula, so this oracle takes
the plainest reading that a Blackwell block-scaled tensor-core kernel computes:

* Format: OCP Microscaling (MX) with FP8 E4M3 elements. Blocks of 32 consecutive values along
  the contraction axis share one power-of-two scale X = 2^(floor(log2 amax) - 8). Here 8 is the
  exponent of E4M3's largest normal (448 = 1.75 * 2^8). Each element is the E4M3 value nearest
  to v / X (ties to even), clamped to +-448.
* Routing is unchanged: q_bar, k_bar and the threshold come from the unquantized inputs, exactly
  as in the bf16 definition (sol_attn_oracle), so the kept set is the same.
* QK^T of kept tiles and of the correction tiles. The keys are first smoothed, K - mu with mu the
  head's mean key, as SageAttention's outlier smoothing does. Subtracting mu moves every logit of
  a query row by the same amount, so in exact arithmetic it changes nothing. The pooled keys of
  the correction are k_bar - mu. Two formats:
  - "int8" (the default, SageAttention's choice for Q and K): symmetric 8-bit integers with one
    scale amax / 127 per 128-row tile. Those are the unit's query block, each key block, and each
    chunk of 128 pooled keys. Rounding is to nearest, ties to even. A per-tile scale is a single
    factor on a whole score tile.
  - "mxfp8": MX E4M3 along the head dimension (blocks of 32 channels of one row).
* PV: V is quantized along the token axis (32 consecutive tokens per channel), and v_bar along
  the pooled-block axis. P is quantized along the key columns of each 128-column tile: the
  kept block's keys, or a chunk of 128 pooled blocks for the correction. Masked columns are 0.
* Weights: P_rt = w_t 2^(l_t log2(e) - M_r), with w = 1 for a kept key and n_j for a skipped
  block. M_r is an integer (the ceiling of the row's largest l log2(e)). With an integer
  reference the running maximum of an online kernel changes P only by powers of two, which the
  MX block scales absorb exactly. So the result does not depend on the order in which tiles are
  met. The row sum is the sum of the quantized weights, the same values the PV product uses.
  O_r = sum_tiles Pq_tile Vq_tile / sum_tiles sum(Pq_tile).

A second PV reading, "e4m3_channel" (SageAttention's own PV layout, where V is FP8 with one scale
per channel): V is E4M3 with one scale per channel, s_c = amax_c / 448 over all of the head's
tokens, and the pooled values v_bar use the same channel scales (their entries lie within each
channel's range). P carries no block scale: each weight keeps E4M3's 3 stored mantissa bits (round
to nearest even), with its exponent left to the kernel. An online kernel keeps P's exponent inside
E4M3's normal range relative to its own integer running maximum, so this rounding is the one it
applies to every weight that matters; and it commutes with any power-of-two reference, so the
result does not depend on the reference or the order of the tiles. A channel scale is one factor
on an output column: O_rc = s_c sum_t Pq_rt Vcode_tc / sum_t Pq_rt.

Parity with an upstream low-precision kernel is unpinned: the pages give no formula. The pins
in tests/test_oracle_lowp_pins.py tie this oracle to the OCP formats' definitions and to the bf16
definition.

Every function takes and returns float64 arrays.
"""
from __future__ import annotations

import math

import numpy as np

from .sol_attn_oracle import block_counts, pool_blocks, proxy_scores, route

E4M3_MAX = 448.0   # largest finite E4M3 value (S.1111.110)
E4M3_EMAX = 8      # its exponent
E4M3_EMIN = -6     # smallest normal exponent; subnormals are multiples of 2^-9
E4M3_MANT = 3      # stored mantissa bits
MX_BLOCK = 32      # values sharing one scale
TILE = 128         # columns of one P tile (one key block, or one chunk of pooled blocks)


def round_e4m3(x):
    """x rounded to the nearest E4M3 value (ties to even), clamped to +-448."""
    x = np.asarray(x, dtype=np.float64)
    ax = np.abs(x)
    _, e = np.frexp(ax)                                  # ax = f 2^e with f in [0.5, 1)
    binade = np.maximum(e - 1, E4M3_EMIN)                # floor(log2 ax), or the subnormal range
    step = np.ldexp(1.0, binade - E4M3_MANT)             # spacing of E4M3 values there
    q = np.minimum(np.round(ax / step) * step, E4M3_MAX)  # np.round: half to even
    return np.copysign(q, x)


def mx_quantize(x, axis=-1):
    """The values x takes after MXFP8 (E4M3) quantization along `axis` in blocks of 32 consecutive
    entries (a short last block is padded with zeros), returned dequantized."""
    x = np.moveaxis(np.asarray(x, dtype=np.float64), axis, -1)
    n = x.shape[-1]
    pad = (-n) % MX_BLOCK
    xp = np.concatenate([x, np.zeros(x.shape[:-1] + (pad,))], axis=-1) if pad else x
    blocks = xp.reshape(xp.shape[:-1] + (-1, MX_BLOCK))
    amax = np.abs(blocks).max(axis=-1, keepdims=True)
    _, e = np.frexp(amax)
    shared = np.clip(np.where(amax > 0, e - 1 - E4M3_EMAX, -127), -127, 127)  # E8M0 exponent
    X = np.ldexp(1.0, shared)
    q = (round_e4m3(blocks / X) * X).reshape(xp.shape)[..., :n]
    return np.moveaxis(q, -1, axis)


def int8_quantize_tiles(x, rows=TILE):
    """The values x [L, d] takes after symmetric int8 quantization with one scale amax / 127 per
    tile of `rows` consecutive rows (round to nearest, ties to even), returned dequantized."""
    x = np.asarray(x, dtype=np.float64)
    out = np.empty_like(x)
    for r0 in range(0, x.shape[0], rows):
        t = x[r0:r0 + rows]
        amax = np.abs(t).max()
        s = amax / 127.0 if amax > 0 else 1.0
        out[r0:r0 + rows] = np.round(t / s) * s
    return out


def channel_scales(V):
    """One scale per channel (column) of V [rows, d]: amax_c / 448, or 1 for an all-zero channel."""
    amax = np.abs(np.asarray(V, dtype=np.float64)).max(axis=0)
    return np.where(amax > 0, amax / E4M3_MAX, 1.0)


def e4m3_channel_quantize(x, scales):
    """x [rows, d] after E4M3 quantization with the given per-channel scales (round to nearest
    even of x / s_c, clamped to +-448), returned dequantized."""
    s = np.asarray(scales, dtype=np.float64)[None, :]
    return round_e4m3(np.asarray(x, dtype=np.float64) / s) * s


def round_mantissa(x, bits=E4M3_MANT):
    """x with its significand rounded to 1 + `bits` bits (round to nearest, ties to even) and an
    unbounded exponent: no underflow, no saturation."""
    x = np.asarray(x, dtype=np.float64)
    f, e = np.frexp(x)                                   # x = f 2^e, |f| in [0.5, 1)
    return np.ldexp(np.round(np.ldexp(f, bits + 1)), e - bits - 1)


def e4m3_plain(x, axis=-1):
    """The P of the "e4m3_channel" reading: E4M3's mantissa rounding with the exponent left to the
    kernel (axis is unused; the signature matches mx_quantize)."""
    return round_mantissa(x)


def no_quantize(x, axis=-1):
    """Identity in place of mx_quantize: the variant's arithmetic with exact operands."""
    return np.asarray(x, dtype=np.float64)


def unit_forward_mx(qq, Kq, Vq, kbq, vbq, block, n, keep, quant, m_shift=0):
    """Output rows [m, d] of one query block from its quantized rows qq [m, d], the quantized keys
    and values Kq, Vq [L, d] and pooled ones kbq, vbq [N_kb, d], the valid counts n [N_kb] and
    the routing decision keep [N_kb] (see the module docstring)."""
    m, d = qq.shape
    nkb = n.size
    scale = math.log2(math.e) / math.sqrt(d)
    tiles = []  # (x2 = logits * log2(e) [m, 128], weights [128], values [128, d])
    for j in np.flatnonzero(keep):
        t0, t1 = j * block, j * block + n[j]
        x2 = np.full((m, TILE), -np.inf)
        x2[:, : n[j]] = (qq @ Kq[t0:t1].T) * scale
        w = np.zeros(TILE)
        w[: n[j]] = 1.0
        vals = np.zeros((TILE, d))
        vals[: n[j]] = Vq[t0:t1]
        tiles.append((x2, w, vals))
    skipped = ~keep
    for c in range(-(-nkb // TILE)):
        cols = np.arange(c * TILE, min(nkb, (c + 1) * TILE))
        if not skipped[cols].any():
            continue
        x2 = np.full((m, TILE), -np.inf)
        w = np.zeros(TILE)
        vals = np.zeros((TILE, d))
        x2[:, : cols.size] = (qq @ kbq[cols].T) * scale
        w[: cols.size] = np.where(skipped[cols], n[cols].astype(np.float64), 0.0)
        vals[: cols.size] = vbq[cols]  # the whole chunk of pooled values, kept blocks' rows included
        tiles.append((x2, w, vals))
    # integer reference per row: the ceiling of the largest logit * log2(e) over the used columns
    top = np.max([np.max(np.where(w[None, :] > 0, x2, -np.inf), axis=1) for x2, w, _ in tiles], axis=0)
    M = np.ceil(top)[:, None] + m_shift
    num = np.zeros((m, d))
    den = np.zeros((m, 1))
    for x2, w, vals in tiles:
        P = np.where(w[None, :] > 0, w[None, :] * np.exp2(np.where(w[None, :] > 0, x2, 0.0) - M), 0.0)
        Pq = quant(P, axis=1)
        num += Pq @ vals
        den += Pq.sum(axis=1, keepdims=True)
    return num / den


def forward_head_mx(Q, K, V, tau, block, n_force=0, smooth_k=True, quant=mx_quantize, units=None, m_shift=0,
                    qk="int8", pv="mx"):
    """One (batch, head): returns (O [L, d], keep [N_qb, N_kb]). Rows outside `units` are NaN.

    qk: "int8" or "mxfp8", the format of the QK^T operands (module docstring), or "none" for
    exact ones. pv: "mx", where `quant` quantizes P and V (mx_quantize, or no_quantize for exact
    ones); or "e4m3_channel", P plain E4M3 and V, v_bar E4M3 with V's channel scales (`quant`
    unused)."""
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    L, d = Q.shape
    nqb, nq = block_counts(L, block)
    nkb, n = block_counts(L, block)
    kbar = pool_blocks(K, block)
    vbar = pool_blocks(V, block)
    mu = K.mean(axis=0) if smooth_k else np.zeros(d)
    if qk == "int8":
        Qq, Kq, kbq = (int8_quantize_tiles(x, block) for x in (Q, K - mu, kbar - mu))
    elif qk == "mxfp8":
        Qq, Kq, kbq = (mx_quantize(x, axis=1) for x in (Q, K - mu, kbar - mu))
    elif qk == "none":
        Qq, Kq, kbq = Q, K - mu, kbar - mu
    else:
        raise ValueError(f"unknown QK format {qk!r}")
    if pv == "mx":
        Vq = quant(V, axis=0)
        vbq = quant(vbar, axis=0)
        pq = quant
    elif pv == "e4m3_channel":
        sc = channel_scales(V)
        Vq = e4m3_channel_quantize(V, sc)
        vbq = e4m3_channel_quantize(vbar, sc)
        pq = e4m3_plain
    else:
        raise ValueError(f"unknown PV format {pv!r}")
    O = np.full((L, d), np.nan)
    keep_all = np.zeros((nqb, nkb), dtype=bool)
    for i in (range(nqb) if units is None else units):
        r0, r1 = i * block, i * block + nq[i]
        qbar = Q[r0:r1].sum(axis=0) / nq[i]
        keep, _ = route(proxy_scores(qbar, kbar, d), tau, n_force)
        keep_all[i] = keep
        O[r0:r1] = unit_forward_mx(Qq[r0:r1], Kq, Vq, kbq, vbq, block, n, keep, pq, m_shift)
    return O, keep_all
