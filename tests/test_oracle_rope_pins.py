"""Pins of the QK-norm + RoPE + pooling oracle against closed forms and independent restatements.

Each check would fail for a plausible slip in ``oracle/qknorm_rope_oracle.py``: a dropped eps or
gain, the mean replaced by a sum, a flipped rotation sign, swapped pair members, cos and sin
exchanged, or pooling of the unrounded keys.
"""
import math

import numpy as np
import pytest

import oracle
from block_sparse_attention_41_b200 import workloads as wl
from block_sparse_attention_41_b200.workloads import round_to_bf16


def _rows(L=7, d=16, seed=0):
    return np.random.default_rng(seed).standard_normal((L, d)) * 3.0


# ---- RMS norm -------------------------------------------------------------------------------

def test_rms_norm_unit_gain_gives_unit_rms():
    X = _rows()
    Y = oracle.rms_norm(X, np.ones(16), 0.0)
    assert np.allclose(np.sqrt(np.mean(Y * Y, axis=1)), 1.0, atol=1e-12)


def test_rms_norm_hand_values():
    # (2, 0, 0, 0): mean square 1, so the row is unchanged; (1, 1, 1, 1) with gain (1, 2, 3, 4)
    # gives the gain itself; (3, 4) with eps = 0.5: mean square 12.5, root of 13 under the bar
    g = np.array([1.0, 2.0, 3.0, 4.0])
    Y = oracle.rms_norm(np.array([[2.0, 0, 0, 0], [1.0, 1, 1, 1]]), g, 0.0)
    assert np.allclose(Y, [[2.0, 0, 0, 0], [1.0, 2, 3, 4]], atol=1e-15)
    Y = oracle.rms_norm(np.array([[3.0, 4.0]]), np.ones(2), 0.5)
    assert np.allclose(Y, [[3.0 / math.sqrt(13.0), 4.0 / math.sqrt(13.0)]], atol=1e-15)


def test_rms_norm_is_scale_invariant_without_eps():
    X = _rows(seed=1)
    g = np.random.default_rng(2).standard_normal(16)
    assert np.allclose(oracle.rms_norm(X * 7.5, g, 0.0), oracle.rms_norm(X, g, 0.0), atol=1e-12)


# ---- rotary embedding -------------------------------------------------------------------------

def _angles(L, half, seed=3):
    return np.random.default_rng(seed).uniform(-7.0, 7.0, (L, half))


def test_rope_zero_angle_is_identity():
    Y = _rows()
    assert np.array_equal(oracle.rope(Y, np.ones((7, 8)), np.zeros((7, 8))), Y)


def test_rope_quarter_turn_maps_pair_to_its_perpendicular():
    Y = np.array([[1.0, 2.0, -3.0, 0.5]])
    out = oracle.rope(Y, np.zeros((1, 2)), np.ones((1, 2)))  # angle pi/2
    assert np.allclose(out, [[-2.0, 1.0, -0.5, -3.0]], atol=1e-15)


def test_rope_equals_complex_multiplication():
    # independent restatement: pair (a, b) as a + ib times e^{i phi}
    Y = _rows(L=5, d=12, seed=4)
    phi = _angles(5, 6)
    z = (Y[:, 0::2] + 1j * Y[:, 1::2]) * np.exp(1j * phi)
    ref = np.empty_like(Y)
    ref[:, 0::2], ref[:, 1::2] = z.real, z.imag
    assert np.allclose(oracle.rope(Y, np.cos(phi), np.sin(phi)), ref, atol=1e-12)


def test_rope_preserves_pair_norms_and_composes():
    Y = _rows(L=6, d=10, seed=5)
    p1, p2 = _angles(6, 5, seed=6), _angles(6, 5, seed=7)
    once = oracle.rope(Y, np.cos(p1), np.sin(p1))
    n0 = Y[:, 0::2] ** 2 + Y[:, 1::2] ** 2
    n1 = once[:, 0::2] ** 2 + once[:, 1::2] ** 2
    assert np.allclose(n0, n1, atol=1e-10)
    twice = oracle.rope(once, np.cos(p2), np.sin(p2))
    assert np.allclose(twice, oracle.rope(Y, np.cos(p1 + p2), np.sin(p1 + p2)), atol=1e-10)


def test_rope_scores_depend_only_on_relative_position():
    d, L = 16, 40
    theta = 10000.0 ** (-np.arange(d // 2) / (d // 2))
    ang = np.arange(L)[:, None] * theta[None, :]
    c, s = np.cos(ang), np.sin(ang)
    rng = np.random.default_rng(8)
    q, k = rng.standard_normal(d), rng.standard_normal(d)
    Q = oracle.rope(np.tile(q, (L, 1)), c, s)
    K = oracle.rope(np.tile(k, (L, 1)), c, s)
    for t, u, shift in ((3, 11, 5), (20, 2, 17), (0, 0, 31)):
        assert math.isclose(Q[t] @ K[u], Q[t + shift] @ K[u + shift], rel_tol=1e-9, abs_tol=1e-9)


# ---- the fused step ----------------------------------------------------------------------------

def test_fused_step_pools_the_rounded_keys():
    rng = np.random.default_rng(9)
    L, d, blk = 300, 16, 64
    Q, K, V = (rng.standard_normal((L, d)) for _ in range(3))
    c, s = np.cos(_angles(L, 8)), np.sin(_angles(L, 8))
    g = np.ones(d)
    Qn, Kn, kbar, vbar = oracle.qknorm_rope_pool_head(Q, K, V, g, g, c, s, 1e-6, blk,
                                                      lambda x: round_to_bf16(x).astype(np.float64))
    # block size 1 turns pooling into the identity, so each pooled key is one rounded key
    _, _, kbar1, vbar1 = oracle.qknorm_rope_pool_head(Q, K, V, g, g, c, s, 1e-6, 1,
                                                      lambda x: round_to_bf16(x).astype(np.float64))
    assert np.array_equal(kbar1, round_to_bf16(Kn).astype(np.float64))
    assert np.array_equal(vbar1, V)
    # the ragged last block (300 = 4 * 64 + 44) averages its 44 rows only
    assert np.allclose(kbar[4], round_to_bf16(Kn[256:]).astype(np.float64).mean(axis=0), atol=1e-12)
    assert np.allclose(vbar[4], V[256:].mean(axis=0), atol=1e-12)
    # queries: normed then rotated, row RMS 1 before the rotation, and rotation keeps it
    assert np.allclose(np.sqrt(np.mean(Qn * Qn, axis=1)), np.sqrt(1.0 / (1.0 + 1e-6 / np.mean(Q * Q, axis=1))),
                       atol=1e-12)


# ---- the seeded tables (inputs) ----------------------------------------------------------------

@pytest.mark.parametrize("d", [64, 128])
def test_rope_tables_are_unit_rotations_on_the_grid_axes(d):
    grid = (3, 4, 5)
    c, s = wl.rope_tables(grid, d)
    assert c.shape == (60, d // 2) and c.dtype == np.float32
    assert np.allclose(c.astype(np.float64) ** 2 + s.astype(np.float64) ** 2, 1.0, atol=1e-6)
    half, ny = d // 2, (d // 2) // 3
    nt = half - 2 * ny
    # token (0, 0, 1): only the x pairs turn, pair j by base^(-j/ny)
    ang = np.arctan2(s[1].astype(np.float64), c[1].astype(np.float64))
    assert np.allclose(ang[: nt + ny], 0.0, atol=1e-7)
    assert np.allclose(ang[nt + ny:], 10000.0 ** (-np.arange(ny) / ny), atol=1e-6)
