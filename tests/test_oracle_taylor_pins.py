"""Pins of the first-order Taylor correction oracle (PISA reading) against closed forms (no GPU).

Each pin fixes a property the reading implies on its own terms:
  * identical keys inside every block: the cross moments vanish and the result is dense attention;
  * values constant inside every block: the cross moments vanish again, so the result equals the
    zeroth-order (Sol-Attn) correction exactly;
  * a one-dimensional block of two keys a -/+ delta, worked by hand;
  * the defining property of a first-order expansion: against dense attention the error falls by
    about 4x when the key spread inside each block halves, the zeroth-order correction's by 2x;
  * tau = +inf keeps every block, so the result is dense attention;
  * order 0 is the Sol-Attn oracle's unit computation.
Planted mistakes (the cross-moment term dropped, its sign flipped, 1/d instead of 1/sqrt(d), and
the moment built from v_bar instead of v_t) must each fail at least one pin.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import taylor_correction_oracle as tc


def sdpa(q, k, v):
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64))[None, None]  # noqa: E731
    return torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v))[0, 0].numpy()


def spread_inputs(L, d, blk, eps, seed):
    """Keys = a per-block centre plus eps times a fixed per-token deviation; values and queries fixed."""
    rng = np.random.default_rng(seed)
    nb = -(-L // blk)
    centre = rng.standard_normal((nb, d)) * 1.2
    dev = rng.standard_normal((L, d))
    K = centre[np.arange(L) // blk] + eps * dev
    V = rng.standard_normal((L, d))
    Q = rng.standard_normal((L, d)) * 1.2
    return Q, K, V


def test_identical_keys_per_block_is_dense():
    L, d, blk = 300, 8, 32
    Q, K, V = spread_inputs(L, d, blk, 0.0, 1)
    O, keep = oracle.forward_head_taylor(Q, K, V, 0.2, blk)
    assert not keep.all()
    assert np.abs(O - sdpa(Q, K, V)).max() < 1e-12


def test_block_constant_values_equal_the_zeroth_order_correction():
    L, d, blk = 300, 8, 32
    Q, K, _ = spread_inputs(L, d, blk, 0.7, 2)
    V = np.random.default_rng(3).standard_normal((-(-L // blk), d))[np.arange(L) // blk]
    O1, keep = oracle.forward_head_taylor(Q, K, V, 0.3, blk, order=1)
    O0, keep0, _, _ = oracle.forward_head(Q, K, V, 0.3, blk, blk)
    assert (keep == keep0).all() and not keep.all()
    assert np.abs(O1 - O0).max() < 1e-12


def test_order_zero_is_the_sol_attn_unit():
    L, d, blk = 257, 8, 16
    Q, K, V = spread_inputs(L, d, blk, 0.5, 4)
    O0, _ = oracle.forward_head_taylor(Q, K, V, 0.5, blk, order=0)
    ref, _, _, _ = oracle.forward_head(Q, K, V, 0.5, blk, blk)
    assert np.abs(O0 - ref).max() < 1e-12


def test_tau_inf_is_dense():
    Q, K, V = spread_inputs(200, 8, 32, 0.6, 5)
    O, keep = oracle.forward_head_taylor(Q, K, V, math.inf, 32)
    assert keep.all()
    assert np.abs(O - sdpa(Q, K, V)).max() < 1e-12


def test_hand_example_one_dimension():
    # d = 1, one query q = 1 against two blocks: block 0 = one key 3.0 (kept, the argmax), block 1 =
    # keys a - delta, a + delta (skipped) with values v1, v2. With sqrt(d) = 1:
    #   numerator   = e^3 * 5 + e^a * [(v1 + v2) + (-delta v1 + delta v2)]
    #   denominator = e^3 + 2 e^a
    a, delta, v1, v2 = 0.5, 0.1, 2.0, -1.0
    K = np.array([[3.0], [3.0], [a - delta], [a + delta]])
    V = np.array([[5.0], [5.0], [v1], [v2]])
    Q = np.array([[1.0], [1.0], [1.0], [1.0]])
    O, keep = oracle.forward_head_taylor(Q, K, V, 1.0, 2)
    assert keep[0].tolist() == [True, False]
    num = 2 * math.exp(3.0) * 5.0 + math.exp(a) * ((v1 + v2) + (-delta * v1 + delta * v2))
    den = 2 * math.exp(3.0) + 2 * math.exp(a)
    assert abs(O[0, 0] - num / den) < 1e-14


def _errors(eps, order):
    L, d, blk = 384, 16, 32
    Q, K, V = spread_inputs(L, d, blk, eps, 6)
    O, keep = oracle.forward_head_taylor(Q, K, V, 0.4, blk, order=order)
    assert not keep.all()
    return np.abs(O - sdpa(Q, K, V)).max()


def test_first_order_error_is_quadratic_in_the_key_spread():
    e1 = [_errors(eps, 1) for eps in (0.04, 0.02, 0.01)]
    e0 = [_errors(eps, 0) for eps in (0.04, 0.02, 0.01)]
    r1 = [e1[k] / e1[k + 1] for k in range(2)]
    r0 = [e0[k] / e0[k + 1] for k in range(2)]
    assert all(3.3 < r < 4.7 for r in r1), r1
    assert all(1.7 < r < 2.4 for r in r0), r0
    assert e1[-1] < 0.1 * e0[-1]


def test_cross_moment_of_a_ramp():
    # block of 4 keys 0, 1, 2, 3 (d = 1) with values 1, 1, 1, 5: k - k_bar = -1.5, -0.5, 0.5, 1.5
    K = np.arange(4.0)[:, None]
    V = np.array([[1.0], [1.0], [1.0], [5.0]])
    C = tc.cross_moments(K, V, 4)
    assert C.shape == (1, 1, 1)
    assert abs(C[0, 0, 0] - (-1.5 - 0.5 + 0.5 + 7.5)) < 1e-15


# ---------------------------------------------------------------------------------------------
# planted mistakes
# ---------------------------------------------------------------------------------------------

def _pins():
    failed = []
    for name, fn in {"hand": test_hand_example_one_dimension, "quad": test_first_order_error_is_quadratic_in_the_key_spread,
                     "const": test_block_constant_values_equal_the_zeroth_order_correction,
                     "ramp": test_cross_moment_of_a_ramp}.items():
        try:
            fn()
        except AssertionError:
            failed.append(name)
    return failed


def test_pins_pass_on_the_unmodified_oracle():
    assert _pins() == []


def _patched_unit(scale_fn):
    orig = tc.unit_forward_taylor

    def unit(q_rows, K, V, kbar, vbar, C, keep, block, order=1):
        return orig(q_rows, K, V, kbar, vbar, scale_fn(C, K.shape[1]), keep, block, order)
    return unit


def test_planted_dropped_cross_moment_is_caught(monkeypatch):
    monkeypatch.setattr(tc, "unit_forward_taylor", _patched_unit(lambda C, d: 0.0 * C))
    assert {"hand", "quad"} <= set(_pins())


def test_planted_sign_flip_is_caught(monkeypatch):
    monkeypatch.setattr(tc, "unit_forward_taylor", _patched_unit(lambda C, d: -C))
    assert {"hand", "quad"} <= set(_pins())


def test_planted_one_over_d_scale_is_caught(monkeypatch):
    # the correction term divided by d instead of sqrt(d): C scaled by 1/sqrt(d) more
    monkeypatch.setattr(tc, "unit_forward_taylor", _patched_unit(lambda C, d: C / math.sqrt(d)))
    assert "quad" in _pins()


def test_planted_moment_from_mean_values_is_caught(monkeypatch):
    orig = tc.cross_moments

    def wrong(K, V, block):
        nb, n = oracle.block_counts(K.shape[0], block)
        vbar = oracle.pool_blocks(np.asarray(V, dtype=np.float64), block)
        Vb = vbar[np.arange(K.shape[0]) // block]
        return orig(K, Vb, block)
    monkeypatch.setattr(tc, "cross_moments", wrong)
    assert {"ramp", "quad"} <= set(_pins())
