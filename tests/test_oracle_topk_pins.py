"""Pins of the fixed-sparsity (top-k) routing oracle, ``oracle/topk_routing_oracle.py``.

Each pin fails for a plausible slip: keeping the k smallest scores, an off-by-one in k, ties
broken by the higher index, forced blocks left out or counted against k, or a kept-count rule
that rounds the wrong way.
"""
import itertools
import math

import numpy as np
import pytest

import oracle


def test_keep_count_rule():
    assert oracle.keep_count(64, 0.9) == 7       # ceil(6.4)
    assert oracle.keep_count(591, 0.9) == 60     # ceil(59.1)
    assert oracle.keep_count(10, 0.9) == 1       # exactly 1.0, no rounding up past it
    assert oracle.keep_count(3, 0.99) == 1       # never fewer than one
    assert oracle.keep_count(16, 0.0) == 16
    with pytest.raises(ValueError):
        oracle.keep_count(16, 1.0)


def test_topk_is_the_k_largest_by_brute_force():
    rng = np.random.default_rng(0)
    for n in (1, 5, 9):
        s = rng.standard_normal(n)
        for k in range(1, n + 1):
            keep = oracle.route_topk(s, k)
            assert keep.sum() == k
            # brute force: the kept set has the largest score sum of all k-subsets (distinct scores)
            best = max(itertools.combinations(range(n), k), key=lambda c: s[list(c)].sum())
            assert set(np.flatnonzero(keep)) == set(best)


def test_ties_go_to_the_lower_index_and_forced_blocks_are_added():
    s = np.array([1.0, 3.0, 3.0, 2.0, 3.0])
    assert np.flatnonzero(oracle.route_topk(s, 2)).tolist() == [1, 2]
    assert np.flatnonzero(oracle.route_topk(s, 4)).tolist() == [1, 2, 3, 4]
    # forced blocks are OR-ed in after the selection, not counted against k
    assert np.flatnonzero(oracle.route_topk(s, 2, n_force=1)).tolist() == [0, 1, 2]


def test_topk_sets_are_nested_and_match_the_threshold_routing():
    rng = np.random.default_rng(1)
    s = rng.standard_normal(40)
    prev = np.zeros(40, dtype=bool)
    order = np.argsort(-s)
    M = s.max()
    for k in range(1, 41):
        keep = oracle.route_topk(s, k)
        assert np.all(keep >= prev)
        prev = keep
        # the threshold routing keeps a top prefix; tau between the k-th and (k+1)-th gaps keeps k
        if k < 40:
            tau = M - (s[order[k - 1]] + s[order[k]]) / 2
            kp, _ = oracle.route(s, tau)
            assert np.array_equal(kp, keep)


def _inputs(L, d, seed):
    rng = np.random.default_rng(seed)
    t = np.arange(L)[:, None] / 30.0
    feat = np.sin(t * (1 + np.arange(d)[None, :] % 4))
    return (rng.standard_normal((L, d)) + 2.0 * feat, rng.standard_normal((L, d)) + 2.0 * feat,
            rng.standard_normal((L, d)))


def test_all_blocks_kept_is_dense_attention():
    Q, K, V = _inputs(700, 32, 2)
    nkb = 6
    O, keep = oracle.forward_head_topk(Q, K, V, nkb, 128)
    assert keep.all()
    dense, _, _, _ = oracle.forward_head(Q, K, V, math.inf, 128, 128)
    assert np.max(np.abs(O - dense)) <= 1e-12


def test_fixed_sparsity_keeps_k_per_query_block_and_uses_the_common_correction():
    Q, K, V = _inputs(64 * 40, 16, 3)  # 40 blocks of 64, as in the pages' block size
    k = oracle.keep_count(40, 0.9)
    O, keep = oracle.forward_head_topk(Q, K, V, k, 64, n_force=0)
    assert k == 4 and np.all(keep.sum(axis=1) == 4)
    # with the same kept sets, the rest of the path is the bf16 definition's unit computation
    kbar, vbar = oracle.pool_blocks(K, 64), oracle.pool_blocks(V, 64)
    for i in range(keep.shape[0]):
        rows = slice(i * 64, (i + 1) * 64)
        direct = oracle.unit_forward(Q[rows], K, V, kbar, vbar, keep[i], 64)
        assert np.max(np.abs(O[rows] - direct)) <= 1e-12


# ---- planted mistakes -----------------------------------------------------------------------

def _run_topk_pins():
    checks = {
        "count": test_keep_count_rule,
        "brute": test_topk_is_the_k_largest_by_brute_force,
        "ties": test_ties_go_to_the_lower_index_and_forced_blocks_are_added,
        "threshold": test_topk_sets_are_nested_and_match_the_threshold_routing,
    }
    failed = []
    for name, fn in checks.items():
        try:
            fn()
        except (AssertionError, ValueError):
            failed.append(name)
    return failed


def test_topk_pins_pass_on_the_unmodified_oracle():
    assert _run_topk_pins() == []


def test_planted_smallest_scores_are_caught(monkeypatch):
    from oracle import topk_routing_oracle as tk
    orig = tk.route_topk
    monkeypatch.setattr(oracle, "route_topk", lambda s, k, n_force=0: orig(-s, k, n_force))
    assert {"brute", "threshold"} <= set(_run_topk_pins())


def test_planted_higher_index_tie_break_is_caught(monkeypatch):
    def higher_first(s, k, n_force=0):
        n = s.size
        order = np.lexsort((-np.arange(n), -s))
        keep = np.zeros(n, dtype=bool)
        keep[order[:k]] = True
        keep[:n_force] = True
        return keep

    monkeypatch.setattr(oracle, "route_topk", higher_first)
    assert "ties" in _run_topk_pins()


def test_planted_floor_in_the_keep_count_is_caught(monkeypatch):
    monkeypatch.setattr(oracle, "keep_count", lambda nkb, sp: max(1, math.floor((1 - sp) * nkb)))
    assert "count" in _run_topk_pins()
