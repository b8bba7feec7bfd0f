"""Pins of the CPU oracle against what the definition and the mathematics fix (no GPU).

Each pin is chosen so that a plausible slip in the oracle fails at least one of them. The
slips covered are a dropped correction term, a wrong multiplicity, a wrong scale, a reversed
threshold, pooling along the wrong axis, and a wrong max reference. The mutation tests at the
end plant those slips in the oracle and check that a pin catches each one.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import sol_attn_oracle as so


def _rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def sdpa(q, k, v):
    """Dense softmax attention by torch's library routine (float64, CPU), scale 1/sqrt(d)."""
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64))[None, None]
    return torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v))[0, 0].numpy()


def local_inputs(L, d, seed, pos=1.5):
    """Inputs with spatial locality so that finite tau leaves a mix of kept and skipped blocks."""
    rng = np.random.default_rng(seed)
    t = np.arange(L)[:, None] / 7.0
    c = np.arange(d)[None, :]
    feat = np.where(c % 2 == 0, np.sin(t * (1 + c % 5)), np.cos(t * (1 + c % 3)))
    Q = rng.standard_normal((L, d)) + pos * feat
    K = rng.standard_normal((L, d)) + pos * feat
    V = rng.standard_normal((L, d))
    return Q, K, V


# ---------------------------------------------------------------------------------------------
# pooling
# ---------------------------------------------------------------------------------------------

def test_pool_closed_form_ramp_with_ragged_block():
    # X[t, c] = t + 10 c; blocks of 4 over L = 10: token means 1.5, 5.5 and (8 + 9) / 2 = 8.5
    L, d = 10, 3
    X = np.arange(L)[:, None] + 10.0 * np.arange(d)[None, :]
    P = oracle.pool_blocks(X, 4)
    expect = np.array([1.5, 5.5, 8.5])[:, None] + 10.0 * np.arange(d)[None, :]
    assert P.shape == (3, d)
    assert np.array_equal(P, expect)
    nb, n = oracle.block_counts(L, 4)
    assert nb == 3 and list(n) == [4, 4, 2]


def test_pool_constant_blocks():
    X = np.repeat(np.array([[1.0, -2.0], [3.0, 0.5], [7.0, 7.0]]), [5, 5, 3], axis=0)
    assert np.array_equal(oracle.pool_blocks(X, 5), np.array([[1.0, -2.0], [3.0, 0.5], [7.0, 7.0]]))


# ---------------------------------------------------------------------------------------------
# special cases that reduce to dense softmax attention (library routine)
# ---------------------------------------------------------------------------------------------

@pytest.mark.parametrize("L,d,bq,bk", [(300, 16, 64, 64), (257, 8, 32, 16), (64, 4, 64, 64), (5, 3, 4, 4)])
def test_tau_inf_is_dense_attention(L, d, bq, bk):
    Q, K, V = _rand((L, d), 1), _rand((L, d), 2), _rand((L, d), 3)
    O, keep, _, _ = oracle.forward_head(Q, K, V, math.inf, bq, bk)
    assert keep.all()
    assert np.max(np.abs(O - sdpa(Q, K, V))) < 1e-12


@pytest.mark.parametrize("tau", [0.0, 0.3, 1.0, 4.0])
def test_identical_keys_and_values_per_block_is_dense_for_any_tau(tau):
    L, d, blk = 203, 8, 16  # ragged last block of 11 tokens
    nb = -(-L // blk)
    base_k, base_v = _rand((nb, d), 5, 2.0), _rand((nb, d), 6)
    tok_block = np.arange(L) // blk
    K, V = base_k[tok_block], base_v[tok_block]
    Q = _rand((L, d), 7, 1.5)
    O, keep, _, _ = oracle.forward_head(Q, K, V, tau, blk, blk)
    assert not keep.all() or tau >= 4.0  # the correction is really exercised at small tau
    assert np.max(np.abs(O - sdpa(Q, K, V))) < 1e-12


@pytest.mark.parametrize("tau", [0.0, 0.5, 2.0])
def test_key_block_size_one_is_dense_for_any_tau(tau):
    L, d = 37, 5
    Q, K, V = _rand((L, d), 8, 1.5), _rand((L, d), 9, 1.5), _rand((L, d), 10)
    O, keep, _, _ = oracle.forward_head(Q, K, V, tau, 8, 1)
    assert not keep.all()
    assert np.max(np.abs(O - sdpa(Q, K, V))) < 1e-12


# ---------------------------------------------------------------------------------------------
# the correction = n_j duplicated pooled columns (independent library formulation)
# ---------------------------------------------------------------------------------------------

def duplicated_column_output(Q_rows, K, V, keep, blk):
    """A skipped block j contributes like n_j copies of (k_bar_j, v_bar_j): build those copies
    with numpy's mean and run the library's dense attention on the modified key set."""
    K2, V2 = K.copy(), V.copy()
    for j in np.flatnonzero(~keep):
        sl = slice(j * blk, min((j + 1) * blk, K.shape[0]))
        K2[sl] = np.mean(K[sl], axis=0)
        V2[sl] = np.mean(V[sl], axis=0)
    return sdpa(Q_rows, K2, V2)


@pytest.mark.parametrize("L,d,blk,tau,seed", [(300, 16, 32, 0.5, 0), (250, 8, 16, 1.0, 1),
                                              (129, 32, 64, 0.2, 2), (1000, 16, 64, 0.0, 3)])
def test_correction_equals_duplicated_pooled_columns(L, d, blk, tau, seed):
    Q, K, V = local_inputs(L, d, seed)
    O, keep, _, _ = oracle.forward_head(Q, K, V, tau, blk, blk)
    assert (~keep).any() and keep.any()
    for i in range(keep.shape[0]):
        rows = slice(i * blk, min((i + 1) * blk, L))
        ref = duplicated_column_output(Q[rows], K, V, keep[i], blk)
        assert np.max(np.abs(O[rows] - ref)) < 1e-12


# ---------------------------------------------------------------------------------------------
# routing
# ---------------------------------------------------------------------------------------------

def test_proxy_score_special_case_constant_rows():
    # every query row of block i equals a_i and every key of block j equals b_j:
    # then q_bar = a_i, k_bar = b_j and s_bar = a_i . b_j / sqrt(d)
    d, blk = 9, 4
    A, Bv = _rand((3, d), 11), _rand((3, d), 12)
    Q, K = np.repeat(A, blk, axis=0), np.repeat(Bv, blk, axis=0)
    V = _rand((3 * blk, d), 13)
    _, _, sbar, M = oracle.forward_head(Q, K, V, 1.0, blk, blk)
    assert np.allclose(sbar, (A @ Bv.T) / 3.0, rtol=0, atol=1e-13)
    assert np.allclose(M, ((A @ Bv.T) / 3.0).max(axis=1), rtol=0, atol=1e-13)


def test_tau_zero_keeps_only_the_argmax_block():
    L, d, blk = 512, 16, 32
    Q, K, V = local_inputs(L, d, 4)
    _, keep, sbar, _ = oracle.forward_head(Q, K, V, 0.0, blk, blk)
    for i in range(keep.shape[0]):
        assert list(np.flatnonzero(keep[i])) == [int(np.argmax(sbar[i]))]


def test_tau_sweep_gives_nested_top_prefixes():
    # sweeping tau over the gaps gives the N_kb prefixes of the blocks sorted by descending score
    L, d, blk = 16, 4, 4
    Q, K, V = local_inputs(L, d, 5, pos=2.0)
    _, _, sbar, M = oracle.forward_head(Q, K, V, math.inf, blk, blk)
    for i in range(sbar.shape[0]):
        order = np.argsort(-sbar[i], kind="stable")
        gaps = np.sort(M[i] - sbar[i])
        mids = [(gaps[c] + gaps[c + 1]) / 2 for c in range(len(gaps) - 1)] + [gaps[-1] + 1.0]
        prev = None
        for c, tau in enumerate(mids):
            _, keep, _, _ = oracle.forward_head(Q, K, V, float(tau), blk, blk, units=[i])
            kept = set(np.flatnonzero(keep[i]))
            assert kept == set(order[: c + 1].tolist())
            assert prev is None or prev < kept
            prev = kept


def test_brute_force_subset_enumeration_tiny():
    # L=16, B_q=B_k=4, d=4: among all subsets that contain the top block, the oracle's output
    # equals the duplicated-column output of exactly one subset, namely the thresholded one.
    L, d, blk = 16, 4, 4
    Q, K, V = local_inputs(L, d, 6, pos=2.0)
    for tau in [0.0, 0.4, 1.1, 3.0]:
        O, keep, sbar, M = oracle.forward_head(Q, K, V, tau, blk, blk)
        for i in range(4):
            rows = slice(i * blk, (i + 1) * blk)
            hits = []
            for bits in itertools.product([False, True], repeat=4):
                S = np.array(bits)
                if not S[np.argmax(sbar[i])]:
                    continue
                ref = duplicated_column_output(Q[rows], K, V, S, blk)
                if np.max(np.abs(O[rows] - ref)) < 1e-12:
                    hits.append(S)
            assert len(hits) == 1
            assert np.array_equal(hits[0], sbar[i] >= sbar[i].max() - tau)


def test_forced_blocks_are_kept_and_max_includes_them():
    L, d, blk = 512, 16, 32
    Q, K, V = local_inputs(L, d, 7)
    K[:blk] += 3.0  # make the forced block the most attractive one for some query blocks
    _, keep0, sbar, M = oracle.forward_head(Q, K, V, 0.0, blk, blk, n_force=0)
    _, keep2, _, M2 = oracle.forward_head(Q, K, V, 0.0, blk, blk, n_force=2)
    assert keep2[:, :2].all()
    assert np.array_equal(M, M2) and np.array_equal(M, sbar.max(axis=1))
    assert np.array_equal(keep2[:, 2:], keep0[:, 2:])


def test_invalid_tau_rejected():
    with pytest.raises(ValueError):
        oracle.route(np.zeros(3), -0.1)
    with pytest.raises(ValueError):
        oracle.route(np.zeros(3), float("nan"))


# ---------------------------------------------------------------------------------------------
# invariants
# ---------------------------------------------------------------------------------------------

def test_key_block_permutation_permutes_mask_and_keeps_output():
    L, d, blk = 256, 16, 32  # 8 full blocks
    Q, K, V = local_inputs(L, d, 8)
    O, keep, _, _ = oracle.forward_head(Q, K, V, 0.6, blk, blk)
    perm = np.random.default_rng(0).permutation(L // blk)
    tok = (perm[:, None] * blk + np.arange(blk)[None, :]).reshape(-1)
    O2, keep2, _, _ = oracle.forward_head(Q, K[tok], V[tok], 0.6, blk, blk)
    assert np.array_equal(keep2, keep[:, perm])
    assert np.max(np.abs(O2 - O)) < 1e-12


def test_token_permutation_inside_key_blocks_changes_nothing():
    L, d, blk = 200, 8, 32  # ragged last block
    Q, K, V = local_inputs(L, d, 9)
    O, keep, _, _ = oracle.forward_head(Q, K, V, 0.8, blk, blk)
    rng = np.random.default_rng(1)
    tok = np.concatenate([j * blk + rng.permutation(min(blk, L - j * blk)) for j in range(-(-L // blk))])
    O2, keep2, _, _ = oracle.forward_head(Q, K[tok], V[tok], 0.8, blk, blk)
    assert np.array_equal(keep2, keep)
    assert np.max(np.abs(O2 - O)) < 1e-12


def test_output_is_a_convex_combination():
    L, d, blk = 300, 8, 32
    Q, K, V = local_inputs(L, d, 10)
    O, _, _, _ = oracle.forward_head(Q, K, V, 0.5, blk, blk)
    assert (O <= V.max(axis=0) + 1e-12).all() and (O >= V.min(axis=0) - 1e-12).all()
    # constant values pass through unchanged (weights sum to one)
    O1, _, _, _ = oracle.forward_head(Q, K, np.full_like(V, 0.37), 0.5, blk, blk)
    assert np.max(np.abs(O1 - 0.37)) < 1e-14


def test_sampled_units_equal_full_run():
    L, d, blk = 400, 16, 64
    Q, K, V = local_inputs(L, d, 11)
    O, keep, _, _ = oracle.forward_head(Q, K, V, 0.7, blk, blk)
    units = [1, 4, 6]
    Os, keeps, _, _ = oracle.forward_head(Q, K, V, 0.7, blk, blk, units=units)
    for i in units:
        rows = slice(i * blk, min((i + 1) * blk, L))
        assert np.array_equal(Os[rows], O[rows]) and np.array_equal(keeps[i], keep[i])
    assert np.isnan(Os[0:blk]).all()


def test_forward_batched_density():
    B, H, L, d, blk = 2, 3, 160, 8, 32
    Q, K, V = (_rand((B, H, L, d), s, 1.5) for s in (20, 21, 22))
    tau = np.array([0.0, 0.5, math.inf])
    O, keep, dens = oracle.forward(Q, K, V, tau, blk, blk)
    assert dens.shape == (B, H)
    assert np.allclose(dens[:, 2], 1.0)
    assert np.allclose(dens, keep.mean(axis=(2, 3)))
    O1, _, _, _ = oracle.forward_head(Q[1, 1], K[1, 1], V[1, 1], 0.5, blk, blk)
    assert np.array_equal(O1, O[1, 1])


# ---------------------------------------------------------------------------------------------
# hand-derived golden example
# ---------------------------------------------------------------------------------------------

def test_hand_derived_example(golden_dir):
    with open(os.path.join(golden_dir, "hand_example.json")) as f:
        g = json.load(f)
    Q, K, V = (np.array(g[k], dtype=np.float64) for k in ("Q", "K", "V"))
    for case in g["cases"]:
        O, keep, _ = oracle.forward(Q[None, None], K[None, None], V[None, None], [case["tau"]],
                                    g["block"], g["block"], case["n_force"])[:3]
        assert np.array_equal(keep[0, 0], np.array(case["keep"]))
        for r, expr in enumerate(case["O"]):
            num, den = expr.split(" / ")
            vec = np.array(eval(num, {"e": math.e})) / eval(den, {"e": math.e})
            assert np.max(np.abs(O[0, 0, r] - vec)) < 1e-15, (case["tau"], r)


# ---------------------------------------------------------------------------------------------
# planted mistakes: each must be caught by at least one pin above
# ---------------------------------------------------------------------------------------------

def _run_pins(golden_dir):
    """Run a set of pins, return the names that failed."""
    failed = []
    checks = {
        "pool": test_pool_closed_form_ramp_with_ragged_block,
        "dense": lambda: test_tau_inf_is_dense_attention(257, 8, 32, 16),
        "identical": lambda: test_identical_keys_and_values_per_block_is_dense_for_any_tau(0.3),
        "duplicated": lambda: test_correction_equals_duplicated_pooled_columns(250, 8, 16, 1.0, 1),
        "tau0": test_tau_zero_keeps_only_the_argmax_block,
        "hand": lambda: test_hand_derived_example(golden_dir),
    }
    for name, fn in checks.items():
        try:
            fn()
        except (AssertionError, ValueError, IndexError):
            failed.append(name)
    return failed


def test_pins_pass_on_the_unmodified_oracle(golden_dir):
    assert _run_pins(golden_dir) == []


def test_planted_dropped_correction_is_caught(monkeypatch, golden_dir):
    orig = so.unit_terms

    def dropped(q_rows, K, V, kbar, vbar, keep, block):
        w, logits, vals = orig(q_rows, K, V, kbar, vbar, keep, block)
        w = w.copy()
        w[w.size - int((~keep).sum()):] = 0.0
        return w, logits, vals

    monkeypatch.setattr(so, "unit_terms", dropped)
    assert {"identical", "duplicated", "hand"} & set(_run_pins(golden_dir))


def test_planted_block_size_multiplicity_is_caught(monkeypatch, golden_dir):
    orig = so.unit_terms

    def full_block(q_rows, K, V, kbar, vbar, keep, block):
        w, logits, vals = orig(q_rows, K, V, kbar, vbar, keep, block)
        w = w.copy()
        w[w.size - int((~keep).sum()):] = float(block)
        return w, logits, vals

    monkeypatch.setattr(so, "unit_terms", full_block)
    assert {"identical", "duplicated"} & set(_run_pins(golden_dir))


def test_planted_wrong_scale_is_caught(monkeypatch, golden_dir):
    monkeypatch.setattr(so, "proxy_scores", lambda qb, kb, d: (kb @ qb) / d)
    assert "hand" in _run_pins(golden_dir)


def test_planted_strict_threshold_is_caught(monkeypatch, golden_dir):
    def strict(sbar, tau, n_force=0):
        M = float(np.max(sbar))
        keep = sbar > M - tau
        keep[:n_force] = True
        return keep, M

    monkeypatch.setattr(so, "route", strict)
    assert {"tau0", "hand"} & set(_run_pins(golden_dir))


def test_planted_pooling_axis_is_caught(monkeypatch, golden_dir):
    orig = so.pool_blocks
    monkeypatch.setattr(so, "pool_blocks", lambda X, block: orig(X, block)[:, ::-1].copy())
    assert {"pool", "identical", "duplicated", "hand"} & set(_run_pins(golden_dir))


def test_planted_min_reference_is_caught(monkeypatch, golden_dir):
    def min_ref(sbar, tau, n_force=0):
        M = float(np.min(sbar))
        keep = sbar >= M - tau
        keep[:n_force] = True
        return keep, M

    monkeypatch.setattr(so, "route", min_ref)
    assert {"tau0", "hand"} & set(_run_pins(golden_dir))
