"""Pins of the oracle's routing acceptance logic (no GPU).

The GPU parity tests accept a kept-block mask when (1) it equals the oracle's decision outside
the band |s_bar - (max - tau)| < BAND, where float32 and float64 routing may both be right,
and (2) every row is a kept set that a float32 evaluation of the threshold routing could
produce (oracle.routing_violations, with the float32 error bound oracle.proxy_error_bound).
Inside the band the oracle then adopts the GPU's decision (forward_head's keep_override)
before O is compared. These pins tie each of those helpers to hand cases and to float32
arithmetic, and the planted mistakes at the end check that a pin catches a band that is too
wide, an override applied outside the band, and forced blocks left in the band.
"""
import math

import numpy as np
import pytest

import oracle
from oracle import sol_attn_oracle as so

U = 2.0 ** -24


def local_inputs(L, d, seed, pos=1.5):
    rng = np.random.default_rng(seed)
    t = np.arange(L)[:, None] / 7.0
    c = np.arange(d)[None, :]
    feat = np.where(c % 2 == 0, np.sin(t * (1 + c % 5)), np.cos(t * (1 + c % 3)))
    Q = rng.standard_normal((L, d)) + pos * feat
    K = rng.standard_normal((L, d)) + pos * feat
    V = rng.standard_normal((L, d))
    return (np.float32(Q).astype(np.float64), np.float32(K).astype(np.float64), V)


# ---------------------------------------------------------------------------------------------
# band_mask: a hand case around one threshold
# ---------------------------------------------------------------------------------------------

# M = 2, tau = 0.5: threshold 1.5. Column 0 is forced (n_force = 1) and sits in the band.
HAND_SBAR = np.array([[1.5002, 2.0, 1.5, 1.5004, 1.4996, 1.5009, 1.4991, 1.5015, 1.4985, 1.506, 0.3]])
HAND_M = np.array([2.0])
HAND_BAND = np.array([[False, False, True, True, True, True, True, False, False, False, False]])


def test_band_mask_hand_case():
    band = oracle.band_mask(HAND_SBAR, HAND_M, 0.5, n_force=1)
    assert band.dtype == bool and band.shape == HAND_SBAR.shape
    assert (band == HAND_BAND).all()


def test_band_mask_forced_column_only_excluded_when_forced():
    band = oracle.band_mask(HAND_SBAR, HAND_M, 0.5, n_force=0)
    want = HAND_BAND.copy()
    want[0, 0] = True  # 1.5002 is 2e-4 from the threshold
    assert (band == want).all()


def test_band_mask_tau_inf_is_empty():
    assert not oracle.band_mask(HAND_SBAR, HAND_M, math.inf).any()


def test_band_mask_per_row_maximum():
    # two rows with different maxima: the band follows each row's own threshold
    sbar = np.array([[1.0, 0.6004, 0.59], [3.0, 2.5995, 0.6004]])
    band = oracle.band_mask(sbar, np.array([1.0, 3.0]), 0.4)
    assert (band == np.array([[False, True, False], [False, True, False]])).all()


def test_adopt_in_band_takes_override_only_in_band():
    keep = np.array([True, True, False, False])
    band = np.array([False, True, True, False])
    over = np.array([False, False, True, True])
    assert (oracle.adopt_in_band(keep, band, over) == np.array([True, False, True, False])).all()


# ---------------------------------------------------------------------------------------------
# keep_override in forward_head: a real input with entries placed in the band on purpose
# ---------------------------------------------------------------------------------------------

def _band_case(n_force=0):
    """Inputs and a tau that puts two non-forced blocks of unit 1 at 3e-4 and 6e-4 from the
    threshold (inside the band); every other entry of that unit stays outside it."""
    L, d, blk = 640, 16, 64
    Q, K, V = local_inputs(L, d, seed=41)
    _, _, sbar, M = oracle.forward_head(Q, K, V, math.inf, blk, blk)
    s = np.sort(sbar[1])[::-1]
    gaps = M[1] - s
    j = 4  # the 5th highest block sits at the threshold - 3e-4
    tau = float(gaps[j] - 3e-4)
    return Q, K, V, blk, tau, n_force


def test_keep_override_changes_only_band_entries():
    Q, K, V, blk, tau, nf = _band_case()
    O0, keep0, sbar, M = oracle.forward_head(Q, K, V, tau, blk, blk, nf)
    band = oracle.band_mask(sbar, M, tau, nf)
    assert band[1].sum() >= 1  # the planted near-threshold entry
    flipped = ~keep0
    O1, keep1, _, _ = oracle.forward_head(Q, K, V, tau, blk, blk, nf, keep_override=flipped)
    assert (keep1[~band] == keep0[~band]).all()
    assert (keep1[band] == flipped[band]).all()
    # O follows the adopted decisions: rows of units without band entries are unchanged
    for i in range(keep0.shape[0]):
        rows = slice(i * blk, (i + 1) * blk)
        if band[i].any():
            ref = oracle.unit_forward(Q[rows], K, V, oracle.pool_blocks(K, blk), oracle.pool_blocks(V, blk),
                                      keep1[i], blk)
            assert np.abs(O1[rows] - ref).max() < 1e-12
            assert np.abs(O1[rows] - O0[rows]).max() > 0
        else:
            assert np.array_equal(O1[rows], O0[rows])


def test_keep_override_never_drops_forced_blocks():
    Q, K, V, blk, tau, _ = _band_case()
    _, _, sbar, M = oracle.forward_head(Q, K, V, tau, blk, blk, 0)
    # force the planted near-threshold block: it is then out of the band and stays kept
    j = int(np.flatnonzero(oracle.band_mask(sbar, M, tau, 0)[1])[0])
    nf = j + 1
    none = np.zeros_like(oracle.forward_head(Q, K, V, tau, blk, blk, nf)[1])
    _, keep, _, _ = oracle.forward_head(Q, K, V, tau, blk, blk, nf, keep_override=none)
    assert keep[:, :nf].all()


def test_keep_override_ignored_at_tau_inf():
    Q, K, V, blk, _, _ = _band_case()
    nb = -(-Q.shape[0] // blk)
    O, keep, _, _ = oracle.forward_head(Q, K, V, math.inf, blk, blk, keep_override=np.zeros((nb, nb), bool))
    assert keep.all()


# ---------------------------------------------------------------------------------------------
# proxy_error_bound: float32 evaluations in several orders stay inside it, and it is not loose
# ---------------------------------------------------------------------------------------------

def _fp32_scores(Q, K, blk_q, blk_k, order):
    """s_bar in float32 with a given summation order ("seq", "rev" or "pair")."""
    def fsum(X):
        X = X.astype(np.float32)
        if order == "seq":
            acc = np.zeros(X.shape[1:], np.float32)
            for x in X:
                acc = np.float32(acc + x)
            return acc
        if order == "rev":
            acc = np.zeros(X.shape[1:], np.float32)
            for x in X[::-1]:
                acc = np.float32(acc + x)
            return acc
        while X.shape[0] > 1:  # pairwise tree
            if X.shape[0] % 2:
                X = np.concatenate([X, np.zeros((1,) + X.shape[1:], np.float32)])
            X = np.float32(X[0::2] + X[1::2])
        return X[0]
    L, d = Q.shape
    nqb, nq = oracle.block_counts(L, blk_q)
    nkb, nk = oracle.block_counts(K.shape[0], blk_k)
    kb = np.stack([fsum(K[j * blk_k: j * blk_k + nk[j]]) * np.float32(1.0 / nk[j]) for j in range(nkb)])
    inv = np.float32(1.0 / math.sqrt(d))
    S = np.empty((nqb, nkb))
    for i in range(nqb):
        qb = fsum(Q[i * blk_q: i * blk_q + nq[i]]) / np.float32(nq[i])
        S[i] = (fsum((kb * qb[None, :]).T) * inv).astype(np.float64)
    return S


@pytest.mark.parametrize("order", ["seq", "rev", "pair"])
def test_fp32_routing_error_within_bound(order):
    Q, K, _ = local_inputs(700, 64, seed=5, pos=3.0)
    K[::97] += 4.0  # sink-like keys with a large common offset
    eps = oracle.proxy_error_bound(Q, K, 64, 64)
    _, _, sbar, _ = oracle.forward_head(Q, K, K, math.inf, 64, 64)
    err = np.abs(_fp32_scores(Q, K, 64, 64, order) - sbar)
    assert (err <= eps).all()
    assert err.max() > 0  # float32 really differs from float64 here


def test_error_bound_holds_under_cancellation():
    # a query block whose rows cancel: 1e8 + 1 - 1e8 loses the 1 in float32 sequential order
    d = 4
    Q = np.zeros((3, d))
    Q[:, 0] = [1e8, 1.0, -1e8]
    K = np.ones((3, d))
    eps = oracle.proxy_error_bound(Q, K, 3, 3)
    exact = (1.0 / 3.0) * 1.0 / math.sqrt(d)
    got = _fp32_scores(Q, K, 3, 3, "seq")[0, 0]
    assert abs(got - exact) > 0.1 * exact  # float32 lost most of it
    assert abs(got - exact) <= eps[0, 0]


def test_error_bound_scale_is_first_order_in_u():
    # all-positive exactly representable inputs: sum_c A_c B_jc / sqrt(d) is the score itself, and
    # the relative bound is about (m + n + d + 5) u to first order: not loose by orders of magnitude
    m = n = 8
    d = 16
    Q = np.full((m, d), 0.5)
    K = np.full((n, d), 0.25)
    eps = oracle.proxy_error_bound(Q, K, m, n)[0, 0]
    s = 0.5 * 0.25 * d / math.sqrt(d)
    assert (m + n + d) * U * s < eps < (m + n + d + 8) * U * s * 1.001


def test_error_bound_is_far_below_the_band_on_small_workloads():
    Q, K, _ = local_inputs(1024, 64, seed=2)
    eps = oracle.proxy_error_bound(Q, K, 128, 128)
    assert eps.max() < 0.5 * oracle.BAND


# ---------------------------------------------------------------------------------------------
# routing_violations: the oracle's own mask passes; each kind of wrong GPU mask is flagged
# ---------------------------------------------------------------------------------------------

def _rows(tau, n_force=0, seed=3):
    Q, K, V = local_inputs(1200, 32, seed=seed)
    _, keep, sbar, M = oracle.forward_head(Q, K, V, tau, 64, 64, n_force)
    eps = oracle.proxy_error_bound(Q, K, 64, 64)
    return keep, sbar, M, eps


@pytest.mark.parametrize("tau,n_force", [(0.0, 0), (0.08, 0), (0.08, 3), (math.inf, 0), (0.15, 2)])
def test_oracle_mask_has_no_violations(tau, n_force):
    keep, sbar, M, eps = _rows(tau, n_force)
    v = oracle.routing_violations(sbar, M, tau, keep, eps, n_force)
    assert v == {"forced": 0, "outside_band": 0, "max_kept": 0, "threshold": 0}


def test_shifted_threshold_within_band_is_accepted():
    # a float32 evaluation may move the threshold by less than the band: any such threshold set passes
    keep, sbar, M, eps = _rows(0.08)
    for delta in (-4e-4, 4e-4):
        alt = sbar >= (M[:, None] - 0.08 + delta)
        v = oracle.routing_violations(sbar, M, 0.08, alt, eps)
        assert v["outside_band"] == 0 and v["max_kept"] == 0 and v["threshold"] == 0


def test_dropped_argmax_at_tau_zero_is_flagged():
    keep, sbar, M, eps = _rows(0.0)
    assert (keep.sum(axis=1) == 1).all()  # tau = 0 keeps only the argmax (no ties here)
    bad = keep.copy()
    bad[2] = False  # the argmax is in the band at tau = 0, so only max_kept can see this
    v = oracle.routing_violations(sbar, M, 0.0, bad, eps)
    assert v["outside_band"] == 0 and v["max_kept"] == 1


def test_dropped_forced_block_is_flagged():
    keep, sbar, M, eps = _rows(0.08, n_force=3)
    bad = keep.copy()
    bad[4, 1] = False
    assert oracle.routing_violations(sbar, M, 0.08, bad, eps, 3)["forced"] == 1


def test_non_threshold_set_inside_the_band_is_flagged():
    # keep a lower in-band block while skipping a higher in-band one: both within BAND of the
    # threshold 1.5 (so the band comparison cannot see it), but no single threshold gives that set
    sbar = np.array([[2.0, 1.5003, 1.4998, 0.2]])
    M = np.array([2.0])
    eps = np.full_like(sbar, 1e-5)
    ok = np.array([[True, True, False, False]])
    bad = np.array([[True, False, True, False]])
    v_ok = oracle.routing_violations(sbar, M, 0.5, ok, eps)
    v_bad = oracle.routing_violations(sbar, M, 0.5, bad, eps)
    assert v_ok == {"forced": 0, "outside_band": 0, "max_kept": 0, "threshold": 0}
    assert v_bad == {"forced": 0, "outside_band": 0, "max_kept": 0, "threshold": 1}
    # within the error bound the same swap is a legitimate float32 outcome
    wide = np.full_like(sbar, 3e-4)
    assert oracle.routing_violations(sbar, M, 0.5, bad, wide)["threshold"] == 0


def test_flip_outside_band_is_flagged():
    keep, sbar, M, eps = _rows(0.08)
    band = oracle.band_mask(sbar, M, 0.08)
    i, j = np.argwhere(~keep & ~band)[0]  # a skipped block well below the threshold
    bad = keep.copy()
    bad[i, j] = True
    v = oracle.routing_violations(sbar, M, 0.08, bad, eps)
    assert v["outside_band"] == 1 and v["threshold"] == 1


def test_empty_row_is_flagged():
    keep, sbar, M, eps = _rows(0.08)
    bad = keep.copy()
    bad[3] = False
    assert oracle.routing_violations(sbar, M, 0.08, bad, eps)["max_kept"] == 1


# ---------------------------------------------------------------------------------------------
# planted mistakes in the oracle's band logic: a pin above must catch each one
# ---------------------------------------------------------------------------------------------

def _band_pins():
    failed = []
    checks = {
        "hand": test_band_mask_hand_case,
        "rows": test_band_mask_per_row_maximum,
        "override": test_keep_override_changes_only_band_entries,
        "forced": test_keep_override_never_drops_forced_blocks,
        "inf": test_keep_override_ignored_at_tau_inf,
        "shift": test_shifted_threshold_within_band_is_accepted,
    }
    for name, fn in checks.items():
        try:
            fn()
        except (AssertionError, IndexError, ValueError):
            failed.append(name)
    return failed


def test_band_pins_pass_on_the_unmodified_oracle():
    assert _band_pins() == []


def test_planted_band_ten_times_too_wide_is_caught(monkeypatch):
    monkeypatch.setattr(so, "BAND", 10 * so.BAND)
    assert "hand" in _band_pins()


def test_planted_override_outside_band_is_caught(monkeypatch):
    wrong = lambda keep, band, over: np.asarray(over, dtype=bool)  # noqa: E731
    monkeypatch.setattr(so, "adopt_in_band", wrong)
    monkeypatch.setattr(oracle, "adopt_in_band", wrong)
    assert {"override", "forced", "inf"} & set(_band_pins())


def test_planted_forced_columns_left_in_band_is_caught(monkeypatch):
    def no_force_clear(sbar, M, tau, n_force=0):
        if math.isinf(tau):
            return np.zeros_like(sbar, dtype=bool)
        return np.abs(sbar - (np.asarray(M)[:, None] - tau)) < so.BAND

    monkeypatch.setattr(so, "band_mask", no_force_clear)
    monkeypatch.setattr(oracle, "band_mask", no_force_clear)
    assert "hand" in _band_pins()
