"""Pins of the low-precision (8-bit) oracle, ``oracle/mxfp8_oracle.py``.

The quantizers are checked against the formats' own definitions: every E4M3 code decoded from
its sign, exponent and mantissa fields, hand-derived MX and int8 examples, and the scale rules.
The variant's structure is checked against the bf16 definition: with exact operands it must
reproduce ``forward_head``. Its invariances are checked too: key smoothing, and the integer
softmax reference. Each pin fails for a plausible slip. Examples: a wrong E4M3 exponent
range, rounding half up, a ceiling in place of the floor in the MX scale, a missing clamp, P or
V quantized along the wrong axis, a dropped multiplicity, routing on quantized operands.
"""
import math

import numpy as np
import pytest

import oracle
from oracle import mxfp8_oracle as mx


def e4m3_table():
    """(value, code) of every finite non-negative E4M3 code: 1 sign, 4 exponent (bias 7) and 3
    mantissa bits; exponent field 0 is subnormal; S.1111.111 is NaN."""
    out = []
    for code in range(0x7F):  # 0x7F = 0.1111.111 is NaN
        e, m = code >> 3, code & 7
        v = (m / 8.0) * 2.0 ** -6 if e == 0 else (1.0 + m / 8.0) * 2.0 ** (e - 7)
        out.append((v, code))
    return out


def test_every_e4m3_value_is_a_fixed_point_and_the_range_is_right():
    vals = np.array([v for v, _ in e4m3_table()])
    assert np.array_equal(oracle.round_e4m3(vals), vals)
    assert np.array_equal(oracle.round_e4m3(-vals), -vals)
    assert vals.max() == 448.0 and sorted(vals)[1] == 2.0 ** -9


def test_e4m3_midpoints_round_to_the_even_code_and_large_values_saturate():
    tab = sorted(e4m3_table())
    for (a, ca), (b, _cb) in zip(tab, tab[1:]):
        mid = (a + b) / 2
        want = a if ca % 2 == 0 else b
        assert oracle.round_e4m3(mid) == want, (a, b)
        assert oracle.round_e4m3(np.nextafter(mid, 0)) == a and oracle.round_e4m3(np.nextafter(mid, 1e9)) == b
    assert oracle.round_e4m3(2.0 ** -10) == 0.0 and oracle.round_e4m3(1.5 * 2.0 ** -10) == 2.0 ** -9
    assert oracle.round_e4m3(1e6) == 448.0 and oracle.round_e4m3(-500.0) == -448.0


def test_mx_hand_example_scale_rule_and_clamp():
    # amax 5: floor(log2 5) = 2, scale 2^(2-8) = 2^-6. Scaled: 64, 19.2 -> 20 (spacing 2 in [16, 32)),
    # -320 (exact). Dequantized: 1, 0.3125, -5, 0
    assert np.array_equal(oracle.mx_quantize(np.array([1.0, 0.3, -5.0, 0.0])), [1.0, 0.3125, -5.0, 0.0])
    # amax 1.99: scale 2^-8, 1.99 * 256 = 509.4 is clamped to 448, so 1.75 comes back
    assert oracle.mx_quantize(np.array([1.99]))[0] == 1.75
    # an all-zero block stays zero
    assert np.array_equal(oracle.mx_quantize(np.zeros(40)), np.zeros(40))


def test_mx_blocks_axis_and_power_of_two_scaling():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((6, 80)) * np.exp(rng.uniform(-4, 4, (6, 1)))
    q = oracle.mx_quantize(x)
    # blocks of 32 along the axis, independent of each other; a short last block is zero-padded
    parts = [oracle.mx_quantize(x[:, a:a + 32]) for a in (0, 32, 64)]
    assert np.array_equal(q, np.concatenate(parts, axis=1))
    assert np.array_equal(oracle.mx_quantize(x.T, axis=0), q.T)
    for k in (-20, -3, 5, 30):
        assert np.array_equal(oracle.mx_quantize(x * 2.0 ** k), q * 2.0 ** k)
    assert np.array_equal(oracle.mx_quantize(q), q)
    # each element lies within half an E4M3 step of x / X (X the block's scale), or at the clamp
    for r in range(6):
        for a in (0, 32, 64):
            xb, qb = x[r, a:a + 32], q[r, a:a + 32]
            X = 2.0 ** (math.floor(math.log2(np.abs(xb).max())) - 8)
            sc = np.abs(xb) / X
            binade = np.maximum(np.floor(np.log2(np.maximum(sc, 1e-300))), -6)
            bound = np.where(sc > 448.0, sc - 448.0, 2.0 ** (binade - 4))
            assert np.all(np.abs(qb - xb) <= bound * X * (1 + 1e-12))


def test_int8_hand_example_and_tiles():
    # amax 1, scale 1/127: 0.5 -> 63.5 -> 64 (ties to even), 0.25 -> 31.75 -> 32
    q = oracle.int8_quantize_tiles(np.array([[1.0, -0.5, 0.25]]))
    assert np.allclose(q, [[1.0, -64 / 127, 32 / 127]], rtol=0, atol=1e-15)
    rng = np.random.default_rng(2)
    x = rng.standard_normal((300, 16))
    x[130:140] *= 50.0  # a loud second tile must not change the first tile's scale
    q = oracle.int8_quantize_tiles(x, 128)
    assert np.array_equal(q[:128], oracle.int8_quantize_tiles(x[:128], 128))
    for t0 in (0, 128, 256):
        t = x[t0:t0 + 128]
        s = np.abs(t).max() / 127
        assert np.all(np.abs(q[t0:t0 + 128] - t) <= s / 2 + 1e-15)
    assert np.array_equal(oracle.int8_quantize_tiles(np.zeros((5, 4))), np.zeros((5, 4)))


def _inputs(L, d, seed, offset=0.0):
    rng = np.random.default_rng(seed)
    t = np.arange(L)[:, None] / 30.0
    feat = np.sin(t * (1 + np.arange(d)[None, :] % 4))
    Q = rng.standard_normal((L, d)) + 2.0 * feat
    K = rng.standard_normal((L, d)) + 2.0 * feat + offset
    V = rng.standard_normal((L, d))
    return Q, K, V


@pytest.mark.parametrize("L,d,tau,n_force", [(700, 64, 0.0, 0), (700, 64, 0.8, 1), (1000, 32, math.inf, 0),
                                             (300, 16, 1.5, 2)])
@pytest.mark.parametrize("smooth", [True, False])
def test_exact_operands_reproduce_the_bf16_definition(L, d, tau, n_force, smooth):
    Q, K, V = _inputs(L, d, L + d)
    ref, keep, _, _ = oracle.forward_head(Q, K, V, tau, 128, 128, n_force)
    O, keep_lp = oracle.forward_head_mx(Q, K, V, tau, 128, n_force, smooth_k=smooth, quant=oracle.no_quantize,
                                        qk="none")
    assert np.array_equal(keep_lp, keep)
    assert np.max(np.abs(O - ref)) <= 1e-12


@pytest.mark.parametrize("qk", ["int8", "mxfp8"])
def test_routing_is_the_bf16_routing(qk):
    Q, K, V = _inputs(700, 64, 5)
    _, keep, _, _ = oracle.forward_head(Q, K, V, 0.5, 128, 128, 0)
    _, keep_lp = oracle.forward_head_mx(Q, K, V, 0.5, 128, 0, qk=qk)
    assert np.array_equal(keep_lp, keep)


def test_smoothing_removes_a_common_key_offset():
    Q, K, V = _inputs(700, 64, 6)
    a, _ = oracle.forward_head_mx(Q, K, V, 0.8, 128, qk="none", quant=oracle.no_quantize, smooth_k=True)
    b, _ = oracle.forward_head_mx(Q, K, V, 0.8, 128, qk="none", quant=oracle.no_quantize, smooth_k=False)
    assert np.max(np.abs(a - b)) <= 1e-12  # exact arithmetic: the shift cancels in the softmax
    # with int8 operands, keys offset by a constant vector give the same result once smoothed
    Q2, K2, V2 = _inputs(700, 64, 6, offset=np.linspace(-3, 3, 64))
    c, _ = oracle.forward_head_mx(Q, K, V, 0.8, 128)
    e, _ = oracle.forward_head_mx(Q2, K2, V2, 0.8, 128)
    assert np.max(np.abs(c - e)) <= 1e-9


def test_integer_softmax_reference_makes_p_quantization_order_free():
    Q, K, V = _inputs(700, 64, 7)
    base, _ = oracle.forward_head_mx(Q, K, V, 0.8, 128, 1)
    for shift in (-3, 7):
        O, _ = oracle.forward_head_mx(Q, K, V, 0.8, 128, 1, m_shift=shift)
        assert np.array_equal(O, base)


def test_p_and_v_are_quantized_along_the_contraction_axis():
    calls = []

    def spy(x, axis=-1):
        calls.append((np.shape(x), axis))
        return np.asarray(x, dtype=np.float64)

    L, d = 300, 16
    Q, K, V = _inputs(L, d, 8)
    oracle.forward_head_mx(Q, K, V, 0.5, 128, quant=spy, units=[1])
    nkb = 3
    assert ((L, d), 0) in calls and ((nkb, d), 0) in calls  # V along tokens, v_bar along pooled blocks
    p_calls = [c for c in calls if c[0] == (128, 128)]
    assert p_calls and all(a == 1 for _, a in p_calls)  # P along each 128-column tile's keys


def test_weights_of_skipped_blocks_enter_before_quantization():
    # identical keys and values inside each block: pooled = actual, so with exact operands the
    # variant is dense attention for any tau, and a dropped multiplicity would break it
    rng = np.random.default_rng(9)
    L, d, blk = 640, 16, 128
    tok = np.arange(L) // blk
    K = rng.standard_normal((5, d))[tok] * 1.5
    V = rng.standard_normal((5, d))[tok]
    Q = rng.standard_normal((L, d)) * 1.5
    O, keep = oracle.forward_head_mx(Q, K, V, 0.3, blk, qk="none", quant=oracle.no_quantize)
    assert not keep.all()
    dense, _, _, _ = oracle.forward_head(Q, K, V, math.inf, blk, blk, 0)
    assert np.max(np.abs(O - dense)) <= 1e-12


def test_error_against_the_exact_definition_on_a_seeded_case():
    # a regression record of the formats' accuracy on one seeded case, not a law: int8 scores
    # with MX weights and values stay within these figures; MX E4M3 scores are coarser
    Q, K, V = _inputs(1000, 128, 10)
    ref, _, _, _ = oracle.forward_head(Q, K, V, 0.8, 128, 128, 0)
    e8 = np.abs(oracle.forward_head_mx(Q, K, V, 0.8, 128)[0] - ref)
    efp = np.abs(oracle.forward_head_mx(Q, K, V, 0.8, 128, qk="mxfp8")[0] - ref)
    assert e8.mean() < 0.02 and e8.max() < 0.4
    assert efp.mean() > e8.mean()


# ---- the "e4m3_channel" PV reading: plain E4M3 weights, E4M3 values with one scale per channel ----

def test_channel_scales_hand_example():
    V = np.array([[896.0, 0.0, 0.25],
                  [-3.0, 0.0, -1.0],
                  [5.0, 0.0, 0.5]])
    s = oracle.channel_scales(V)
    assert np.array_equal(s, [2.0, 1.0, 1.0 / 448.0])  # amax / 448 per column; 1 for a zero column


def test_e4m3_channel_quantize_hand_example():
    s = np.array([2.0, 0.5])
    x = np.array([[896.0, 224.0],    # 448 * s: the top code exactly
                  [19.0, 4.5],       # 9.5 -> 9.5 is not E4M3 (8..16 step 1): tie -> 10 (even); 9 -> 9
                  [-3.0, 0.0],       # -1.5 exact; 0 exact
                  [2000.0, -500.0]])  # beyond 448 s: clamped to +-448 s
    q = oracle.e4m3_channel_quantize(x, s)
    assert np.array_equal(q, [[896.0, 224.0], [20.0, 4.5], [-3.0, 0.0], [896.0, -224.0]])
    # channels are independent: changing channel 1 leaves channel 0 as it was
    x2 = x.copy()
    x2[:, 1] *= 3
    assert np.array_equal(oracle.e4m3_channel_quantize(x2, s)[:, 0], q[:, 0])


def _two_level_case(d=16, L=256):
    """Identical queries; keys 0 in block 0 and e_0 in block 1, scaled so the log2-domain logits
    are exactly 0 and 1; V integers with a 448 in every channel (exact E4M3, scale 1)."""
    rng = np.random.default_rng(31)
    q = np.zeros(d)
    q[0] = math.sqrt(d) * math.log(2.0)
    Q = np.tile(q, (L, 1))
    K = np.zeros((L, d))
    K[128:, 0] = 1.0
    V = rng.integers(-7, 8, size=(L, d)).astype(np.float64)  # |v| <= 7: at most 3 significant bits
    V[5] = 448.0
    return Q, K, V


def test_e4m3_channel_reading_is_exact_on_a_closed_form_case():
    # weights 2^(0-1) = 0.5 for block 0 and 2^(1-1) = 1 for block 1, both exact in E4M3; values
    # exact under their channel scales (amax 448 -> scale 1): the reading reproduces the definition
    Q, K, V = _two_level_case()
    O, keep = oracle.forward_head_mx(Q, K, V, math.inf, 128, qk="none", pv="e4m3_channel")
    assert keep.all()
    closed = (0.5 * V[:128].sum(axis=0) + V[128:].sum(axis=0)) / (0.5 * 128 + 128)
    assert np.max(np.abs(O - closed[None, :])) <= 1e-12
    ref, _, _, _ = oracle.forward_head(Q, K, V, math.inf, 128, 128, 0)
    assert np.max(np.abs(O - ref)) <= 1e-12


def test_e4m3_channel_values_take_the_channel_scale_and_pooled_values_take_v_scales():
    # a column of V scaled by 2^k: its scale is 2^k times larger, so its codes and the output's
    # column scale by exactly 2^k (v_bar included), the other columns are unchanged
    Q, K, V = _inputs(700, 32, 12)
    a, _ = oracle.forward_head_mx(Q, K, V, 0.8, 128, pv="e4m3_channel")
    V2 = V.copy()
    V2[:, 3] *= 8.0
    b, _ = oracle.forward_head_mx(Q, K, V2, 0.8, 128, pv="e4m3_channel")
    assert np.array_equal(b[:, 3], 8.0 * a[:, 3])
    assert np.array_equal(np.delete(b, 3, axis=1), np.delete(a, 3, axis=1))


def test_mantissa_rounding_hand_values_and_no_underflow():
    x = np.array([0.3, 1.0, 17.0, 19.0, -2.0 ** -20 * 1.3, 1000.0, 0.0])
    # 0.3 = 1.2 * 2^-2 -> 1.25 * 2^-2; 17 = 1.0625 * 2^4 -> tie -> 1.0 (even); 19 = 1.1875 * 2^4 ->
    # 1.25 * 2^4 = 20; a tiny value keeps its 4 significant bits (no flush); 1000 -> 1024 (no clamp)
    want = np.array([0.3125, 1.0, 16.0, 20.0, -2.0 ** -20 * 1.25, 1024.0, 0.0])
    assert np.array_equal(oracle.round_mantissa(x), want)
    # inside E4M3's normal range it is E4M3's own rounding
    v = np.linspace(2.0 ** -6, 448.0, 4001)
    assert np.array_equal(oracle.round_mantissa(v), oracle.round_e4m3(v))


def test_e4m3_channel_result_does_not_depend_on_the_reference():
    # the weights' rounding commutes with any power-of-two reference: shifting the reference leaves
    # O bitwise unchanged (an online kernel's running maximum may sit anywhere)
    Q, K, V = _inputs(700, 64, 13)
    base, _ = oracle.forward_head_mx(Q, K, V, 0.8, 128, 1, pv="e4m3_channel")
    for shift in (-7, -1, 3, 9):
        O, _ = oracle.forward_head_mx(Q, K, V, 0.8, 128, 1, pv="e4m3_channel", m_shift=shift)
        assert np.array_equal(O, base)


def test_e4m3_channel_error_against_the_exact_definition_on_a_seeded_case():
    # a regression record of this reading's accuracy on one seeded case (int8 scores)
    Q, K, V = _inputs(1000, 128, 10)
    ref, _, _, _ = oracle.forward_head(Q, K, V, 0.8, 128, 128, 0)
    e = np.abs(oracle.forward_head_mx(Q, K, V, 0.8, 128, pv="e4m3_channel")[0] - ref)
    assert e.mean() < 0.03 and e.max() < 0.5


# ---- planted mistakes: each must make at least one pin above fail ------------------------------

def _run_lowp_pins():
    checks = {
        "e4m3_values": test_every_e4m3_value_is_a_fixed_point_and_the_range_is_right,
        "e4m3_midpoints": test_e4m3_midpoints_round_to_the_even_code_and_large_values_saturate,
        "mx_hand": test_mx_hand_example_scale_rule_and_clamp,
        "mx_blocks": test_mx_blocks_axis_and_power_of_two_scaling,
        "int8": test_int8_hand_example_and_tiles,
        "routing": lambda: test_routing_is_the_bf16_routing("int8"),
        "exact": lambda: test_exact_operands_reproduce_the_bf16_definition(700, 64, 0.8, 1, True),
        "exact_tau0": lambda: test_exact_operands_reproduce_the_bf16_definition(700, 64, 0.0, 0, True),
        "channel_scales": test_channel_scales_hand_example,
        "channel_quantize": test_e4m3_channel_quantize_hand_example,
        "channel_closed_form": test_e4m3_channel_reading_is_exact_on_a_closed_form_case,
        "mantissa": test_mantissa_rounding_hand_values_and_no_underflow,
        "channel_columns": test_e4m3_channel_values_take_the_channel_scale_and_pooled_values_take_v_scales,
    }
    failed = []
    for name, fn in checks.items():
        try:
            fn()
        except (AssertionError, ValueError, IndexError):
            failed.append(name)
    return failed


def test_lowp_pins_pass_on_the_unmodified_oracle():
    assert _run_lowp_pins() == []


def test_planted_round_half_away_from_zero_is_caught(monkeypatch):
    def half_up(x):
        x = np.asarray(x, dtype=np.float64)
        ax = np.abs(x)
        _, e = np.frexp(ax)
        step = np.ldexp(1.0, np.maximum(e - 1, mx.E4M3_EMIN) - mx.E4M3_MANT)
        return np.copysign(np.minimum(np.floor(ax / step + 0.5) * step, mx.E4M3_MAX), x)

    monkeypatch.setattr(mx, "round_e4m3", half_up)
    monkeypatch.setattr(oracle, "round_e4m3", half_up)
    assert "e4m3_midpoints" in _run_lowp_pins()


def test_planted_wrong_element_exponent_is_caught(monkeypatch):
    monkeypatch.setattr(mx, "E4M3_EMAX", 7)
    assert "mx_hand" in _run_lowp_pins()


def test_planted_strict_threshold_in_the_variant_is_caught(monkeypatch):
    def strict(sbar, tau, n_force=0):
        M = float(np.max(sbar))
        keep = sbar > M - tau
        keep[:n_force] = True
        return keep, M

    monkeypatch.setattr(mx, "route", strict)
    assert "exact_tau0" in _run_lowp_pins()  # tau = 0: the argmax block sits on the threshold


def test_planted_int8_scale_is_caught(monkeypatch):
    def wrong(x, rows=128):
        x = np.asarray(x, dtype=np.float64)
        out = np.empty_like(x)
        for r0 in range(0, x.shape[0], rows):
            t = x[r0:r0 + rows]
            sc = np.abs(t).max() / 128.0 or 1.0
            out[r0:r0 + rows] = np.round(t / sc) * sc
        return out

    monkeypatch.setattr(mx, "int8_quantize_tiles", wrong)
    monkeypatch.setattr(oracle, "int8_quantize_tiles", wrong)
    assert "int8" in _run_lowp_pins()


def test_planted_int8_style_channel_scale_is_caught(monkeypatch):
    def wrong(V):
        amax = np.abs(np.asarray(V, dtype=np.float64)).max(axis=0)
        return np.where(amax > 0, amax / 127.0, 1.0)

    monkeypatch.setattr(mx, "channel_scales", wrong)
    monkeypatch.setattr(oracle, "channel_scales", wrong)
    assert "channel_scales" in _run_lowp_pins()


def test_planted_per_tensor_channel_scale_is_caught(monkeypatch):
    def per_tensor(V):
        a = float(np.abs(np.asarray(V, dtype=np.float64)).max())
        return np.full(np.shape(V)[1], a / 448.0 if a > 0 else 1.0)

    monkeypatch.setattr(mx, "channel_scales", per_tensor)
    monkeypatch.setattr(oracle, "channel_scales", per_tensor)
    assert "channel_scales" in _run_lowp_pins()


def test_planted_e4m3_range_on_the_weights_is_caught(monkeypatch):
    # clamping and flushing the weights to E4M3's own range would tie the result to the reference
    monkeypatch.setattr(mx, "e4m3_plain", lambda x, axis=-1: oracle.round_e4m3(x))
    with pytest.raises(AssertionError):
        test_e4m3_channel_result_does_not_depend_on_the_reference()
