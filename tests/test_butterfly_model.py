"""Lane-level emulation, in float32, of the routing pass's transposing butterfly reduction
(csrc/route.cu, butterfly_sum<N>) and of the per-lane partial dot products around it.

The routing pass and the fused kernel's own router must keep the same blocks bit for bit. The
fused kernel sums each proxy score with a plain xor butterfly (five steps, every lane adding its
own value and its partner's); the routing pass sums R scores at once with a butterfly that halves
the values a lane carries at every step. These tests check, on the CPU, that the second gives the
first's float32 sums exactly and leaves value r on the lanes the kernel reads it from."""
import numpy as np
import pytest

F32 = np.float32


def xor_reduce(vals):
    """Plain butterfly over 32 lanes: at offsets 16, 8, 4, 2, 1 each lane adds its partner's value
    to its own. Returns the 32 lane values afterwards."""
    x = [F32(v) for v in vals]
    for o in (16, 8, 4, 2, 1):
        x = [F32(x[l] + x[l ^ o]) for l in range(32)]
    return x


def butterfly_sum(v, o=16):
    """v[lane][k], N values per lane. Mirrors the kernel: at offset o a lane with bit o set keeps
    the upper half of its values and sends the lower half, the other lane the reverse; each kept
    value gains the partner's copy of the same value. Then the kept half recurses at o / 2."""
    n = len(v[0])
    if o < 1:
        return v
    if n == 1:
        return butterfly_sum([[F32(v[l][0] + v[l ^ o][0])] for l in range(32)], o // 2)
    h = n // 2
    out = []
    for l in range(32):
        hi = (l & o) != 0
        partner = l ^ o
        # the partner sends what this lane keeps: its lower half if this lane is low, and v.v.
        keep = v[l][h:] if hi else v[l][:h]
        recv = v[partner][h:] if hi else v[partner][:h]
        out.append([F32(keep[k] + recv[k]) for k in range(h)])
    return butterfly_sum(out, o // 2)


def partial_dots(q, kvec, dpl):
    """Lane l's partial product over components [l dpl, (l+1) dpl), in the kernel's fma order:
    fma(q0, k0, fma(q1, k1, fma(q2, k2, q3 * k3))) for dpl = 4, fma(q0, k0, q1 * k1) for 2."""
    def fma(a, b, c):
        return F32(np.float64(a) * np.float64(b) + np.float64(c))  # one rounding, as fmaf
    out = []
    for l in range(32):
        a = q[l * dpl:(l + 1) * dpl]
        b = kvec[l * dpl:(l + 1) * dpl]
        acc = F32(a[dpl - 1] * b[dpl - 1])
        for c in range(dpl - 2, -1, -1):
            acc = fma(a[c], b[c], acc)
        out.append(acc)
    return out


@pytest.mark.parametrize("n", [1, 2, 4, 8, 16])
def test_butterfly_equals_plain_xor_tree_bit_for_bit(n):
    rng = np.random.default_rng(n)
    for trial in range(40):
        scale = 10.0 ** rng.integers(-6, 7)
        vals = (rng.standard_normal((32, n)) * scale).astype(F32)
        if trial % 5 == 0:
            vals[rng.integers(0, 32, 6), rng.integers(0, n, 6)] = F32(0.0)
        got = butterfly_sum([[vals[l, k] for k in range(n)] for l in range(32)])
        logn = n.bit_length() - 1
        for l in range(32):
            r = l >> (5 - logn) if n > 1 else 0
            want = xor_reduce(vals[:, r])[l]
            assert np.array_equal(np.array([got[l][0]], F32).view(np.uint32), np.array([want], F32).view(np.uint32)), \
                (n, trial, l, r)


@pytest.mark.parametrize("d,r_blocks", [(128, 16), (128, 8), (128, 4), (64, 16), (64, 8), (64, 4)])
def test_proxy_scores_of_both_routers_agree(d, r_blocks):
    """R query-block means against one pooled key: the routing pass (R scores through the
    transposing butterfly) and the fused kernel's router (one score per plain butterfly) give the
    same float32 scores."""
    rng = np.random.default_rng(d * 100 + r_blocks)
    dpl = d // 32
    for _ in range(10):
        qbar = (rng.standard_normal((r_blocks, d)) * rng.uniform(0.01, 3.0)).astype(F32)
        kbar = (rng.standard_normal(d) * rng.uniform(0.01, 3.0)).astype(F32)
        parts = [partial_dots(qbar[r], kbar, dpl) for r in range(r_blocks)]  # [r][lane]
        v = [[parts[r][l] for r in range(r_blocks)] for l in range(32)]
        got = butterfly_sum(v)
        logr = r_blocks.bit_length() - 1
        for r in range(r_blocks):
            one = xor_reduce(parts[r])[0]
            lanes = [l for l in range(32) if (l >> (5 - logr)) == r]
            for l in lanes:
                assert np.float32(got[l][0]).view(np.uint32) == np.float32(one).view(np.uint32)
            # and both are the float32 dot product up to rounding
            assert abs(float(one) - float(np.dot(qbar[r].astype(np.float64), kbar.astype(np.float64)))) <= \
                1e-5 * (np.abs(qbar[r]).astype(np.float64) @ np.abs(kbar).astype(np.float64)) + 1e-30


def test_a_wrong_lane_map_is_caught():
    """Planted mistake: reading value r from lane r instead of lane r << (5 - log2 R) picks another
    query block's score."""
    rng = np.random.default_rng(3)
    vals = rng.standard_normal((32, 8)).astype(F32)
    got = butterfly_sum([[vals[l, k] for k in range(8)] for l in range(32)])
    wrong = [got[r][0] for r in range(8)]
    right = [xor_reduce(vals[:, r])[0] for r in range(8)]
    assert any(np.float32(a).view(np.uint32) != np.float32(b).view(np.uint32) for a, b in zip(wrong, right))
