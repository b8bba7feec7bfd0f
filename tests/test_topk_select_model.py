"""Lane-level emulation of the routing pass's top-k selection (csrc/route.cu, radix_select_kth
and the ballot pass), checked against the top-k oracle: random scores, heavy ties, signed zeros
and a wide range of magnitudes. It checks the algorithm the kernel implements, on the CPU."""
import numpy as np
import pytest

import oracle

def ordered_key(f):
    f = np.float32(f) + np.float32(0.0)
    u = int(np.array([f], dtype=np.float32).view(np.uint32)[0])
    return (~u & 0xffffffff) if (u & 0x80000000) else (u | 0x80000000)

def radix_select_kth(sc, k):
    keys = [ordered_key(x) for x in sc]
    prefix, pmask, kk = 0, 0, k
    for shift in (24, 16, 8, 0):
        hist = [0] * 256
        for key in keys:
            if (key & pmask) == prefix:
                hist[(key >> shift) & 255] += 1
        lsum = [sum(hist[8 * l: 8 * l + 8]) for l in range(32)]
        suf = [sum(lsum[l:]) for l in range(32)]
        above = [suf[l] - lsum[l] for l in range(32)]
        mine = [above[l] < kk <= suf[l] for l in range(32)]
        assert sum(mine) == 1, (shift, kk, suf)
        src = mine.index(True)
        acc, qsel, higher = above[src], -1, 0
        for q in range(7, -1, -1):
            c = hist[8 * src + q]
            if qsel < 0 and acc + c >= kk:
                qsel, higher = q, acc
            acc += c
        prefix |= (8 * src + qsel) << shift
        pmask |= 255 << shift
        kk -= higher
    return prefix, kk, keys

def select(sc, k, n_force):
    kth, take, keys = radix_select_kth(sc, k)
    n = len(sc)
    keep = np.zeros(n, bool)
    for i in range((n + 31) // 32):
        js = range(32 * i, min(n, 32 * i + 32))
        gt = [j for j in js if keys[j] > kth]
        eq = [j for j in js if keys[j] == kth]
        eq_kept = eq[:max(0, take)]
        take -= len(eq_kept)
        for j in gt + eq_kept:
            keep[j] = True
        for j in js:
            if j < n_force:
                keep[j] = True
    return keep



@pytest.mark.parametrize("kind", range(4))
def test_emulated_selection_equals_the_oracle(kind):
    rng = np.random.default_rng(kind)
    for _ in range(400):
        n = int(rng.integers(1, 300))
        if kind == 0:
            sc = rng.standard_normal(n).astype(np.float32)
        elif kind == 1:
            sc = rng.integers(-3, 4, n).astype(np.float32)
        elif kind == 2:
            sc = rng.choice(np.array([-0.0, 0.0, 1.0, -1.0], np.float32), n)
        else:
            sc = (rng.standard_normal(n) * 10.0 ** rng.integers(-30, 30, n)).astype(np.float32)
        k = int(rng.integers(1, n + 1))
        nf = int(rng.integers(0, 3))
        assert np.array_equal(select(sc, k, nf), oracle.route_topk(sc.astype(np.float64), k, nf))
