"""GPU parity of the fused QK-norm + RoPE + block pooling step against the float64 oracle.

Pass criteria: every stored query/key element lies within one bf16 rounding (relative 2^-8) plus
1e-5 (the fp32 error of a rotated value near zero) of the float64 result, and at least 99.9 % of
them equal its bf16 rounding exactly; the pooled keys match
the oracle's means of its rounded keys to 1e-4 and the pooled values its means to 1e-5; the bf16
mirrors are the fp32 means rounded; in-place and out-of-place calls agree bit for bit; and the
pooled vectors agree with pooling the stored keys in a separate pass.
"""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_41_b200 import sol_attn as sa
from block_sparse_attention_41_b200 import workloads as wl
from block_sparse_attention_41_b200.workloads import round_to_bf16

pytestmark = pytest.mark.gpu

EPS = 1e-6


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from block_sparse_attention_41_b200 import build
    build.build()
    sa.load_library()


def _bf16_64(x):
    return round_to_bf16(x).astype(np.float64)


def _check_rows(got, ref):
    # one bf16 rounding (relative 2^-8) plus the fp32 arithmetic's absolute error: a rotated pair
    # member near zero comes from a difference of O(1) products, so its fp32 error is absolute
    err = np.abs(got - ref)
    assert np.all(err <= 2.0 ** -8 * np.abs(ref) + 1e-5), float(err.max())
    exact = np.mean(got == _bf16_64(ref))
    assert exact >= 0.999, exact


def _run(Qh, Kh, Vh, grid, d, blk, seed, in_place=False):
    cos, sin = wl.rope_tables(grid, d)
    gq, gk = wl.qk_norm_gains(d, seed)
    Q, K, V = (torch.from_numpy(x).to(torch.bfloat16).cuda() for x in (Qh, Kh, Vh))
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()  # noqa: E731
    kw = dict(Q_out=Q, K_out=K) if in_place else {}
    outs = sa.sol_attn_qknorm_rope_pool(Q, K, V, dev(gq), dev(gk), dev(cos), dev(sin), blk, EPS, **kw)
    torch.cuda.synchronize()
    return outs, (cos, sin, gq, gk)


@pytest.mark.parametrize("grid,d,blk", [((5, 10, 20), 128, 128), ((3, 7, 13), 64, 128), ((5, 10, 20), 128, 64),
                                        ((1, 1, 77), 64, 64)])
def test_qknorm_rope_pool_matches_oracle(grid, d, blk):
    B, H = 1, 3
    L = grid[0] * grid[1] * grid[2]
    rng = np.random.default_rng(L + d + blk)
    Qh, Kh, Vh = (round_to_bf16(rng.standard_normal((B, H, L, d)) * s) for s in (2.0, 0.7, 1.0))
    (Qo, Ko, kbar, vbar, klp, vlp), (cos, sin, gq, gk) = _run(Qh, Kh, Vh, grid, d, blk, seed=L)
    Qg, Kg = Qo.double().cpu().numpy(), Ko.double().cpu().numpy()
    for h in range(H):
        Qr, Kr, kb, vb = oracle.qknorm_rope_pool_head(Qh[0, h], Kh[0, h], Vh[0, h], gq, gk, cos, sin, EPS, blk,
                                                       _bf16_64)
        _check_rows(Qg[0, h], Qr)
        _check_rows(Kg[0, h], Kr)
        assert np.max(np.abs(kbar[0, h].double().cpu().numpy() - kb)) <= 1e-4
        assert np.max(np.abs(vbar[0, h].double().cpu().numpy() - vb)) <= 1e-5
    assert torch.equal(klp, kbar.to(torch.bfloat16)) and torch.equal(vlp, vbar.to(torch.bfloat16))
    # the same call in place
    (Qi, Ki, kbi, vbi, _, _), _ = _run(Qh, Kh, Vh, grid, d, blk, seed=L, in_place=True)
    assert torch.equal(Qi, Qo) and torch.equal(Ki, Ko) and torch.equal(kbi, kbar) and torch.equal(vbi, vbar)
    # the fused pooling equals pooling the stored keys in a separate pass (fp32 sums, other order)
    kbar2, vbar2, _, _ = sa.sol_attn_pool(Ko, torch.from_numpy(Vh).to(torch.bfloat16).cuda(), blk)
    assert torch.allclose(kbar2, kbar, rtol=0, atol=2e-6) and torch.allclose(vbar2, vbar, rtol=0, atol=2e-6)


def test_qknorm_rope_pool_full_720p_shape_sampled():
    """The benchmark's shape (40 heads x 75600 tokens, d 128): every output is produced, and
    sampled heads and key blocks are checked against the oracle."""
    w = wl.WORKLOADS["video720p_L75600"]
    d, blk = w.d, w.block
    cos, sin = wl.rope_tables(w.grid, d)
    gq, gk = wl.qk_norm_gains(d, 2)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()  # noqa: E731
    Q = torch.empty((1, w.H, w.L, d), dtype=torch.bfloat16, device="cuda")
    K, V = torch.empty_like(Q), torch.empty_like(Q)
    heads = [0, 17, 39]
    raw = {}
    for h in range(w.H):
        if h in heads:
            raw[h] = wl.head_tensors(w, 0, h)
            for T, a in zip((Q, K, V), raw[h]):
                T[0, h].copy_(torch.from_numpy(a).to(torch.bfloat16))
        else:
            for T in (Q, K, V):
                T[0, h].normal_()
    Qo, Ko, kbar, vbar, _, _ = sa.sol_attn_qknorm_rope_pool(Q, K, V, dev(gq), dev(gk), dev(cos), dev(sin), blk, EPS)
    torch.cuda.synchronize()
    assert bool(torch.isfinite(Qo.float()).all()) and bool(torch.isfinite(kbar).all())
    blocks = [0, 300, w.n_blocks - 1]
    for h in heads:
        Qh, Kh, Vh = (a.astype(np.float64) for a in raw[h])
        rows = np.concatenate([np.arange(j * blk, min(w.L, (j + 1) * blk)) for j in blocks])
        Qr, Kr, kb, vb = oracle.qknorm_rope_pool_head(Qh[rows], Kh[rows], Vh[rows], gq, gk, cos[rows], sin[rows], EPS,
                                                       blk, _bf16_64)
        _check_rows(Qo[0, h].double().cpu().numpy()[rows], Qr)
        _check_rows(Ko[0, h].double().cpu().numpy()[rows], Kr)
        # the sampled rows are whole blocks, so the oracle's block means line up with the kernel's
        got_k = kbar[0, h].double().cpu().numpy()[blocks]
        got_v = vbar[0, h].double().cpu().numpy()[blocks]
        assert np.max(np.abs(got_k - kb)) <= 1e-4 and np.max(np.abs(got_v - vb)) <= 1e-5
