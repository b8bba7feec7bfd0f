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


# ------------------------------------------------------------------------------------------------
# the query-block means written by the same pass, and the forward whose routing takes them
# ------------------------------------------------------------------------------------------------

@pytest.mark.parametrize("grid,d,blk", [((5, 10, 20), 128, 128), ((3, 7, 13), 64, 128), ((1, 1, 77), 64, 64)])
def test_qbar_output_is_the_mean_of_the_stored_query_rows(grid, d, blk):
    """q_bar is the mean of each block's stored (bf16) query rows over its valid rows; asking for it
    changes no other output of the pass."""
    B, H = 1, 3
    L = grid[0] * grid[1] * grid[2]
    rng = np.random.default_rng(L + 7 * d + blk)
    Qh, Kh, Vh = (round_to_bf16(rng.standard_normal((B, H, L, d)) * s) for s in (2.0, 0.7, 1.0))
    cos, sin = wl.rope_tables(grid, d)
    gq, gk = wl.qk_norm_gains(d, L)
    Q, K, V = (torch.from_numpy(x).to(torch.bfloat16).cuda() for x in (Qh, Kh, Vh))
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()  # noqa: E731
    args = (Q, K, V, dev(gq), dev(gk), dev(cos), dev(sin), blk, EPS)
    plain = sa.sol_attn_qknorm_rope_pool(*args)
    withq = sa.sol_attn_qknorm_rope_pool(*args, want_qbar=True)
    torch.cuda.synchronize()
    assert len(withq) == 7
    for a, b in zip(plain, withq[:6]):
        assert torch.equal(a, b)
    qbar = withq[6].double().cpu().numpy()
    Qg = withq[0].double().cpu().numpy()
    for h in range(H):
        ref = oracle.pool_blocks(Qg[0, h], blk)  # the stored rows, pooled in float64
        assert qbar[0, h].shape == ref.shape
        assert np.max(np.abs(qbar[0, h] - ref)) <= 2e-6 * max(1.0, float(np.abs(Qg).max()))
        # and against the means of the oracle's own stored rows: a difference of means is at most
        # the mean of the row differences (the rare last-bit bf16 roundings), plus fp32 summation
        Qr, _, _, _ = oracle.qknorm_rope_pool_head(Qh[0, h], Kh[0, h], Vh[0, h], gq, gk, cos, sin, EPS, blk, _bf16_64)
        bound = oracle.pool_blocks(np.abs(Qg[0, h] - Qr), blk) + 2e-6 * max(1.0, float(np.abs(Qg).max()))
        assert np.all(np.abs(qbar[0, h] - oracle.pool_blocks(Qr, blk)) <= bound)


@pytest.mark.parametrize("L,d,tau,n_force", [(3000, 128, [0.4, 1.0], 0), (1111, 64, [0.0, 2.0], 2),
                                             (16_500, 128, [0.6, 0.3], 0)])
def test_forward_with_given_qbar_matches_the_oracle(L, d, tau, n_force):
    """The pass's q_bar fed to sol_attn_fwd_qbar: the routing pass reads no Q, the kept sets meet
    the oracle's routing acceptance, O is within the bf16 tolerance of the oracle, and the result
    agrees with sol_attn_fwd on the same stored inputs (masks may differ only where the proxy score
    lies within rounding of the threshold)."""
    from test_parity_gpu import local_inputs, full_compare, check_bf16, check_mask_density, report
    B, H = 1, 2
    Qh, Kh, Vh = local_inputs(B, H, L, d, seed=L + d)
    grid = (1, 1, L)
    cos, sin = wl.rope_tables(grid, d)
    gq, gk = wl.qk_norm_gains(d, L)
    Q, K, V = (torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16).cuda() for x in (Qh, Kh, Vh))
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()  # noqa: E731
    Qs, Ks, kbar, vbar, klp, vlp, qbar = sa.sol_attn_qknorm_rope_pool(Q, K, V, dev(gq), dev(gk), dev(cos), dev(sin),
                                                                      128, EPS, want_qbar=True)
    nb = -(-L // 128)
    masks, outs = [], []
    for use_qbar in (True, False):
        mask = torch.empty((B, H, nb, nb), dtype=torch.uint8, device="cuda")
        dens = torch.empty((B, H), dtype=torch.float32, device="cuda")
        ws = sa.new_workspace(B, H, L, 128, Q.device)
        if use_qbar:
            O = sa.sol_attn_fwd_qbar(Qs, Ks, V, kbar, vbar, klp, vlp, qbar, tau, n_force=n_force, kept_mask=mask,
                                     density=dens, workspace=ws)
        else:
            O = sa.sol_attn_fwd(Qs, Ks, V, kbar, vbar, klp, vlp, tau, 128, 128, n_force=n_force, kept_mask=mask,
                                density=dens, workspace=ws)
        sa.sol_attn_check_device_error(ws)
        check_mask_density(mask, dens, n_force)
        masks.append(mask)
        outs.append(O)
    Qsh, Ksh = Qs.double().cpu().numpy(), Ks.double().cpu().numpy()
    st = full_compare(Qsh, Ksh, Vh.astype(np.float64), outs[0], masks[0], tau, 128, n_force=n_force)
    report(f"fwd with given q_bar L={L} d={d}", st)
    check_bf16(st)
    differ = int((masks[0] != masks[1]).sum())
    assert differ <= st["band_entries"], (differ, st["band_entries"])
    if differ == 0:
        diff = (outs[0].double() - outs[1].double()).abs()
        assert float(diff.max()) <= 2e-2 and float(diff.mean()) <= 2e-3
