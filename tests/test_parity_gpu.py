"""GPU parity: the CUDA path, called through the C ABI, against the float64 CPU oracle on the same
seeded inputs.

Pass criteria:
  * kept-block mask: bit-exact except in the near-threshold band |s_bar - (max - tau)| < 1e-3,
    where fp32 and float64 routing may legitimately differ; the band count is reported.
  * O: bf16 inputs (fp32 accumulation): max-abs <= 2e-2 and mean-abs <= 2e-3. fp32 inputs:
    max-abs <= 1e-4.
The large workloads run in the same launch configuration as the benchmark, at full size, and
are checked on seeded samples of query blocks (query blocks are independent).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_41_b200 import sol_attn as sa
from block_sparse_attention_41_b200 import workloads as wl
from block_sparse_attention_41_b200.workloads import round_to_bf16

from parity_harness import (TOL_BF16_MAX, TOL_BF16_MEAN, TOL_F32_MAX, compare_units, device_inputs,
                            merge_violations, run_path, taus)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from block_sparse_attention_41_b200 import build
    build.build()
    sa.load_library()


def report(name, st):
    print(f"\n[{name}] max_abs={st['max_abs']:.3e} mean_abs={st['mean_abs']:.3e} "
          f"band={st['band_entries']} mismatches={st['mask_mismatch_outside_band']} units={st['units']} "
          f"routing_violations={st['routing_violations']}")


def check_routing(st):
    """The mask equals the oracle's outside the band and, inside it, is a kept set that a float32
    evaluation of the routing could produce (every count of oracle.routing_violations is 0)."""
    assert st["mask_mismatch_outside_band"] == 0
    assert set(st["routing_violations"]) == {"forced", "outside_band", "max_kept", "threshold"}
    assert all(n == 0 for n in st["routing_violations"].values()), st["routing_violations"]


def check_bf16(st):
    check_routing(st)
    assert st["max_abs"] <= TOL_BF16_MAX
    assert st["mean_abs"] <= TOL_BF16_MEAN


def check_mask_density(mask, dens, n_force=0):
    m = mask.float()
    assert torch.equal(m.mean(dim=(2, 3)), dens) or torch.allclose(m.mean(dim=(2, 3)), dens, rtol=0, atol=1e-7)
    if n_force:
        assert bool(mask[:, :, :, :n_force].all())


# ------------------------------------------------------------------------------------------------
# pooling
# ------------------------------------------------------------------------------------------------

@pytest.mark.parametrize("dtype,L,d,blk", [("bf16", 1000, 128, 128), ("bf16", 77, 64, 128), ("f32", 1000, 64, 64),
                                           ("bf16", 4096, 128, 128), ("f32", 130, 128, 32), ("bf16", 300, 256, 128),
                                           ("bf16", 260, 8, 64), ("f32", 99, 4, 16), ("f32", 500, 32, 128)])
def test_pool_matches_oracle(dtype, L, d, blk):
    rng = np.random.default_rng(L + d)
    B, H = 2, 3
    X = [rng.standard_normal((B, H, L, d)) * 2 + 1 for _ in range(2)]
    X = [round_to_bf16(x) if dtype == "bf16" else x.astype(np.float32) for x in X]
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    K, V = (torch.from_numpy(x).to(tdt).cuda() for x in X)
    kbar, vbar, klp, vlp = sa.sol_attn_pool(K, V, blk)
    torch.cuda.synchronize()
    for t, x, lp in ((kbar, X[0], klp), (vbar, X[1], vlp)):
        ref = np.stack([np.stack([oracle.pool_blocks(x[b, h].astype(np.float64), blk) for h in range(H)])
                        for b in range(B)])
        assert np.max(np.abs(t.double().cpu().numpy() - ref)) < 2e-6
        if dtype == "bf16":
            assert torch.equal(lp, t.to(torch.bfloat16))
        else:
            assert lp is None


# ------------------------------------------------------------------------------------------------
# the five workloads
# ------------------------------------------------------------------------------------------------

@pytest.mark.parametrize("tau", [math.inf, 2.0, 0.5])
def test_tiny_f32_workload_full(tau):
    w = wl.WORKLOADS["tiny_f32_L1024"]
    Q, K, V = device_inputs(w)
    t = [tau] * w.H
    O, mask, dens = run_path(Q, K, V, t, w.block)
    units = [(b, h, i) for b in range(w.B) for h in range(w.H) for i in range(w.n_blocks)]
    st = compare_units(w, t, units, O, mask)
    report(f"tiny f32 tau={tau}", st)
    check_routing(st)
    assert st["max_abs"] <= TOL_F32_MAX
    check_mask_density(mask, dens)
    if math.isinf(tau):
        assert bool(mask.all())


def test_small_dit_workload_full():
    w = wl.WORKLOADS["small_dit_L8192"]
    Q, K, V = device_inputs(w)
    t = taus(w, "0.25")
    O, mask, dens = run_path(Q, K, V, t, w.block)
    units = [(b, h, i) for b in range(w.B) for h in range(w.H) for i in range(w.n_blocks)]
    st = compare_units(w, t, units, O, mask)
    report("small DiT 25%", st)
    check_bf16(st)
    check_mask_density(mask, dens)
    assert abs(float(dens.mean()) - 0.25) < 0.01


@pytest.fixture(scope="module")
def video720p():
    w = wl.WORKLOADS["video720p_L75600"]
    return (w, *device_inputs(w))


@pytest.mark.parametrize("density", ["0.1", "0.2", "0.4", "1.0"])
def test_video720p_workload_sampled(video720p, density):
    w, Q, K, V = video720p
    t = taus(w, density)
    O, mask, dens = run_path(Q, K, V, t, w.block)
    units = wl.sample_units(w, 24, seed_offset=int(float(density) * 100))
    st = compare_units(w, t, units, O, mask)
    report(f"720p {density}", st)
    check_bf16(st)
    check_mask_density(mask, dens)
    assert abs(float(dens.mean()) - float(density)) < 0.01


def test_video1080p_workload_sampled():
    w = wl.WORKLOADS["video1080p_L252960"]
    Q, K, V = device_inputs(w)
    t = taus(w, "0.15")
    O, mask, dens = run_path(Q, K, V, t, w.block)
    units = wl.sample_units(w, 64)
    st = compare_units(w, t, units, O, mask)
    report("1080p 15%", st)
    check_bf16(st)
    check_mask_density(mask, dens)
    assert abs(float(dens.mean()) - 0.15) < 0.01
    del Q, K, V, O
    torch.cuda.empty_cache()


def test_text_video_cfg_workload_sampled():
    w = wl.WORKLOADS["text_video_cfg_L33272"]
    Q, K, V = device_inputs(w)
    t = taus(w, "per_head")
    O, mask, dens = run_path(Q, K, V, t, w.block, n_force=w.n_force)
    units = wl.sample_units(w, 48)
    st = compare_units(w, t, units, O, mask, n_force=w.n_force)
    report("text+video CFG", st)
    check_bf16(st)
    check_mask_density(mask, dens, n_force=w.n_force)
    spread = dens[0].cpu().numpy()
    assert spread.max() - spread.min() > 0.2  # densities really vary across heads


# ------------------------------------------------------------------------------------------------
# edge cases on small synthetic inputs (compared in full)
# ------------------------------------------------------------------------------------------------

def local_inputs(B, H, L, d, seed, pos=2.0, dtype="bf16"):
    rng = np.random.default_rng(seed)
    t = np.arange(L)[:, None] / 40.0
    c = np.arange(d)[None, :]
    feat = np.where(c % 2 == 0, np.sin(t * (1 + c % 5)), np.cos(t * (1 + c % 3)))
    Q = rng.standard_normal((B, H, L, d)) + pos * feat
    K = rng.standard_normal((B, H, L, d)) + pos * feat
    V = rng.standard_normal((B, H, L, d))
    rnd = round_to_bf16 if dtype == "bf16" else (lambda a: a.astype(np.float32))
    return rnd(Q), rnd(K), rnd(V)


def full_compare(Qh, Kh, Vh, O, mask, tau, blk, n_force=0):
    B, H, L, d = Qh.shape
    max_err, sum_err, n, mism, band_n = 0.0, 0.0, 0, 0, 0
    viol = {}
    mk = mask.cpu().numpy().astype(bool)
    Og = O.double().cpu().numpy()
    for b in range(B):
        for h in range(H):
            O_ref, keep, sbar, M = oracle.forward_head(Qh[b, h], Kh[b, h], Vh[b, h], tau[h], blk, blk, n_force,
                                                       keep_override=mk[b, h])
            band = oracle.band_mask(sbar, M, tau[h], n_force)
            eps = oracle.proxy_error_bound(Qh[b, h], Kh[b, h], blk, blk)
            merge_violations(viol, oracle.routing_violations(sbar, M, tau[h], mk[b, h], eps, n_force))
            mism += int((mk[b, h][~band] != keep[~band]).sum())
            band_n += int(band.sum())
            e = np.abs(Og[b, h] - O_ref)
            max_err = max(max_err, float(e.max()))
            sum_err += float(e.sum())
            n += e.size
    return {"max_abs": max_err, "mean_abs": sum_err / n, "mask_mismatch_outside_band": mism, "band_entries": band_n,
            "units": B * H, "routing_violations": viol}


@pytest.mark.parametrize("L", [1, 5, 100, 128, 129, 383, 1000, 2049])
@pytest.mark.parametrize("d", [64, 128])
def test_bf16_ragged_lengths(L, d):
    Qh, Kh, Vh = local_inputs(2, 3, L, d, seed=L * 7 + d)
    Q, K, V = (torch.from_numpy(x).to(torch.bfloat16).cuda() for x in (Qh, Kh, Vh))
    tau = [0.0, 1.5, math.inf]
    O, mask, dens = run_path(Q, K, V, tau, 128)
    st = full_compare(Qh, Kh, Vh, O, mask, tau, 128)
    report(f"ragged L={L} d={d}", st)
    check_bf16(st)
    check_mask_density(mask, dens)


@pytest.mark.parametrize("n_force", [1, 3, 8])
def test_bf16_forced_blocks(n_force):
    Qh, Kh, Vh = local_inputs(1, 2, 1000, 128, seed=5 + n_force)
    Q, K, V = (torch.from_numpy(x).to(torch.bfloat16).cuda() for x in (Qh, Kh, Vh))
    tau = [0.0, 0.8]
    O, mask, dens = run_path(Q, K, V, tau, 128, n_force=n_force)
    st = full_compare(Qh, Kh, Vh, O, mask, tau, 128, n_force=n_force)
    report(f"n_force={n_force}", st)
    check_bf16(st)
    check_mask_density(mask, dens, n_force=n_force)


def test_bf16_identical_block_keys_give_dense_attention():
    # every key block holds one repeated key and value: the corrected sparse output is dense attention
    rng = np.random.default_rng(11)
    B, H, L, d, blk = 1, 2, 1500, 128, 128
    nb = -(-L // blk)
    tok = np.arange(L) // blk
    Kh = round_to_bf16(rng.standard_normal((B, H, nb, d)) * 1.5)[:, :, tok]
    Vh = round_to_bf16(rng.standard_normal((B, H, nb, d)))[:, :, tok]
    Qh = round_to_bf16(rng.standard_normal((B, H, L, d)) * 1.5)
    Q, K, V = (torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16).cuda() for x in (Qh, Kh, Vh))
    O, mask, _ = run_path(Q, K, V, [0.0, 0.5], blk)
    assert not bool(mask.all())
    dense = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(Qh).double(), torch.from_numpy(np.ascontiguousarray(Kh)).double(),
        torch.from_numpy(np.ascontiguousarray(Vh)).double()).numpy()
    err = np.abs(O.double().cpu().numpy() - dense)
    assert err.max() <= TOL_BF16_MAX and err.mean() <= TOL_BF16_MEAN


# ------------------------------------------------------------------------------------------------
# routing pass (full workspace) against the fused kernel's own routing (header-only workspace)
# ------------------------------------------------------------------------------------------------

def _header_only_workspace(B, H, device):
    return torch.zeros(((4 + B * H) * 4 + 255) // 256 * 256, dtype=torch.uint8, device=device)


@pytest.mark.parametrize("L,d,H", [(3000, 128, 3), (1500, 64, 2), (150_000, 128, 1), (140_000, 64, 1),
                                   (262_221, 128, 1), (524_288, 64, 1)])
def test_routing_pass_matches_in_kernel_routing(L, d, H):
    """Both routing paths do the same fp32 arithmetic in the same order, so the mask, the density
    and O agree bit for bit. The routing pass takes 16 query blocks per CTA up to N_kb = 1024, 8 up
    to 2048 (N_kb = 1172 and 1094 here) and 4 beyond (N_kb = 2049 and 4096, the limit); sampled
    query blocks of the long cases are also checked against the oracle."""
    Qh, Kh, Vh = local_inputs(1, H, L, d, seed=L % 997 + d)
    Q, K, V = (torch.from_numpy(x).to(torch.bfloat16).cuda() for x in (Qh, Kh, Vh))
    kbar, vbar, klp, vlp = sa.sol_attn_pool(K, V, 128)
    nb = -(-L // 128)
    tau = {1: [0.3], 2: [0.4, 1.2], 3: [0.0, 1.0, math.inf]}[H]
    outs = []
    for ws in (sa.new_workspace(1, H, L, 128, Q.device), _header_only_workspace(1, H, Q.device)):
        mask = torch.empty((1, H, nb, nb), dtype=torch.uint8, device="cuda")
        dens = torch.empty((1, H), dtype=torch.float32, device="cuda")
        O = sa.sol_attn_fwd(Q, K, V, kbar, vbar, klp, vlp, tau, 128, 128, kept_mask=mask, density=dens, workspace=ws)
        sa.sol_attn_check_device_error(ws)
        outs.append((O, mask, dens))
    assert torch.equal(outs[0][1], outs[1][1])
    assert torch.equal(outs[0][2], outs[1][2])
    assert torch.equal(outs[0][0], outs[1][0])
    O, mask, dens = outs[0]
    check_mask_density(mask, dens)
    if nb <= 64:
        st = full_compare(Qh, Kh, Vh, O, mask, tau, 128)
    else:
        units = sorted(set(np.random.default_rng(d).choice(nb, size=3, replace=False).tolist()) | {0, nb - 1})
        mk = mask.cpu().numpy().astype(bool)[0, 0]
        O_ref, keep, sbar, M = oracle.forward_head(Qh[0, 0], Kh[0, 0], Vh[0, 0], tau[0], 128, 128, 0, units=units,
                                                   keep_override=mk)
        band = oracle.band_mask(sbar[units], M[units], tau[0], 0)
        eps = oracle.proxy_error_bound(Qh[0, 0], Kh[0, 0], 128, 128, units=units)
        rows = np.concatenate([np.arange(i * 128, min(L, i * 128 + 128)) for i in units])
        e = np.abs(O[0, 0].double().cpu().numpy()[rows] - O_ref[rows])
        st = {"max_abs": float(e.max()), "mean_abs": float(e.mean()),
              "mask_mismatch_outside_band": int((mk[units][~band] != keep[units][~band]).sum()),
              "band_entries": int(band.sum()), "units": len(units),
              "routing_violations": oracle.routing_violations(sbar[units], M[units], tau[0], mk[units], eps[units])}
    report(f"routing pass L={L} d={d}", st)
    check_bf16(st)


@pytest.mark.parametrize("blk,d", [(32, 32), (64, 64), (128, 128), (64, 128)])
def test_f32_path_shapes(blk, d):
    Qh, Kh, Vh = local_inputs(1, 2, 700, d, seed=blk + d, dtype="f32")
    Q, K, V = (torch.from_numpy(x).cuda() for x in (Qh, Kh, Vh))
    tau = [0.3, 2.0]
    O, mask, dens = run_path(Q, K, V, tau, blk)
    st = full_compare(Qh, Kh, Vh, O, mask, tau, blk)
    report(f"f32 blk={blk} d={d}", st)
    check_routing(st)
    assert st["max_abs"] <= TOL_F32_MAX
    check_mask_density(mask, dens)


def test_repeat_calls_are_bitwise_deterministic():
    Qh, Kh, Vh = local_inputs(1, 4, 3000, 128, seed=3)
    Q, K, V = (torch.from_numpy(x).to(torch.bfloat16).cuda() for x in (Qh, Kh, Vh))
    ws = sa.new_workspace(1, 4, 3000, 128, Q.device)
    outs = [sa.sol_attn(Q, K, V, [0.5, 1.0, 2.0, math.inf], want_mask=True, workspace=ws) for _ in range(3)]
    torch.cuda.synchronize()
    for O, m, _ in outs[1:]:
        assert torch.equal(O, outs[0][0]) and torch.equal(m, outs[0][1])


def test_nondefault_stream():
    Qh, Kh, Vh = local_inputs(1, 2, 900, 64, seed=9)
    Q, K, V = (torch.from_numpy(x).to(torch.bfloat16).cuda() for x in (Qh, Kh, Vh))
    ref, _, _ = sa.sol_attn(Q, K, V, [0.7, 0.7])
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        O, _, _ = sa.sol_attn(Q, K, V, [0.7, 0.7])
    s.synchronize()
    torch.cuda.synchronize()
    assert torch.equal(O, ref)


# ------------------------------------------------------------------------------------------------
# failure detection: a bounded on-device wait expires, the host reads the status, the context lives
# ------------------------------------------------------------------------------------------------

def test_expired_wait_is_reported_and_context_survives():
    Qh, Kh, Vh = local_inputs(1, 2, 2000, 128, seed=21)
    Q, K, V = (torch.from_numpy(x).to(torch.bfloat16).cuda() for x in (Qh, Kh, Vh))
    ws = sa.new_workspace(1, 2, 2000, 128, Q.device)
    sa.sol_attn_check_device_error(ws)  # clean start
    sa.sol_attn_debug_drop_one_load(1)
    sa.sol_attn(Q, K, V, [0.5, 0.5], workspace=ws)
    with pytest.raises(sa.SolAttnError) as ei:
        sa.sol_attn_check_device_error(ws)
    assert ei.value.status == sa.SOL_ETIMEOUT
    sa.sol_attn_check_device_error(ws)  # the error word was cleared
    O, mask, _ = sa.sol_attn(Q, K, V, [0.5, 0.5], want_mask=True, workspace=ws)
    sa.sol_attn_check_device_error(ws)
    st = full_compare(Qh, Kh, Vh, O, mask, [0.5, 0.5], 128)
    check_bf16(st)
