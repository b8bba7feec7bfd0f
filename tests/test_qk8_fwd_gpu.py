"""GPU parity of the forward with 8-bit QK^T (sol_attn_fwd_qk8) against the oracle's int8 variant.

The oracle (oracle/mxfp8_oracle.py with qk="int8" and exact PV) quantizes Q, K - mu and the pooled
keys k_bar - mu per 128-row tile and otherwise computes the bf16 definition. The kernel runs the
same products on int8 tensor cores and folds the tile scales into the softmax scale. Routing is the
bf16 routing, so the kept sets agree outside the near-threshold band; units whose kept set differs
(a near-threshold decision) are not compared.
"""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_41_b200 import sol_attn as sa

from test_parity_gpu import local_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from block_sparse_attention_41_b200 import build
    build.build()
    sa.load_library()


# ------------------------------------------------------------------------------------------------
# the forward with 8-bit QK^T against the oracle's int8 variant (exact PV)
# ------------------------------------------------------------------------------------------------

TOL_MAX, TOL_MEAN = 2e-2, 2e-3  # as the bf16 path: P is rounded to bf16, v_bar is bf16


def _fwd_qk8(Q, K, V, tau, n_force=0, mask=None):
    kbar, vbar, klp, vlp = sa.sol_attn_pool(K, V, 128)
    q8, k8, kb8, qs, ks, kbs, mu = sa.sol_attn_quantize_qk8(Q, K, kbar)
    O = sa.sol_attn_fwd_qk8(Q, q8, k8, kb8, qs, ks, kbs, V, kbar, vlp, tau, n_force=n_force, kept_mask=mask)
    torch.cuda.synchronize()
    return O


@pytest.mark.parametrize("L,tau,n_force", [(1000, [0.0, 1.0], 0), (3000, [0.6, 2.0], 2), (129, [0.3, float("inf")], 0),
                                           (16_500, [0.4, 0.8], 0)])
def test_qk8_forward_matches_the_int8_oracle(L, tau, n_force):
    B, H, d = 1, 2, 128
    Qh, Kh, Vh = local_inputs(B, H, L, d, seed=L + 11)
    Q, K, V = (torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16).cuda() for x in (Qh, Kh, Vh))
    nb = -(-L // 128)
    mask = torch.empty((B, H, nb, nb), dtype=torch.uint8, device="cuda")
    O = _fwd_qk8(Q, K, V, tau, n_force, mask)
    mk = mask.cpu().numpy().astype(bool)
    units = range(nb) if nb <= 40 else sorted(set(np.random.default_rng(L).choice(nb, 10, replace=False).tolist()) | {nb - 1})
    errs = []
    for h in range(H):
        q, k, v = (x[0, h].astype(np.float64) for x in (Qh, Kh, Vh))
        ref, keep = oracle.forward_head_mx(q, k, v, tau[h], 128, n_force, qk="int8", quant=oracle.no_quantize,
                                           units=list(units))
        _, keep_bf, sbar, M = oracle.forward_head(q, k, v, tau[h], 128, 128, n_force, units=list(units))
        band = oracle.band_mask(sbar[list(units)], M[list(units)], tau[h], n_force)
        # routing is the bf16 routing: the kept sets agree outside the band
        assert (mk[0, h][list(units)][~band] == keep_bf[list(units)][~band]).all()
        for i in units:
            if not np.array_equal(mk[0, h, i], keep[i]):
                continue  # a near-threshold decision: the oracle row was computed with the other set
            rows = slice(i * 128, min(L, i * 128 + 128))
            errs.append(np.abs(O[0, h, rows].double().cpu().numpy() - ref[rows]))
    e = np.concatenate([x.ravel() for x in errs])
    print(f"\n[qk8 fwd L={L}] max_abs={e.max():.3e} mean_abs={e.mean():.3e} units={len(errs)}")
    assert e.max() <= TOL_MAX and e.mean() <= TOL_MEAN


def test_qk8_forward_is_close_to_the_bf16_forward():
    # the 8-bit variant's own error against the exact definition, measured on the GPU: about the
    # oracle's figure for int8 QK^T with exact PV (mean 0.005, max 0.07 on seeded inputs)
    Qh, Kh, Vh = local_inputs(1, 2, 3000, 128, seed=5)
    Q, K, V = (torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16).cuda() for x in (Qh, Kh, Vh))
    O8 = _fwd_qk8(Q, K, V, [0.5, 1.5])
    O16, _, _ = sa.sol_attn(Q, K, V, [0.5, 1.5])
    torch.cuda.synchronize()
    diff = (O8.double() - O16.double()).abs()
    assert float(diff.mean()) < 0.02 and float(diff.max()) < 0.3
