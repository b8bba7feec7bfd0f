"""GPU check of the 8-bit QK^T operands (sol_attn_quantize_qk8) against the oracle's int8 tiles.

The oracle (oracle/mxfp8_oracle.py, int8 QK^T) quantizes Q, K - mu and k_bar - mu per 128-row tile
with scale amax / 127 and round-half-even, in float64. The kernel takes the same decision in
float32 (x * 127 / amax, round to nearest even) from its own float32 mean key and pooled keys. So a
code is unique except where the float64 value x / s lies within a hair of a .5 tie: there the two
may differ by one, and the test counts those. Everywhere else the codes must be equal, and the
scales agree to float32 rounding.
"""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_41_b200 import sol_attn as sa

from test_parity_gpu import local_inputs

pytestmark = pytest.mark.gpu
TIE_WINDOW = 1e-4  # float32 rounding of x * 127 / amax, in units of the code (127 * 2^-23 ~ 1.5e-5, padded)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from block_sparse_attention_41_b200 import build
    build.build()
    sa.load_library()


def oracle_codes(x, rows=128):
    """Codes and scales of symmetric int8 tiles (the oracle's quantizer, written out per tile)."""
    codes = np.empty(x.shape, dtype=np.int64)
    ratio = np.empty(x.shape)
    scales = []
    for r0 in range(0, x.shape[0], rows):
        t = x[r0:r0 + rows]
        amax = np.abs(t).max()
        s = amax / 127.0 if amax > 0 else 1.0
        scales.append(s)
        ratio[r0:r0 + rows] = t / s
        codes[r0:r0 + rows] = np.round(t / s)
    # the oracle's dequantized values are these codes times the scales
    deq = oracle.int8_quantize_tiles(x, rows)
    rep = np.repeat(np.array(scales), rows)[: x.shape[0]][:, None]
    assert np.allclose(deq, codes * rep, rtol=0, atol=1e-12)
    return codes, np.array(scales), ratio


def compare(gpu_codes, gpu_scales, x, dx=0.0):
    """dx bounds how far the kernel's float32 input may be from x (its own mean key and pooled
    keys): a tie window of dx / s + TIE_WINDOW codes around every .5."""
    codes, scales, ratio = oracle_codes(x)
    assert np.allclose(gpu_scales, scales, rtol=2e-6, atol=dx / 127)
    diff = gpu_codes.astype(np.int64) - codes
    window = TIE_WINDOW + dx / np.repeat(scales, 128)[: x.shape[0]][:, None]
    near_tie = np.abs(np.abs(ratio - np.floor(ratio)) - 0.5) < window
    assert (diff[~near_tie] == 0).all()
    assert (np.abs(diff[near_tie]) <= 1).all()
    return int((diff != 0).sum()), int(near_tie.sum())


@pytest.mark.parametrize("L,d", [(1000, 128), (300, 64), (16_500, 128)])
def test_qk8_codes_match_the_oracle(L, d):
    B, H = 1, 2
    Qh, Kh, Vh = local_inputs(B, H, L, d, seed=L + 3 * d)
    Kh = Kh + 0.7  # a common key offset, removed by the mean-key smoothing
    Q, K, V = (torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16).cuda() for x in (Qh, Kh, Vh))
    Kh = K.float().cpu().numpy()  # the bf16 values the kernel reads
    kbar, _, _, _ = sa.sol_attn_pool(K, V, 128)
    q8, k8, kb8, qs, ks, kbs, mu = sa.sol_attn_quantize_qk8(Q, K, kbar)
    torch.cuda.synchronize()
    flips = 0
    for h in range(H):
        k64 = Kh[0, h].astype(np.float64)
        mu_ref = k64.mean(axis=0)
        assert np.allclose(mu[0, h].double().cpu().numpy(), mu_ref, rtol=0, atol=2e-6)
        f, _ = compare(q8[0, h].cpu().numpy(), qs[0, h].cpu().numpy(), Qh[0, h].astype(np.float64))
        flips += f
        # the kernel's mean key is within 2e-6 (asserted above) and its pooled keys within 2e-6
        # (the pooling test's bound) of the float64 values
        f, _ = compare(k8[0, h].cpu().numpy(), ks[0, h].cpu().numpy(), k64 - mu_ref, dx=2e-6)
        flips += f
        kb = oracle.pool_blocks(k64, 128) - mu_ref
        f, _ = compare(kb8[0, h].cpu().numpy(), kbs[0, h].cpu().numpy(), kb, dx=4e-6)
        flips += f
    print(f"\n[qk8 L={L} d={d}] near-tie codes that differ by one: {flips}")
    assert int(q8.abs().max()) <= 127 and int(k8.abs().max()) <= 127


def test_qk8_all_zero_tile_has_scale_one():
    Q = torch.zeros((1, 1, 256, 64), dtype=torch.bfloat16, device="cuda")
    K = torch.zeros_like(Q)
    kbar, _, _, _ = sa.sol_attn_pool(K, K, 128)
    q8, k8, kb8, qs, ks, kbs, mu = sa.sol_attn_quantize_qk8(Q, K, kbar)
    torch.cuda.synchronize()
    assert int(q8.abs().max()) == 0 and int(k8.abs().max()) == 0 and int(kb8.abs().max()) == 0
    assert torch.equal(qs, torch.ones_like(qs)) and torch.equal(ks, torch.ones_like(ks))
    assert torch.equal(kbs, torch.ones_like(kbs)) and float(mu.abs().max()) == 0.0

