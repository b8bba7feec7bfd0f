"""GPU checks of sol_attn_fwd_host: the whole path on host buffers, pipelined by head chunks.

Heads are independent, and every chunk runs the same kernels as the device-resident call on a
slice of the heads. So the output and the per-head densities must equal those of sol_attn (pool +
sol_attn_fwd on device tensors) bit for bit, for every chunk size, for pinned and for pageable
host memory. One case is also compared with the float64 oracle directly.
"""
import math

import numpy as np
import pytest
import torch

from block_sparse_attention_41_b200 import sol_attn as sa
from block_sparse_attention_41_b200 import workloads as wl

from parity_harness import taus
from test_parity_gpu import check_bf16, full_compare, local_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from block_sparse_attention_41_b200 import build
    build.build()
    sa.load_library()


def _device_path(Qc, Kc, Vc, tau, blk, n_force):
    Q, K, V = (t.cuda() for t in (Qc, Kc, Vc))
    O, mask, dens = sa.sol_attn(Q, K, V, tau, block=blk, n_force=n_force, want_mask=True, want_density=True)
    torch.cuda.synchronize()
    return O.cpu(), mask, dens.cpu()


def _host(arrays, dtype, pinned):
    out = []
    for a in arrays:
        t = torch.from_numpy(np.ascontiguousarray(a)).to(dtype)
        out.append(t.pin_memory() if pinned else t)
    return out


@pytest.mark.parametrize("dtype,B,H,L,d,blk,n_force", [
    ("bf16", 2, 3, 1000, 128, 128, 0),
    ("bf16", 2, 3, 1000, 64, 128, 2),
    ("bf16", 1, 3, 77, 128, 128, 0),
    ("f32", 1, 3, 700, 64, 64, 1),
])
@pytest.mark.parametrize("chunk", [1, 2, 3, 5])
@pytest.mark.parametrize("pinned", [True, False])
def test_host_path_equals_device_path(dtype, B, H, L, d, blk, n_force, chunk, pinned):
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    Qh, Kh, Vh = local_inputs(B, H, L, d, seed=L + d + chunk, dtype=dtype)
    tau = [0.0, 1.5, math.inf]
    Qc, Kc, Vc = _host((Qh, Kh, Vh), tdt, pinned)
    O_dev, mask, dens_dev = _device_path(Qc, Kc, Vc, tau, blk, n_force)
    O, dens = sa.sol_attn_fwd_host(Qc, Kc, Vc, tau, block=blk, n_force=n_force, heads_per_chunk=chunk,
                                   want_density=True)
    assert O.device.type == "cpu" and O.is_pinned() == pinned
    assert torch.equal(O, O_dev)
    assert torch.equal(dens, dens_dev)
    if dtype == "bf16" and chunk == 2 and pinned and L == 1000 and d == 128:
        st = full_compare(Qh, Kh, Vh, O, mask, tau, blk, n_force=n_force)
        check_bf16(st)


def test_host_path_reuses_a_given_scratch_and_output():
    Qh, Kh, Vh = local_inputs(1, 4, 1500, 128, seed=3)
    Qc, Kc, Vc = _host((Qh, Kh, Vh), torch.bfloat16, True)
    tau = [0.2, 0.7, 1.1, 0.0]
    n = sa.sol_attn_fwd_host_scratch_bytes(torch.bfloat16, 1, 4, 1500, 128, 128, 3)
    scratch = torch.full((n,), 0xAB, dtype=torch.uint8, device="cuda")  # no zeroing needed
    O = torch.empty_like(Qc).pin_memory()
    first, _ = sa.sol_attn_fwd_host(Qc, Kc, Vc, tau, heads_per_chunk=3, O=O, scratch=scratch)
    assert first.data_ptr() == O.data_ptr()
    ref = O.clone()
    again, _ = sa.sol_attn_fwd_host(Qc, Kc, Vc, tau, heads_per_chunk=3, O=O, scratch=scratch)
    assert torch.equal(again, ref)
    O_dev, _, _ = _device_path(Qc, Kc, Vc, tau, 128, 0)
    assert torch.equal(ref, O_dev)


def test_host_path_full_sequence_length_of_the_720p_workload():
    """L = 75,600 tokens (591 key blocks), d = 128, four heads of the benchmark's inputs at its
    calibrated 20 % thresholds, two heads per chunk: equal to the device path bit for bit."""
    w = wl.WORKLOADS["video720p_L75600"]
    heads = range(4)
    arrs = [wl.head_tensors(w, 0, h) for h in heads]
    Qh, Kh, Vh = (np.stack([a[i] for a in arrs])[None] for i in range(3))
    tau = taus(w, "0.2")[:4]
    Qc, Kc, Vc = _host((Qh, Kh, Vh), torch.bfloat16, True)
    O_dev, _, dens_dev = _device_path(Qc, Kc, Vc, tau, w.block, w.n_force)
    O, dens = sa.sol_attn_fwd_host(Qc, Kc, Vc, tau, block=w.block, n_force=w.n_force, heads_per_chunk=2,
                                   want_density=True)
    assert torch.equal(O, O_dev) and torch.equal(dens, dens_dev)
    assert 0.1 < float(dens.mean()) < 0.3


def test_host_path_reports_an_expired_wait_and_recovers():
    Qh, Kh, Vh = local_inputs(1, 2, 3000, 128, seed=9)
    Qc, Kc, Vc = _host((Qh, Kh, Vh), torch.bfloat16, True)
    tau = [0.5, 1.0]
    sa.sol_attn_debug_drop_one_load(1)  # the first chunk's fused launch skips one K tile
    with pytest.raises(sa.SolAttnError) as e:
        sa.sol_attn_fwd_host(Qc, Kc, Vc, tau, heads_per_chunk=1)
    assert e.value.status == sa.SOL_ETIMEOUT
    O, _ = sa.sol_attn_fwd_host(Qc, Kc, Vc, tau, heads_per_chunk=1)
    O_dev, _, _ = _device_path(Qc, Kc, Vc, tau, 128, 0)
    assert torch.equal(O, O_dev)
