"""Context-parallel layer on CPU: gloo process groups of 2 to 4 ranks, the float64 oracle standing in
for the per-rank attention call.

Each rank holds a token range of Q, K, V for all heads. After the all-to-all, the oracle runs on
that rank's whole-sequence heads, and the output returns to the token ranges. Every head is then
computed by the same float64 code on the same values as a single-process oracle run, so the
gathered output must equal that run exactly. The cases cover ragged ranges (one of them empty),
uneven head groups (one rank without a head), forced blocks and a shape mismatch that every rank
must report.
"""
import math
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from block_sparse_attention_41_b200 import context_parallel as cp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(B, H, L, d, seed):
    rng = np.random.default_rng(seed)
    t = np.arange(L)[:, None] / 30.0
    feat = np.sin(t * (1 + np.arange(d)[None, :] % 4))
    Q = rng.standard_normal((B, H, L, d)) + 2.0 * feat
    K = rng.standard_normal((B, H, L, d)) + 2.0 * feat
    V = rng.standard_normal((B, H, L, d))
    return Q, K, V


def _oracle_attn(Q, K, V, tau, block, n_force):
    O, _, _ = oracle.forward(Q.numpy(), K.numpy(), V.numpy(), tau, block, block, n_force)
    return torch.from_numpy(O)


def _rank(rank, world, port, case, mismatch, out, chunk=None):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        B, H, L, d, blk, n_force, lens, tau, seed = case
        Q, K, V = (torch.from_numpy(x) for x in _inputs(B, H, L, d, seed))
        a = sum(lens[:rank])
        sl = slice(a, a + lens[rank])
        Hr = H - 1 if mismatch == "heads" and rank == 1 else H
        q, k, v = (x[:, :Hr, sl].contiguous() for x in (Q, K, V))
        if mismatch == "k_shape" and rank == 1:
            k = k[:, :, : max(0, k.shape[2] - 1)].contiguous()
        try:
            o = cp.sol_attn_context_parallel(q, k, v, tau[:Hr], block=blk, n_force=n_force, attn=_oracle_attn,
                                             heads_per_chunk=chunk)
            out[rank] = o.numpy()
        except ValueError as e:
            out[rank] = f"ValueError: {e}"
    finally:
        dist.destroy_process_group()


def _run(world, case, mismatch=None, chunk=None):
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_rank, args=(world, _free_port(), case, mismatch, out, chunk), nprocs=world, join=True)
    return dict(out)


def test_head_groups_and_sequence_ranges():
    assert cp.head_groups(5, 2) == [(0, 3), (3, 5)]
    assert cp.head_groups(3, 4) == [(0, 1), (1, 2), (2, 3), (3, 3)]
    assert cp.head_groups(40, 8) == [(5 * g, 5 * g + 5) for g in range(8)]
    # 700 tokens in blocks of 64: 11 blocks as 4 + 4 + 3, the last range ends at the ragged tail
    assert cp.seq_shard_ranges(700, 3, 64) == [(0, 256), (256, 512), (512, 700)]
    assert cp.seq_shard_ranges(75600, 8, 128)[-1] == (518 * 128, 75600)  # 591 blocks = 7 x 74 + 73
    assert cp.seq_shard_ranges(100, 4, 64) == [(0, 64), (64, 100), (100, 100), (100, 100)]


@pytest.mark.parametrize("world,H,lens,n_force,chunk", [
    (2, 5, [300, 400], 0, None),
    (3, 5, [128, 250, 322], 2, None),
    (4, 3, [100, 0, 350, 250], 1, None),  # an empty token range, and a rank without a head
    (2, 5, [300, 400], 0, 1),             # groups of 3 and 2 heads in 3 pipelined chunks
    (3, 5, [128, 250, 322], 1, 1),        # the third rank's group runs out after one chunk
    (2, 5, [350, 350], 0, 2),             # chunks of 2 and 1 heads
])
def test_context_parallel_equals_the_single_process_oracle(world, H, lens, n_force, chunk):
    B, d, blk = 1, 16, 64
    L = sum(lens)
    tau = [0.0, 0.7, math.inf, 1.3, 0.2][:H]
    case = (B, H, L, d, blk, n_force, lens, tau, 17 + world)
    got = _run(world, case, chunk=chunk)
    Q, K, V = _inputs(B, H, L, d, 17 + world)
    ref, keep, _ = oracle.forward(Q, K, V, tau, blk, blk, n_force)
    assert not keep.all()  # the thresholds skip blocks, so the correction takes part
    full = np.concatenate([got[r] for r in range(world)], axis=2)
    assert full.shape == ref.shape
    assert np.array_equal(full, ref)


@pytest.mark.parametrize("mismatch", ["heads", "k_shape"])
def test_shape_mismatch_is_reported_on_every_rank(mismatch):
    # rank 1 passes one head fewer, or a K shorter than its Q: every rank sees the gathered shapes
    # and raises before any exchange, so none is left waiting in a collective
    case = (1, 4, 700, 16, 64, 0, [300, 400], [0.5] * 4, 3)
    got = _run(2, case, mismatch=mismatch)
    assert all(isinstance(got[r], str) and got[r].startswith("ValueError") for r in range(2)), got


def test_default_attention_is_the_cuda_path_with_no_cpu_fallback():
    # one gloo rank, CPU tensors: the exchange works, and the default attention call refuses them
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("gloo", rank=0, world_size=1)
    try:
        x = torch.zeros(1, 2, 64, 16)
        with pytest.raises(TypeError, match="CUDA tensor"):
            cp.sol_attn_context_parallel(x, x, x, [0.5, 0.5], block=64)
    finally:
        dist.destroy_process_group()
