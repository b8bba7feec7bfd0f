"""Context-parallel layer on one GPU: a world-size-1 NCCL group, the default CUDA attention path.

The CPU tests run the layer over gloo groups of 2 to 4 ranks with the float64 oracle as the
per-rank attention. Here the same code runs with its default attention, the library's CUDA path
(pooling, routing pass, fused forward), through NCCL collectives on a single rank. So the
exchange is a local all-to-all and the computed heads are the whole sequence. Checks:
  * the output equals the single-GPU call bit for bit, unchunked and in head chunks;
  * it matches the float64 oracle within the bf16 parity tolerances, on a ragged length with
    forced blocks, with every mask row a valid kept set.
More than one rank is not run here: every call in this environment holds one GPU.
"""
import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

from block_sparse_attention_41_b200 import context_parallel as cp
from block_sparse_attention_41_b200 import sol_attn as sa

from test_parity_gpu import check_bf16, full_compare, local_inputs, report

pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.fixture(scope="module")
def nccl_group():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from block_sparse_attention_41_b200 import build
    build.build()
    sa.load_library()
    torch.cuda.set_device(0)
    os.environ.setdefault("NCCL_NVLS_ENABLE", "0")
    import datetime
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60), device_id=torch.device("cuda", 0))
    yield dist.group.WORLD
    dist.destroy_process_group()


@pytest.mark.parametrize("chunk", [None, 1, 2])
def test_world_one_nccl_equals_single_gpu_and_oracle(nccl_group, chunk):
    B, H, L, d, blk, n_force = 1, 3, 2_561, 128, 128, 2
    Qh, Kh, Vh = local_inputs(B, H, L, d, seed=77)
    Q, K, V = (torch.from_numpy(x).to(torch.bfloat16).cuda() for x in (Qh, Kh, Vh))
    tau = [0.0, 0.9, math.inf]
    O = cp.sol_attn_context_parallel(Q, K, V, tau, block=blk, n_force=n_force, group=nccl_group,
                                     heads_per_chunk=chunk)
    torch.cuda.synchronize()
    ref, mask, _ = sa.sol_attn(Q, K, V, tau, block=blk, n_force=n_force, want_mask=True)
    torch.cuda.synchronize()
    assert torch.equal(O, ref)
    st = full_compare(Qh, Kh, Vh, O, mask, tau, blk, n_force=n_force)
    report(f"context parallel world=1 chunk={chunk}", st)
    check_bf16(st)
    assert np.isfinite(O.float().cpu().numpy()).all()
