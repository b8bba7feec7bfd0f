"""Context-parallel Sol-Attn over several GPUs: sequence-sharded inputs, head-sharded attention.

The Sol-Engine README ("To-do", the MiniMax-H3 entry) deploys Sol-Attn together with context
parallelism: the attention of one long video sequence runs on several GPUs, each holding a
contiguous range of the tokens. Routing needs every key block of a head (the threshold is relative to the maximum proxy
score over all of them), and so do the exact tiles a query block keeps. This module makes every
head whole on one rank:

1. one all-to-all per tensor turns each rank's token range of all H heads into the full sequence
   of a contiguous group of heads (about H / world of them);
2. the single-GPU path (pooling, routing pass, fused forward) runs unchanged on those heads, so
   each head's output equals the single-GPU output bit for bit;
3. one all-to-all turns the output back into each rank's token range of all heads.

Every rank sends (world - 1) / world of its Q, K, V shard out and receives as much, and the
same again for O. The collectives are torch.distributed's (NCCL over NVLink on GPUs; gloo
in the CPU tests). Each rank's token range may have any length; head groups differ in size by
at most one head, and a rank with no head (world > H) only forwards data.
"""
from __future__ import annotations

from typing import Callable, List, Optional, Sequence, Tuple

import torch
import torch.distributed as dist


def head_groups(H: int, world: int) -> List[Tuple[int, int]]:
    """Contiguous head ranges [h0, h1) per rank; the first H % world ranks get one head more."""
    q, r = divmod(H, world)
    out, h0 = [], 0
    for g in range(world):
        n = q + (1 if g < r else 0)
        out.append((h0, h0 + n))
        h0 += n
    return out


def seq_shard_ranges(L: int, world: int, block: int) -> List[Tuple[int, int]]:
    """A split of L tokens into `world` contiguous ranges of whole blocks (the last range takes the
    ragged tail); ranges differ in size by at most one block. Any other split works too."""
    nb = -(-L // block)
    q, r = divmod(nb, world)
    out, b0 = [], 0
    for g in range(world):
        n = q + (1 if g < r else 0)
        out.append((min(b0 * block, L), min((b0 + n) * block, L)))
        b0 += n
    return out


def _gather_meta(x: torch.Tensor, group) -> List[List[int]]:
    """(B, H, L_r, d) of every rank, on every rank."""
    world = dist.get_world_size(group)
    mine = torch.tensor(list(x.shape), dtype=torch.int64, device=x.device)
    allm = [torch.empty_like(mine) for _ in range(world)]
    dist.all_gather(allm, mine, group=group)
    return [[int(v) for v in m.tolist()] for m in allm]


def seq_to_heads(x: torch.Tensor, lens: Sequence[int], groups: Sequence[Tuple[int, int]], rank: int,
                 group=None) -> torch.Tensor:
    """[B, H, L_rank, d] token range of all heads -> [B, h1 - h0, L, d] whole sequence of this
    rank's head group (token ranges concatenated in rank order)."""
    B, _, Lr, d = x.shape
    send = torch.cat([x[:, h0:h1].reshape(-1) for h0, h1 in groups])
    in_splits = [B * (h1 - h0) * Lr * d for h0, h1 in groups]
    hg = groups[rank][1] - groups[rank][0]
    out_splits = [B * hg * n * d for n in lens]
    recv = torch.empty(sum(out_splits), dtype=x.dtype, device=x.device)
    dist.all_to_all_single(recv, send, output_split_sizes=out_splits, input_split_sizes=in_splits, group=group)
    parts = [p.view(B, hg, n, d) for p, n in zip(recv.split(out_splits), lens)]
    return torch.cat(parts, dim=2)


def heads_to_seq(o: torch.Tensor, lens: Sequence[int], groups: Sequence[Tuple[int, int]], rank: int,
                 group=None) -> torch.Tensor:
    """Inverse of seq_to_heads: [B, h1 - h0, L, d] of this rank's heads -> [B, H, L_rank, d]."""
    B, hg, _, d = o.shape
    offs = [0]
    for n in lens:
        offs.append(offs[-1] + n)
    send = torch.cat([o[:, :, offs[s]:offs[s + 1]].reshape(-1) for s in range(len(lens))])
    in_splits = [B * hg * n * d for n in lens]
    Lr = lens[rank]
    out_splits = [B * (h1 - h0) * Lr * d for h0, h1 in groups]
    recv = torch.empty(sum(out_splits), dtype=o.dtype, device=o.device)
    dist.all_to_all_single(recv, send, output_split_sizes=out_splits, input_split_sizes=in_splits, group=group)
    parts = [p.view(B, h1 - h0, Lr, d) for p, (h0, h1) in zip(recv.split(out_splits), groups)]
    return torch.cat(parts, dim=1)


def _cuda_path(Q, K, V, tau, block, n_force):
    from . import sol_attn as sa
    O, _, _ = sa.sol_attn(Q, K, V, tau, block=block, n_force=n_force)
    return O


def sol_attn_context_parallel(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, tau: Sequence[float],
                              block: int = 128, n_force: int = 0, group=None,
                              attn: Optional[Callable] = None) -> torch.Tensor:
    """Sol-Attn forward of one sequence sharded over the ranks of `group` by tokens.

    Q, K, V: this rank's contiguous token range [B, H, L_rank, d] (ranges in rank order make up
    the sequence; any lengths). tau: H thresholds (the same on every rank). n_force counts key
    blocks of the whole sequence. Returns this rank's token range of O, [B, H, L_rank, d].

    `attn(Q, K, V, tau, block, n_force) -> O` computes one rank's whole-sequence heads; the
    default is the library's CUDA path (pooling + fused forward).
    """
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    meta = _gather_meta(Q, group)
    B, H, _, d = meta[0]
    # every rank checks the same gathered shapes, so a bad call fails on all of them together
    for m in meta:
        if m[0] != B or m[1] != H or m[3] != d:
            raise ValueError(f"ranks disagree on (B, H, d): {[tuple(x[i] for i in (0, 1, 3)) for x in meta]}")
    if K.shape != Q.shape or V.shape != Q.shape:
        raise ValueError("Q, K and V must have the same shape on each rank")
    tau = [float(t) for t in tau]
    if len(tau) != H:
        raise ValueError(f"tau must hold H={H} values")
    lens = [m[2] for m in meta]
    groups = head_groups(H, world)
    h0, h1 = groups[rank]
    Qh, Kh, Vh = (seq_to_heads(x.contiguous(), lens, groups, rank, group) for x in (Q, K, V))
    if h1 > h0:
        Oh = (attn or _cuda_path)(Qh, Kh, Vh, tau[h0:h1], block, n_force)
    else:
        Oh = torch.empty((B, 0, sum(lens), d), dtype=Q.dtype, device=Q.device)
    return heads_to_seq(Oh.contiguous(), lens, groups, rank, group)
