"""Context-parallel Sol-Attn over several GPUs: sequence-sharded inputs, head-sharded attention.

The Sol-Engine README ("To-do", the MiniMax-H3 entry) deploys Sol-Attn together with context
parallelism: the attention of one long video sequence runs on several GPUs, each holding a
contiguous range of the tokens. Routing needs every key block of a head (the threshold is
relative to the maximum proxy score over all of them), and so do the exact tiles a query block
keeps. This module makes every head whole on one rank:

1. one all-to-all per tensor turns each rank's token range of all H heads into the full sequence
   of a contiguous group of heads (about H / world of them);
2. the single-GPU path (pooling, routing pass, fused forward) runs unchanged on those heads, so
   each head's output equals the single-GPU output bit for bit;
3. one all-to-all turns the output back into each rank's token range of all heads.

Every rank sends (world - 1) / world of its Q, K, V shard out and receives as much, and the
same again for O. The collectives are torch.distributed's (NCCL over NVLink on GPUs; gloo
in the CPU tests). Each rank's token range may have any length; head groups differ in size by
at most one head, and a rank with no head (world > H) only forwards data. Optionally the heads
go in chunks, so that one chunk's exchange overlaps another chunk's compute. Before any
exchange, every rank checks every rank's shapes, so a bad call raises on all ranks together
rather than leaving some waiting in a collective.
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


def _gather_meta(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, n_tau: int, group) -> List[List[int]]:
    """The shapes of Q, K and V and the number of thresholds of every rank, on every rank."""
    world = dist.get_world_size(group)
    mine = torch.tensor(list(Q.shape) + list(K.shape) + list(V.shape) + [n_tau], dtype=torch.int64,
                        device=Q.device)
    allm = [torch.empty_like(mine) for _ in range(world)]
    dist.all_gather(allm, mine, group=group)
    return [[int(v) for v in m.tolist()] for m in allm]


def _seq_to_heads_start(x: torch.Tensor, lens: Sequence[int], ranges: Sequence[Tuple[int, int]], rank: int, group):
    """Start the all-to-all that turns [B, H, L_rank, d] into [B, h1 - h0, L, d] for this rank's
    head range; returns a function that waits for it and assembles the result."""
    B, _, Lr, d = x.shape
    send = torch.cat([x[:, a:b].reshape(-1) for a, b in ranges])
    in_splits = [B * (b - a) * Lr * d for a, b in ranges]
    hc = ranges[rank][1] - ranges[rank][0]
    out_splits = [B * hc * n * d for n in lens]
    recv = torch.empty(sum(out_splits), dtype=x.dtype, device=x.device)
    work = dist.all_to_all_single(recv, send, output_split_sizes=out_splits, input_split_sizes=in_splits,
                                  group=group, async_op=True)

    def finish(_send=send) -> torch.Tensor:  # _send keeps the send buffer alive until the exchange ends
        work.wait()
        parts = [t.view(B, hc, n, d) for t, n in zip(recv.split(out_splits), lens)]
        return torch.cat(parts, dim=2)
    return finish


def _heads_to_seq_start(o: torch.Tensor, lens: Sequence[int], ranges: Sequence[Tuple[int, int]], rank: int, group):
    """Start the inverse exchange: [B, h1 - h0, L, d] of this rank's head range out, this rank's
    token range of every rank's head range in. The returned function waits and gives one
    [B, b - a, L_rank, d] piece per rank, in rank order."""
    B, hc, _, d = o.shape
    offs = [0]
    for n in lens:
        offs.append(offs[-1] + n)
    send = torch.cat([o[:, :, offs[s]:offs[s + 1]].reshape(-1) for s in range(len(lens))])
    in_splits = [B * hc * n * d for n in lens]
    Lr = lens[rank]
    out_splits = [B * (b - a) * Lr * d for a, b in ranges]
    recv = torch.empty(sum(out_splits), dtype=o.dtype, device=o.device)
    work = dist.all_to_all_single(recv, send, output_split_sizes=out_splits, input_split_sizes=in_splits,
                                  group=group, async_op=True)

    def finish(_send=send) -> List[torch.Tensor]:
        work.wait()
        return [t.view(B, b - a, Lr, d) for t, (a, b) in zip(recv.split(out_splits), ranges)]
    return finish


def seq_to_heads(x: torch.Tensor, lens: Sequence[int], groups: Sequence[Tuple[int, int]], rank: int,
                 group=None) -> torch.Tensor:
    """[B, H, L_rank, d] token range of all heads -> [B, h1 - h0, L, d] whole sequence of this
    rank's head group (token ranges concatenated in rank order)."""
    return _seq_to_heads_start(x, lens, groups, rank, group)()


def heads_to_seq(o: torch.Tensor, lens: Sequence[int], groups: Sequence[Tuple[int, int]], rank: int,
                 group=None) -> torch.Tensor:
    """Inverse of seq_to_heads: [B, h1 - h0, L, d] of this rank's heads -> [B, H, L_rank, d]."""
    return torch.cat(_heads_to_seq_start(o, lens, groups, rank, group)(), dim=1)


def _cuda_path(Q, K, V, tau, block, n_force):
    from . import sol_attn as sa
    O, _, _ = sa.sol_attn(Q, K, V, tau, block=block, n_force=n_force)
    return O


def sol_attn_context_parallel(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, tau: Sequence[float],
                              block: int = 128, n_force: int = 0, group=None,
                              attn: Optional[Callable] = None, heads_per_chunk: Optional[int] = None) -> torch.Tensor:
    """Sol-Attn forward of one sequence sharded over the ranks of `group` by tokens.

    Q, K, V: this rank's contiguous token range [B, H, L_rank, d] (ranges in rank order make up
    the sequence; any lengths). tau: H thresholds (the same on every rank). n_force counts key
    blocks of the whole sequence. Returns this rank's token range of O, [B, H, L_rank, d].

    `attn(Q, K, V, tau, block, n_force) -> O` computes one rank's whole-sequence heads; the
    default is the library's CUDA path (pooling + fused forward).

    heads_per_chunk: None exchanges and computes each rank's whole head group at once. A number c
    cuts every group into chunks of c heads and pipelines them: the exchange of chunk k+1 is in
    flight while chunk k is computed, and chunk k's output travels back while chunk k+1 is
    computed. Every rank runs the same number of chunks (set by the largest group), so all ranks
    issue the same collectives in the same order; a rank whose group has run out of heads
    sends and computes empty chunks.
    """
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    tau = [float(t) for t in tau]
    meta = _gather_meta(Q, K, V, len(tau), group)
    B, H, _, d = meta[0][:4]
    # every rank checks every rank's arguments, so a bad call fails on all of them at this point
    for m in meta:
        qs, ks, vs, n_tau = m[0:4], m[4:8], m[8:12], m[12]
        if ks != qs or vs != qs:
            raise ValueError(f"Q, K and V differ in shape on some rank: {meta}")
        if qs[0] != B or qs[1] != H or qs[3] != d:
            raise ValueError(f"ranks disagree on (B, H, d): {[tuple(x[i] for i in (0, 1, 3)) for x in meta]}")
        if n_tau != H:
            raise ValueError(f"every rank must pass H={H} thresholds: {[x[12] for x in meta]}")
    if heads_per_chunk is not None and heads_per_chunk < 1:
        raise ValueError("heads_per_chunk must be >= 1")
    lens = [m[2] for m in meta]
    groups = head_groups(H, world)
    gmax = max(b - a for a, b in groups)
    c = gmax if heads_per_chunk is None else heads_per_chunk
    n_chunks = max(1, -(-gmax // max(c, 1)))

    def ranges(k):
        return [(min(a + k * c, b), min(a + (k + 1) * c, b)) for a, b in groups]

    run = attn or _cuda_path
    xs = [x.contiguous() for x in (Q, K, V)]
    inflight = [_seq_to_heads_start(x, lens, ranges(0), rank, group) for x in xs]
    returning = []
    for k in range(n_chunks):
        nxt = [_seq_to_heads_start(x, lens, ranges(k + 1), rank, group) for x in xs] if k + 1 < n_chunks else None
        Qh, Kh, Vh = (f() for f in inflight)
        a, b = ranges(k)[rank]
        if b > a:
            Oh = run(Qh, Kh, Vh, tau[a:b], block, n_force)
        else:
            Oh = torch.empty((B, 0, sum(lens), d), dtype=Q.dtype, device=Q.device)
        returning.append((ranges(k), _heads_to_seq_start(Oh.contiguous(), lens, ranges(k), rank, group)))
        inflight = nxt
    out = torch.empty((B, H, lens[rank], d), dtype=Q.dtype, device=Q.device)
    for rg, finish in returning:
        for (a, b), piece in zip(rg, finish()):
            if b > a:
                out[:, a:b] = piece
    return out
