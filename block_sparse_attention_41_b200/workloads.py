"""Seeded synthetic inputs shaped like the video-DiT attention workloads of the Sol-Attn pages.

This module only draws tensors. It holds no step of the attention method (no pooling, no
scores, no softmax), so both the CPU oracle and the CUDA library can take their inputs from it.

Recipe (identical for every consumer):

* One NumPy PCG64 stream per (workload seed, batch b, head h, tensor id), built directly from
  ``SeedSequence(seed, spawn_key=(b, h, tensor_id))``. Draws are float64 N(0, 1).
* Positional feature of channel c at video grid position (t, y, x):
  axis = c mod 3 picks t, y or x; frequency = (1/4, 1/8, 1/16)[(c div 3) mod 3];
  the function is sin when (c div 9) is even, cos otherwise; feat = fn(2*pi*f*pos).
  Token order is row-major over (t, y, x) with x fastest.
* Q = N + s*feat, K = N' + s*feat (same feature, independent noise), V = N''.
* Sinks: ``n_sinks`` seeded video positions per (b, h) get ``sink_boost`` added to every key
  channel (a key aligned with the all-ones direction, 4 sigma per channel).
* Joint text+video workloads prepend ``n_text`` text tokens drawn N(0, 1) per batch entry with
  no positional feature; the video part is drawn once and shared by every batch entry
  (a classifier-free-guidance pair differs only in its text tokens).
* Rounding: float64 -> float32 (round to nearest even) and, for bf16 workloads, float32 -> bf16
  (round to nearest even). Returned arrays are float32 holding exactly representable values.

The workloads stand in for the pages' real-model shapes: the Sol-Engine README lists
Wan2.1 at 720x1280, 81 frames and LTX at 1088x1920; the grids below are those videos after
a 4x temporal / 16x spatial token compression (an inference, not stated on the pages).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

# tensor ids inside one (seed, b, h) family of streams
_TID_Q, _TID_K, _TID_V, _TID_SINK = 0, 1, 2, 3
_TID_TEXT_Q, _TID_TEXT_K, _TID_TEXT_V = 4, 5, 6
_TID_DENSITY = 7  # per-head target density draw (joint text+video workload)


@dataclass(frozen=True)
class Workload:
    """One synthetic attention problem: shapes, dtype, seed and the routing targets."""

    name: str
    B: int
    H: int
    d: int
    grid: tuple  # (T, Y, X) video token grid
    block: int  # B_q = B_k
    dtype: str  # "f32" or "bf16"
    seed: int
    pos_scale: float
    n_text: int = 0
    n_sinks: int = 0
    sink_boost: float = 4.0
    n_force: int = 0  # leading key blocks that are always kept (text blocks)
    # routing targets: either fixed thresholds broadcast to all heads, or target densities
    taus: tuple = ()
    densities: tuple = ()
    per_head_density: tuple = ()  # (lo, hi) for a seeded uniform draw per head
    description: str = ""

    @property
    def n_video(self) -> int:
        T, Y, X = self.grid
        return T * Y * X

    @property
    def L(self) -> int:
        return self.n_text + self.n_video

    @property
    def n_blocks(self) -> int:
        return -(-self.L // self.block)


WORKLOADS = {
    w.name: w
    for w in [
        Workload(
            name="tiny_f32_L1024",
            B=1, H=2, d=64, grid=(4, 16, 16), block=64, dtype="f32", seed=0, pos_scale=2.0,
            taus=(math.inf, 2.0, 0.5),
            description="tiny oracle case, fp32, tau in {inf, 2.0, 0.5}",
        ),
        Workload(
            name="small_dit_L8192",
            B=1, H=12, d=64, grid=(8, 32, 32), block=128, dtype="bf16", seed=1, pos_scale=2.0,
            densities=(0.25,),
            description="small video DiT layer, bf16, ~25% kept blocks per head",
        ),
        Workload(
            name="video720p_L75600",
            B=1, H=40, d=128, grid=(21, 45, 80), block=128, dtype="bf16", seed=2, pos_scale=3.0,
            n_sinks=8, densities=(0.10, 0.20, 0.40, 1.0),
            description="720p-like long video, bf16, density sweep 10/20/40/100%",
        ),
        Workload(
            name="video1080p_L252960",
            B=1, H=40, d=128, grid=(31, 68, 120), block=128, dtype="bf16", seed=3, pos_scale=3.0,
            n_sinks=8, densities=(0.15,),
            description="1080p-like very long sequence, bf16, ~15% density",
        ),
        Workload(
            name="text_video_cfg_L33272",
            B=2, H=32, d=128, grid=(13, 42, 60), block=128, dtype="bf16", seed=4, pos_scale=3.0,
            n_text=512, n_sinks=8, n_force=4, per_head_density=(0.05, 0.50),
            description="joint text+video with a CFG pair, text blocks forced, per-head density 5-50%",
        ),
    ]
}


def _rng(seed: int, b: int, h: int, tid: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(seed, spawn_key=(b, h, tid))))


_FEATURE_CACHE: dict = {}


def positional_feature(grid: tuple, d: int) -> np.ndarray:
    """float64 [T*Y*X, d] sinusoidal 3-D positional feature (recipe in the module docstring)."""
    key = (tuple(grid), d)
    if key in _FEATURE_CACHE:
        return _FEATURE_CACHE[key]
    T, Y, X = grid
    n = T * Y * X
    tok = np.arange(n)
    pos = np.stack([tok // (Y * X), (tok // X) % Y, tok % X], axis=1).astype(np.float64)  # [n, 3]
    freqs = np.array([1.0 / 4, 1.0 / 8, 1.0 / 16])
    feat = np.empty((n, d), dtype=np.float64)
    for c in range(d):
        arg = 2.0 * math.pi * freqs[(c // 3) % 3] * pos[:, c % 3]
        feat[:, c] = np.sin(arg) if (c // 9) % 2 == 0 else np.cos(arg)
    _FEATURE_CACHE.clear()
    _FEATURE_CACHE[key] = feat
    return feat


def rope_tables(grid: tuple, d: int, base: float = 10000.0):
    """cos, sin float32 [T*Y*X, d/2] of 3-D rotary angles for the QK-norm + RoPE step's inputs.

    The d/2 interleaved pairs are split over the axes (t, y, x): n_y = n_x = (d/2) // 3 pairs, the
    rest to t. Pair j of an axis with n pairs turns by pos_axis * base^(-j/n). Tokens run
    row-major over the grid, x fastest. These are inputs handed to the kernel and to the oracle.
    """
    T, Y, X = grid
    n = T * Y * X
    tok = np.arange(n)
    pos = np.stack([tok // (Y * X), (tok // X) % Y, tok % X], axis=1).astype(np.float64)
    half = d // 2
    ny = half // 3
    counts = (half - 2 * ny, ny, ny)
    ang = np.empty((n, half), dtype=np.float64)
    col = 0
    for axis, cnt in enumerate(counts):
        theta = base ** (-np.arange(cnt, dtype=np.float64) / cnt)
        ang[:, col:col + cnt] = pos[:, axis:axis + 1] * theta[None, :]
        col += cnt
    return np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)


def qk_norm_gains(d: int, seed: int):
    """Seeded RMS-norm gains (float32 [d] each) for queries and keys: 1 + N(0, 0.1^2)."""
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence(seed, spawn_key=(99,))))
    return tuple((1.0 + 0.1 * rng.standard_normal(d)).astype(np.float32) for _ in range(2))


def round_to_bf16(x) -> np.ndarray:
    """float -> float32 (nearest even) -> bf16 (nearest even); returned as float32 values."""
    x32 = np.ascontiguousarray(x, dtype=np.float32)
    u = x32.view(np.uint32).astype(np.uint64)
    u = (u + (((u >> 16) & 1) + 0x7FFF)) >> 16
    return (u << 16).astype(np.uint32).view(np.float32)


def head_tensors(w: Workload, b: int, h: int):
    """Q, K, V of one (batch, head) as float32 [L, d] arrays exactly representable in w.dtype."""
    d = w.d
    vb = 0 if w.n_text else b  # video part is shared by the CFG pair
    feat = positional_feature(w.grid, d)
    nv = w.n_video
    q = _rng(w.seed, vb, h, _TID_Q).standard_normal((nv, d)) + w.pos_scale * feat
    k = _rng(w.seed, vb, h, _TID_K).standard_normal((nv, d)) + w.pos_scale * feat
    v = _rng(w.seed, vb, h, _TID_V).standard_normal((nv, d))
    if w.n_sinks:
        pos = _rng(w.seed, vb, h, _TID_SINK).choice(nv, size=w.n_sinks, replace=False)
        k[pos] += w.sink_boost
    if w.n_text:
        tq = _rng(w.seed, b, h, _TID_TEXT_Q).standard_normal((w.n_text, d))
        tk = _rng(w.seed, b, h, _TID_TEXT_K).standard_normal((w.n_text, d))
        tv = _rng(w.seed, b, h, _TID_TEXT_V).standard_normal((w.n_text, d))
        q = np.concatenate([tq, q])
        k = np.concatenate([tk, k])
        v = np.concatenate([tv, v])
    rnd = round_to_bf16 if w.dtype == "bf16" else (lambda a: np.ascontiguousarray(a, dtype=np.float32))
    return rnd(q), rnd(k), rnd(v)


def target_densities(w: Workload) -> np.ndarray:
    """Per-head target kept-block densities for workloads drawn per head (seeded uniform)."""
    lo, hi = w.per_head_density
    return _rng(w.seed, 0, 0, _TID_DENSITY).uniform(lo, hi, size=w.H)


def _head_job(args):
    name, b, h = args
    return b, h, head_tensors(WORKLOADS[name], b, h)


def all_tensors(w: Workload, heads=None, workers: int = 0):
    """Q, K, V as float32 [B, H, L, d] (or only the listed (b, h) pairs, others zero).

    ``workers > 1`` draws heads in a spawn-started process pool (safe after CUDA is initialised).
    """
    pairs = [(b, h) for b in range(w.B) for h in range(w.H)] if heads is None else list(heads)
    out = [np.zeros((w.B, w.H, w.L, w.d), dtype=np.float32) for _ in range(3)]
    jobs = [(w.name, b, h) for (b, h) in pairs]
    if workers and workers > 1 and len(jobs) > 1:
        import multiprocessing as mp
        from concurrent.futures import ProcessPoolExecutor

        with ProcessPoolExecutor(max_workers=workers, mp_context=mp.get_context("spawn")) as ex:
            for b, h, qkv in ex.map(_head_job, jobs):
                for t in range(3):
                    out[t][b, h] = qkv[t]
    else:
        for job in jobs:
            b, h, qkv = _head_job(job)
            for t in range(3):
                out[t][b, h] = qkv[t]
    return out


def sample_units(w: Workload, count: int, seed_offset: int = 0):
    """Seeded sample of distinct (b, h, query_block) units, sorted."""
    total = w.B * w.H * w.n_blocks
    rng = _rng(w.seed, 1000 + seed_offset, 0, 0)
    idx = np.sort(rng.choice(total, size=min(count, total), replace=False))
    return [(int(u // (w.H * w.n_blocks)), int((u // w.n_blocks) % w.H), int(u % w.n_blocks)) for u in idx]
