"""Shared helpers of the GPU parity tests: device inputs from the seeded generator, the tau table,
and the comparison of the CUDA path's outputs with the float64 oracle.

The oracle side regenerates each needed head from the seeded generator inside a spawn-started
worker process. So no oracle input comes from device memory, and host memory stays bounded on
the longest workload.
"""
from __future__ import annotations

import json
import math
import multiprocessing as mp
import os
from concurrent.futures import ProcessPoolExecutor

import numpy as np
import torch

import oracle
from block_sparse_attention_41_b200 import workloads as wl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
TOL_BF16_MAX, TOL_BF16_MEAN = 2e-2, 2e-3  # bf16 inputs, fp32 accumulation
TOL_F32_MAX = 1e-4                         # fp32 inputs


def tau_table():
    with open(os.path.join(ROOT, "tests", "golden", "tau.json")) as f:
        return json.load(f)["workloads"]


def taus(w: wl.Workload, key: str):
    vals = tau_table()[w.name][key]["tau"]
    return [math.inf if v == "inf" else float(v) for v in vals]


def _pool(workers):
    os.environ.setdefault("OPENBLAS_NUM_THREADS", "1")
    os.environ.setdefault("OMP_NUM_THREADS", "1")
    os.environ.setdefault("MKL_NUM_THREADS", "1")
    return ProcessPoolExecutor(max_workers=workers, mp_context=mp.get_context("spawn"))


def _workers(n_jobs):
    return max(1, min(n_jobs, os.cpu_count() or 1, 32))


def _gen_job(args):
    name, b, h = args
    return b, h, wl.head_tensors(wl.WORKLOADS[name], b, h)


def device_inputs(w: wl.Workload, device="cuda"):
    """Q, K, V on the device in the workload's dtype, filled head by head from the generator."""
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    shape = (w.B, w.H, w.L, w.d)
    Q, K, V = (torch.empty(shape, dtype=dt, device=device) for _ in range(3))
    jobs = [(w.name, b, h) for b in range(w.B) for h in range(w.H)]
    with _pool(_workers(len(jobs))) as ex:
        for b, h, qkv in ex.map(_gen_job, jobs):
            for T, a in zip((Q, K, V), qkv):
                T[b, h].copy_(torch.from_numpy(a).to(dt))
    return Q, K, V


def _oracle_job(args):
    """Worker: regenerate one head, run the oracle on its units with the GPU's band decisions."""
    name, b, h, tau, n_force, qbs, gpu_mask_rows = args
    w = wl.WORKLOADS[name]
    q, k, v = wl.head_tensors(w, b, h)
    nkb = w.n_blocks
    override = np.zeros((nkb, nkb), dtype=bool)
    for i, row in zip(qbs, gpu_mask_rows):
        override[i] = row
    O, keep, sbar, M = oracle.forward_head(q, k, v, tau, w.block, w.block, n_force, units=qbs,
                                           keep_override=override)
    band = oracle.band_mask(sbar, M, tau, n_force)
    eps = oracle.proxy_error_bound(q, k, w.block, w.block, units=qbs)
    viol = oracle.routing_violations(sbar[qbs], M[qbs], tau, override[qbs], eps[qbs], n_force)
    out = []
    for i in qbs:
        rows = slice(i * w.block, min((i + 1) * w.block, w.L))
        out.append((i, O[rows], keep[i], band[i]))
    return b, h, out, viol


def merge_violations(total, v):
    for key, n in v.items():
        total[key] = total.get(key, 0) + n
    return total


def compare_units(w, tau, units, O_gpu, mask_gpu, n_force=0):
    """Oracle vs CUDA path on the listed (b, h, i) units. The mask is compared bit for bit outside
    the near-threshold band, and every mask row must be a kept set that a float32 evaluation of the
    routing could produce (oracle.routing_violations: forced blocks kept, the argmax kept, the kept
    set closed upward in the score up to the float32 error bound). O is compared after the oracle
    adopts the GPU's decision for band entries. Returns a dict of error statistics."""
    blk = w.block
    by_head = {}
    for b, h, i in units:
        by_head.setdefault((b, h), []).append(i)
    mask_host = mask_gpu.cpu().numpy().astype(bool)
    jobs = [(w.name, b, h, float(tau[h]), n_force, sorted(qbs), [mask_host[b, h, i] for i in sorted(qbs)])
            for (b, h), qbs in sorted(by_head.items())]
    max_err, sum_err, count, band_total, mism = 0.0, 0.0, 0, 0, 0
    viol = {}
    with _pool(_workers(len(jobs))) as ex:
        for b, h, res, v in ex.map(_oracle_job, jobs):
            merge_violations(viol, v)
            for i, O_ref, keep_ref, band in res:
                g = mask_host[b, h, i]
                mism += int((g[~band] != keep_ref[~band]).sum())
                band_total += int(band.sum())
                rows = slice(i * blk, min((i + 1) * blk, w.L))
                err = np.abs(O_gpu[b, h, rows].double().cpu().numpy() - O_ref)
                max_err = max(max_err, float(err.max()))
                sum_err += float(err.sum())
                count += err.size
    return {"max_abs": max_err, "mean_abs": sum_err / max(count, 1), "mask_mismatch_outside_band": mism,
            "band_entries": band_total, "units": len(units), "routing_violations": viol}


def run_path(Q, K, V, tau, block, n_force=0):
    """The whole CUDA path through the C ABI (pool + fused forward) with mask and density."""
    from block_sparse_attention_41_b200 import sol_attn as sa
    O, mask, dens = sa.sol_attn(Q, K, V, tau, block=block, n_force=n_force, want_mask=True, want_density=True)
    torch.cuda.synchronize()
    return O, mask, dens
