"""Write tests/golden/tau.json: per-head routing thresholds that give each workload's target
kept-block density. Only the float64 CPU oracle (pooling and proxy scores) and the seeded
input generator are used.

Calibration per head (and per target density D):
  1. Pool every query block and key block of the head, then take every proxy score
     s_bar_ij and each row max M_i.
  2. Collect the gaps g_ij = M_i - s_bar_ij over the non-forced key blocks and sort them.
  3. Non-forced pairs must be kept at rate r = (D - f) / (1 - f), with f = n_force / N_kb.
     Take the gap at rank ceil(r * count) - 1 (0-based).
  4. Set tau to the midpoint between that gap and the next larger distinct gap. A midpoint
     leaves as few entries as possible within the +-1e-3 near-threshold band.
D >= 1 gives tau = +inf (dense). The joint text+video workload draws D per head
(seeded, uniform 5-50%), calibrates on batch entry 0 and shares tau over the batch.

Run:  python tests/golden/make_tau.py [--workers N]
"""
import argparse
import json
import math
import multiprocessing as mp
import os
import sys
from concurrent.futures import ProcessPoolExecutor

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from block_sparse_attention_41_b200 import workloads as wl  # noqa: E402


def head_gaps(name, b, h):
    w = wl.WORKLOADS[name]
    q, k, _ = wl.head_tensors(w, b, h)
    qbar = oracle.pool_blocks(q.astype(np.float64), w.block)
    kbar = oracle.pool_blocks(k.astype(np.float64), w.block)
    sbar = np.stack([oracle.proxy_scores(qbar[i], kbar, w.d) for i in range(qbar.shape[0])])
    M = sbar.max(axis=1)
    gaps = (M[:, None] - sbar)[:, w.n_force:]
    return h, np.sort(gaps.reshape(-1)), sbar, M


def calibrate(gaps_sorted, D, n_force, nkb):
    if D >= 1.0:
        return math.inf
    f = n_force / nkb
    r = (D - f) / (1.0 - f)
    k = max(0, math.ceil(r * gaps_sorted.size) - 1)
    g = gaps_sorted[k]
    larger = gaps_sorted[gaps_sorted > g]
    return float((g + larger[0]) / 2) if larger.size else float(g + 1.0)


def achieved(sbar, M, tau, n_force):
    keep, band = np.zeros_like(sbar, dtype=bool), 0
    for i in range(sbar.shape[0]):
        keep[i], _ = oracle.route(sbar[i], tau, n_force)
    if not math.isinf(tau):
        band = int((oracle.band_mask(sbar, M, tau, n_force)).sum())
    return float(keep.mean()), band


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--workers", type=int, default=os.cpu_count())
    ap.add_argument("--only", default=None)
    args = ap.parse_args()
    out_path = os.path.join(ROOT, "tests", "golden", "tau.json")
    table = {}
    if os.path.exists(out_path):
        with open(out_path) as f:
            table = json.load(f).get("workloads", {})
    ctx = mp.get_context("spawn")
    for name, w in wl.WORKLOADS.items():
        if not w.densities and not w.per_head_density:
            continue
        if args.only and name != args.only:
            continue
        with ProcessPoolExecutor(max_workers=args.workers, mp_context=ctx) as ex:
            res = list(ex.map(head_gaps, [name] * w.H, [0] * w.H, range(w.H)))
        res.sort(key=lambda r: r[0])
        entry = {}
        targets = {str(D): [D] * w.H for D in w.densities}
        if w.per_head_density:
            targets = {"per_head": [float(x) for x in wl.target_densities(w)]}
        for key, Ds in targets.items():
            taus, dens, bands = [], [], []
            for (h, gaps, sbar, M), D in zip(res, Ds):
                tau = calibrate(gaps, D, w.n_force, w.n_blocks)
                a, band = achieved(sbar, M, tau, w.n_force)
                taus.append("inf" if math.isinf(tau) else tau)
                dens.append(a)
                bands.append(band)
            entry[key] = {"target": Ds, "tau": taus, "density_b0": dens, "band_b0": bands}
            print(f"{name} {key}: mean density {np.mean(dens):.4f}, band entries {sum(bands)}", flush=True)
        table[name] = entry
    doc = {
        "what": "per-head routing thresholds tau for the synthetic workloads (see make_tau.py)",
        "written_by": "tests/golden/make_tau.py (float64 oracle pooling and proxy scores only)",
        "workloads": table,
    }
    with open(out_path, "w") as f:
        json.dump(doc, f, indent=1)


if __name__ == "__main__":
    main()
