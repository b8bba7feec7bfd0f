"""Host-side checks of bench.py that need no GPU: the max-over-ranks reduction with world size 2
(gloo on CPU) and the reference arm's JSON line."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, values, out):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        out[rank] = bench.reduce_max_over_ranks(values[rank], world, torch.device("cpu"))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world_2():
    mgr = mp.Manager()
    out = mgr.dict()
    values = [3.5, 7.25]
    mp.spawn(_rank, args=(2, _free_port(), values, out), nprocs=2, join=True)
    assert dict(out) == {0: 7.25, 1: 7.25}


def test_single_rank_reduction_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_max_over_ranks(1.5, 1, None) == 1.5


def test_reference_arm_prints_contract_line():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "small_dit_L8192",
                        "--steps", "1", "--warmup", "3", "--ref-budget", "0.5"],
                       cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in line, k
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2")
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "small_dit_L8192"],
                       cwd=ROOT, capture_output=True, text=True, timeout=300, env=env)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_kernel_code_hash_ignores_comments_but_not_code():
    sys.path.insert(0, ROOT)
    import bench
    base = 'int a = 1;  // note\n/* block\n comment */\nconst char* s = "x // y";\n'
    assert bench.code_tokens(base) == bench.code_tokens(base.replace("note", "other note") + "\n// more\n")
    assert bench.code_tokens(base) != bench.code_tokens(base.replace("a = 1", "a = 2"))
    assert '"x // y"' in bench.code_tokens(base)  # a string literal is code, not a comment


def test_captured_traffic_is_dropped_once_the_kernel_code_changes(monkeypatch):
    # the ncu summary's DRAM traffic is reported only while the kernel code is the captured one
    sys.path.insert(0, ROOT)
    import bench
    from block_sparse_attention_41_b200 import workloads as wl
    w = wl.WORKLOADS["video720p_L75600"]
    got = bench.captured_traffic(w, "0.2")
    assert got is None or got > 0
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "0000000000000000")
    assert bench.captured_traffic(w, "0.2") is None


def test_sampled_parity_report_compares_only_units_with_the_same_kept_set():
    # the oracle's own sampled rows, collected outside its timed part, against themselves plus a
    # known error; a unit whose mask row differs is counted but not compared
    import numpy as np
    sys.path.insert(0, ROOT)
    import bench
    from block_sparse_attention_41_b200 import workloads as wl
    w = wl.WORKLOADS["small_dit_L8192"]
    tau = bench.tau_for(w, bench.density_keys(w)[0])
    got = []
    _, _, n, _ = bench.oracle_sample(w, tau, budget_s=0.5, max_units=4, collect=got)
    assert len(got) == n >= 1
    b, h, i, rows, keep = got[0]
    assert rows.shape == (w.block, w.d) and np.isfinite(rows).all() and keep.dtype == bool and keep.any()
    gpu = {(b_, h_, i_): r + 1e-3 for b_, h_, i_, r, _ in got}
    masks = {(b_, h_, i_): k.copy() for b_, h_, i_, _, k in got}
    rep = bench.sample_parity(got, gpu, masks)
    assert rep["units"] == n and rep["units_compared"] == n
    assert abs(rep["max_abs"] - 1e-3) < 1e-12 and abs(rep["mean_abs"] - 1e-3) < 1e-12
    masks[(b, h, i)] = ~masks[(b, h, i)]
    assert bench.sample_parity(got, gpu, masks)["units_compared"] == n - 1


def test_cpu_sample_units_come_from_a_few_fixed_heads():
    sys.path.insert(0, ROOT)
    import bench
    from block_sparse_attention_41_b200 import workloads as wl
    w = wl.WORKLOADS["video720p_L75600"]
    a = bench.cpu_sample_units(w, 192, 77)
    assert a == bench.cpu_sample_units(w, 192, 77) and a == sorted(a) and len(set(a)) == 192
    b = bench.cpu_sample_units(w, 192, 100)
    heads = {(u[0], u[1]) for u in a}
    assert len(heads) == bench.CPU_SAMPLE_HEADS and {(u[0], u[1]) for u in b} == heads and a != b
    assert all(0 <= u[2] < w.n_blocks for u in a)
