"""C-ABI checks that need no GPU: the library loads, exports every function the header declares,
and rejects invalid arguments on the host before launching anything."""
import ctypes
import math
import os
import re

import pytest

from block_sparse_attention_41_b200 import build as builder
from block_sparse_attention_41_b200 import sol_attn as sa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    builder.build()
    return sa.load_library()


def declared_functions():
    with open(os.path.join(ROOT, "include", "sol_attn.h")) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sol_attn_\w+)\s*\(", text)))


def test_header_declares_the_binding_names():
    assert declared_functions() == sorted(sa.EXPORTED)


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_status_strings(lib):
    for s in range(5):
        assert sa.status_string(s).startswith("SOL_")
    assert "unknown" in sa.status_string(99)


def test_workspace_size(lib):
    n = sa.sol_attn_fwd_workspace_bytes(2, 32, 33272, 128)
    assert n % 256 == 0 and n >= 4 * (4 + 64)
    assert sa.sol_attn_fwd_workspace_bytes(0, 1, 1, 1) == 0
    # header (error, where, counter, done, 40 per-head counts) + keep bits 40 x 591 x ceil(591/32) words
    # + query-block means 40 x 591 x 128 floats
    header = ((4 + 40) * 4 + 255) // 256 * 256
    bits = -(-(40 * 591 * 19 * 4) // 256) * 256
    qbar = -(-(40 * 591 * 128 * 4) // 256) * 256
    assert sa.sol_attn_fwd_workspace_bytes(1, 40, 75600, 128) == header + bits + qbar


# fake, 16-byte aligned device addresses: validation must reject before any of them is used
P = [ctypes.c_void_p(0x1000 * (i + 1)) for i in range(12)]


def fwd(lib, dt=sa.SOL_BF16, B=1, H=2, L=1000, d=128, bq=128, bk=128, n_force=0, tau=(1.0, 1.0), ws=4096,
        ptrs=None):
    p = list(ptrs or P)
    tau_c = (ctypes.c_float * len(tau))(*tau)
    return lib.sol_attn_fwd(p[0], p[1], p[2], p[3], p[4], p[5], p[6], tau_c, dt, B, H, L, d, bq, bk, n_force,
                            p[7], None, None, p[8], ws, None)


def test_fwd_rejects_invalid_arguments(lib):
    assert fwd(lib, tau=(1.0, -0.5)) == sa.SOL_EINVAL
    assert fwd(lib, tau=(math.nan, 1.0)) == sa.SOL_EINVAL
    assert "tau" in lib.sol_attn_last_error().decode()
    assert fwd(lib, L=0) == sa.SOL_EINVAL
    assert fwd(lib, n_force=9) == sa.SOL_EINVAL  # N_kb = 8
    assert fwd(lib, n_force=-1) == sa.SOL_EINVAL
    assert fwd(lib, ws=16) == sa.SOL_EINVAL
    misaligned = list(P)
    misaligned[1] = ctypes.c_void_p(0x1008)
    assert fwd(lib, ptrs=misaligned) == sa.SOL_EINVAL
    nulls = list(P)
    nulls[0] = None
    assert fwd(lib, ptrs=nulls) == sa.SOL_EINVAL
    assert fwd(lib, dt=7) == sa.SOL_EINVAL


def test_fwd_rejects_unsupported_shapes(lib):
    assert fwd(lib, d=96) == sa.SOL_EUNSUPPORTED
    assert fwd(lib, bq=64, bk=64) == sa.SOL_EUNSUPPORTED           # bf16 needs 128
    assert fwd(lib, bq=128, bk=64) == sa.SOL_EUNSUPPORTED
    assert fwd(lib, dt=sa.SOL_F32, d=48, bq=64, bk=64) == sa.SOL_EUNSUPPORTED
    assert fwd(lib, L=4096 * 128 + 1) == sa.SOL_EUNSUPPORTED      # N_kb > 4096
    assert fwd(lib, H=300, tau=tuple([1.0] * 300)) == sa.SOL_EUNSUPPORTED


def test_pool_rejects_invalid_arguments(lib):
    p = P
    assert lib.sol_attn_pool(p[0], p[1], sa.SOL_BF16, 1, 1, 100, 64, 128, p[2], p[3], None, None, None) == sa.SOL_EINVAL
    assert lib.sol_attn_pool(p[0], p[1], sa.SOL_F32, 1, 1, 100, 64, 128, p[2], p[3], p[4], p[5], None) == sa.SOL_EINVAL
    assert lib.sol_attn_pool(p[0], p[1], sa.SOL_BF16, 1, 1, 100, 60, 128, p[2], p[3], p[4], p[5], None) == sa.SOL_EUNSUPPORTED
    # rows of 12 or 64 16-byte vectors: not a power of two <= 32
    assert lib.sol_attn_pool(p[0], p[1], sa.SOL_BF16, 1, 1, 100, 96, 128, p[2], p[3], p[4], p[5], None) == sa.SOL_EUNSUPPORTED
    assert lib.sol_attn_pool(p[0], p[1], sa.SOL_F32, 1, 1, 100, 256, 128, p[2], p[3], None, None, None) == sa.SOL_EUNSUPPORTED
    assert lib.sol_attn_pool(p[0], p[1], sa.SOL_BF16, 1, 1, 0, 64, 128, p[2], p[3], p[4], p[5], None) == sa.SOL_EINVAL


def rope_pool(lib, eps=1e-6, d=128, blk=128, B=1, H=2, L=1000, ptrs=None):
    p = list(ptrs or P) + [ctypes.c_void_p(0x20000), ctypes.c_void_p(0x30000)]
    return lib.sol_attn_qknorm_rope_pool(p[0], p[1], p[2], p[3], p[4], p[5], p[6], ctypes.c_float(eps), B, H, L, d, blk,
                                         p[7], p[8], p[9], p[10], p[11], p[12], None)


def test_qknorm_rope_pool_rejects_invalid_arguments(lib):
    assert rope_pool(lib, eps=0.0) == sa.SOL_EINVAL
    assert rope_pool(lib, eps=-1.0) == sa.SOL_EINVAL
    assert rope_pool(lib, eps=math.inf) == sa.SOL_EINVAL
    assert rope_pool(lib, L=0) == sa.SOL_EINVAL
    nulls = list(P)
    nulls[5] = None
    assert rope_pool(lib, ptrs=nulls) == sa.SOL_EINVAL
    misaligned = list(P)
    misaligned[3] = ctypes.c_void_p(0x1004)
    assert rope_pool(lib, ptrs=misaligned) == sa.SOL_EINVAL
    assert rope_pool(lib, d=96) == sa.SOL_EUNSUPPORTED
    assert rope_pool(lib, blk=8192) == sa.SOL_EUNSUPPORTED
    assert rope_pool(lib, B=300, H=300) == sa.SOL_EUNSUPPORTED
    assert rope_pool(lib, L=4 * 65535 + 1, blk=1) == sa.SOL_EUNSUPPORTED  # the grid's second dimension


def test_check_device_error_rejects_null(lib):
    assert lib.sol_attn_check_device_error(None, None) == sa.SOL_EINVAL


def test_binding_fails_loudly_without_cuda_tensors(lib):
    import torch
    x = torch.zeros(1, 1, 8, 64)
    with pytest.raises(TypeError):
        sa.sol_attn_pool(x, x, 128)


def test_host_entry_scratch_size(lib):
    # two slots of Q, K, V, O for 2 heads, pooled fp32 + bf16 vectors for 2 heads, the workspace
    # of a 2-head call and 40 density words, each rounded up to 256 bytes
    r = lambda x: -(-x // 256) * 256  # noqa: E731
    L, d, c, H, nkb = 75600, 128, 2, 40, 591
    ws = r(r((4 + c) * 4) + r(c * nkb * 19 * 4) + r(c * nkb * 128 * 4))  # header, keep bits, q_bar
    want = 8 * r(c * L * d * 2) + 2 * r(c * nkb * d * 4) + 2 * r(c * nkb * d * 2) + ws + r(H * 4)
    assert lib.sol_attn_fwd_host_scratch_bytes(sa.SOL_BF16, 1, H, L, d, 128, c) == want
    # fp32: 4-byte elements, no bf16 mirrors
    want32 = (8 * r(c * 1000 * 64 * 4) + 2 * r(c * 16 * 64 * 4) +
              r(r((4 + c) * 4) + r(c * 16 * 1 * 4) + r(c * 16 * 128 * 4)) + r(3 * 4))
    assert lib.sol_attn_fwd_host_scratch_bytes(sa.SOL_F32, 1, 3, 1000, 64, 64, c) == want32
    # more heads per chunk than heads: one chunk of H heads
    assert (lib.sol_attn_fwd_host_scratch_bytes(sa.SOL_BF16, 2, 3, 1000, 64, 128, 99) ==
            lib.sol_attn_fwd_host_scratch_bytes(sa.SOL_BF16, 2, 3, 1000, 64, 128, 3))
    for bad in ((7, 1, 3, 1000, 64, 128, 1), (sa.SOL_BF16, 0, 3, 1000, 64, 128, 1),
                (sa.SOL_BF16, 1, 3, 1000, 64, 128, 0)):
        assert lib.sol_attn_fwd_host_scratch_bytes(*bad) == 0


def fwd_host(lib, dt=sa.SOL_BF16, B=1, H=2, L=1000, d=128, blk=128, n_force=0, tau=(1.0, 1.0), chunk=1,
             scratch=ctypes.c_void_p(0x100000), nbytes=1 << 40, o=P[3]):
    tau_c = (ctypes.c_float * len(tau))(*tau)
    return lib.sol_attn_fwd_host(P[0], P[1], P[2], o, tau_c, dt, B, H, L, d, blk, n_force, chunk, None, scratch,
                                 nbytes, None)


def test_host_entry_rejects_invalid_arguments_before_any_copy(lib):
    assert fwd_host(lib, tau=(1.0, -1.0)) == sa.SOL_EINVAL
    assert fwd_host(lib, chunk=0) == sa.SOL_EINVAL
    assert "heads_per_chunk" in lib.sol_attn_last_error().decode()
    assert fwd_host(lib, o=None) == sa.SOL_EINVAL
    assert fwd_host(lib, scratch=ctypes.c_void_p(0x100010)) == sa.SOL_EINVAL  # not 256-byte aligned
    assert fwd_host(lib, nbytes=4096) == sa.SOL_EINVAL
    assert "scratch too small" in lib.sol_attn_last_error().decode()
    assert fwd_host(lib, n_force=9) == sa.SOL_EINVAL
    assert fwd_host(lib, d=96) == sa.SOL_EUNSUPPORTED
    assert fwd_host(lib, dt=sa.SOL_F32, blk=48) == sa.SOL_EUNSUPPORTED
    assert fwd_host(lib, L=4096 * 128 + 1) == sa.SOL_EUNSUPPORTED
    # valid sizes: the next check asks the runtime where the pointers live, which fails without a
    # GPU (SOL_ECUDA) and rejects the fake scratch address with one (SOL_EINVAL); no copy is made
    assert fwd_host(lib) in (sa.SOL_ECUDA, sa.SOL_EINVAL)


def test_host_binding_rejects_non_host_tensors(lib):
    import torch
    with pytest.raises(TypeError):
        sa.sol_attn_fwd_host([1.0], [1.0], [1.0], [1.0])
    x = torch.zeros(1, 1, 8, 64)
    with pytest.raises(ValueError):
        sa.sol_attn_fwd_host(x, x, torch.zeros(1, 1, 8, 32), [1.0])


def test_topk_entry_rejects_invalid_arguments(lib):
    def call(k=3, L=1000, ws=1 << 30, workspace=P[8], B=1, H=2):
        return lib.sol_attn_fwd_topk(P[0], P[1], P[2], P[3], P[4], P[5], k, B, H, L, 128, 0, P[7], None, None,
                                     workspace, ws, None)
    assert call(k=0) == sa.SOL_EINVAL
    assert call(k=9) == sa.SOL_EINVAL  # N_kb = 8
    assert call(ws=16) == sa.SOL_EINVAL
    assert "full workspace" in lib.sol_attn_last_error().decode()
    assert call(workspace=None) == sa.SOL_EINVAL
    assert call(L=0) == sa.SOL_EINVAL
    assert call(H=300) == sa.SOL_EUNSUPPORTED


def test_qbar_entries_reject_invalid_arguments(lib):
    tau = (ctypes.c_float * 2)(0.5, 0.5)

    def fwd(qbar=P[9], ws=1 << 30, workspace=P[8], L=1000):
        return lib.sol_attn_fwd_qbar(P[0], P[1], P[2], P[3], P[4], P[5], P[6], qbar, tau, 1, 2, L, 128, 0, P[7], None,
                                     None, workspace, ws, None)
    assert fwd(qbar=None) == sa.SOL_EINVAL
    assert "qbar" in lib.sol_attn_last_error().decode()
    assert fwd(qbar=ctypes.c_void_p(0x1008)) == sa.SOL_EINVAL  # not 16-byte aligned
    assert fwd(ws=256) == sa.SOL_EINVAL
    assert "full workspace" in lib.sol_attn_last_error().decode()
    assert fwd(workspace=None) == sa.SOL_EINVAL
    assert fwd(L=0) == sa.SOL_EINVAL

    def pool(qbar=P[9]):
        return lib.sol_attn_qknorm_rope_pool_qbar(P[0], P[1], P[2], P[3], P[4], P[5], P[6], ctypes.c_float(1e-6), 1, 2,
                                                  1000, 128, 128, P[7], P[8], P[9], P[10], P[11], P[11], qbar, None)
    assert pool(qbar=None) == sa.SOL_EINVAL
    assert "qbar" in lib.sol_attn_last_error().decode()


def test_8bit_value_and_forward_entries_reject_invalid_arguments(lib):
    def quant(d=128, L=1000, ptrs=None):
        p = list(ptrs or P)
        return lib.sol_attn_quantize_v8(p[0], p[1], 1, 2, L, d, p[2], p[3], p[4], None)
    assert quant(d=64) == sa.SOL_EUNSUPPORTED
    assert quant(L=0) == sa.SOL_EINVAL
    nulls = list(P)
    nulls[3] = None
    assert quant(ptrs=nulls) == sa.SOL_EINVAL
    assert quant(L=4097 * 128) == sa.SOL_EUNSUPPORTED
    tau = (ctypes.c_float * 2)(0.5, 0.5)

    def fwd(d=128, ws=1 << 30, ptrs=None):
        p = list(ptrs or P)
        return lib.sol_attn_fwd_8bit(p[0], p[1], p[2], p[3], p[4], p[5], p[6], p[7], p[8], p[9], p[10], tau, 1, 2,
                                     1000, d, 0, p[11], None, None, p[11], ws, None)
    assert fwd(d=64) == sa.SOL_EUNSUPPORTED
    assert fwd(ws=256) == sa.SOL_EINVAL
    assert "full workspace" in lib.sol_attn_last_error().decode()
    nulls = list(P)
    nulls[8] = None  # vbar8t
    assert fwd(ptrs=nulls) == sa.SOL_EINVAL
