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
    header = ((4 + 40) * 4 + 255) // 256 * 256
    bits = -(-(40 * 591 * 19 * 4) // 256) * 256
    assert sa.sol_attn_fwd_workspace_bytes(1, 40, 75600, 128) == header + bits


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


def test_check_device_error_rejects_null(lib):
    assert lib.sol_attn_check_device_error(None, None) == sa.SOL_EINVAL


def test_binding_fails_loudly_without_cuda_tensors(lib):
    import torch
    x = torch.zeros(1, 1, 8, 64)
    with pytest.raises(TypeError):
        sa.sol_attn_pool(x, x, 128)
