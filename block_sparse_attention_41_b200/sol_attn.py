"""Thin ctypes binding of libsolattn.so (C ABI in include/sol_attn.h), with the same call names.

This module only marshals arguments: it checks tensor placement, dtype and contiguity,
allocates output tensors with torch when the caller passes none, passes raw pointers and
the current CUDA stream, and turns status codes into exceptions. All compute runs in the
library's CUDA kernels. There is no fallback: if the library is missing or no sm_100 GPU is
present, the calls raise.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Sequence

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsolattn.so")

SOL_OK, SOL_EINVAL, SOL_EUNSUPPORTED, SOL_ECUDA, SOL_ETIMEOUT = range(5)
SOL_F32, SOL_BF16 = 0, 1

# symbols declared in include/sol_attn.h
EXPORTED = (
    "sol_attn_status_string",
    "sol_attn_last_error",
    "sol_attn_pool",
    "sol_attn_fwd_workspace_bytes",
    "sol_attn_fwd",
    "sol_attn_check_device_error",
    "sol_attn_debug_drop_one_load",
    "sol_attn_debug_record_cta_times",
    "sol_attn_fwd_noalloc",
    "sol_attn_qknorm_rope_pool",
    "sol_attn_fwd_host_scratch_bytes",
    "sol_attn_fwd_host",
    "sol_attn_fwd_topk",
    "sol_attn_quantize_qk8",
    "sol_attn_fwd_qk8",
    "sol_attn_qknorm_rope_pool_qbar",
    "sol_attn_fwd_qbar",
    "sol_attn_quantize_v8",
    "sol_attn_fwd_8bit",
)


class SolAttnError(RuntimeError):
    """A library call returned a status other than SOL_OK."""

    def __init__(self, status: int, call: str, detail: str):
        self.status = status
        super().__init__(f"{call}: {status_string(status)}: {detail}")


_lib = None


def load_library() -> ctypes.CDLL:
    """Load libsolattn.so once; raise if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"{LIB_PATH} is missing: build it with `python -m block_sparse_attention_41_b200.build` "
            "(there is no non-CUDA implementation)")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, f32p = ctypes.c_void_p, ctypes.c_int, ctypes.POINTER(ctypes.c_float)
    lib.sol_attn_status_string.argtypes = [i32]
    lib.sol_attn_status_string.restype = ctypes.c_char_p
    lib.sol_attn_last_error.argtypes = []
    lib.sol_attn_last_error.restype = ctypes.c_char_p
    lib.sol_attn_pool.argtypes = [vp, vp, i32, i32, i32, i32, i32, i32, vp, vp, vp, vp, vp]
    lib.sol_attn_pool.restype = i32
    lib.sol_attn_fwd_workspace_bytes.argtypes = [i32, i32, i32, i32]
    lib.sol_attn_fwd_workspace_bytes.restype = ctypes.c_size_t
    lib.sol_attn_fwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, f32p, i32, i32, i32, i32, i32, i32, i32, i32,
                                 vp, vp, vp, vp, ctypes.c_size_t, vp]
    lib.sol_attn_fwd.restype = i32
    lib.sol_attn_fwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, f32p, i32, i32, i32, i32, i32, i32, i32, i32,
                                         vp, vp, vp, vp]
    lib.sol_attn_fwd_noalloc.restype = i32
    lib.sol_attn_qknorm_rope_pool.argtypes = [vp, vp, vp, vp, vp, vp, vp, ctypes.c_float, i32, i32, i32, i32, i32,
                                              vp, vp, vp, vp, vp, vp, vp]
    lib.sol_attn_qknorm_rope_pool.restype = i32
    lib.sol_attn_qknorm_rope_pool_qbar.argtypes = [vp, vp, vp, vp, vp, vp, vp, ctypes.c_float, i32, i32, i32, i32,
                                                   i32, vp, vp, vp, vp, vp, vp, vp, vp]
    lib.sol_attn_qknorm_rope_pool_qbar.restype = i32
    lib.sol_attn_fwd_qbar.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, f32p, i32, i32, i32, i32, i32, vp, vp, vp, vp,
                                      ctypes.c_size_t, vp]
    lib.sol_attn_fwd_qbar.restype = i32
    lib.sol_attn_quantize_v8.argtypes = [vp, vp, i32, i32, i32, i32, vp, vp, vp, vp]
    lib.sol_attn_quantize_v8.restype = i32
    lib.sol_attn_fwd_8bit.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, f32p, i32, i32, i32, i32, i32, vp, vp,
                                      vp, vp, ctypes.c_size_t, vp]
    lib.sol_attn_fwd_8bit.restype = i32
    lib.sol_attn_quantize_qk8.argtypes = [vp, vp, vp, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp, vp, vp]
    lib.sol_attn_quantize_qk8.restype = i32
    lib.sol_attn_fwd_qk8.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, f32p, i32, i32, i32, i32, i32, vp, vp,
                                     vp, vp, ctypes.c_size_t, vp]
    lib.sol_attn_fwd_qk8.restype = i32
    lib.sol_attn_fwd_host_scratch_bytes.argtypes = [i32, i32, i32, i32, i32, i32, i32]
    lib.sol_attn_fwd_host_scratch_bytes.restype = ctypes.c_size_t
    lib.sol_attn_fwd_host.argtypes = [vp, vp, vp, vp, f32p, i32, i32, i32, i32, i32, i32, i32, i32, vp, vp,
                                      ctypes.c_size_t, vp]
    lib.sol_attn_fwd_host.restype = i32
    lib.sol_attn_fwd_topk.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, vp, vp, vp, vp,
                                      ctypes.c_size_t, vp]
    lib.sol_attn_fwd_topk.restype = i32
    lib.sol_attn_check_device_error.argtypes = [vp, vp]
    lib.sol_attn_check_device_error.restype = i32
    lib.sol_attn_debug_drop_one_load.argtypes = [i32]
    lib.sol_attn_debug_drop_one_load.restype = None
    lib.sol_attn_debug_record_cta_times.argtypes = [vp, i32]
    lib.sol_attn_debug_record_cta_times.restype = None
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load_library().sol_attn_status_string(int(status)).decode()


def _check(status: int, call: str) -> None:
    if status != SOL_OK:
        raise SolAttnError(status, call, load_library().sol_attn_last_error().decode())


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return SOL_BF16
    if t.dtype == torch.float32:
        return SOL_F32
    raise TypeError(f"unsupported dtype {t.dtype}: use torch.bfloat16 or torch.float32")


def _need_cuda(name: str, t: torch.Tensor, dtype=None) -> None:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must have dtype {dtype}, got {t.dtype}")


def sol_attn_pool(K: torch.Tensor, V: torch.Tensor, block_k: int, kbar=None, vbar=None, kbar_lp=None,
                  vbar_lp=None, stream=None):
    """Block means of K and V. Returns (kbar, vbar, kbar_lp, vbar_lp); the bf16 mirrors are None
    for fp32 inputs."""
    _need_cuda("K", K)
    _need_cuda("V", V, K.dtype)
    B, H, L, d = K.shape
    if V.shape != K.shape:
        raise ValueError("K and V must have the same shape")
    nkb = -(-L // block_k)
    dt = _dtype_code(K)
    dev = K.device
    if kbar is None:
        kbar = torch.empty((B, H, nkb, d), dtype=torch.float32, device=dev)
    if vbar is None:
        vbar = torch.empty((B, H, nkb, d), dtype=torch.float32, device=dev)
    if dt == SOL_BF16:
        if kbar_lp is None:
            kbar_lp = torch.empty((B, H, nkb, d), dtype=torch.bfloat16, device=dev)
        if vbar_lp is None:
            vbar_lp = torch.empty((B, H, nkb, d), dtype=torch.bfloat16, device=dev)
    for n, t in (("kbar", kbar), ("vbar", vbar)):
        _need_cuda(n, t, torch.float32)
    st = load_library().sol_attn_pool(_ptr(K), _ptr(V), dt, B, H, L, d, block_k, _ptr(kbar), _ptr(vbar),
                                      _ptr(kbar_lp), _ptr(vbar_lp), _stream(stream))
    _check(st, "sol_attn_pool")
    return kbar, vbar, kbar_lp, vbar_lp


def sol_attn_qknorm_rope_pool(Q, K, V, gain_q, gain_k, rope_cos, rope_sin, block_k: int, eps: float = 1e-6,
                              Q_out=None, K_out=None, kbar=None, vbar=None, kbar_lp=None, vbar_lp=None, stream=None,
                              qbar=None, want_qbar: bool = False):
    """QK RMS norm + rotary embedding of Q and K, and the block means of the stored K and of V, in
    one pass. Returns (Q_out, K_out, kbar, vbar, kbar_lp, vbar_lp), plus qbar (the block means of
    the stored Q, for sol_attn_fwd_qbar) when want_qbar or a qbar tensor is given. Pass Q_out=Q,
    K_out=K to work in place."""
    for n, t in (("Q", Q), ("K", K), ("V", V)):
        _need_cuda(n, t, torch.bfloat16)
    B, H, L, d = Q.shape
    if K.shape != Q.shape or V.shape != Q.shape:
        raise ValueError("Q, K and V must have the same shape [B, H, L, d]")
    for n, t in (("gain_q", gain_q), ("gain_k", gain_k), ("rope_cos", rope_cos), ("rope_sin", rope_sin)):
        _need_cuda(n, t, torch.float32)
    if rope_cos.shape != (L, d // 2) or rope_sin.shape != (L, d // 2):
        raise ValueError(f"rope tables must be [L, d/2] = [{L}, {d // 2}]")
    nkb = -(-L // block_k)
    dev = Q.device
    Q_out = torch.empty_like(Q) if Q_out is None else Q_out
    K_out = torch.empty_like(K) if K_out is None else K_out
    kbar = torch.empty((B, H, nkb, d), dtype=torch.float32, device=dev) if kbar is None else kbar
    vbar = torch.empty((B, H, nkb, d), dtype=torch.float32, device=dev) if vbar is None else vbar
    kbar_lp = torch.empty((B, H, nkb, d), dtype=torch.bfloat16, device=dev) if kbar_lp is None else kbar_lp
    vbar_lp = torch.empty((B, H, nkb, d), dtype=torch.bfloat16, device=dev) if vbar_lp is None else vbar_lp
    if qbar is None and not want_qbar:
        st = load_library().sol_attn_qknorm_rope_pool(
            _ptr(Q), _ptr(K), _ptr(V), _ptr(gain_q), _ptr(gain_k), _ptr(rope_cos), _ptr(rope_sin),
            ctypes.c_float(eps), B, H, L, d, block_k, _ptr(Q_out), _ptr(K_out), _ptr(kbar), _ptr(vbar), _ptr(kbar_lp),
            _ptr(vbar_lp), _stream(stream))
        _check(st, "sol_attn_qknorm_rope_pool")
        return Q_out, K_out, kbar, vbar, kbar_lp, vbar_lp
    qbar = torch.empty((B, H, nkb, d), dtype=torch.float32, device=dev) if qbar is None else qbar
    _need_cuda("qbar", qbar, torch.float32)
    st = load_library().sol_attn_qknorm_rope_pool_qbar(
        _ptr(Q), _ptr(K), _ptr(V), _ptr(gain_q), _ptr(gain_k), _ptr(rope_cos), _ptr(rope_sin), ctypes.c_float(eps),
        B, H, L, d, block_k, _ptr(Q_out), _ptr(K_out), _ptr(kbar), _ptr(vbar), _ptr(kbar_lp), _ptr(vbar_lp),
        _ptr(qbar), _stream(stream))
    _check(st, "sol_attn_qknorm_rope_pool_qbar")
    return Q_out, K_out, kbar, vbar, kbar_lp, vbar_lp, qbar


def sol_attn_quantize_qk8(Q, K, kbar, stream=None):
    """8-bit QK^T operands (blocks of 128): returns (q8, k8, kbar8, q_scale, k_scale, kbar_scale, mu),
    the int8 codes of Q, K - mu and kbar - mu with one scale per 128-row tile, and the mean key mu."""
    for n, t in (("Q", Q), ("K", K)):
        _need_cuda(n, t, torch.bfloat16)
    _need_cuda("kbar", kbar, torch.float32)
    B, H, L, d = Q.shape
    nkb = -(-L // 128)
    if K.shape != Q.shape or tuple(kbar.shape) != (B, H, nkb, d):
        raise ValueError("Q, K must be [B, H, L, d] and kbar [B, H, ceil(L/128), d]")
    dev = Q.device
    q8 = torch.empty((B, H, L, d), dtype=torch.int8, device=dev)
    k8 = torch.empty_like(q8)
    kbar8 = torch.empty((B, H, nkb, d), dtype=torch.int8, device=dev)
    q_scale = torch.empty((B, H, nkb), dtype=torch.float32, device=dev)
    k_scale = torch.empty_like(q_scale)
    kbar_scale = torch.empty((B, H, -(-nkb // 128)), dtype=torch.float32, device=dev)
    mu = torch.empty((B, H, d), dtype=torch.float32, device=dev)
    st = load_library().sol_attn_quantize_qk8(
        _ptr(Q), _ptr(K), _ptr(kbar), B, H, L, d, _ptr(q8), _ptr(k8), _ptr(kbar8), _ptr(q_scale), _ptr(k_scale),
        _ptr(kbar_scale), _ptr(mu), _stream(stream))
    _check(st, "sol_attn_quantize_qk8")
    return q8, k8, kbar8, q_scale, k_scale, kbar_scale, mu


def sol_attn_fwd_qk8(Q, q8, k8, kbar8, q_scale, k_scale, kbar_scale, V, kbar, vbar_lp, tau: Sequence[float],
                     n_force: int = 0, O=None, kept_mask=None, density=None, workspace=None, stream=None):
    """The forward with 8-bit QK^T from the operands of sol_attn_quantize_qk8 (d = 128). Returns O."""
    _need_cuda("Q", Q, torch.bfloat16)
    _need_cuda("V", V, torch.bfloat16)
    B, H, L, d = Q.shape
    for n, t in (("q8", q8), ("k8", k8), ("kbar8", kbar8)):
        _need_cuda(n, t, torch.int8)
    for n, t in (("q_scale", q_scale), ("k_scale", k_scale), ("kbar_scale", kbar_scale), ("kbar", kbar)):
        _need_cuda(n, t, torch.float32)
    _need_cuda("vbar_lp", vbar_lp, torch.bfloat16)
    tau = [float(x) for x in tau]
    if len(tau) != H:
        raise ValueError(f"tau must hold H={H} values")
    if O is None:
        O = torch.empty_like(Q)
    if workspace is None:
        workspace = new_workspace(B, H, L, 128, Q.device)
    tau_c = (ctypes.c_float * H)(*tau)
    st = load_library().sol_attn_fwd_qk8(
        _ptr(Q), _ptr(q8), _ptr(k8), _ptr(kbar8), _ptr(q_scale), _ptr(k_scale), _ptr(kbar_scale), _ptr(V), _ptr(kbar),
        _ptr(vbar_lp), tau_c, B, H, L, d, int(n_force), _ptr(O), _ptr(kept_mask), _ptr(density), _ptr(workspace),
        workspace.numel(), _stream(stream))
    _check(st, "sol_attn_fwd_qk8")
    return O


def sol_attn_fwd_workspace_bytes(B: int, H: int, L: int, block_q: int) -> int:
    return int(load_library().sol_attn_fwd_workspace_bytes(B, H, L, block_q))


def new_workspace(B: int, H: int, L: int, block_q: int, device) -> torch.Tensor:
    """A zeroed workspace buffer of the size sol_attn_fwd needs."""
    return torch.zeros(sol_attn_fwd_workspace_bytes(B, H, L, block_q), dtype=torch.uint8, device=device)


def sol_attn_fwd(Q, K, V, kbar, vbar, kbar_lp, vbar_lp, tau: Sequence[float], block_q: int, block_k: int,
                 n_force: int = 0, O=None, kept_mask=None, density=None, workspace=None, stream=None):
    """Fused routing + exact kept-block attention + skipped-block correction. Returns O.

    `tau` is a host sequence of H floats (>= 0, +inf = dense). `kept_mask` (uint8
    [B,H,N_qb,N_kb]) and `density` (float32 [B,H]) are optional output tensors.
    """
    _need_cuda("Q", Q)
    for n, t in (("K", K), ("V", V)):
        _need_cuda(n, t, Q.dtype)
    B, H, L, d = Q.shape
    if K.shape != Q.shape or V.shape != Q.shape:
        raise ValueError("Q, K and V must have the same shape [B, H, L, d]")
    dt = _dtype_code(Q)
    tau = [float(x) for x in tau]
    if len(tau) != H:
        raise ValueError(f"tau must hold H={H} values")
    if O is None:
        O = torch.empty_like(Q)
    if workspace is None:
        workspace = new_workspace(B, H, L, block_q, Q.device)
    tau_c = (ctypes.c_float * H)(*tau)
    st = load_library().sol_attn_fwd(
        _ptr(Q), _ptr(K), _ptr(V), _ptr(kbar), _ptr(vbar), _ptr(kbar_lp), _ptr(vbar_lp), tau_c, dt, B, H, L, d,
        block_q, block_k, int(n_force), _ptr(O), _ptr(kept_mask), _ptr(density), _ptr(workspace),
        workspace.numel(), _stream(stream))
    _check(st, "sol_attn_fwd")
    return O


def sol_attn_fwd_noalloc(Q, K, V, kbar, vbar, kbar_lp, vbar_lp, tau: Sequence[float], block_q: int, block_k: int,
                         n_force: int = 0, O=None, kept_mask=None, density=None, stream=None):
    """sol_attn_fwd without a workspace argument: the library uses its own static device array
    (B*H <= 4096; calls that overlap on the GPU race on it). For callers that cannot allocate
    device memory; pass a preallocated `O` to allocate nothing here either."""
    _need_cuda("Q", Q)
    for n, t in (("K", K), ("V", V)):
        _need_cuda(n, t, Q.dtype)
    B, H, L, d = Q.shape
    if K.shape != Q.shape or V.shape != Q.shape:
        raise ValueError("Q, K and V must have the same shape [B, H, L, d]")
    tau = [float(x) for x in tau]
    if len(tau) != H:
        raise ValueError(f"tau must hold H={H} values")
    if O is None:
        O = torch.empty_like(Q)
    tau_c = (ctypes.c_float * H)(*tau)
    st = load_library().sol_attn_fwd_noalloc(
        _ptr(Q), _ptr(K), _ptr(V), _ptr(kbar), _ptr(vbar), _ptr(kbar_lp), _ptr(vbar_lp), tau_c, _dtype_code(Q), B, H,
        L, d, block_q, block_k, int(n_force), _ptr(O), _ptr(kept_mask), _ptr(density), _stream(stream))
    _check(st, "sol_attn_fwd_noalloc")
    return O


def sol_attn_fwd_topk(Q, K, V, kbar, kbar_lp, vbar_lp, k_keep: int, n_force: int = 0, O=None, kept_mask=None,
                      density=None, workspace=None, stream=None):
    """Fused forward with fixed-sparsity routing: each query block keeps its k_keep highest-scoring
    key blocks (bf16, blocks of 128). Returns O."""
    _need_cuda("Q", Q, torch.bfloat16)
    for n, t in (("K", K), ("V", V)):
        _need_cuda(n, t, torch.bfloat16)
    B, H, L, d = Q.shape
    if K.shape != Q.shape or V.shape != Q.shape:
        raise ValueError("Q, K and V must have the same shape [B, H, L, d]")
    if O is None:
        O = torch.empty_like(Q)
    if workspace is None:
        workspace = new_workspace(B, H, L, 128, Q.device)
    st = load_library().sol_attn_fwd_topk(
        _ptr(Q), _ptr(K), _ptr(V), _ptr(kbar), _ptr(kbar_lp), _ptr(vbar_lp), int(k_keep), B, H, L, d, int(n_force),
        _ptr(O), _ptr(kept_mask), _ptr(density), _ptr(workspace), workspace.numel(), _stream(stream))
    _check(st, "sol_attn_fwd_topk")
    return O


def sol_attn_fwd_qbar(Q, K, V, kbar, vbar, kbar_lp, vbar_lp, qbar, tau, n_force: int = 0, O=None, kept_mask=None,
                      density=None, workspace=None, stream=None):
    """Fused forward whose routing pass takes the query-block means qbar (fp32 [B, H, N_qb, d],
    from sol_attn_qknorm_rope_pool(..., want_qbar=True)) instead of reading Q for them (bf16,
    blocks of 128). Returns O."""
    _need_cuda("Q", Q, torch.bfloat16)
    for n, t in (("K", K), ("V", V)):
        _need_cuda(n, t, torch.bfloat16)
    _need_cuda("qbar", qbar, torch.float32)
    B, H, L, d = Q.shape
    if K.shape != Q.shape or V.shape != Q.shape:
        raise ValueError("Q, K and V must have the same shape [B, H, L, d]")
    if tuple(qbar.shape) != (B, H, -(-L // 128), d):
        raise ValueError("qbar must be [B, H, ceil(L/128), d]")
    tau = [float(x) for x in tau]
    if len(tau) != H:
        raise ValueError(f"tau must hold H={H} values")
    tau_arr = (ctypes.c_float * H)(*tau)
    if O is None:
        O = torch.empty_like(Q)
    if workspace is None:
        workspace = new_workspace(B, H, L, 128, Q.device)
    st = load_library().sol_attn_fwd_qbar(
        _ptr(Q), _ptr(K), _ptr(V), _ptr(kbar), _ptr(vbar), _ptr(kbar_lp), _ptr(vbar_lp), _ptr(qbar), tau_arr, B, H, L,
        d, int(n_force), _ptr(O), _ptr(kept_mask), _ptr(density), _ptr(workspace), workspace.numel(), _stream(stream))
    _check(st, "sol_attn_fwd_qbar")
    return O


def sol_attn_quantize_v8(V, vbar, stream=None):
    """8-bit PV values (d = 128, blocks of 128): returns (v8t, vbar8t, v_scale), the E4M3 codes of V
    and of the pooled values vbar with one scale amax_c / 448 per channel, stored transposed
    ([B, H, d, N_kb * 128] and [B, H, d, 128 * ceil(N_kb / 128)], uint8)."""
    _need_cuda("V", V, torch.bfloat16)
    _need_cuda("vbar", vbar, torch.float32)
    B, H, L, d = V.shape
    nkb = -(-L // 128)
    if tuple(vbar.shape) != (B, H, nkb, d):
        raise ValueError("vbar must be [B, H, ceil(L/128), d]")
    dev = V.device
    v8t = torch.empty((B, H, d, nkb * 128), dtype=torch.uint8, device=dev)
    vbar8t = torch.empty((B, H, d, -(-nkb // 128) * 128), dtype=torch.uint8, device=dev)
    v_scale = torch.empty((B, H, d), dtype=torch.float32, device=dev)
    st = load_library().sol_attn_quantize_v8(_ptr(V), _ptr(vbar), B, H, L, d, _ptr(v8t), _ptr(vbar8t),
                                             _ptr(v_scale), _stream(stream))
    _check(st, "sol_attn_quantize_v8")
    return v8t, vbar8t, v_scale


def sol_attn_fwd_8bit(Q, q8, k8, kbar8, q_scale, k_scale, kbar_scale, v8t, vbar8t, v_scale, kbar, tau,
                      n_force: int = 0, O=None, kept_mask=None, density=None, workspace=None, stream=None):
    """Fused forward with 8-bit kept tiles and correction: int8 QK^T (sol_attn_quantize_qk8) and E4M3
    PV (sol_attn_quantize_v8); routing from the bf16 Q and the fp32 pooled keys. Returns O (bf16)."""
    _need_cuda("Q", Q, torch.bfloat16)
    B, H, L, d = Q.shape
    tau = [float(x) for x in tau]
    if len(tau) != H:
        raise ValueError(f"tau must hold H={H} values")
    tau_c = (ctypes.c_float * H)(*tau)
    if O is None:
        O = torch.empty_like(Q)
    if workspace is None:
        workspace = new_workspace(B, H, L, 128, Q.device)
    st = load_library().sol_attn_fwd_8bit(
        _ptr(Q), _ptr(q8), _ptr(k8), _ptr(kbar8), _ptr(q_scale), _ptr(k_scale), _ptr(kbar_scale), _ptr(v8t),
        _ptr(vbar8t), _ptr(v_scale), _ptr(kbar), tau_c, B, H, L, d, int(n_force), _ptr(O), _ptr(kept_mask),
        _ptr(density), _ptr(workspace), workspace.numel(), _stream(stream))
    _check(st, "sol_attn_fwd_8bit")
    return O


def sol_attn_check_device_error(workspace: torch.Tensor, stream=None) -> None:
    """Synchronise and raise SolAttnError(SOL_ETIMEOUT) if a bounded device wait expired."""
    _check(load_library().sol_attn_check_device_error(_ptr(workspace), _stream(stream)),
           "sol_attn_check_device_error")


def sol_attn_debug_drop_one_load(mode: int) -> None:
    load_library().sol_attn_debug_drop_one_load(int(mode))


def sol_attn_debug_record_cta_times(times: torch.Tensor, capacity: int) -> None:
    """Arm the next bf16 fused launch to write each CTA's (start, finish) globaltimer stamps into
    `times` (int64 device tensor of at least 2 * capacity elements)."""
    _need_cuda("times", times, torch.int64)
    if times.numel() < 2 * capacity:
        raise ValueError("times must hold 2 * capacity values")
    load_library().sol_attn_debug_record_cta_times(_ptr(times), int(capacity))


def sol_attn(Q, K, V, tau, block: int = 128, n_force: int = 0, want_mask: bool = False,
             want_density: bool = False, workspace=None, stream=None):
    """The whole path for one call: pool K/V, then the fused forward.

    Returns (O, kept_mask or None, density or None).
    """
    B, H, L, d = Q.shape
    kbar, vbar, kbar_lp, vbar_lp = sol_attn_pool(K, V, block, stream=stream)
    nb = -(-L // block)
    mask = torch.empty((B, H, nb, nb), dtype=torch.uint8, device=Q.device) if want_mask else None
    dens = torch.empty((B, H), dtype=torch.float32, device=Q.device) if want_density else None
    O = sol_attn_fwd(Q, K, V, kbar, vbar, kbar_lp, vbar_lp, tau, block, block, n_force, kept_mask=mask,
                     density=dens, workspace=workspace, stream=stream)
    return O, mask, dens


def sol_attn_fwd_host_scratch_bytes(dtype: torch.dtype, B: int, H: int, L: int, d: int, block: int,
                                    heads_per_chunk: int) -> int:
    code = SOL_BF16 if dtype == torch.bfloat16 else SOL_F32 if dtype == torch.float32 else -1
    return int(load_library().sol_attn_fwd_host_scratch_bytes(code, B, H, L, d, block, heads_per_chunk))


def default_heads_per_chunk(H: int) -> int:
    """About 20 chunks per batch entry: the pipeline fills after one small upload."""
    return max(1, -(-H // 20))


def sol_attn_fwd_host(Q, K, V, tau, block: int = 128, n_force: int = 0, heads_per_chunk: Optional[int] = None,
                      O=None, want_density: bool = False, scratch=None, stream=None):
    """The whole path (pool + forward) on HOST tensors, pipelined by head chunks through device
    scratch. Synchronous: returns (O, density or None) with both in host memory.

    Q, K, V: CPU tensors [B, H, L, d] (pinned for copy/compute overlap). `scratch`: a CUDA uint8
    tensor of at least sol_attn_fwd_host_scratch_bytes(...) bytes on the current device.
    """
    for n, t in (("Q", Q), ("K", K), ("V", V)):
        if not isinstance(t, torch.Tensor) or t.device.type != "cpu":
            raise TypeError(f"{n} must be a CPU tensor")
        if not t.is_contiguous():
            raise ValueError(f"{n} must be contiguous")
        if t.dtype != Q.dtype or t.shape != Q.shape:
            raise ValueError("Q, K and V must have the same dtype and shape [B, H, L, d]")
    B, H, L, d = Q.shape
    dt = _dtype_code(Q)
    tau = [float(x) for x in tau]
    if len(tau) != H:
        raise ValueError(f"tau must hold H={H} values")
    c = default_heads_per_chunk(H) if heads_per_chunk is None else int(heads_per_chunk)
    pinned = Q.is_pinned()
    if O is None:
        O = torch.empty(Q.shape, dtype=Q.dtype, pin_memory=pinned)
    elif O.device.type != "cpu" or not O.is_contiguous() or O.dtype != Q.dtype or O.shape != Q.shape:
        raise ValueError("O must be a contiguous CPU tensor of Q's dtype and shape")
    dens = torch.empty((B, H), dtype=torch.float32, pin_memory=pinned) if want_density else None
    if scratch is None:
        scratch = torch.empty(sol_attn_fwd_host_scratch_bytes(Q.dtype, B, H, L, d, block, c), dtype=torch.uint8,
                              device=torch.device("cuda", torch.cuda.current_device()))
    else:
        _need_cuda("scratch", scratch, torch.uint8)
    tau_c = (ctypes.c_float * H)(*tau)
    st = load_library().sol_attn_fwd_host(
        _ptr(Q), _ptr(K), _ptr(V), _ptr(O), tau_c, dt, B, H, L, d, block, int(n_force), c, _ptr(dens),
        _ptr(scratch), scratch.numel(), _stream(stream))
    _check(st, "sol_attn_fwd_host")
    return O, dens


def tau_list(values) -> list:
    """Turn a JSON-style tau list ("inf" strings allowed) into floats."""
    return [math.inf if (isinstance(v, str) and v.lower() == "inf") else float(v) for v in values]
