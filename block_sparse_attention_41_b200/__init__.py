"""Sol-Attn block-sparse attention forward for NVIDIA B200 (sm_100a).

The compute path lives in the C-ABI shared library ``libsolattn.so`` (CUDA kernels under
``csrc/``); :mod:`.sol_attn` is the thin ctypes binding with the same call names, including the
host-buffer entry point ``sol_attn_fwd_host``. :mod:`.context_parallel` runs one token-sharded
sequence over several GPUs (head-sharded by all-to-all, the single-GPU path per head group).
:mod:`.workloads` draws the seeded synthetic inputs and does not touch the library.
"""
