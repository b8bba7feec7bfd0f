"""CPU oracle of the Sol-Attn forward. TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import
this package. The CUDA library never calls it.
"""
from .sol_attn_oracle import (  # noqa: F401
    BAND,
    adopt_in_band,
    band_mask,
    block_counts,
    forward,
    forward_head,
    pool_blocks,
    proxy_error_bound,
    proxy_scores,
    route,
    routing_violations,
    unit_forward,
    unit_terms,
)
from .qknorm_rope_oracle import qknorm_rope_pool_head, rms_norm, rope  # noqa: F401
from .mxfp8_oracle import (  # noqa: F401
    channel_scales,
    e4m3_channel_quantize,
    e4m3_plain,
    forward_head_mx,
    int8_quantize_tiles,
    mx_quantize,
    no_quantize,
    round_e4m3,
    round_mantissa,
)
from .topk_routing_oracle import forward_head_topk, keep_count, route_topk  # noqa: F401
from .taylor_correction_oracle import cross_moments, forward_head_taylor, unit_forward_taylor  # noqa: F401
