"""B200-native R-SWA / SR-SWA decode attention.

The compute lives in ``librswa.so`` (hand-written CUDA for sm_100a behind the
C ABI of ``include/rswa.h``); this package is its Python binding plus the
seeded synthetic-input generators. There is no CPU fallback.
"""
from .binding import (  # noqa: F401
    EXPORTED, LIB_PATH, OP_DECODE, OP_PREFILL, OP_ROUTE, OP_SRSWA_DECODE, OP_SRSWA_ROUTED, Dims, RswaError, check_status, dims_of,
    fp8_prefix_buffers, fp8_ring_buffers, load, new_workspace, route_workspace, rswa_append, rswa_append_fp8,
    rswa_append_rope, rswa_decode, rswa_decode_append, rswa_decode_fp8, rswa_decode_fp8kv, rswa_prefill,
    rswa_rope_page2d, srswa_decode_fp8kv,
    rswa_quantize_prefix, srswa_decode, srswa_decode_append, srswa_decode_fp8, srswa_index_pool, srswa_prefill,
    srswa_route,
    srswa_route_tokens, test_arm_wait_timeout, workspace_bytes, srswa_decode_routed, srswa_step,
    srswa_prefill_workspace, rswa_decode_append_rope, srswa_step_rope,
)

__all__ = ["load", "Dims", "RswaError", "rswa_append", "rswa_decode", "rswa_prefill", "srswa_index_pool", "srswa_route",
           "srswa_decode", "rswa_quantize_prefix", "rswa_decode_fp8", "srswa_decode_fp8", "fp8_prefix_buffers",
           "srswa_route_tokens", "srswa_prefill", "rswa_decode_append", "srswa_decode_append",
           "rswa_rope_page2d", "rswa_append_rope", "rswa_append_fp8", "rswa_decode_fp8kv", "srswa_decode_fp8kv",
           "fp8_ring_buffers", "test_arm_wait_timeout", "srswa_decode_routed", "srswa_step",
           "srswa_prefill_workspace", "rswa_decode_append_rope", "srswa_step_rope",
           "workspace_bytes", "new_workspace", "route_workspace", "check_status", "dims_of"]
