"""B200-native Hierarchical Global Attention (HGA) layer.

The compute lives in ``libhga.so`` (hand-written sm_100a CUDA, C ABI in
include/hga.h); this package is its ctypes binding and the in-tree build
script (``build.py``).
"""
from .binding import (  # noqa: F401
    HGA_BF16, HGA_FP32, HGA_DEV_BAD_INDEX, HGA_DEV_TIMEOUT, HGA_DEV_STAGE_FULL, HGA_TIER_RESET, HGA_TIER_CHAIN,
    EXPORTED, HGAError, Params, TierSched, lib,
    hga_build_summaries, hga_route, hga_route_causal, hga_route_groups, hga_route_groups_tiered, hga_attn_fwd,
    hga_route_attn_fwd,
    hga_attn_bwd_workspace_size,
    hga_attn_bwd, hga_attn_bwd_noalloc, hga_attn_decode_workspace_size, hga_attn_decode,
    hga_attn_fwd_groups, hga_attn_bwd_groups, hga_attn_causal_workspace_size, hga_attn_fwd_causal,
    hga_attn_bwd_causal,
    hga_tier_scratch_size, hga_tier_reset, hga_fetch_tiered, hga_tier_offload, hga_attn_fwd_tiered,
    hga_segment_fwd_tiered, hga_segment_fwd,
    hga_get_device_status, hga_selftest_wait_timeout,
)
