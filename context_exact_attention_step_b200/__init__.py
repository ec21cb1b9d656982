"""B200 (sm_100a) context-parallel exact attention: ring-step block attention
with partial (O, LSE), fp32 LSE merge, zigzag and striped reorders, Ulysses
sequence<->head transpose and the Ulysses-inside / Ring-across hybrid, with P
virtual ranks on one GPU.

The compute lives in ``libcp_attn.so`` (C ABI in ``include/cp_attn.h``);
``api`` is a thin PyTorch binding over it.
"""
from .api import (  # noqa: F401
    attn_bwd_prep,
    block_attn_bwd,
    block_attn_fwd,
    count_live_pairs,
    device_error,
    kernel_launch_count,
    set_profile_events,
    striped_reorder,
    lse_merge,
    ring_attn_bwd,
    ring_attn_bwd_workspace_size,
    ring_attn_fwd,
    ring_attn_workspace_size,
    ring_schedule,
    ulysses_attn_bwd,
    ulysses_attn_fwd,
    ulysses_attn_workspace_size,
    ulysses_permute,
    usp_attn_bwd,
    usp_attn_fwd,
    usp_attn_workspace_size,
    zigzag_reorder,
)

__version__ = "0.1.0"
