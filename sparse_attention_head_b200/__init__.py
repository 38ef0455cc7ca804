"""Elastic Attention prefill hot path for B200 (sm_100a).

A per-head Attention Router (mean-pooled keys -> two-layer MLP -> hard
threshold) routes each (batch, head) to full causal attention or to
streaming sparse attention (sink + local window); one fused tcgen05 kernel
computes both kinds of heads in a single launch.  All compute runs in
libea.so; this package only marshals arguments.
"""
from ._lib import (EA_OK, EA_ERR_CUDA, EA_ERR_INVALID_ARG, EA_ERR_MISALIGNED,  # noqa: F401
                   EA_ERR_TIMEOUT, EA_ERR_UNSUPPORTED, EA_ERR_WORKSPACE, EA_SELECT_ALL,
                   EA_SELECT_FA, EA_SELECT_SA, EaAttnParams, EaError, LIB_PATH)
from .api import (HostPrefill, attn_workspace, decode_workspace, ea_decode_kv_policy,  # noqa: F401
                  ea_hybrid_attn_decode, make_decode_params, ea_attn_grid_size, ea_get_device_status,  # noqa: F401
                  ea_hybrid_attn_prefill, ea_hybrid_attn_workspace_size, ea_router_decide,
                  ea_router_workspace_size, ea_schedule_unit_tiles, ea_schedule_units,
                  make_params, ea_hybrid_attn_prefill_varlen, ea_schedule_units_varlen,
                  make_varlen_params, ea_router_decide_varlen, ea_hybrid_attn_prefill_routed,
                  ea_hybrid_attn_prefill_varlen_routed, ea_hybrid_attn_prefill_lse,
                  ea_hybrid_attn_backward, ea_router_decide_gumbel, ea_router_ste_backward,
                  ea_hybrid_attn_prefill_train, ea_quantize_fp8, ea_hybrid_attn_prefill_fp8,
                  ea_fp8_vt_stride)
from .flops import attn_visible_pairs, effective_flops, tile_flops  # noqa: F401
