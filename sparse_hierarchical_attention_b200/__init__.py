"""Lighthouse selection layer on NVIDIA B200 (sm_100a).

The layer pools Q, K and V into an L-level pyramid, scores every cell with max-pooled l2 norms,
keeps a stratified top-K per chunk (always with the chunk's coarsest cell), runs dense causal
attention on the S gathered rows and scatters the outputs back to the tokens. Source: "Long
Context Pre-Training with Lighthouse Attention" (gist.science summary), technical summary
sections 2.A-2.C. All arithmetic runs in the CUDA kernels of liblh.so (include/lh.h); this
package only allocates device memory through PyTorch and marshals arguments.
"""
from ._lib import (LighthouseError, Shape, lh_attn_bwd, lh_attn_fwd, lh_build_pyramid,
                   lh_check, lh_gather, lh_gather_bwd, lh_launches, lh_layer_bwd, lh_layer_fwd,
                   lh_saved_bytes, lh_saved_offsets, lh_scatter, lh_scatter_bwd, lh_score,
                   lh_select_topk, lh_set_wait_limit_ns, lh_validate, lh_version,
                   lh_workspace_bytes, lh_workspace_init)
from .layer import LighthouseAttention, LighthouseLayer, saved_views

__all__ = [
    "LighthouseAttention", "LighthouseError", "LighthouseLayer", "Shape", "lh_attn_bwd",
    "lh_attn_fwd", "lh_build_pyramid", "lh_check", "lh_gather", "lh_gather_bwd",
    "lh_launches", "lh_layer_bwd", "lh_layer_fwd", "lh_saved_bytes", "lh_saved_offsets", "lh_scatter",
    "lh_scatter_bwd", "lh_score", "lh_select_topk", "lh_set_wait_limit_ns", "lh_validate", "lh_version",
    "lh_workspace_bytes", "lh_workspace_init", "saved_views",
]
