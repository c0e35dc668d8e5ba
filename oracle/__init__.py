"""CPU oracle of the Lighthouse selection layer: test infrastructure, never the product path.

Only the tests, the smoke check and the benchmark's CPU-baseline leg import this package.
"""
from .lighthouse_ref import (Geometry, attn_bwd, attn_fwd, build_pyramid, gather, gather_bwd,
                             layer_bwd, layer_fwd, pool_stored, round_to, row_norm_f32, scatter, scatter_bwd,
                             score, select_topk)

__all__ = ["Geometry", "attn_bwd", "attn_fwd", "build_pyramid", "gather", "gather_bwd",
           "layer_bwd", "layer_fwd", "pool_stored", "round_to", "row_norm_f32", "scatter", "scatter_bwd", "score",
           "select_topk"]
