"""CPU oracle of the Lighthouse selection layer: test infrastructure, never the product path.

Only the tests, the smoke check and the benchmark's CPU-baseline leg import this package.
"""
from .lighthouse_ref import (Geometry, attn_bwd, attn_fwd, build_pyramid, gather, gather_bwd,
                             kv_head_of, layer_bwd, layer_fwd, pool_stored, round_to, row_norm_f32,
                             scatter, scatter_bwd, score, select_topk)

__all__ = ["Geometry", "attn_bwd", "attn_fwd", "build_pyramid", "gather", "gather_bwd",
           "kv_head_of", "layer_bwd", "layer_fwd", "pool_stored", "round_to", "row_norm_f32",
           "scatter", "scatter_bwd", "score", "select_topk"]

# The same operations under the C ABI's names (lh_<stage> -> lh_ref_<stage>), on host arrays.
lh_ref_build_pyramid = build_pyramid
lh_ref_score = score
lh_ref_select_topk = select_topk
lh_ref_gather = gather
lh_ref_attn_fwd = attn_fwd
lh_ref_attn_bwd = attn_bwd
lh_ref_scatter = scatter
lh_ref_scatter_bwd = scatter_bwd
lh_ref_gather_bwd = gather_bwd
lh_ref_layer_fwd = layer_fwd
lh_ref_layer_bwd = layer_bwd
__all__ += [n for n in dir() if n.startswith("lh_ref_")]
