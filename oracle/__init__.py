"""fp64 CPU oracle for the spacetime-attention hot path.

TEST INFRASTRUCTURE ONLY: imported by the test suite, ``__graft_entry__.smoke()`` and the
CPU-baseline legs of ``bench.py``.  The CUDA library neither imports nor calls it.
"""

from .spacetime_oracle import (  # noqa: F401
    SKIP_GROUP,
    SKIP_SINGLE,
    attention_head_backward_ref,
    attention_head_backward_rows_ref,
    attention_head_lse_ref,
    attention_head_ref,
    attn_backward_ref,
    attn_ref,
    cross_attn_ref,
    default_scale,
    frame_causal_attn_ref,
    frame_causal_backward_ref,
    frame_causal_limit,
    packed_attn_ref,
    packed_backward_ref,
    rope3d_packed_ref,
    rope3d_positions_ref,
    rope3d_ref,
    rope_frequencies,
    round_to_bf16,
    segment_bounds,
    skiparse_attn_ref,
    skiparse_backward_ref,
    skiparse_gather_ref,
    skiparse_index_map,
    skiparse_scatter_ref,
    skiparse_sets,
    skiparse_text_attn_ref,
    skiparse_text_backward_ref,
    skiparse_text_backward_rows_ref,
    softmax_rows,
    spatial_attn_ref,
    spatial_backward_ref,
    temporal_attn_ref,
    temporal_backward_ref,
    video_positions,
)
