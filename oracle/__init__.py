"""fp64 CPU oracle (test infrastructure only; see bsa_oracle.py's header)."""

from .bsa_oracle import (  # noqa: F401
    BLOCK, VARIANTS, block_bounds, pooled_means, video_query_anchor,
    block_summaries, block_scores, select_blocks, attend, forward_head, forward,
    effective_pairs,
)
