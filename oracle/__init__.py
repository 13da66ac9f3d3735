"""fp64 CPU oracle (test infrastructure only; never on the product path).

Only the tests, the package smoke check and the benchmark's CPU-baseline leg
may import this package.
"""
from .ssa_oracle import (  # noqa: F401
    attention_probs,
    block_summary,
    decode,
    decode_append,
    decode_route,
    pool_query_blocks,
    route,
    select_topk,
    sparse_attention,
    sparse_attention_backward,
    summary_scores,
)
from .dash_oracle import (  # noqa: F401
    entmax,
    entmax_route,
    learned_block_summary,
    prior_sparse_attention,
)
from .hier_oracle import (  # noqa: F401
    decode_per_head,
    decode_route_per_head,
    hierarchical_route,
    segment_summaries,
)
from .paged_oracle import (  # noqa: F401
    decode_append_paged,
    decode_paged,
    gather_pages,
)
