"""CPU oracle (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg import this
package. It computes, slowly and in fp64, what the jagged candidate-isolated attention path
computes, restating the source pages' rules; it imports nothing from the CUDA package.
"""

from . import jagged_oracle, brute, rope, stack, backward, variants, ug_sep, seqpack  # noqa: F401
from .jagged_oracle import (  # noqa: F401
    offsets_from_lengths,
    split_by_offsets,
    packing_counts,
    attention_segment_ids,
    segment_ids,
    bounds_from_segment_ids,
    history_candidate_mask,
    masked_softmax_attention,
    jagged_cand_attn,
    jagged_cand_attn_rows,
    cand_only_attn,
    allowed_pairs,
    work_items,
    SEG_HISTORY,
    SEG_CANDIDATE,
    SEG_PADDING,
)
from .rope import (  # noqa: F401
    right_anchored_positions,
    rope_inverse_frequencies,
    apply_rope,
    cand_only_positions,
    round_to_bf16,
)
