"""Float64 CPU oracle (test infrastructure only; see attention_f64's header).

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline / reference
arm may import it. It shares no code with the CUDA library.
"""
from .attention_f64 import (  # noqa: F401
    backward, backward_blocked, backward_head, backward_head_with_shift, backward_row_block,
    block_mask_keep, causal_pair_count, forward, forward_head, keep_mask, key_tail, query_rows,
)
from .mha_layer_f64 import layer as mha_layer  # noqa: F401,E402
from .double_backward_f64 import double_backward, double_backward_head  # noqa: F401,E402
