"""fp64 CPU oracle (test infrastructure only; never on the product path)."""
from .sparsed_oracle import *  # noqa: F401,F403
from .sparsed_oracle import (DENSE, SELECT, SPARSE, block_mass, dense_attention,  # noqa: F401
                             entropy_budget, head_entropy, kept_keys, largest_remainder,
                             masked_attention, n_blocks, run_steps, schedule,
                             select_pattern, softmax_attention, topk_blocks,
                             uniform_keep)
