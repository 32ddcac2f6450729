"""CPU oracle of the PBSA hot path (test infrastructure; see pbsa_oracle)."""
from .pbsa_oracle import *  # noqa: F401,F403
from .pbsa_oracle import (EVICT, MERGE_MEAN, MASK_CHUNK, MASK_TOKEN, round_bf16, round_storage,
                          query_block_lengths, pool_queries, pool_keys, block_scores,
                          memory_scores, score_blocks, update_memory, select_local,
                          lists_to_arrays, attention_fwd, attention_bwd)
