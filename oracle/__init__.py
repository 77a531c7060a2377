"""fp64 CPU oracle for RecSA (test infrastructure only; see recsa_oracle)."""
from .recsa_oracle import (  # noqa: F401
    build_tree, pool_level, pool_alpha, round_bf16, round_f32, storage_round,
    rope, rope_theta, level_logits, select_and_attend, list_sizes, is_near_tie,
    NEAR_TIE_REL, NEAR_TIE_ABS, LevelTrace, QueryResult,
)
