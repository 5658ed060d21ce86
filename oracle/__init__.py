"""fp64 CPU oracle - test infrastructure only (tests, smoke check, CPU baseline).

The product path never imports this package.
"""
from .oracle import _f64
from .oracle import (window_scores, chunk_keys, chunk_scores, top_b, mass_count,
                     local_indices, special_indices, full_indices, chunk_select,
                     allocate_budgets, layout, compact, append, decode_attention,
                     retained_mass, attention_loss, profile_head, chunk_select_local, icac_decode,
                     sliding_local_indices)
from .pipeline import run_workload, OracleResult

__all__ = ["window_scores", "chunk_keys", "chunk_scores", "top_b", "mass_count",
           "local_indices", "special_indices", "full_indices", "chunk_select",
           "allocate_budgets", "layout", "compact", "append", "decode_attention",
           "retained_mass", "attention_loss", "profile_head", "chunk_select_local", "icac_decode",
           "sliding_local_indices",
           "run_workload", "OracleResult"]
