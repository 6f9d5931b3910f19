"""fp64 CPU oracle (test infrastructure; never imported by the product path)."""
from .arl2_oracle import (  # noqa: F401
    NORM_EPS, Layer, attention_matrix, feature_map, frame_commit, frame_commit_gated, frame_query,
    frame_commit_token, frame_query_token, gates_from_hidden, intra_attention, kv_cache_attention,
    l2_normalize_rows, readout, softmax_rows, token_level_scan,
)
