"""Float64 CPU oracle for HCA (test infrastructure only; see hca_oracle)."""

from .hca_oracle import (  # noqa: F401
    attend_position,
    compress_blocks,
    compressed_entry_count,
    hca_decode,
    hca_prefill,
    mask_table,
    visible_compressed_count,
    visible_pairs,
    window_bounds,
)
