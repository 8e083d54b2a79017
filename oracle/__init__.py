"""CPU oracle for the token-sparse decode step (test infrastructure only).

Plain float64 numpy restatement of what the decode step computes.  Only the
tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline and
reference legs may import it; the product path never does.
"""

from .reference import (  # noqa: F401
    ROLE_SPARSE,
    ROLE_DENSE,
    ROLE_STREAM,
    rope,
    dominant_dims,
    tip_scores,
    select_top,
    attend,
    focused_attention,
    stream_positions,
    dense_positions,
    decode_row,
    decode_step,
    shared_index_step,
    tie_band,
    ring_slot,
    ring_contents,
    to_bf16_bits,
    bf16_bits_to_f64,
    append_token_rows,
    pack_dominant_row,
    rest_dims,
    head_rows,
    qk_kernel,
    proxy_matrix,
    proxy_singular_values,
    effective_rank,
    head_effective_ranks,
    group_effective_ranks,
    classify_heads,
    tie_band_check,
)
