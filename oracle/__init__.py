"""Plain, slow, obviously-correct CPU oracle for the head-weighted ReLU indexer.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or
execute anything in this package: only the test suite, the package smoke check
and the CPU-baseline leg of the benchmark use it.  It shares no code with the
CUDA path (no kernels, headers, helpers, tables or constants); the two meet
only through the seeded input generators, which hold none of the method's
arithmetic.

All floating point here is IEEE binary64.  Every function names the passage
of the source pages that it follows.
"""

from .indexer_oracle import (  # noqa: F401
    TOKEN,
    COMPRESSED,
    POOLED,
    decode_bf16,
    decode_e4m3,
    round_to_bf16_bits,
    visible_keys,
    incomplete_tail,
    pooled_keys,
    score_keys,
    select_topk,
    out_width,
    topk_rows,
    topk_rows_docs,
    topk_rows_padded,
    witness_seed_keys,
    witness_threshold,
    decode_keys_for,
    pair_shared_counts,
    pair_regions,
)
