"""CPU fp64 oracle for block-sparse top-k attention (pool -> score -> top-k -> attention).

TEST INFRASTRUCTURE ONLY.  Only `tests/`, `__graft_entry__.smoke()` and `bench.py`'s
CPU-baseline / reference leg may import this package.  The product path (the CUDA
library and its Python binding) never imports, calls or falls back to it.

It shares no code with the CUDA path: it is plain numpy in float64, written step by
step from the method's definition (see `msa_oracle.py` for the citations), slow on
purpose, and checked against pins that come from outside itself (tests/test_oracle_*).
"""
from .msa_oracle import (  # noqa: F401
    pool_keys, group_query_sum, prefill_block_scores, select_prefill_row,
    select_decode_row, attend_row, prefill_rows, decode_rows, PrefillRow, DecodeRow,
    rel_gap, prefill_keys_of, decode_keys_of,
)
from .msa_sharded import (  # noqa: F401
    shard_blocks, local_candidates, merge_candidates, attend_owned, merge_partials,
    decode_rows_sharded,
)
from .msa_backward import attend_row_backward, prefill_backward  # noqa: F401
from .msa_docs import doc_positions, prefill_varlen_rows, rope_angles, rope_docwise  # noqa: F401
