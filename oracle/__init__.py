"""CPU fp64 oracle of the chunked H2O attention step.

Test infrastructure only: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline legs of ``bench.py``; never by the product path.
"""
from .h2o_oracle import (OracleCache, Placement, attention_one_cache,  # noqa: F401
                         bf16_round, dequantize_q8, evict_one_head, gap_at_boundary,
                         kv_head_of, quantize_row_q8, visible_mask)
