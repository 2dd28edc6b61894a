"""Float64 CPU oracle of the sparse+linear attention layer.

TEST INFRASTRUCTURE: only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference leg of ``bench.py`` may import this package. It shares
no code with the CUDA path.
"""
from .sla_oracle import (CRITICAL, MARGINAL, NEGLIGIBLE, TIE_REL, Layer, OracleCfg,  # noqa: F401
                         block_order, classify_threeway, combine, forward, linear_attention,
                         linear_states, phi, pool_blocks, pooled_scores, select_topn, sigmoid,
                         softmax, softmax_attention, threeway_tie_rows)
