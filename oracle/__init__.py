"""CPU oracle of the RTPurbo inference path (test infrastructure only).

Importable by the test-suite, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` -- never by the product path.
"""
from .rtp_oracle import (  # noqa: F401
    D_IDX, INDEXER_SCALE, LayerOracle, QueryResult, Selection, attend, attend_lse, combine_partials,
    index_project,
    indexer_scores, local_query, needle_recall, retrieval_query, round_bf16, round_storage,
    topk_select, topp_select, window_keys,
)
