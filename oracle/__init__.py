"""fp64 CPU oracle for the DSA forward path and its training-stage gradients
(test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package; the CUDA library never does.
"""
from .dsa_oracle import (  # noqa: F401
    e4m3_table, decode_e4m3, decode_bf16, to_f64, index_scores, topk_select,
    sparse_mla, dense_causal_mqa, forward_rows, numpy_inputs, indexer_kl_target,
    index_scores_dequantised, indexer_kl_score_grad, sparse_mla_backward, indexer_backward,
)
