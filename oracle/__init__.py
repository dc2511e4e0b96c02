"""CPU oracle for the sparse decode path (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline and
reference legs import this package; the library never does.
"""
from .sd_oracle import (  # noqa: F401
    attend_rows,
    bf16_bits_to_f64,
    decode_step,
    dense_attention,
    expand_csr,
    gather_token_rows,
    indexer_scores,
    sparse_attention,
    sparse_attention_csr,
    topk_indices,
    topk_row,
)
from .tri_oracle import PER_HEAD as TRI_PER_HEAD  # noqa: F401
from .tri_oracle import UNION as TRI_UNION  # noqa: F401
from .tri_oracle import PER_LAYER_PER_HEAD as TRI_PER_LAYER_PER_HEAD  # noqa: F401
from .tri_oracle import tri_compact, tri_evict, tri_evict_layers, tri_logits, tri_scores, tri_select  # noqa: F401
