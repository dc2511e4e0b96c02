"""Top-k sparse decode attention over a paged KV cache, for NVIDIA B200 (sm_100a).

The computation lives in ``libsd.so`` (hand-written CUDA kernels behind the C
ABI of ``include/sd_api.h``); this package is a thin ctypes binding over it
plus the seeded synthetic-input generator used by tests and benchmarks.
"""
from .api import (  # noqa: F401
    EXPORTED,
    NOALLOC_MAX_SCORES,
    SD_DEVERR_INDEX,
    SD_DEVERR_PAGE,
    SD_DEVERR_SEQLEN,
    SD_DEVERR_TIMEOUT,
    SdError,
    TRI_PER_HEAD,
    TRI_PER_LAYER_PER_HEAD,
    TRI_UNION,
    StageTimer,
    alloc_workspace,
    device_errors,
    last_launch_count,
    load_library,
    sd_decode_step,
    sd_decode_step_hinted,
    sd_indexer_topk,
    sd_indexer_topk_hinted,
    sd_indexer_topk_noalloc,
    sd_sparse_attn,
    sd_sparse_attn_csr,
    sd_sparse_attn_layers,
    sd_tri_compact,
    sd_tri_compact_layers,
    set_wait_limit,
    workspace_size,
)

__all__ = [
    "sd_indexer_topk", "sd_indexer_topk_hinted", "sd_indexer_topk_noalloc", "sd_decode_step_hinted", "sd_sparse_attn", "sd_sparse_attn_layers", "sd_sparse_attn_csr",
    "sd_decode_step", "sd_tri_compact", "sd_tri_compact_layers", "TRI_UNION", "TRI_PER_HEAD",
    "TRI_PER_LAYER_PER_HEAD",
    "workspace_size", "alloc_workspace", "device_errors", "set_wait_limit", "load_library", "SdError", "StageTimer",
]
