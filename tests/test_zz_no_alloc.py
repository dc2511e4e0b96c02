"""The allocation-free indexer + top-k entry point, through the C ABI.

sd_indexer_topk_noalloc serves callers that cannot allocate device memory (a
plugin inside an application that owns every device allocation, or a serving
loop that must not allocate after start-up): it keeps the scores in a fixed
scratch array inside the library instead of a caller workspace. It must give
exactly the indices of sd_indexer_topk (the tolerance for indices is zero), on
two calls in a row with different inputs, since the scratch array keeps the
previous call's contents. This file is collected last on purpose.
"""
import numpy as np
import pytest

from top_sparse_decode_paged_b200 import workloads as W

from helpers import to_device

pytestmark = pytest.mark.gpu


def _both(spec):
    import torch
    import top_sparse_decode_paged_b200 as sd
    wl = W.make(spec)
    d = to_device(wl)
    B, G, k, L = wl.seqlens.shape[0], spec.G, spec.k, wl.max_seqlen
    ref = sd.sd_indexer_topk(d["qi"], d["w"], d["ki_pages"], d["block_table"], d["seqlens"], k, L,
                             workspace=sd.alloc_workspace(B, G, L, k, G, 1))
    got = torch.full((B, G, k), -7, dtype=torch.int32, device="cuda")
    sd.sd_indexer_topk_noalloc(d["qi"], d["w"], d["ki_pages"], d["block_table"], d["seqlens"], k, L, got)
    torch.cuda.synchronize()
    return got.cpu().numpy(), ref.cpu().numpy()


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    import top_sparse_decode_paged_b200 as sd
    sd.device_errors(clear=True)
    # first call: long rows; second call: shorter, ragged rows and another
    # head layout, so that stale scores from the first call would show up
    got1, ref1 = _both(W.spec("b4_l4096_mla", seqlens=(4096, 3001, 2049, 700), seed=31))
    got2, ref2 = _both(W.spec("perhead_b16_gqa", seqlens=(3000, 1500, 5000), seed=32))
    assert np.array_equal(got1, ref1)
    assert np.array_equal(got2, ref2)
    assert sd.device_errors() == 0


def test_noalloc_limit_is_on_scratch_size():
    """B * G * max_seqlen at the limit runs; one token per row more is rejected
    with SD_ERR_WORKSPACE before anything is enqueued."""
    import torch
    import top_sparse_decode_paged_b200 as sd
    spec = W.spec("perhead_b16_gqa", seqlens=(3000,), seed=33)      # B=1, G=8
    wl = W.make(spec)
    d = to_device(wl)
    # 8 * 524288 == NOALLOC_MAX_SCORES, and at_limit + 1 is still below the
    # library's max_seqlen limit (1 << 20), so only the scratch check can
    # reject the second call
    at_limit = sd.NOALLOC_MAX_SCORES // 8
    idx = torch.empty((1, 8, spec.k), dtype=torch.int32, device="cuda")
    sd.sd_indexer_topk_noalloc(d["qi"], d["w"], d["ki_pages"], d["block_table"], d["seqlens"], spec.k,
                               at_limit, idx)
    ref = sd.sd_indexer_topk(d["qi"], d["w"], d["ki_pages"], d["block_table"], d["seqlens"], spec.k,
                             wl.max_seqlen)
    torch.cuda.synchronize()
    assert np.array_equal(idx.cpu().numpy(), ref.cpu().numpy())
    with pytest.raises(sd.SdError) as e:
        sd.sd_indexer_topk_noalloc(d["qi"], d["w"], d["ki_pages"], d["block_table"], d["seqlens"], spec.k,
                                   at_limit + 1, idx)
    assert e.value.name == "SD_ERR_WORKSPACE"


def test_noalloc_allocates_no_device_memory():
    """The property the entry point exists for: after one warm-up call (which
    loads every kernel it uses), a call at the scratch limit changes neither
    the device's free memory nor torch's allocated bytes."""
    import torch
    import top_sparse_decode_paged_b200 as sd
    spec = W.spec("perhead_b16_gqa", seqlens=(3000,), seed=34)      # B=1, G=8
    wl = W.make(spec)
    d = to_device(wl)
    at_limit = sd.NOALLOC_MAX_SCORES // 8
    idx = torch.empty((1, 8, spec.k), dtype=torch.int32, device="cuda")

    def call():
        sd.sd_indexer_topk_noalloc(d["qi"], d["w"], d["ki_pages"], d["block_table"], d["seqlens"], spec.k,
                                   at_limit, idx)
        torch.cuda.synchronize()

    call()
    free0, alloc0 = torch.cuda.mem_get_info()[0], torch.cuda.memory_allocated()
    call()
    assert torch.cuda.mem_get_info()[0] == free0
    assert torch.cuda.memory_allocated() == alloc0
