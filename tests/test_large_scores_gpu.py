"""Score scratch past 2^31 elements ("Add TriAttention KV-cache compression
method", Test Plan: score buffers beyond 2^31 elements).

The scores are [B, G, max_seqlen] int32, row r = b * G + g at offset
r * max_seqlen. With max_seqlen = 2^20, rows r >= 2048 start past 2^31
elements (8 GiB), so any 32-bit product in an offset would land them on
earlier rows. Most requests here are one page long and share a small key
pool; the last requests are long, and their scores and indices are compared
with the oracle bit for bit. Both indexer kernels run (one KV head of 128-byte
keys with 64 heads: the tensor-core kernel; eight KV heads of 64-byte keys:
the dp4a kernel), and the top-k runs over L2 (rows longer than a cluster
holds).
"""
import numpy as np
import pytest

import oracle

pytestmark = pytest.mark.gpu

MAX_SEQLEN = 1 << 20


def _case(B, G, Hi, Di, k, long_lens, seed):
    rng = np.random.default_rng(seed)
    P, max_pages = 64, 2048
    n_pages = 4096
    seqlens = np.full(B, 16, dtype=np.int32)
    seqlens[B - len(long_lens):] = long_lens
    qi = rng.integers(-64, 65, size=(B, G, Hi, Di), dtype=np.int8)
    w = rng.integers(1, 9, size=(B, G, Hi), dtype=np.int32)
    ki = rng.integers(-64, 65, size=(n_pages, P, G, Di), dtype=np.int8)
    bt = np.full((B, max_pages), -1, dtype=np.int32)
    for b in range(B):
        n = (int(seqlens[b]) + P - 1) // P
        bt[b, :n] = rng.permutation(n_pages)[:n]  # requests may share pages: they only read them
    return qi, w, ki, bt, seqlens


@pytest.mark.parametrize("B,G,Hi,Di,k,long_lens", [
    (2052, 1, 64, 128, 2048, (30000, 65536, 4097, 100)),   # rows 2048..2051 past 2^31
    (260, 8, 4, 64, 1024, (65536, 20000)),                 # rows 2064..2079 past 2^31
])
def test_scores_past_2_31_elements(B, G, Hi, Di, k, long_lens):
    import torch
    import top_sparse_decode_paged_b200 as sd
    assert (B - 1) * G * MAX_SEQLEN >= 1 << 31
    qi, w, ki, bt, seqlens = _case(B, G, Hi, Di, k, long_lens, seed=B + G)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()  # noqa: E731
    scores = torch.empty((B, G, MAX_SEQLEN), dtype=torch.int32, device="cuda")
    idx = sd.sd_indexer_topk(t(qi), t(w), t(ki), t(bt), t(seqlens), k, MAX_SEQLEN, scores=scores)
    torch.cuda.synchronize()
    assert sd.device_errors() == 0
    last = list(range(B - len(long_lens) - 1, B))  # the long requests and one short one before them
    ref_s = oracle.indexer_scores(qi, w, ki, bt, seqlens, requests=last)
    ref_i = oracle.topk_indices(ref_s, k)
    got_i = idx.cpu().numpy()
    for j, b in enumerate(last):
        L = int(seqlens[b])
        got = scores[b, :, :L].cpu().numpy()
        assert np.array_equal(got, ref_s[j]), f"request {b}: scores differ"
        assert np.array_equal(got_i[b], ref_i[j]), f"request {b}: indices differ"
    del scores
    torch.cuda.empty_cache()
