"""GPU parity of the TriAttention eviction (sd_tri_compact) against the oracle.

The oracle scores in fp64; the library sums in fp32. The GPU's kept set is
read back from the compacted pool and must be a valid top-`budget` set under
the oracle's scores within the fp32 error bound of the scoring (tests/
tri_check.py derives it); where the boundary is separated by more than that
bound the set is unique and must equal the oracle's. Then the new lengths and
every byte of the K and V pools must equal the oracle's compaction with the
GPU's kept set ("Add TriAttention KV-cache compression method", Summary and
Test Plan: a fast scoring kernel checked against an oracle, union and
per-head modes, ragged lengths and unaligned final tokens, heavy ties).
"""
import dataclasses

import numpy as np
import pytest

from oracle import tri_oracle as T
from top_sparse_decode_paged_b200.workloads import bf16_bits_from_f32, make_tri, tri_spec

from tri_check import check_eviction, score_bounds, separated

pytestmark = pytest.mark.gpu


def _dev(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _bf16(a):
    import torch
    return _dev(a.view(np.int16)).view(torch.bfloat16)


def _bits(t):
    import torch
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def _run_gpu(w, mode, budget=None):
    import torch
    import top_sparse_decode_paged_b200 as sd
    s = w.spec
    budget = s.budget if budget is None else budget
    kp, vp = _bf16(w.k_pages), None if w.v_pages is None else _bf16(w.v_pages)
    nl = sd.sd_tri_compact(_dev(w.q_cal), kp, vp, _dev(w.block_table), _dev(w.seqlens), w.max_seqlen, s.n_sink,
                           s.n_recent, budget, mode)
    torch.cuda.synchronize()
    assert sd.device_errors() == 0
    return _bits(kp), None if vp is None else _bits(vp), nl.cpu().numpy()


def _check(w, mode, budget=None):
    s = w.spec
    budget = s.budget if budget is None else budget
    k, v, nl = _run_gpu(w, mode, budget)
    check_eviction([w.q_cal], [w.k_pages], None if w.v_pages is None else [w.v_pages], w.block_table, w.seqlens,
                   s.n_sink, s.n_recent, budget, mode, [k], None if v is None else [v], nl)
    return nl


def _check_exact(w, mode, budget=None):
    """The oracle's whole eviction, byte for byte (for inputs whose kept set
    is unique under the bound, or whose scores tie exactly in any arithmetic)."""
    s = w.spec
    budget = s.budget if budget is None else budget
    k_ref, v_ref, nl_ref, _ = T.tri_evict(w.q_cal, w.k_pages, w.v_pages, w.block_table, w.seqlens, s.n_sink,
                                          s.n_recent, budget, mode)
    k, v, nl = _run_gpu(w, mode, budget)
    assert np.array_equal(nl, nl_ref)
    assert np.array_equal(k, k_ref)
    if v_ref is not None:
        assert np.array_equal(v, v_ref)


@pytest.mark.parametrize("mode", [T.UNION, T.PER_HEAD])
@pytest.mark.parametrize("with_v", [True, False])
def test_tiny_ragged(mode, with_v):
    """Lengths 100, 20, 37 (region 88, 8, 25 against budget 24): one request
    keeps everything, one evicts a single token, pages end unaligned."""
    w = make_tri(tri_spec("tri_tiny", with_v=with_v))
    nl = _check(w, mode)
    assert nl.tolist() == [4 + 24 + 8, 20, 4 + 24 + 8]


@pytest.mark.parametrize("H,G,D", [(32, 8, 128), (8, 8, 64), (16, 8, 64), (16, 2, 128), (4, 1, 64)])
@pytest.mark.parametrize("mode", [T.UNION, T.PER_HEAD])
def test_shapes_span_tiles(H, G, D, mode):
    """Regions of several 128-position score tiles with ragged tails, every
    supported query-heads-per-KV-head ratio (4, 1, 2, 8) and both widths."""
    s = tri_spec("tri_ragged_b16", B=5, H=H, G=G, D=D, page_size=16, n_sink=40, n_recent=9, budget=200,
                 ragged=(0, 700), seed=20 + H + G + D)
    _check(make_tri(s), mode)


def test_misaligned_queries():
    """A q_cal that is not 16-byte aligned (the score pass reads it element by
    element) gives the same result bit for bit."""
    import torch
    import top_sparse_decode_paged_b200 as sd
    w = make_tri(tri_spec("tri_ragged_b16", B=3, page_size=16, n_sink=40, n_recent=9, budget=200, ragged=(0, 700),
                          seed=35))
    s = w.spec
    flat = torch.zeros(s.H * s.D + 1, dtype=torch.int16, device="cuda")
    flat[1:] = torch.from_numpy(w.q_cal.view(np.int16).reshape(-1)).cuda()
    q = flat[1:].view(s.H, s.D).view(torch.bfloat16)
    assert q.data_ptr() % 16 != 0
    kp, vp = _bf16(w.k_pages), _bf16(w.v_pages)
    nl = sd.sd_tri_compact(q, kp, vp, _dev(w.block_table), _dev(w.seqlens), w.max_seqlen, s.n_sink, s.n_recent,
                           s.budget, T.UNION)
    torch.cuda.synchronize()
    assert sd.device_errors() == 0
    check_eviction([w.q_cal], [w.k_pages], [w.v_pages], w.block_table, w.seqlens, s.n_sink, s.n_recent, s.budget,
                   T.UNION, [_bits(kp)], [_bits(vp)], nl.cpu().numpy())


def test_heavy_ties_on_gpu():
    """Every key row equal: all scores tie at 0 in any arithmetic (identical
    inputs), so the kept set is the lowest positions, exactly."""
    s = tri_spec("tri_tiny", B=2, seqlens=(300, 129), budget=50, n_sink=3, n_recent=5, seed=30)
    w = make_tri(s)
    for b, L in enumerate(w.seqlens):
        for t in range(int(L)):
            w.k_pages[w.block_table[b, t // s.page_size], t % s.page_size] = bf16_bits_from_f32(
                np.full((s.G, s.D), 0.5, np.float32))
    for mode in (T.UNION, T.PER_HEAD):
        _check_exact(dataclasses.replace(w, k_pages=w.k_pages.copy(),
                                         v_pages=None if w.v_pages is None else w.v_pages.copy()), mode)


@pytest.mark.parametrize("budget", [1, 2048])
def test_budget_extremes(budget):
    s = tri_spec("tri_tiny", B=3, seqlens=(2100, 64, 5), n_sink=2, n_recent=3, budget=budget, seed=31)
    _check(make_tri(s), T.UNION)


def test_nothing_evictable_and_empty_batch():
    import torch
    import top_sparse_decode_paged_b200 as sd
    s = tri_spec("tri_tiny", B=3, seqlens=(0, 12, 30), budget=24, seed=32)  # regions 0, 0, 18
    w = make_tri(s)
    k, v, nl = _run_gpu(w, T.UNION)
    assert nl.tolist() == [0, 12, 30]
    assert np.array_equal(k, w.k_pages) and np.array_equal(v, w.v_pages)
    kp = _bf16(w.k_pages)
    empty = torch.zeros((0,), dtype=torch.int32, device="cuda")
    out = sd.sd_tri_compact(_dev(w.q_cal), kp, None, _dev(w.block_table[:0]), empty, 0, 4, 8, 24)
    torch.cuda.synchronize()
    assert out.numel() == 0


def test_bad_page_is_reported_without_fault():
    import torch
    import top_sparse_decode_paged_b200 as sd
    w = make_tri(tri_spec("tri_tiny"))
    bt = w.block_table.copy()
    bt[0, 2] = w.k_pages.shape[0] + 5  # out of the pool, inside the request
    kp = _bf16(w.k_pages)
    sd.sd_tri_compact(_dev(w.q_cal), kp, None, _dev(bt), _dev(w.seqlens), w.max_seqlen, 4, 8, 24)
    torch.cuda.synchronize()
    assert sd.device_errors() & sd.SD_DEVERR_PAGE


def test_full_size_sampled_requests():
    """The measured workload (32 requests, Qwen3-8B attention shape, region
    4096, budget 2048) in the launch configuration the benchmark times; the
    oracle scores every request and the check covers sampled requests (their
    pages are disjoint from the others')."""
    w = make_tri(tri_spec("tri_b32_qwen3_8b"))
    s = w.spec
    k, v, nl = _run_gpu(w, T.UNION)
    assert np.all(nl == s.n_sink + s.budget + s.n_recent)
    check_eviction([w.q_cal], [w.k_pages], [w.v_pages], w.block_table, w.seqlens, s.n_sink, s.n_recent, s.budget,
                   T.UNION, [k], [v], nl, requests=(0, 13, 31))


@pytest.mark.parametrize("mode", [T.UNION, T.PER_HEAD])
def test_separated_boundary_is_exact(mode):
    """Keys of a planted set of `budget` positions per selection row (union:
    one set, raised in every KV head) are moved along the sign of their head's
    query, which lifts their logits far above the rest: the boundary is then
    separated by much more than the fp32 bound, the kept set is unique, and
    the GPU must keep exactly the oracle's."""
    s = tri_spec("tri_ragged_b16", B=3, H=2, G=2, D=128, page_size=16, n_sink=8, n_recent=4, budget=60,
                 ragged=(300, 500), seed=77)
    w = make_tri(s)
    rng = np.random.default_rng(78)
    q = (w.q_cal.astype(np.uint32) << 16).view(np.float32)
    P = s.page_size
    for b, L in enumerate(w.seqlens):
        E = int(L) - s.n_sink - s.n_recent
        planted = rng.choice(E, size=s.budget, replace=False)
        for g in range(s.G):  # query head g reads KV head g here (H = G)
            if mode == T.PER_HEAD:
                planted = rng.choice(E, size=s.budget, replace=False)
            for p in planted:
                t = s.n_sink + int(p)
                row = w.k_pages[w.block_table[b, t // P], t % P, g]
                kv = (row.astype(np.uint32) << 16).view(np.float32) + 8.0 * np.sign(q[g])
                w.k_pages[w.block_table[b, t // P], t % P, g] = bf16_bits_from_f32(kv.astype(np.float32))
    for sc, sl in score_bounds(w.q_cal, w.k_pages, w.block_table, w.seqlens, s.n_sink, s.n_recent, mode):
        assert all(separated(sc[r], sl[r], s.budget) for r in range(sc.shape[0]))
    _check_exact(w, mode)


@pytest.mark.parametrize("mode", [T.UNION, T.PER_HEAD, T.PER_LAYER_PER_HEAD])
@pytest.mark.parametrize("with_v", [True, False])
def test_layers_every_mode(mode, with_v):
    """Three layers sharing the block table ("Add TriAttention KV-cache
    compression method", Summary: union / per_head / per_layer_perhead): one
    selection across layers, or one per layer, every layer compacted."""
    import torch
    import top_sparse_decode_paged_b200 as sd
    from top_sparse_decode_paged_b200.workloads import make_tri_layers
    s = tri_spec("tri_ragged_b16", B=4, page_size=16, n_sink=24, n_recent=7, budget=150, ragged=(0, 600),
                 with_v=with_v, seed=41 + mode)
    ws = make_tri_layers(s, 3)
    kps = [_bf16(w.k_pages) for w in ws]
    vps = None if not with_v else [_bf16(w.v_pages) for w in ws]
    nl = sd.sd_tri_compact_layers([_bf16(w.q_cal) for w in ws], kps, vps, _dev(ws[0].block_table),
                                  _dev(ws[0].seqlens), ws[0].max_seqlen, s.n_sink, s.n_recent, s.budget, mode)
    torch.cuda.synchronize()
    assert sd.device_errors() == 0
    check_eviction([w.q_cal for w in ws], [w.k_pages for w in ws], None if not with_v else [w.v_pages for w in ws],
                   ws[0].block_table, ws[0].seqlens, s.n_sink, s.n_recent, s.budget, mode, [_bits(k) for k in kps],
                   None if not with_v else [_bits(v) for v in vps], nl.cpu().numpy())


def test_layers_one_layer_matches_single_call():
    import torch
    import top_sparse_decode_paged_b200 as sd
    w = make_tri(tri_spec("tri_tiny"))
    s = w.spec
    a, b = _bf16(w.k_pages), _bf16(w.k_pages)
    sd.sd_tri_compact(_dev(w.q_cal), a, None, _dev(w.block_table), _dev(w.seqlens), w.max_seqlen, s.n_sink,
                      s.n_recent, s.budget, T.PER_HEAD)
    sd.sd_tri_compact_layers([_dev(w.q_cal)], [b], None, _dev(w.block_table), _dev(w.seqlens), w.max_seqlen,
                             s.n_sink, s.n_recent, s.budget, T.PER_LAYER_PER_HEAD)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_compaction_wait_runs_out_and_the_device_stays_usable():
    """Failure path of the bounded cross-CTA waits, made to happen from the
    host: with the wait limit at 0 polls every unit that waits on an earlier
    one gives up at once. The call returns, SD_DEVERR_TIMEOUT is set, and the
    next call with the default limit evicts a fresh copy correctly. No unit
    has a copy in flight when it gives up, and nothing waits without bound."""
    import torch
    import top_sparse_decode_paged_b200 as sd
    s = tri_spec("tri_ragged_b16", B=4, H=32, G=8, D=128, page_size=16, n_sink=40, n_recent=9, budget=200,
                 ragged=(300, 700), seed=51)
    w = make_tri(s)
    # 2048 bytes per union token (K and V: 4096), so a 32 KB unit holds 8 kept tokens and every
    # row has many units; later units read destinations that earlier units hold
    assert (s.budget + s.n_recent) > 2 * (32768 // (2 * s.G * s.D * 2))
    assert sd.device_errors() == 0
    try:
        sd.set_wait_limit(0)
        kp, vp = _bf16(w.k_pages), _bf16(w.v_pages)
        sd.sd_tri_compact(_dev(w.q_cal), kp, vp, _dev(w.block_table), _dev(w.seqlens), w.max_seqlen, s.n_sink,
                          s.n_recent, s.budget, T.UNION)
        torch.cuda.synchronize()
        assert sd.device_errors() & sd.SD_DEVERR_TIMEOUT
    finally:
        sd.set_wait_limit(-1)
    _check(w, T.UNION)  # default limit: fresh pools, the full check, no error bit
