"""Pins of the TriAttention eviction oracle to facts outside itself.

The steps follow "Add TriAttention KV-cache compression method" (Summary: score
the evictable decode region with per-head calibrated queries, keep `budget`
tokens, compact in place; Key Design Decisions: in-place compaction inside the
same pools, prompt and protected tails preserved; Test Plan: union and
per-head modes, ragged lengths, deterministic heavy-tie settlement).
"""
import itertools

import numpy as np
import pytest

from oracle import tri_oracle as T
from top_sparse_decode_paged_b200.workloads import bf16_bits_from_f32, make_tri, tri_spec


def _pool_from_values(vals: np.ndarray, P: int, perm=None):
    """Pages [n_pages, P, G, D] holding token rows vals [L, G, D] (bf16 bits),
    with a page permutation; returns (pool, block_table_row)."""
    L = vals.shape[0]
    n = (L + P - 1) // P
    perm = np.arange(n) if perm is None else np.asarray(perm)
    pool = np.zeros((n, P) + vals.shape[1:], dtype=np.uint16)
    for t in range(L):
        pool[perm[t // P], t % P] = vals[t]
    return pool, perm.astype(np.int32)


def _bf(x):
    return (bf16_bits_from_f32(np.asarray(x, np.float32)).astype(np.uint32) << 16).view(np.float32)


def test_logits_equal_the_exact_rational_dot_product():
    """z[h, p] equals q_cal[h] . K[p, h // (H/G)] summed exactly in rationals
    (bf16 values are dyadic), up to the fp64 rounding of the sum; a transposed
    operand, a wrong head map or a dropped term is off by far more."""
    from fractions import Fraction
    rng = np.random.default_rng(0)
    H, G, D, E = 6, 3, 64, 12
    q = _bf(rng.standard_normal((H, D), dtype=np.float32)).astype(np.float64)
    Kf = _bf(rng.standard_normal((E, G, D), dtype=np.float32)).astype(np.float64)
    z = T.tri_logits(q, Kf, G)
    assert z.dtype == np.float64
    for h in range(H):
        g = h // (H // G)
        for p in range(E):
            exact = sum(Fraction(float(q[h, d])) * Fraction(float(Kf[p, g, d])) for d in range(D))
            scale = float(np.abs(q[h]) @ np.abs(Kf[p, g]))
            assert abs(Fraction(float(z[h, p])) - exact) <= Fraction(D * 2.0 ** -53 * scale)


def _fp32_scores_reverse_order(w, mode):
    """Scores as an fp32 kernel could take them: products summed in fp32 in
    reverse index order (one rounding per step), shift and maxima in fp32. A
    different evaluation from the oracle's, inside the bound the GPU check
    allows."""
    s = w.spec
    from oracle.sd_oracle import bf16_bits_to_f64, gather_token_rows
    q = bf16_bits_to_f64(w.q_cal)
    H, D = q.shape
    qpk = H // s.G
    out = []
    for b, L in enumerate(w.seqlens):
        E = max(0, int(L) - s.n_sink - s.n_recent)
        K = bf16_bits_to_f64(gather_token_rows(w.k_pages, w.block_table[b], np.arange(s.n_sink, s.n_sink + E)))
        z = np.zeros((H, E), dtype=np.float32)
        for h in range(H):
            acc = np.zeros(E, dtype=np.float32)
            for d in range(D - 1, -1, -1):
                acc = (acc.astype(np.float64) + K[:, h // qpk, d] * q[h, d]).astype(np.float32)
            z[h] = acc
        zs = (z - z.max(axis=1, keepdims=True)).astype(np.float32) if E else z
        per_g = np.stack([zs[g * qpk:(g + 1) * qpk].max(axis=0) for g in range(s.G)])
        out.append(per_g if mode == T.PER_HEAD else per_g.max(axis=0, keepdims=True))
    return out


@pytest.mark.parametrize("mode", [T.UNION, T.PER_HEAD])
def test_gpu_check_accepts_an_fp32_evaluation_and_rejects_planted_mistakes(mode):
    """The validity check the GPU tests use (tests/tri_check.py): a selection
    from an fp32 evaluation in another order passes; swapping one kept
    position for the worst dropped one fails; the bound is far below the
    spread of the scores, so it does not accept everything."""
    from tri_check import score_bounds, valid_selection
    s = tri_spec("tri_ragged_b16", B=3, H=8, G=4, D=128, page_size=16, n_sink=8, n_recent=4, budget=100,
                 ragged=(200, 400), seed=5)
    w = make_tri(s)
    bounds = score_bounds(w.q_cal, w.k_pages, w.block_table, w.seqlens, s.n_sink, s.n_recent, mode)
    f32 = _fp32_scores_reverse_order(w, mode)
    for (sc, slack), sc32 in zip(bounds, f32):
        assert np.median(slack) < 1e-3 * np.std(sc)
        assert np.all(np.abs(sc32.astype(np.float64) - sc) <= slack)
        sel32 = T.tri_select(sc32, s.budget)
        for r in range(sc.shape[0]):
            assert valid_selection(sc[r], slack[r], sel32[r], s.budget)
            bad = sel32[r].copy()
            dropped = np.setdiff1d(np.arange(sc.shape[1]), bad)
            bad[np.argmax(sc[r][bad])] = dropped[np.argmin(sc[r][dropped])]
            assert not valid_selection(sc[r], slack[r], np.sort(bad), s.budget)
            assert not valid_selection(sc[r], slack[r], sel32[r][:-1], s.budget)


def test_one_hot_queries_closed_form_and_independent_sort():
    """q_cal[h] = 2 e_{d_h}: z[h, p] = 2 K[p, g, d_h] exactly; with one head the
    selection is the `budget` largest K[., d_0], ties to the lower position."""
    rng = np.random.default_rng(1)
    E, D, budget = 50, 64, 17
    vals = rng.integers(-6, 7, size=(E, 1, D)).astype(np.float32)  # many ties
    K = bf16_bits_from_f32(vals)
    q = np.zeros((1, D), dtype=np.float32)
    q[0, 5] = 2.0
    z = T.tri_logits(q, vals, 1)
    assert np.array_equal(z[0], 2.0 * vals[:, 0, 5])
    pool, bt = _pool_from_values(K, P=8, perm=[3, 0, 6, 1, 5, 2, 4])
    s = T.tri_scores(bf16_bits_from_f32(q), pool, bt[None], np.array([E]), 0, 0, T.UNION)[0]
    sel = T.tri_select(s, budget)[0]
    expect = sorted(sorted(range(E), key=lambda p: (-vals[p, 0, 5], p))[:budget])
    assert sel.tolist() == expect


def test_each_head_normalised_by_its_own_maximum():
    """A constant key column seen by one head only shifts that head's logits;
    after the per-head shift the union selection is unchanged, and each head's
    best token (score 0, the maximum) is kept. Without the shift the offset
    head would take every slot."""
    rng = np.random.default_rng(2)
    E, D, H = 24, 64, 2
    vals = rng.integers(-4, 5, size=(E, 1, D)).astype(np.float32)
    vals[:, 0, 63] = 8.0  # constant column
    q = np.zeros((H, D), dtype=np.float32)
    q[0, 3] = 1.0
    q[1, 7] = 1.0
    q_shift = q.copy()
    q_shift[1, 63] = 16.0  # head 1 logits + 128 everywhere
    pool, bt = _pool_from_values(bf16_bits_from_f32(vals), P=8)
    budget = 6
    sel = T.tri_select(T.tri_scores(bf16_bits_from_f32(q), pool, bt[None], np.array([E]), 0, 0, T.UNION)[0],
                       budget)[0]
    sel2 = T.tri_select(T.tri_scores(bf16_bits_from_f32(q_shift), pool, bt[None], np.array([E]), 0, 0,
                                     T.UNION)[0], budget)[0]
    assert sel.tolist() == sel2.tolist()
    for h, d in ((0, 3), (1, 7)):
        best = min(range(E), key=lambda p: (-vals[p, 0, d], p))
        assert best in sel.tolist()


def test_union_is_max_of_per_head_and_selection_is_a_threshold_set():
    w = make_tri(tri_spec("tri_tiny"))
    s = w.spec
    per = T.tri_scores(w.q_cal, w.k_pages, w.block_table, w.seqlens, s.n_sink, s.n_recent, T.PER_HEAD)
    uni = T.tri_scores(w.q_cal, w.k_pages, w.block_table, w.seqlens, s.n_sink, s.n_recent, T.UNION)
    for a, b in zip(per, uni):
        assert np.array_equal(a.max(axis=0), b[0])
        for row in a:
            if row.size:
                assert row.max() == 0.0 and np.all(row <= 0.0)
    # every kept score >= every dropped score; among equal scores the lower position is kept
    for sc in per:
        sel = T.tri_select(sc, s.budget)
        for r in range(sel.shape[0]):
            kept = set(sel[r].tolist())
            for p, q in itertools.product(range(sc.shape[1]), repeat=2):
                if p in kept and q not in kept:
                    assert sc[r, p] > sc[r, q] or (sc[r, p] == sc[r, q] and p < q)


def test_heavy_ties_keep_the_lowest_positions():
    E, D = 30, 64
    vals = np.ones((E, 2, D), dtype=np.float32)
    pool, bt = _pool_from_values(bf16_bits_from_f32(vals), P=4)
    q = bf16_bits_from_f32(np.ones((4, D), dtype=np.float32))
    for mode in (T.UNION, T.PER_HEAD):
        sc = T.tri_scores(q, pool, bt[None], np.array([E]), 2, 3, mode)[0]
        sel = T.tri_select(sc, 7)
        assert np.all(sel == np.arange(7))


def test_hand_worked_compaction_across_pages():
    """L = 13, prefix 2, tail 3, budget 3, page 4, pages permuted: the evictable
    region is tokens 2..9; keeping region positions {1, 4, 6} (tokens 3, 6, 8)
    leaves tokens [0, 1, 3, 6, 8, 10, 11, 12] at positions 0..7; positions 8..12
    keep their old rows. Per-head: head 1 keeps positions {0, 1, 2} (tokens
    2, 3, 4) by its own selection."""
    L, P, G, D = 13, 4, 2, 8
    vals = np.zeros((L, G, D), dtype=np.float32)
    for t in range(L):
        for g in range(G):
            vals[t, g, :] = 100 * g + t
    K = bf16_bits_from_f32(vals)
    V = bf16_bits_from_f32(-vals)
    kp, bt = _pool_from_values(K, P, perm=[2, 0, 3, 1])
    vp, _ = _pool_from_values(V, P, perm=[2, 0, 3, 1])

    def token_at(pool, pos, g):
        x = pool[bt[pos // P], pos % P, g, 0]
        return float((np.uint32(x) << 16).view(np.float32))

    sel_u = [np.array([[1, 4, 6]])]
    k2, v2, nl = T.tri_compact(kp, vp, bt[None], np.array([L]), sel_u, 2, 3, 3, T.UNION)
    assert nl.tolist() == [8]
    expect = [0, 1, 3, 6, 8, 10, 11, 12, 8, 9, 10, 11, 12]
    for pos, t in enumerate(expect):
        for g in range(G):
            assert token_at(k2, pos, g) == 100 * g + t
            assert token_at(v2, pos, g) == -(100 * g + t)

    sel_h = [np.array([[1, 4, 6], [0, 1, 2]])]
    k3, _, nl = T.tri_compact(kp, None, bt[None], np.array([L]), sel_h, 2, 3, 3, T.PER_HEAD)
    expect1 = [0, 1, 2, 3, 4, 10, 11, 12, 8, 9, 10, 11, 12]
    for pos in range(L):
        assert token_at(k3, pos, 0) == expect[pos]
        assert token_at(k3, pos, 1) == 100 + expect1[pos]


@pytest.mark.parametrize("L", [0, 3, 5, 10, 13])
def test_nothing_moves_when_the_region_fits_the_budget(L):
    """E = max(0, L - 5) <= budget 8: pools and lengths unchanged."""
    rng = np.random.default_rng(L)
    P, G, D = 4, 1, 64
    n = max(1, (L + P - 1) // P)
    kp = bf16_bits_from_f32(rng.standard_normal((n, P, G, D), dtype=np.float32))
    bt = np.arange(n, dtype=np.int32)[None]
    q = bf16_bits_from_f32(rng.standard_normal((2, D), dtype=np.float32))
    k2, v2, nl, sel = T.tri_evict(q, kp, None, bt, np.array([L]), 2, 3, 8, T.UNION)
    assert nl.tolist() == [L]
    assert np.array_equal(k2, kp) and v2 is None
    assert sel[0].shape == (1, 0)


def test_compaction_brute_force_tiny():
    """Every 3-subset of a 6-token region: the compacted request reads back as
    prefix + subset + tail, and bytes past the new length are untouched."""
    L, n_sink, n_recent, budget, P = 10, 1, 3, 3, 4
    vals = np.arange(L, dtype=np.float32)[:, None, None] * np.ones((1, 1, 64), np.float32)
    kp, bt = _pool_from_values(bf16_bits_from_f32(vals), P, perm=[1, 2, 0])
    for sub in itertools.combinations(range(6), 3):
        k2, _, nl = T.tri_compact(kp, None, bt[None], np.array([L]), [np.array([sub])], n_sink, n_recent,
                                  budget, T.UNION)
        assert nl[0] == 7
        got = [float((np.uint32(k2[bt[i // P], i % P, 0, 0]) << 16).view(np.float32)) for i in range(L)]
        assert got[:7] == [0] + [1 + s for s in sub] + [7, 8, 9]
        assert got[7:] == [7, 8, 9]


def test_layers_identical_layers_select_as_one():
    """Two copies of one layer: the union and per-head selections across
    layers equal the single layer's (the maximum of equal scores)."""
    w = make_tri(tri_spec("tri_tiny"))
    s = w.spec
    for mode in (T.UNION, T.PER_HEAD):
        _, _, nl1, sel1 = T.tri_evict(w.q_cal, w.k_pages, w.v_pages, w.block_table, w.seqlens, s.n_sink,
                                      s.n_recent, s.budget, mode)
        _, _, nl2, sel2 = T.tri_evict_layers([w.q_cal] * 2, [w.k_pages] * 2, [w.v_pages] * 2, w.block_table,
                                             w.seqlens, s.n_sink, s.n_recent, s.budget, mode)
        assert np.array_equal(nl1, nl2)
        for a, b in zip(sel1, sel2):
            assert np.array_equal(a, b)


def test_layers_union_keeps_each_layers_favourite():
    """Layer 0's query picks one key column, layer 1's another; with a budget
    of 2 the cross-layer union keeps each layer's best position (score 0, the
    maximum), and per-layer-per-head keeps each layer's own top 2."""
    E, D = 12, 64
    vals = np.zeros((E, 1, D), dtype=np.float32)
    vals[:, 0, 0] = [1, 9, 2, 3, 1, 2, 0, 1, 2, 1, 0, 8]   # layer 0 prefers 1, then 11
    vals[:, 0, 1] = [0, 1, 2, 3, 4, 7, 2, 11, 1, 1, 6, 1]  # layer 1 prefers 7, then 5
    pool, bt = _pool_from_values(bf16_bits_from_f32(vals), P=4)
    q0 = np.zeros((1, D), np.float32)
    q0[0, 0] = 1.0
    q1 = np.zeros((1, D), np.float32)
    q1[0, 1] = 1.0
    qs = [bf16_bits_from_f32(q0), bf16_bits_from_f32(q1)]
    _, _, _, sel = T.tri_evict_layers(qs, [pool, pool], None, bt[None], np.array([E]), 0, 0, 2, T.UNION)
    assert sel[0].tolist() == [[1, 7]]
    _, _, _, sels = T.tri_evict_layers(qs, [pool, pool], None, bt[None], np.array([E]), 0, 0, 2,
                                       T.PER_LAYER_PER_HEAD)
    assert sels[0][0].tolist() == [[1, 11]] and sels[1][0].tolist() == [[5, 7]]


def test_gpu_check_reads_the_kept_set_back_and_compares_every_byte():
    """check_eviction on the oracle's own eviction (standing in for the GPU's
    pools) passes and reads back the oracle's kept sets; a wrong V row in one
    kept slot, or a changed byte in a page no request owns, fails."""
    from tri_check import check_eviction
    w = make_tri(tri_spec("tri_tiny"))
    s = w.spec
    for mode in (T.UNION, T.PER_HEAD):
        k2, v2, nl, sel = T.tri_evict(w.q_cal, w.k_pages, w.v_pages, w.block_table, w.seqlens, s.n_sink,
                                      s.n_recent, s.budget, mode)
        kept = check_eviction([w.q_cal], [w.k_pages], [w.v_pages], w.block_table, w.seqlens, s.n_sink, s.n_recent,
                              s.budget, mode, [k2], [v2], nl)
        for b in range(len(w.seqlens)):
            assert np.array_equal(kept[0][b], sel[b])
        P = s.page_size
        t = s.n_sink + 3  # a kept slot of request 0 (it evicts)
        bad_v = v2.copy()
        bad_v[w.block_table[0, t // P], t % P, 0, 0] ^= 1
        with pytest.raises(AssertionError):
            check_eviction([w.q_cal], [w.k_pages], [w.v_pages], w.block_table, w.seqlens, s.n_sink, s.n_recent,
                           s.budget, mode, [k2], [bad_v], nl)
        spare = w.k_pages.shape[0] - 1  # the workload's spare pages belong to no request
        bad_k = k2.copy()
        bad_k[spare, 0, 0, 0] ^= 1
        with pytest.raises(AssertionError):
            check_eviction([w.q_cal], [w.k_pages], [w.v_pages], w.block_table, w.seqlens, s.n_sink, s.n_recent,
                           s.budget, mode, [bad_k], [v2], nl)
