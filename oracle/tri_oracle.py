"""CPU oracle for TriAttention-style decode-time eviction of one layer.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
module. The library never calls it and shares no code with it.

What it computes ("Add TriAttention KV-cache compression method", Summary and
Key Design Decisions: score the evictable decode region with per-head
calibrated queries, keep ``budget`` tokens, compact the kept K/V entries in
place inside the same paged pools, keep prompt and protected tails; union and
per-head modes; deterministic tie settlement):

1. ``tri_scores``   for request b with length L, evictable positions
   p < E = max(0, L - n_sink - n_recent) (token n_sink + p):
     z[h, p]  = q_cal[h] . K[n_sink + p, g(h)]      (q_cal and K bf16)
     s[g, p]  = max over the query heads h of KV head g of (z[h, p] - max_p' z[h, p'])
     union:     s[p] = max_g s[g, p]
2. ``tri_select``   the ``budget`` largest scores, ties to the lower position,
   in ascending position order (nothing is selected when E <= budget).
3. ``tri_compact``  kept token i takes logical position i: the protected
   prefix [0, n_sink) stays, then the selected positions, then the tail
   [L - n_recent, L); the new length is n_sink + budget + n_recent. Union mode
   moves whole rows, per-head mode each KV head's part by its own selection.

Precision: the scores are the plain definition, computed in fp64. The
factors are bf16 values, so every product q k is exact in fp64; the sum of D
of them is rounded at most D times at 2^-53, far below anything a selection
can depend on, and the shift and the maxima are exact fp64 operations on it.
No summation order is assumed: a kernel that sums in fp32, in any order, is
checked against these scores with the fp32 error bound of its arithmetic
(the tests derive that bound), not against a restatement of its rounding.

Readings where the pages are silent (they name the steps, not the formulas):
the score is the plain dot product with the calibrated query; each head is
shifted by its own maximum before the maximum over heads; the protected prefix
and tail are uniform sizes. The design notes list them.

Parity pins: ``tests/test_tri_pins.py`` (the logits against an exact rational
dot product, one-hot queries against a closed form and an independent sort,
shift invariance of the per-head normalisation, a hand-worked compaction
across pages, brute force over small subsets, the degenerate cases).
"""

from __future__ import annotations

import numpy as np

from .sd_oracle import bf16_bits_to_f64, gather_token_rows

UNION = 0
PER_HEAD = 1
PER_LAYER_PER_HEAD = 2


def _evictable(L: int, n_sink: int, n_recent: int) -> int:
    return max(0, L - n_sink - n_recent)


def tri_logits(q_cal: np.ndarray, K: np.ndarray, G: int) -> np.ndarray:
    """z[h, p] = q_cal[h] . K[p, h * G // H], the plain dot product in fp64
    (each bf16 x bf16 product exact; the sum rounded in fp64).

    q_cal: [H, D] and K: [E, G, D], bf16 values in any float type.
    Returns fp64 [H, E]."""
    q = np.asarray(q_cal, dtype=np.float64)
    H, D = q.shape
    E = K.shape[0]
    z = np.zeros((H, E), dtype=np.float64)
    for h in range(H):
        g = h * G // H
        z[h] = np.asarray(K[:, g, :], dtype=np.float64) @ q[h]
    return z


def tri_scores(q_cal, k_pages, block_table, seqlens, n_sink: int, n_recent: int, mode: int):
    """Per request, its selection rows' scores: fp64 [rows, E_b] with rows = 1
    (union) or G (per-head). q_cal: bf16 bits [H, D]; k_pages: bf16 bits
    [num_pages, P, G, D]."""
    G = k_pages.shape[2]
    q_cal = bf16_bits_to_f64(q_cal)
    H = q_cal.shape[0]
    qpk = H // G
    out = []
    for b, L in enumerate(np.asarray(seqlens)):
        E = _evictable(int(L), n_sink, n_recent)
        tokens = np.arange(n_sink, n_sink + E)
        K = bf16_bits_to_f64(gather_token_rows(k_pages, block_table[b], tokens))
        z = tri_logits(q_cal, K, G)
        zs = z - z.max(axis=1, keepdims=True) if E > 0 else z
        per_g = np.stack([zs[g * qpk:(g + 1) * qpk].max(axis=0) if E > 0 else np.zeros(0, np.float64)
                          for g in range(G)])
        out.append(per_g if mode == PER_HEAD else per_g.max(axis=0, keepdims=True))
    return out


def tri_select(scores_b: np.ndarray, budget: int) -> np.ndarray:
    """Kept evictable positions per selection row: int64 [rows, budget]
    ascending, or [rows, 0] when the region holds at most ``budget`` tokens."""
    rows, E = scores_b.shape
    if E <= budget:
        return np.zeros((rows, 0), dtype=np.int64)
    out = np.zeros((rows, budget), dtype=np.int64)
    for r in range(rows):
        # full sort by (score descending, position ascending); lexsort keys go last-first
        order = np.lexsort((np.arange(E), -np.asarray(scores_b[r], dtype=np.float64)))
        out[r] = np.sort(order[:budget])
    return out


def tri_kept_tokens(L: int, sel_row: np.ndarray, n_sink: int, n_recent: int, budget: int) -> np.ndarray:
    """Old logical positions of the kept tokens, in their new order."""
    if _evictable(L, n_sink, n_recent) <= budget:
        return np.arange(L)
    return np.concatenate([np.arange(n_sink), n_sink + np.asarray(sel_row), np.arange(L - n_recent, L)])


def tri_compact(k_pages, v_pages, block_table, seqlens, selections, n_sink: int, n_recent: int, budget: int,
                mode: int, inplace: bool = False):
    """Compaction on copies of the pools (or, with ``inplace``, on the pools
    given). Returns (k, v, new_seqlens); every byte outside the kept positions
    is left as it was."""
    k = k_pages if inplace else np.array(k_pages, copy=True)
    v = None if v_pages is None else (v_pages if inplace else np.array(v_pages, copy=True))
    P, G = k.shape[1], k.shape[2]
    new_len = np.zeros(len(seqlens), dtype=np.int32)
    for b, L in enumerate(np.asarray(seqlens)):
        L = int(L)
        if _evictable(L, n_sink, n_recent) <= budget:
            new_len[b] = L
            continue
        new_len[b] = n_sink + budget + n_recent
        bt = np.asarray(block_table[b], dtype=np.int64)
        heads = [list(range(G))] if mode == UNION else [[g] for g in range(G)]
        for r, hs in enumerate(heads):
            src = tri_kept_tokens(L, selections[b][r], n_sink, n_recent, budget)
            dst = np.arange(len(src))
            sp, ss = bt[src // P], src % P
            dp, ds = bt[dst // P], dst % P
            for pool in (k, v):
                if pool is None:
                    continue
                rows = pool[sp, ss][:, hs].copy()  # all reads before any write
                for j in range(len(dst)):
                    pool[dp[j], ds[j], hs] = rows[j]
    return k, v, new_len


def tri_evict(q_cal, k_pages, v_pages, block_table, seqlens, n_sink: int, n_recent: int, budget: int, mode: int,
              inplace: bool = False):
    """Scores, selection and compaction of one layer: (k, v, new_seqlens, selections)."""
    scores = tri_scores(q_cal, k_pages, block_table, seqlens, n_sink, n_recent, mode)
    selections = [tri_select(s, budget) for s in scores]
    k, v, new_len = tri_compact(k_pages, v_pages, block_table, seqlens, selections, n_sink, n_recent, budget, mode,
                                inplace)
    return k, v, new_len, selections


def tri_evict_layers(q_cals, k_pools, v_pools, block_table, seqlens, n_sink: int, n_recent: int, budget: int,
                     mode: int):
    """Several layers sharing the block table ("Add TriAttention KV-cache
    compression method", Summary: union, per_head and per_layer_perhead modes).
    UNION / PER_HEAD: one selection for every layer, from the maximum over
    layers of each layer's scores in that mode; PER_LAYER_PER_HEAD: each layer
    evicted on its own, per head. Returns (k_pools, v_pools, new_seqlens,
    selections); v_pools is None without V."""
    n = len(k_pools)
    if mode == PER_LAYER_PER_HEAD:
        ks, vs, sels = [], [], []
        for l in range(n):
            k, v, nl, sel = tri_evict(q_cals[l], k_pools[l], None if v_pools is None else v_pools[l], block_table,
                                      seqlens, n_sink, n_recent, budget, PER_HEAD)
            ks.append(k)
            vs.append(v)
            sels.append(sel)
        return ks, (None if v_pools is None else vs), nl, sels
    per_layer = [tri_scores(q_cals[l], k_pools[l], block_table, seqlens, n_sink, n_recent, mode) for l in range(n)]
    scores = [np.maximum.reduce([per_layer[l][b] for l in range(n)]) for b in range(len(seqlens))]
    selections = [tri_select(sc, budget) for sc in scores]
    ks, vs = [], []
    for l in range(n):
        k, v, nl = tri_compact(k_pools[l], None if v_pools is None else v_pools[l], block_table, seqlens, selections,
                               n_sink, n_recent, budget, mode)
        ks.append(k)
        vs.append(v)
    return ks, (None if v_pools is None else vs), nl, selections
