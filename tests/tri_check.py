"""Validity check of a GPU eviction against the oracle's exact scores.

The eviction's scores only decide an integer selection, and the library sums
its dot products in fp32. So the GPU's kept set is not compared with the
oracle's by replaying the kernel's rounding. It is checked to be a valid
top-`budget` set under the oracle's exact (fp64) scores, allowing each score
the error that any fp32 evaluation of it can carry:

  z_h(p)   = sum_d q[h,d] K[p,d]: every product exact (bf16 factors, fused
             multiply-add or fp32 product of 8-bit significands), D - 1 fp32
             additions in any order: |err| <= gamma_D sum_d |q K| = beta_h(p),
             gamma_D = D u / (1 - D u), u = 2^-24 (recursive summation bound);
  m_h      = max_p z_h(p): off by at most B_h = max_p beta_h(p);
  z_h - m_h, one fp32 subtraction: adds u |z_h - m_h| (with the errors above);
  maxima over heads and layers: exact, so the bound is the largest operand's.

A kept position p and a dropped position q are consistent with some fp32
evaluation iff s(p) + slack(p) >= s(q) - slack(q); that holds for every pair
iff min over kept of (s + slack) >= max over dropped of (s - slack). Where the
boundary is separated by more than the slack, that leaves exactly one valid
set, the oracle's.

The kept set is read back from the compacted K pool: kept slot i holds the
row of region position sel[i], and sel is ascending, so slot rows are matched
to region rows in order (the earliest matching position each time).
"""
from __future__ import annotations

import numpy as np

from oracle import tri_oracle as T
from oracle.sd_oracle import bf16_bits_to_f64, gather_token_rows

U32 = 2.0 ** -24
U64 = 2.0 ** -53


def score_bounds(q_cal, k_pages, block_table, seqlens, n_sink: int, n_recent: int, mode: int):
    """Per request: (scores, slack), each fp64 [rows, E_b]; scores are the
    oracle's, slack the fp32 evaluation bound derived in the module text."""
    scores = T.tri_scores(q_cal, k_pages, block_table, seqlens, n_sink, n_recent, mode)
    q = bf16_bits_to_f64(q_cal)
    H, D = q.shape
    G = k_pages.shape[2]
    qpk = H // G
    gamma = D * U32 / (1.0 - D * U32)
    out = []
    for b, L in enumerate(np.asarray(seqlens)):
        E = max(0, int(L) - n_sink - n_recent)
        sc = scores[b]
        if E == 0:
            out.append((sc, np.zeros_like(sc)))
            continue
        K = bf16_bits_to_f64(gather_token_rows(k_pages, block_table[b], np.arange(n_sink, n_sink + E)))
        err = np.zeros((H, E))
        for h in range(H):
            g = h // qpk
            z = K[:, g, :] @ q[h]
            a = np.abs(K[:, g, :]) @ np.abs(q[h])
            beta = gamma * a
            big_b = beta.max()
            shifted = np.abs(z - z.max())
            e32 = (beta + big_b) * (1.0 + U32) + U32 * shifted
            e64 = 4.0 * D * U64 * (a + a.max())  # the oracle's own fp64 rounding, generously
            err[h] = e32 + e64
        per_g = np.stack([err[g * qpk:(g + 1) * qpk].max(axis=0) for g in range(G)])
        slack = per_g if mode == T.PER_HEAD else per_g.max(axis=0, keepdims=True)
        out.append((sc, slack))
    return out


def combine_layers(per_layer):
    """Cross-layer selection scores (maximum over layers) and their slack."""
    n_req = len(per_layer[0])
    out = []
    for b in range(n_req):
        sc = np.maximum.reduce([per_layer[l][b][0] for l in range(len(per_layer))])
        sl = np.maximum.reduce([per_layer[l][b][1] for l in range(len(per_layer))])
        out.append((sc, sl))
    return out


def valid_selection(scores_row, slack_row, sel, budget: int) -> bool:
    """sel is a valid top-`budget` set of the row under the bound."""
    E = scores_row.shape[0]
    sel = np.asarray(sel, dtype=np.int64)
    if E <= budget:
        return sel.size == 0
    if sel.shape != (budget,) or np.any(np.diff(sel) <= 0) or sel[0] < 0 or sel[-1] >= E:
        return False
    dropped = np.ones(E, dtype=bool)
    dropped[sel] = False
    lo = float((scores_row[sel] + slack_row[sel]).min())
    hi = float((scores_row[dropped] - slack_row[dropped]).max())
    return lo >= hi


def separated(scores_row, slack_row, budget: int) -> bool:
    """The row's boundary leaves exactly one valid set (the oracle's)."""
    E = scores_row.shape[0]
    if E <= budget:
        return True
    sel = T.tri_select(scores_row[None], budget)[0]
    dropped = np.ones(E, dtype=bool)
    dropped[sel] = False
    return float((scores_row[sel] - slack_row[sel]).min()) > float((scores_row[dropped] + slack_row[dropped]).max())


def infer_selection(k_before, k_after, block_table, seqlens, n_sink: int, n_recent: int, budget: int, mode: int):
    """The kept region positions per request and selection row, read back from
    the compacted K pool (raises AssertionError if a kept slot matches no
    region row in order)."""
    P, G = k_before.shape[1], k_before.shape[2]
    sels = []
    for b, L in enumerate(np.asarray(seqlens)):
        L = int(L)
        E = max(0, L - n_sink - n_recent)
        rows = 1 if mode == T.UNION else G
        if E <= budget:
            sels.append(np.zeros((rows, 0), dtype=np.int64))
            continue
        bt = np.asarray(block_table[b], dtype=np.int64)
        region = np.arange(n_sink, n_sink + E)
        slots = np.arange(n_sink, n_sink + budget)
        before = k_before[bt[region // P], region % P]   # [E, G, D]
        after = k_after[bt[slots // P], slots % P]        # [budget, G, D]
        sel = np.zeros((rows, budget), dtype=np.int64)
        for r in range(rows):
            hs = slice(None) if mode == T.UNION else slice(r, r + 1)
            src = before[:, hs].reshape(E, -1)
            dst = after[:, hs].reshape(budget, -1)
            where = {}
            for p in range(E - 1, -1, -1):
                where.setdefault(src[p].tobytes(), []).append(p)  # descending lists: pop() gives the earliest
            last = -1
            for i in range(budget):
                cand = where.get(dst[i].tobytes(), [])
                while cand and cand[-1] <= last:
                    cand.pop()
                assert cand, f"request {b}, row {r}: kept slot {i} holds no region row after position {last}"
                last = cand.pop()
                sel[r, i] = last
        sels.append(sel)
    return sels


def _request_pages(block_table_row, L: int, P: int, num_pages: int) -> np.ndarray:
    n = (int(L) + P - 1) // P
    pages = np.asarray(block_table_row[:n], dtype=np.int64)
    return pages[(pages >= 0) & (pages < num_pages)]


def check_eviction(q_cals, k_pools, v_pools, block_table, seqlens, n_sink: int, n_recent: int, budget: int,
                   mode: int, k_gpu, v_gpu, nl_gpu, requests=None):
    """Checks a GPU eviction of len(k_pools) layers (pools before: k_pools /
    v_pools; after, from the GPU: k_gpu / v_gpu; new lengths nl_gpu): new
    lengths exact, every kept set valid under the bound, and every byte of
    each request's pages equal to the oracle's compaction with the GPU's kept
    sets. With ``requests`` None every request is checked and pages no request
    owns must be unchanged; otherwise only those requests (their pages must be
    disjoint from the others'). Returns the kept sets, [layer][request]."""
    n = len(k_pools)
    P, num_pages = k_pools[0].shape[1], k_pools[0].shape[0]
    seqlens = np.asarray(seqlens)
    reqs = range(len(seqlens)) if requests is None else list(requests)
    if mode == T.PER_LAYER_PER_HEAD:
        groups = [([l], T.PER_HEAD) for l in range(n)]
    else:
        groups = [(list(range(n)), mode)]
    kept = [dict() for _ in range(n)]
    for layers, m in groups:
        bounds = combine_layers([score_bounds(q_cals[l], k_pools[l], block_table, seqlens, n_sink, n_recent, m)
                                 for l in layers])
        l0 = layers[0]
        for b in reqs:
            L = int(seqlens[b])
            sel = infer_selection(k_pools[l0], k_gpu[l0], block_table[b:b + 1], seqlens[b:b + 1], n_sink, n_recent,
                                  budget, m)[0]
            sc, slack = bounds[b]
            for r in range(sc.shape[0]):
                assert valid_selection(sc[r], slack[r], sel[r], budget), (
                    f"request {b}, row {r}: kept set is not a top-{budget} set within the fp32 bound")
            pages = _request_pages(block_table[b], L, P, num_pages)
            local_bt = np.full((1, block_table.shape[1]), -1, dtype=np.int64)
            local_bt[0, :pages.size] = np.arange(pages.size)
            for l in layers:
                k_ref, v_ref, nl_ref = T.tri_compact(k_pools[l][pages], None if v_pools is None else v_pools[l][pages],
                                                     local_bt, seqlens[b:b + 1], [sel], n_sink, n_recent, budget, m)
                assert int(nl_gpu[b]) == int(nl_ref[0]), f"request {b}: new length {nl_gpu[b]} != {nl_ref[0]}"
                assert np.array_equal(k_gpu[l][pages], k_ref), f"layer {l}, request {b}: K pool differs"
                if v_pools is not None:
                    assert np.array_equal(v_gpu[l][pages], v_ref), f"layer {l}, request {b}: V pool differs"
                kept[l][b] = sel
    if requests is None:
        owned = np.zeros(num_pages, dtype=bool)
        for b in range(len(seqlens)):
            owned[_request_pages(block_table[b], int(seqlens[b]), P, num_pages)] = True
        for l in range(n):
            assert np.array_equal(k_gpu[l][~owned], k_pools[l][~owned]), f"layer {l}: a page no request owns changed"
            if v_pools is not None:
                assert np.array_equal(v_gpu[l][~owned], v_pools[l][~owned])
    return kept
