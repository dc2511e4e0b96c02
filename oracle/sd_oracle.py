"""CPU oracle for top-k sparse decode attention over a paged KV cache.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
module. The library (``top_sparse_decode_paged_b200``) never calls it and shares
no code with it.

What it computes, plainly and slowly (integers exactly in int64, floating point
in fp64), following the pages' description of the DSA decode step
("Overlap DSA heuristic prev_topk write-back on the aux stream", Description:
indexer -> top-k buffer -> core sparse attention) and its golden-reference
pattern ("Add DSA Vanilla sparse attention", Walkthrough: rebuild each
request's logical cache from the pages, validate request-local selections,
attend over the selected tokens):

1. ``indexer_scores``  s[b,g,t] = sum_h w[b,g,h] * max(0, sum_d qi[b,g,h,d] * ki[t,g,d])
   for every cached token t < L_b, keys read through the block table.
2. ``topk_indices``    full sort by (score descending, token ascending); keep the
   first min(k, L_b); emit them in ascending token order; pad with -1.
3. ``sparse_attention`` for every query head h (KV head g = h // (H/G)):
   o = sum_j softmax_j(scale * q_h . K_j) V_j over the selected rows j.
4. ``dense_attention``  the same over every cached token (the dense golden case).
5. ``expand_csr`` / ``sparse_attention_csr``  the selection given as CSR
   offsets and block-sized indices ("Unify sparse attention framework with
   clean backend interfaces", runtime parameters), expanded to tokens.

Readings where the pages are silent (the pages never write the formulas):
the per-head ReLU and integer head weights of the indexer; ties broken toward
the lower token index; ascending output order with -1 padding; V as the first
Dv columns of the MLA latent row; contiguous GQA groups. Each is listed in the
design notes with its reason.

Parity pins: every function here is checked in ``tests/test_oracle_pins.py``
against brute force on tiny inputs, closed forms, invariants and independent
library routines (numpy lexsort, torch scaled_dot_product_attention in fp64).
"""

from __future__ import annotations

import numpy as np


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact value of bf16 numbers given as uint16 bits."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def gather_token_rows(pages: np.ndarray, block_table_row: np.ndarray, tokens: np.ndarray) -> np.ndarray:
    """Rows of request-local tokens from a paged pool [num_pages, P, ...].

    Token t of the request lives in physical page block_table_row[t // P] at
    slot t % P (the block-table translation from request-local to global rows
    described in "Unify sparse attention framework...", review notes on DSA
    global index conversion)."""
    P = pages.shape[1]
    tokens = np.asarray(tokens, dtype=np.int64)
    phys = np.asarray(block_table_row, dtype=np.int64)[tokens // P]
    if np.any(phys < 0) or np.any(phys >= pages.shape[0]):
        raise ValueError("block table entry out of range for a valid token")
    return pages[phys, tokens % P]


def indexer_scores(qi, w, ki_pages, block_table, seqlens, requests=None):
    """Exact int64 indexer scores; returns a list (one per request) of [G, L_b] arrays.

    s[b,g,t] = sum_h w[b,g,h] * max(0, sum_d qi[b,g,h,d] * ki[phys(t), slot(t), g, d]).
    The int dot products go through an fp64 matmul, which is exact here because
    every partial sum is an integer far below 2**53 (|q|,|k| <= 127, Di <= 512)."""
    qi = np.asarray(qi)
    B, G, Hi, Di = qi.shape
    req = range(B) if requests is None else requests
    out = []
    for b in req:
        L = int(seqlens[b])
        rows = gather_token_rows(ki_pages, block_table[b], np.arange(L))  # [L, G, Di]
        s = np.zeros((G, L), dtype=np.int64)
        for g in range(G):
            kg = rows[:, g, :].astype(np.float64)                       # [L, Di]
            dots = qi[b, g].astype(np.float64) @ kg.T                   # [Hi, L]
            dots = np.rint(dots).astype(np.int64)
            relu = np.maximum(dots, 0)
            s[g] = (w[b, g].astype(np.int64)[:, None] * relu).sum(axis=0)
        out.append(s)
    return out


def topk_row(scores_row: np.ndarray, k: int) -> np.ndarray:
    """Top-k of one row under the total order (score desc, token asc).

    Returns int32 [k]: the selected tokens in ascending order, then -1 padding."""
    L = int(scores_row.shape[0])
    kk = min(k, L)
    # np.lexsort sorts by the last key first: score descending, then token ascending
    order = np.lexsort((np.arange(L), -np.asarray(scores_row, dtype=np.int64)))
    chosen = np.sort(np.asarray(order[:kk], dtype=np.int64))
    out = np.full(k, -1, dtype=np.int32)
    out[:kk] = chosen
    return out


def topk_indices(scores_per_req, k: int):
    """Per request, per KV head top-k; returns a list of int32 [G, k] arrays."""
    return [np.stack([topk_row(s[g], k) for g in range(s.shape[0])]) for s in scores_per_req]


def attend_rows(qh: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float):
    """softmax(scale * K qh) weighted sum of V, in fp64. Returns (o, lse)."""
    if K.shape[0] == 0:
        return np.zeros(V.shape[1]), -np.inf
    z = scale * (K @ qh)
    m = z.max()
    p = np.exp(z - m)
    l = p.sum()
    return (p @ V) / l, m + np.log(l)


def _kv_rows(wl_k_pages, wl_v_pages, Dv, block_table_row, tokens, g):
    K = bf16_bits_to_f64(gather_token_rows(wl_k_pages, block_table_row, tokens)[:, g, :])
    if wl_v_pages is None:
        V = K[:, :Dv]
    else:
        V = bf16_bits_to_f64(gather_token_rows(wl_v_pages, block_table_row, tokens)[:, g, :])
    return K, V


def sparse_attention(q, k_pages, v_pages, Dv, block_table, seqlens, indices, scale, requests=None):
    """Selected-token attention; returns (out [n_req, H, Dv] fp64, lse [n_req, H]).

    ``indices[b]`` is [G, k] of request-local tokens (ascending, -1 padded); the
    query head h reads KV head g = h // (H // G). ``v_pages`` None means V is the
    first Dv columns of the K row."""
    q = np.asarray(q)
    B, H, Dk = q.shape
    G = indices[0].shape[0] if len(indices) else 1
    qpk = H // G
    req = list(range(B)) if requests is None else list(requests)
    out = np.zeros((len(req), H, Dv))
    lse = np.zeros((len(req), H))
    for i, b in enumerate(req):
        L = int(seqlens[b])
        for g in range(G):
            sel = np.asarray(indices[i][g], dtype=np.int64)
            sel = sel[sel >= 0]
            if np.any(sel >= L):
                raise ValueError("selected token beyond seqlen")
            K, V = _kv_rows(k_pages, v_pages, Dv, block_table[b], sel, g)
            for h in range(g * qpk, (g + 1) * qpk):
                out[i, h], lse[i, h] = attend_rows(bf16_bits_to_f64(q[b, h]), K, V, scale)
    return out, lse


def expand_csr(indices_flat, offsets, block_size, seqlens, G, max_selected):
    """The packed selection of the unified sparse runtime ("Unify sparse
    attention framework with clean backend interfaces", runtime parameters
    sparse_attn_offsets / sparse_attn_indices_block_size), in the padded form.

    Row r = b*G + g owns entries offsets[r] .. offsets[r+1]-1. Entry e covers
    tokens e*bs .. e*bs+bs-1 with bs = max(block_size, 1); entries < 0 are
    skipped and tokens at or past L_b dropped; the valid tokens keep list order
    and the first min(max_selected, L_b) are kept. Returns, per request, int64
    [G, max_selected] padded with -1."""
    bs = max(int(block_size), 1)
    out = []
    for b in range(len(seqlens)):
        L = int(seqlens[b])
        cap = min(int(max_selected), L)
        rows = np.full((G, int(max_selected)), -1, dtype=np.int64)
        for g in range(G):
            r = b * G + g
            toks = []
            for j in range(int(offsets[r]), int(offsets[r + 1])):
                e = int(indices_flat[j])
                if e < 0:
                    continue
                for u in range(bs):
                    t = e * bs + u
                    if t < L:
                        toks.append(t)
            toks = toks[:cap]
            rows[g, :len(toks)] = toks
        out.append(rows)
    return out


def sparse_attention_csr(q, k_pages, v_pages, Dv, block_table, seqlens, indices_flat, offsets, block_size,
                         max_selected, scale, requests=None):
    """Selected-token attention with the selection in CSR / block form
    (``expand_csr``); duplicates are attended as listed."""
    G = k_pages.shape[2]
    sel = expand_csr(indices_flat, offsets, block_size, seqlens, G, max_selected)
    req = list(range(len(seqlens))) if requests is None else list(requests)
    return sparse_attention(q, k_pages, v_pages, Dv, block_table, seqlens, [sel[b] for b in req], scale,
                            requests=req)


def dense_attention(q, k_pages, v_pages, Dv, block_table, seqlens, G, scale, requests=None):
    """Attention over every cached token t < L_b (the dense golden case)."""
    B = q.shape[0]
    req = list(range(B)) if requests is None else list(requests)
    idx = []
    for b in req:
        L = int(seqlens[b])
        idx.append(np.tile(np.arange(L, dtype=np.int64), (G, 1)))
    out = np.zeros((len(req), q.shape[1], Dv))
    lse = np.zeros((len(req), q.shape[1]))
    for i, b in enumerate(req):
        o, l_ = sparse_attention(q[b:b + 1], k_pages, v_pages, Dv, block_table[b:b + 1],
                                 seqlens[b:b + 1], [idx[i]], scale)
        out[i], lse[i] = o[0], l_[0]
    return out, lse


def decode_step(wl, requests=None):
    """The whole step on a workload: scores -> top-k -> sparse attention.

    Returns dict(scores=list of int64 [G, L_b], indices=list of int32 [G, k],
    out=fp64 [n_req, H, Dv], lse=fp64 [n_req, H])."""
    s = wl.spec
    req = list(range(wl.seqlens.shape[0])) if requests is None else list(requests)
    scores = indexer_scores(wl.qi, wl.w, wl.ki_pages, wl.block_table, wl.seqlens, req)
    idx = topk_indices(scores, s.k)
    out, lse = sparse_attention(wl.q, wl.k_pages, wl.v_pages, s.Dv, wl.block_table,
                                wl.seqlens, idx, s.scale, req)
    return dict(scores=scores, indices=idx, out=out, lse=lse)
