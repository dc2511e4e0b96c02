"""Pins for the CPU oracle: each check ties the oracle to something other than
itself (brute force in pure Python, closed forms, invariants, special cases that
reduce to a textbook or library routine). A plausible slip anywhere in the
oracle (a dropped ReLU, a transposed operand, a wrong page/slot split, the wrong
tie direction, a missing max-subtraction, the wrong GQA group) fails one of them;
``test_planted_mistakes_are_caught`` plants such slips and checks exactly that.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from top_sparse_decode_paged_b200 import workloads as W


# ----------------------------------------------------------------------------
# tiny hand-built paged inputs (independent of the workload generator)
# ----------------------------------------------------------------------------
def _tiny_paged(seed=0, B=3, G=2, Hi=3, Di=8, P=4, lens=(5, 11, 1), Dk=6, Dv=4, H=4,
                separate_v=True):
    rng = np.random.default_rng(seed)
    pages_per = [(L + P - 1) // P for L in lens]
    n_pages = sum(pages_per) + 1
    perm = rng.permutation(n_pages)
    bt = np.full((B, max(pages_per)), -1, dtype=np.int32)
    c = 0
    for b, n in enumerate(pages_per):
        bt[b, :n] = perm[c:c + n]
        c += n
    qi = rng.integers(-64, 65, size=(B, G, Hi, Di)).astype(np.int8)
    w = rng.integers(1, 9, size=(B, G, Hi)).astype(np.int32)
    ki = rng.integers(-64, 65, size=(n_pages, P, G, Di)).astype(np.int8)
    q = W.bf16_bits_from_f32(rng.standard_normal((B, H, Dk)).astype(np.float32))
    kp = W.bf16_bits_from_f32(rng.standard_normal((n_pages, P, G, Dk)).astype(np.float32))
    vp = W.bf16_bits_from_f32(rng.standard_normal((n_pages, P, G, Dv)).astype(np.float32)) \
        if separate_v else None
    return dict(qi=qi, w=w, ki=ki, bt=bt, seqlens=np.asarray(lens, dtype=np.int32),
                q=q, kp=kp, vp=vp, P=P, G=G, H=H, Dk=Dk, Dv=Dv)


def _bf16_to_float(bits):
    """Pure-Python bf16 decode (sign, exponent, mantissa), no numpy views."""
    bits = int(bits)
    sign = -1.0 if bits & 0x8000 else 1.0
    e = (bits >> 7) & 0xFF
    m = bits & 0x7F
    if e == 0:
        return sign * m * 2.0 ** (-133)
    if e == 0xFF:
        return float("nan") if m else sign * float("inf")
    return sign * (1.0 + m / 128.0) * 2.0 ** (e - 127)


def _brute_scores(d):
    """Pure-Python loops over the definition, token by token."""
    B, G, Hi, Di = d["qi"].shape
    P = d["P"]
    out = []
    for b in range(B):
        rows = []
        for g in range(G):
            row = []
            for t in range(int(d["seqlens"][b])):
                page = int(d["bt"][b][t // P])
                slot = t % P
                total = 0
                for h in range(Hi):
                    dot = 0
                    for e in range(Di):
                        dot += int(d["qi"][b][g][h][e]) * int(d["ki"][page][slot][g][e])
                    total += int(d["w"][b][g][h]) * (dot if dot > 0 else 0)
                row.append(total)
            rows.append(row)
        out.append(rows)
    return out


def _brute_topk(row, k):
    """Pure-Python selection by repeated arg-max (highest score, lowest token)."""
    remaining = list(range(len(row)))
    chosen = []
    for _ in range(min(k, len(row))):
        best = remaining[0]
        for t in remaining:
            if row[t] > row[best]:
                best = t
        chosen.append(best)
        remaining.remove(best)
    chosen.sort()
    return chosen + [-1] * (k - len(chosen))


def _brute_attention(d, indices, scale):
    """Pure-Python softmax attention with math.exp, no numpy arithmetic."""
    B, H, Dk = d["q"].shape
    G, P, Dv = d["G"], d["P"], d["Dv"]
    qpk = H // G
    out = []
    for b in range(B):
        ob = []
        for h in range(H):
            g = h // qpk
            sel = [t for t in indices[b][g] if t >= 0]
            logits, vrows = [], []
            for t in sel:
                page, slot = int(d["bt"][b][t // P]), t % P
                krow = [_bf16_to_float(x) for x in d["kp"][page][slot][g]]
                if d["vp"] is None:
                    vrow = krow[:Dv]
                else:
                    vrow = [_bf16_to_float(x) for x in d["vp"][page][slot][g]]
                qh = [_bf16_to_float(x) for x in d["q"][b][h]]
                logits.append(scale * sum(a * c for a, c in zip(qh, krow)))
                vrows.append(vrow)
            m = max(logits)
            ps = [math.exp(z - m) for z in logits]
            l = sum(ps)
            ob.append([sum(p * v[j] for p, v in zip(ps, vrows)) / l for j in range(Dv)])
        out.append(ob)
    return np.asarray(out)


# ----------------------------------------------------------------------------
# indexer scores
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_scores_match_python_brute_force(seed):
    d = _tiny_paged(seed)
    got = oracle.indexer_scores(d["qi"], d["w"], d["ki"], d["bt"], d["seqlens"])
    ref = _brute_scores(d)
    for b in range(len(ref)):
        assert got[b].tolist() == ref[b]


def test_scores_closed_form_one_hot_query():
    """qi = e_j in head 0 only (other heads zero): s[t] = w0 * max(0, k[t][j])."""
    d = _tiny_paged(5, B=1, G=1, Hi=3, Di=8, lens=(13,))
    j = 3
    d["qi"][:] = 0
    d["qi"][0, 0, 0, j] = 1
    s = oracle.indexer_scores(d["qi"], d["w"], d["ki"], d["bt"], d["seqlens"])[0][0]
    P = d["P"]
    for t in range(13):
        kv = int(d["ki"][d["bt"][0][t // P]][t % P][0][j])
        assert s[t] == int(d["w"][0, 0, 0]) * max(0, kv)


def test_scores_hand_worked_example():
    """Two heads, Di=2, three tokens on two pages (page size 2, pages swapped).

    q0=(1,2), q1=(-3,1), w=(2,5); tokens k0=(1,1), k1=(2,-1), k2=(-1,4).
    head0 dots: 3, 0, 7      -> relu 3, 0, 7
    head1 dots: -2, -7, 7    -> relu 0, 0, 7
    s = 2*relu0 + 5*relu1 = (6, 0, 14+35=49)."""
    qi = np.array([[[[1, 2], [-3, 1]]]], dtype=np.int8)
    w = np.array([[[2, 5]]], dtype=np.int32)
    ki = np.zeros((2, 2, 1, 2), dtype=np.int8)
    ki[1, 0, 0] = (1, 1)    # token 0 -> page 1 slot 0
    ki[1, 1, 0] = (2, -1)   # token 1 -> page 1 slot 1
    ki[0, 0, 0] = (-1, 4)   # token 2 -> page 0 slot 0
    ki[0, 1, 0] = (99, 99)  # slack slot, beyond seqlen
    bt = np.array([[1, 0]], dtype=np.int32)
    s = oracle.indexer_scores(qi, w, ki, bt, np.array([3], dtype=np.int32))[0][0]
    assert s.tolist() == [6, 0, 49]


def test_scores_int32_range_at_workload_bounds():
    """Largest possible score at the biggest shapes stays inside int32."""
    for name in W.CONFIG_ORDER:
        s = W.spec(name)
        kmax = 64 + s.cluster_shift if s.clusters else 64
        bound = s.Hi * 8 * s.Di * 64 * kmax
        assert bound < 2 ** 31, name


# ----------------------------------------------------------------------------
# top-k
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("seed", range(6))
def test_topk_matches_repeated_argmax(seed):
    rng = np.random.default_rng(seed)
    L = int(rng.integers(1, 40))
    row = rng.integers(0, 6, size=L)  # heavy ties on purpose
    for k in (1, 3, 8, 40, 64):
        assert oracle.topk_row(row, k).tolist() == _brute_topk(row.tolist(), k)


def test_topk_all_equal_takes_lowest_tokens():
    row = np.full(1000, 7, dtype=np.int64)
    assert oracle.topk_row(row, 32).tolist() == list(range(32))


def test_topk_k_at_least_seqlen_takes_all():
    row = np.array([5, 1, 9], dtype=np.int64)
    assert oracle.topk_row(row, 8).tolist() == [0, 1, 2, -1, -1, -1, -1, -1]


def test_topk_invariants_on_generated_workload():
    wl = W.make(W.spec("b4_l4096_mla", B=2))
    sc = oracle.indexer_scores(wl.qi, wl.w, wl.ki_pages, wl.block_table, wl.seqlens)
    idx = oracle.topk_indices(sc, wl.spec.k)
    for b in range(2):
        s, sel = sc[b][0], idx[b][0]
        k = min(wl.spec.k, s.shape[0])
        assert (sel[:k] >= 0).all() and (sel[k:] == -1).all()
        assert np.all(np.diff(sel[:k]) > 0)                      # ascending, unique
        mask = np.zeros(s.shape[0], dtype=bool)
        mask[sel[:k]] = True
        lo, hi = s[mask].min(), s[~mask].max()
        assert lo >= hi                                          # threshold property
        if lo == hi:                                             # ties go to lower tokens
            assert np.flatnonzero(mask & (s == lo)).max() < np.flatnonzero(~mask & (s == lo)).min()


# ----------------------------------------------------------------------------
# attention
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("separate_v", [True, False])
def test_attention_matches_python_brute_force(separate_v):
    d = _tiny_paged(7, separate_v=separate_v, Dv=4)
    rng = np.random.default_rng(1)
    idx = []
    for b, L in enumerate(d["seqlens"]):
        rows = []
        for g in range(d["G"]):
            k = 4
            sel = np.sort(rng.choice(int(L), size=min(k, int(L)), replace=False))
            rows.append(list(sel) + [-1] * (k - len(sel)))
        idx.append(np.asarray(rows, dtype=np.int32))
    out, _ = oracle.sparse_attention(d["q"], d["kp"], d["vp"], d["Dv"], d["bt"], d["seqlens"], idx, 0.37)
    ref = _brute_attention(d, idx, 0.37)
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)


def test_attention_dense_matches_torch_sdpa_fp64():
    """k >= seqlen: the selected-token result equals dense attention, and dense
    attention equals torch's scaled_dot_product_attention in float64 on a
    contiguous cache rebuilt here with plain loops."""
    d = _tiny_paged(11, B=2, G=2, H=6, lens=(9, 14), Dk=16, Dv=16)
    scale = 0.25
    B, H = 2, 6
    dense, _ = oracle.dense_attention(d["q"], d["kp"], d["vp"], d["Dv"], d["bt"], d["seqlens"],
                                      d["G"], scale)
    sc = [np.zeros((d["G"], int(L)), dtype=np.int64) for L in d["seqlens"]]
    full_idx = oracle.topk_indices(sc, 64)                    # k >= L: everything
    sparse, _ = oracle.sparse_attention(d["q"], d["kp"], d["vp"], d["Dv"], d["bt"], d["seqlens"],
                                        full_idx, scale)
    np.testing.assert_allclose(sparse, dense, rtol=1e-13, atol=1e-13)
    P = d["P"]
    for b in range(B):
        L = int(d["seqlens"][b])
        K = torch.zeros(d["G"], L, d["Dk"], dtype=torch.float64)
        V = torch.zeros(d["G"], L, d["Dv"], dtype=torch.float64)
        for t in range(L):
            page, slot = int(d["bt"][b][t // P]), t % P
            for g in range(d["G"]):
                K[g, t] = torch.tensor([_bf16_to_float(x) for x in d["kp"][page][slot][g]])
                V[g, t] = torch.tensor([_bf16_to_float(x) for x in d["vp"][page][slot][g]])
        Q = torch.tensor([[_bf16_to_float(x) for x in d["q"][b][h]] for h in range(H)],
                         dtype=torch.float64).view(d["G"], H // d["G"], 1, d["Dk"])
        ref = torch.nn.functional.scaled_dot_product_attention(
            Q, K[:, None].expand(-1, H // d["G"], -1, -1), V[:, None].expand(-1, H // d["G"], -1, -1),
            scale=scale)
        np.testing.assert_allclose(dense[b], ref.reshape(H, d["Dv"]).numpy(), rtol=1e-12, atol=1e-12)


def test_attention_single_row_returns_that_row_exactly():
    d = _tiny_paged(3, B=1, G=1, H=2, lens=(9,), separate_v=True)
    idx = [np.array([[6, -1, -1]], dtype=np.int32)]
    out, lse = oracle.sparse_attention(d["q"], d["kp"], d["vp"], d["Dv"], d["bt"], d["seqlens"], idx, 1.0)
    page, slot = d["bt"][0][6 // d["P"]], 6 % d["P"]
    v = np.array([_bf16_to_float(x) for x in d["vp"][page][slot][0]])
    assert (out[0] == v[None, :]).all()


def test_attention_zero_query_gives_mean_of_rows():
    d = _tiny_paged(4, B=1, G=1, H=2, lens=(11,), separate_v=False, Dk=6, Dv=4)
    d["q"][:] = 0
    sel = [0, 3, 4, 10]
    idx = [np.array([sel + [-1]], dtype=np.int32)]
    out, lse = oracle.sparse_attention(d["q"], d["kp"], None, 4, d["bt"], d["seqlens"], idx, 0.5)
    P = d["P"]
    rows = np.array([[_bf16_to_float(x) for x in d["kp"][d["bt"][0][t // P]][t % P][0][:4]] for t in sel])
    np.testing.assert_allclose(out[0, 0], rows.mean(axis=0), rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(lse[0], math.log(len(sel)), rtol=1e-13)


def test_attention_constant_values_give_that_constant():
    d = _tiny_paged(8, B=1, G=1, H=3, lens=(12,), separate_v=True)
    d["vp"][:] = W.bf16_bits_from_f32(np.array([1.5], dtype=np.float32))[0]
    idx = [np.array([[1, 2, 7, 11]], dtype=np.int32)]
    out, _ = oracle.sparse_attention(d["q"], d["kp"], d["vp"], d["Dv"], d["bt"], d["seqlens"], idx, 0.9)
    np.testing.assert_allclose(out, 1.5, rtol=1e-14)


def test_gqa_group_mapping_uses_contiguous_heads():
    """With G=2, H=4 heads 0,1 read KV head 0 and heads 2,3 read KV head 1:
    checked by making KV head 1's values a constant."""
    d = _tiny_paged(9, B=1, G=2, H=4, lens=(8,), separate_v=True)
    d["vp"][:, :, 1, :] = W.bf16_bits_from_f32(np.array([-2.0], dtype=np.float32))[0]
    idx = [np.array([[0, 1, 2], [3, 4, 5]], dtype=np.int32)]
    out, _ = oracle.sparse_attention(d["q"], d["kp"], d["vp"], d["Dv"], d["bt"], d["seqlens"], idx, 1.0)
    np.testing.assert_allclose(out[0, 2:], -2.0, rtol=1e-14)
    assert not np.allclose(out[0, :2], -2.0)


def test_attention_large_logits_stay_finite():
    """Logits of order 1e3 need the max-subtraction; the result stays exact."""
    d = _tiny_paged(12, B=1, G=1, H=1, lens=(6,), separate_v=True)
    idx = [np.array([[0, 1, 2, 3, 4, 5]], dtype=np.int32)]
    out, lse = oracle.sparse_attention(d["q"], d["kp"], d["vp"], d["Dv"], d["bt"], d["seqlens"], idx, 500.0)
    ref = _brute_attention(d, idx, 500.0)
    assert np.isfinite(out).all() and np.isfinite(lse).all()
    np.testing.assert_allclose(out, ref, rtol=1e-10, atol=1e-12)


# ----------------------------------------------------------------------------
# the composed step on a generated workload, and planted mistakes
# ----------------------------------------------------------------------------
def test_decode_step_tiny_is_self_consistent():
    wl = W.make(W.spec("tiny"))
    r = oracle.decode_step(wl)
    assert r["scores"][0].shape == (1, 256)
    assert (r["indices"][0] >= 0).sum() == 32
    assert np.isfinite(r["out"]).all()


def _mutants():
    """Plausible slips, each applied to a copy of one oracle function."""
    def no_relu(qi, w, ki, bt, sl, requests=None):
        B, G, Hi, Di = qi.shape
        out = []
        for b in range(B):
            L = int(sl[b])
            rows = oracle.gather_token_rows(ki, bt[b], np.arange(L))
            s = np.zeros((G, L), dtype=np.int64)
            for g in range(G):
                dots = np.rint(qi[b, g].astype(np.float64) @ rows[:, g, :].astype(np.float64).T).astype(np.int64)
                s[g] = (w[b, g].astype(np.int64)[:, None] * dots).sum(axis=0)
            out.append(s)
        return out

    def slot_swapped(qi, w, ki, bt, sl, requests=None):
        B, G, Hi, Di = qi.shape
        P = ki.shape[1]
        out = []
        for b in range(B):
            L = int(sl[b])
            t = np.arange(L)
            rows = ki[bt[b][t // P], (P - 1 - t % P)]
            s = np.zeros((G, L), dtype=np.int64)
            for g in range(G):
                dots = np.rint(qi[b, g].astype(np.float64) @ rows[:, g, :].astype(np.float64).T).astype(np.int64)
                s[g] = (w[b, g].astype(np.int64)[:, None] * np.maximum(dots, 0)).sum(axis=0)
            out.append(s)
        return out

    def ties_high(row, k):
        L = len(row)
        order = np.lexsort((-np.arange(L), -np.asarray(row, dtype=np.int64)))
        out = np.full(k, -1, dtype=np.int32)
        out[:min(k, L)] = np.sort(order[:min(k, L)])
        return out

    return dict(no_relu=no_relu, slot_swapped=slot_swapped, ties_high=ties_high)


def test_planted_mistakes_are_caught():
    m = _mutants()
    d = _tiny_paged(0)
    ref = _brute_scores(d)
    for name in ("no_relu", "slot_swapped"):
        got = m[name](d["qi"], d["w"], d["ki"], d["bt"], d["seqlens"])
        assert any(got[b].tolist() != ref[b] for b in range(len(ref))), name
    rng = np.random.default_rng(0)
    row = rng.integers(0, 3, size=30)
    assert m["ties_high"](row, 8).tolist() != _brute_topk(row.tolist(), 8)


# ----------------------------------------------------------------------------
# CSR offsets and block-sized indices
# ----------------------------------------------------------------------------
def test_csr_expansion_hand_worked():
    """Blocks of 4 tokens, two requests (L = 22 and 9), G = 1:
    request 0 lists blocks 5 and 0 -> tokens 20, 21 (22, 23 are past L) then
    0..3; request 1 lists block 2 -> token 8 (9..11 past L); a negative entry
    is skipped."""
    out = oracle.expand_csr(np.array([5, 0, -3, 2]), np.array([0, 3, 4]), 4, np.array([22, 9]), 1, 8)
    assert out[0].tolist() == [[20, 21, 0, 1, 2, 3, -1, -1]]
    assert out[1].tolist() == [[8, -1, -1, -1, -1, -1, -1, -1]]
    # at most min(max_selected, L) tokens are kept, in list order
    out = oracle.expand_csr(np.array([1, 4, 6]), np.array([0, 3]), 1, np.array([10]), 1, 2)
    assert out[0].tolist() == [[1, 4]]
    out = oracle.expand_csr(np.array([1, 4, 6]), np.array([0, 3]), 0, np.array([5]), 1, 8)
    assert out[0].tolist() == [[1, 4, -1, -1, -1, -1, -1, -1]]


def test_csr_of_a_padded_selection_is_the_same_attention():
    d = _tiny_paged(21, B=3, G=2, lens=(5, 11, 1), separate_v=True)
    sc = oracle.indexer_scores(d["qi"], d["w"], d["ki"], d["bt"], d["seqlens"])
    idx = oracle.topk_indices(sc, 3)
    flat, offs = [], [0]
    for b in range(3):
        for g in range(2):
            row = [int(t) for t in idx[b][g] if t >= 0]
            flat += row
            offs.append(offs[-1] + len(row))
    a = oracle.sparse_attention(d["q"], d["kp"], d["vp"], d["Dv"], d["bt"], d["seqlens"], idx, 0.7)
    c = oracle.sparse_attention_csr(d["q"], d["kp"], d["vp"], d["Dv"], d["bt"], d["seqlens"], np.array(flat),
                                    np.array(offs), 1, 3, 0.7)
    assert np.array_equal(a[0], c[0]) and np.array_equal(a[1], c[1])


def test_csr_duplicates_weigh_twice():
    """q = 0: the output is the mean over the listed rows, with a duplicate
    counted twice: (2 v3 + v7) / 3."""
    d = _tiny_paged(22, B=1, G=1, H=2, lens=(9,), separate_v=True)
    d["q"][:] = 0
    out, _ = oracle.sparse_attention_csr(d["q"], d["kp"], d["vp"], d["Dv"], d["bt"], d["seqlens"],
                                         np.array([3, 7, 3]), np.array([0, 3]), 1, 8, 1.0)
    P = d["P"]
    v = lambda t: np.array([_bf16_to_float(x) for x in d["vp"][d["bt"][0][t // P]][t % P][0]])  # noqa: E731
    np.testing.assert_allclose(out[0, 0], (2 * v(3) + v(7)) / 3, rtol=1e-13, atol=1e-15)
