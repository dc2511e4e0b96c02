"""The previous selection as a top-k hint (sd_indexer_topk_hinted,
sd_decode_step_hinted): the indices equal the oracle's, bit for bit, for an
exact hint, the selection of a perturbed query (the steady state of decode), a
garbage hint (duplicates, negatives, tokens past the seqlen), a partial hint
(fewer than k valid tokens) and an all-ties row; the hinted decode step
matches the oracle; a hint aliasing the output is rejected."""
import dataclasses

import numpy as np
import pytest

from oracle import sd_oracle as oracle
from top_sparse_decode_paged_b200 import workloads as W
from helpers import assert_out_close, to_device

pytestmark = pytest.mark.gpu


def _indices_with_hint(wl, hint_np):
    import torch
    import top_sparse_decode_paged_b200 as sd
    d = to_device(wl)
    s = wl.spec
    hint = torch.from_numpy(np.ascontiguousarray(hint_np, dtype=np.int32)).cuda()
    idx = sd.sd_indexer_topk_hinted(d["qi"], d["w"], d["ki_pages"], d["block_table"], d["seqlens"], s.k,
                                    wl.max_seqlen, hint)
    torch.cuda.synchronize()
    assert sd.device_errors() == 0
    return idx.cpu().numpy()


def _oracle_indices(wl, qi=None, w=None):
    qi = wl.qi if qi is None else qi
    w = wl.w if w is None else w
    sc = oracle.indexer_scores(qi, w, wl.ki_pages, wl.block_table, wl.seqlens)
    return np.stack(oracle.topk_indices(sc, wl.spec.k)).astype(np.int32)


def _perturbed_qi(wl, frac=0.1, seed=5):
    rng = np.random.default_rng(seed)
    qi = wl.qi.astype(np.int16)
    m = rng.random(qi.shape) < frac
    qi[m] += rng.integers(-3, 4, size=int(m.sum())).astype(np.int16)
    return np.clip(qi, -64, 64).astype(np.int8)


@pytest.fixture(scope="module")
def wl():
    return W.make(W.spec("b32_l65536_mla", seqlens=(20000, 9000, 30001), seed=81))


def test_exact_hint(wl):
    ref = _oracle_indices(wl)
    assert np.array_equal(_indices_with_hint(wl, ref), ref)


def test_hint_from_a_perturbed_query(wl):
    ref = _oracle_indices(wl)
    prev = _oracle_indices(wl, qi=_perturbed_qi(wl))
    assert not np.array_equal(prev, ref)      # the hint really differs
    assert np.array_equal(_indices_with_hint(wl, prev), ref)


def test_garbage_and_partial_hints(wl):
    ref = _oracle_indices(wl)
    rng = np.random.default_rng(9)
    B, G, k = ref.shape
    garbage = rng.integers(-5, 40000, size=(B, G, k)).astype(np.int32)
    garbage[:, :, 1::7] = garbage[:, :, ::7][:, :, : garbage[:, :, 1::7].shape[2]]  # duplicates
    assert np.array_equal(_indices_with_hint(wl, garbage), ref)
    partial = ref.copy()
    partial[:, :, ::2] = -1
    assert np.array_equal(_indices_with_hint(wl, partial), ref)


def test_hint_on_an_all_ties_row():
    wl = W.make(W.spec("b32_l65536_mla", seqlens=(5000,), seed=82))
    wl.ki_pages[:] = 1
    ref = _oracle_indices(wl)
    assert (ref[0, 0] == np.arange(wl.spec.k)).all()
    hint = np.full_like(ref, -1)
    hint[0, 0] = np.arange(100, 100 + wl.spec.k)
    assert np.array_equal(_indices_with_hint(wl, hint), ref)
    assert np.array_equal(_indices_with_hint(wl, ref), ref)


def test_hinted_decode_step_and_alias_rejection(wl):
    import torch
    import top_sparse_decode_paged_b200 as sd
    d = to_device(wl)
    s = wl.spec
    prev = torch.from_numpy(_oracle_indices(wl, qi=_perturbed_qi(wl))).cuda()
    idx, out = sd.sd_decode_step_hinted(d["qi"], d["w"], d["ki_pages"], d["q"], d["k_pages"], None,
                                        d["block_table"], d["seqlens"], s.k, wl.max_seqlen, s.scale, s.Dv, prev)
    torch.cuda.synchronize()
    ref = oracle.decode_step(wl)
    assert np.array_equal(idx.cpu().numpy(), np.stack(ref["indices"]))
    assert_out_close(out.float().cpu().numpy(), ref["out"], "hinted step")
    with pytest.raises(sd.SdError):
        sd.sd_indexer_topk_hinted(d["qi"], d["w"], d["ki_pages"], d["block_table"], d["seqlens"], s.k,
                                  wl.max_seqlen, idx, indices=idx)
