"""Edge cases and degenerate inputs on the GPU path (through the C ABI)."""
import numpy as np
import pytest

import oracle
from top_sparse_decode_paged_b200 import workloads as W

from helpers import assert_out_close, run_step, to_device

pytestmark = pytest.mark.gpu


def _sd():
    import top_sparse_decode_paged_b200 as sd
    sd.device_errors(clear=True)
    return sd


def test_heavy_ties_take_lowest_tokens():
    sd = _sd()
    wl = W.make(W.spec("b4_l4096_mla", B=2, seqlens=(4096, 3000)))
    wl.ki_pages[:] = 0          # every score is 0: the first k tokens win
    got = run_step(wl, to_device(wl))
    for b in range(2):
        assert got["indices"][b, 0].tolist() == list(range(2048))
    assert sd.device_errors() == 0


def test_k_at_least_seqlen_equals_dense_attention():
    wl = W.make(W.spec("b4_l4096_mla", seqlens=(2048, 100, 1, 1999), seed=21))
    got = run_step(wl, to_device(wl))
    for b, L in enumerate(wl.seqlens):
        assert got["indices"][b, 0, :L].tolist() == list(range(L))
        assert (got["indices"][b, 0, L:] == -1).all()
    dense, _ = oracle.dense_attention(wl.q, wl.k_pages, None, 512, wl.block_table, wl.seqlens, 1, wl.spec.scale)
    assert_out_close(got["out"], dense, "dense")


def test_empty_request_gives_zero_output_and_minus_one_indices():
    sd = _sd()
    wl = W.make(W.spec("tiny", seqlens=(0,), spare_pages=1))
    # the generator makes a 1-column block table of -1 for an empty request
    got = run_step(wl, to_device(wl))
    assert (got["indices"] == -1).all()
    assert (got["out"] == 0).all()
    assert np.isneginf(got["lse"]).all()
    assert sd.device_errors() == 0


def test_single_selected_row_is_returned_exactly():
    wl = W.make(W.spec("perhead_b16_gqa", seqlens=(300, 77), k=1, seed=22))
    got = run_step(wl, to_device(wl))
    ref = oracle.decode_step(wl)
    for b in range(2):
        assert np.array_equal(got["indices"][b], ref["indices"][b])
        # one row: softmax weight exactly 1, out = V row exactly (bf16 -> bf16)
        assert np.array_equal(got["out"][b], ref["out"][b])


def test_bad_block_table_entry_sets_error_bit_and_masks():
    sd = _sd()
    wl = W.make(W.spec("tiny", seqlens=(200,)))
    wl.block_table[0, 3] = wl.num_pages + 5     # tokens 48..63 point outside the pool
    got = run_step(wl, to_device(wl))
    bits = sd.device_errors()
    assert bits & sd.SD_DEVERR_PAGE
    assert not (set(range(48, 64)) & set(got["indices"][0, 0].tolist()))


def test_seqlen_past_block_table_sets_error_bit():
    import torch
    sd = _sd()
    wl = W.make(W.spec("tiny", seqlens=(64,)))
    d = to_device(wl)
    d["seqlens"] = torch.tensor([10_000], dtype=torch.int32, device="cuda")
    idx = sd.sd_indexer_topk(d["qi"], d["w"], d["ki_pages"], d["block_table"], d["seqlens"], 32, 64)
    torch.cuda.synchronize()
    assert sd.device_errors() & sd.SD_DEVERR_SEQLEN
    assert (idx.cpu().numpy() >= 0).all()


def test_index_past_seqlen_is_skipped_and_flagged():
    import torch
    sd = _sd()
    wl = W.make(W.spec("tiny", seqlens=(100,)))
    d = to_device(wl)
    sel = np.array([[[5, 9, 300, 40] + [-1] * 28]], dtype=np.int32)
    out = sd.sd_sparse_attn(d["q"], d["k_pages"], None, d["block_table"], d["seqlens"],
                            torch.from_numpy(sel).cuda(), wl.spec.scale, 64)
    torch.cuda.synchronize()
    assert sd.device_errors() & sd.SD_DEVERR_INDEX
    ref, _ = oracle.sparse_attention(wl.q, wl.k_pages, None, 64, wl.block_table, wl.seqlens,
                                     [np.array([[5, 9, 40]])], wl.spec.scale)
    assert_out_close(out.float().cpu().numpy(), ref, "skip")


def test_invalid_arguments_raise_before_launch():
    import torch
    sd = _sd()
    wl = W.make(W.spec("tiny"))
    d = to_device(wl)
    with pytest.raises(sd.SdError):
        sd.sd_indexer_topk(d["qi"], d["w"], d["ki_pages"], d["block_table"], d["seqlens"], 4096, 256)
    with pytest.raises(sd.SdError):
        sd.sd_sparse_attn(d["q"], d["k_pages"], None, d["block_table"], d["seqlens"],
                          torch.zeros((1, 1, 4), dtype=torch.int32, device="cuda"), 0.1, 96)


def test_cuda_graph_capture_and_replay_with_new_inputs():
    import torch
    import top_sparse_decode_paged_b200 as sd
    wl = W.make(W.spec("b4_l4096_mla", B=2, seqlens=(4096, 2500), seed=23))
    d = to_device(wl)
    s = wl.spec
    ws = sd.alloc_workspace(2, 1, wl.max_seqlen, s.k, s.H, s.Dv)
    idx = torch.empty((2, 1, s.k), dtype=torch.int32, device="cuda")
    out = torch.empty((2, s.H, s.Dv), dtype=torch.bfloat16, device="cuda")
    run = lambda: sd.sd_decode_step(d["qi"], d["w"], d["ki_pages"], d["q"], d["k_pages"], None,  # noqa: E731
                                    d["block_table"], d["seqlens"], s.k, wl.max_seqlen, s.scale, s.Dv,
                                    indices=idx, out=out, workspace=ws)
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        run()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        run()
    wl2 = W.make(W.spec("b4_l4096_mla", B=2, seqlens=(4096, 2500), seed=24))
    d2 = to_device(wl2)
    for key in ("qi", "w", "q"):
        d[key].copy_(d2[key])
    g.replay()
    torch.cuda.synchronize()
    ref = oracle.decode_step(dict_to_wl(wl, wl2))
    assert np.array_equal(idx.cpu().numpy()[0], ref["indices"][0])
    assert np.array_equal(idx.cpu().numpy()[1], ref["indices"][1])
    assert_out_close(out.float().cpu().numpy(), ref["out"], "graph")


def dict_to_wl(base, queries_from):
    import dataclasses
    return dataclasses.replace(base, qi=queries_from.qi, w=queries_from.w, q=queries_from.q)


def _indices_vs_oracle(wl):
    got = run_step(wl, to_device(wl))
    sc = oracle.indexer_scores(wl.qi, wl.w, wl.ki_pages, wl.block_table, wl.seqlens)
    ref = oracle.topk_indices(sc, wl.spec.k)
    for b in range(wl.seqlens.shape[0]):
        L = int(wl.seqlens[b])
        assert np.array_equal(got["scores"][b][:, :L], sc[b]), f"scores b={b}"
        assert np.array_equal(got["indices"][b], ref[b]), f"indices b={b}"
    return got


@pytest.mark.parametrize("n_hot", [3000, 5000])
def test_topk_two_level_ties_at_the_threshold(n_hot):
    """Scores take two values; more tokens hold the high value than k, so the
    threshold is the high value and the lowest-index ones must win. With 3000
    tied keys the top-k resolves them as candidates in one CTA; with 5000
    (more than its candidate capacity) it takes the full radix passes."""
    wl = W.make(W.spec("b4_l4096_mla", B=2, seqlens=(20000, 9000), seed=41))
    rng = np.random.default_rng(5)
    wl.ki_pages[:] = 0
    row = rng.integers(-64, 65, size=128).astype(np.int8)
    for b, L in enumerate(wl.seqlens):
        hot = rng.choice(int(L), size=n_hot, replace=False)   # > k = 2048
        for t in hot:
            wl.ki_pages[wl.block_table[b, t // 64], t % 64, 0] = row
    _indices_vs_oracle(wl)


def test_topk_cluster_slices_with_ragged_rows():
    """Rows of 4097, 20000 and 131072 tokens in one batch: the top-k runs with
    the largest cluster and slices whose ends fall mid-row and past short rows."""
    _indices_vs_oracle(W.make(W.spec("b4_l4096_mla", seqlens=(4097, 20000, 131072, 2049), seed=42)))


def test_topk_single_cta_fallback_beyond_cluster_capacity():
    """max_seqlen above 8 x 32768 takes the one-CTA-per-row kernel."""
    _indices_vs_oracle(W.make(W.spec("b4_l4096_mla", seqlens=(262145, 5000), seed=43)))


def test_h128_k_at_least_seqlen_equals_dense_and_empty_request():
    """128-head MLA rows (tensor-core attention path) with k >= seqlen, an
    empty request in the middle, and requests shorter than one 256-token tile."""
    sd = _sd()
    wl = W.make(W.spec("b32_l65536_mla", seqlens=(2048, 300, 0, 1, 1999), seed=44))
    got = run_step(wl, to_device(wl))
    live = [b for b in range(5) if wl.seqlens[b] > 0]
    dense, lse = oracle.dense_attention(wl.q, wl.k_pages, None, 512, wl.block_table, wl.seqlens, 1,
                                        wl.spec.scale, requests=live)
    assert_out_close(got["out"][live], dense, "dense h128")
    np.testing.assert_allclose(got["lse"][live], lse, rtol=0, atol=2e-3)
    assert (got["out"][2] == 0).all() and np.isneginf(got["lse"][2]).all()
    assert (got["indices"][2] == -1).all()
    assert sd.device_errors() == 0


def test_h128_single_selected_row_is_exact():
    wl = W.make(W.spec("b32_l65536_mla", seqlens=(3000, 700), k=1, seed=45))
    got = run_step(wl, to_device(wl))
    ref = oracle.decode_step(wl)
    assert np.array_equal(got["indices"][:, :, :1], np.stack(ref["indices"]))
    assert np.array_equal(got["out"], ref["out"])


def test_h128_graph_replay_many_ranges():
    """A captured 128-head step replayed with new queries; every CTA pair of
    the attention covers parts of several requests (B=40 > 74 ranges / 2)."""
    import torch
    import top_sparse_decode_paged_b200 as sd
    wl = W.make(W.spec("b32_l65536_mla", B=40, seqlen=3000, seed=46))
    d = to_device(wl)
    s = wl.spec
    ws = sd.alloc_workspace(40, 1, wl.max_seqlen, s.k, s.H, s.Dv)
    idx = torch.empty((40, 1, s.k), dtype=torch.int32, device="cuda")
    out = torch.empty((40, s.H, s.Dv), dtype=torch.bfloat16, device="cuda")
    run = lambda: sd.sd_decode_step(d["qi"], d["w"], d["ki_pages"], d["q"], d["k_pages"], None,  # noqa: E731
                                    d["block_table"], d["seqlens"], s.k, wl.max_seqlen, s.scale, s.Dv,
                                    indices=idx, out=out, workspace=ws)
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        run()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        run()
    wl2 = W.make(W.spec("b32_l65536_mla", B=40, seqlen=3000, seed=47))
    d2 = to_device(wl2)
    for key in ("qi", "w", "q"):
        d[key].copy_(d2[key])
    g.replay()
    torch.cuda.synchronize()
    import dataclasses
    mixed = dataclasses.replace(wl, qi=wl2.qi, w=wl2.w, q=wl2.q)
    req = [0, 13, 39]
    ref = oracle.decode_step(mixed, requests=req)
    got_idx = idx.cpu().numpy()
    for i, b in enumerate(req):
        assert np.array_equal(got_idx[b], ref["indices"][i])
    assert_out_close(out.float().cpu().numpy()[req], ref["out"], "graph h128")


def test_h128_growing_logits_rescale_mid_request():
    """The rope columns (512..575, which enter S but not V) of the key rows are
    scaled up along the sequence, so every head's running max moves by far
    more than 2^8 between tiles of one request and the lazy rescale of the
    accumulated output runs many times."""
    wl = W.make(W.spec("b32_l65536_mla", seqlens=(4096, 3000, 700), seed=48))
    kf = (wl.k_pages.astype(np.uint32) << 16).view(np.float32)
    for b, L in enumerate(wl.seqlens):
        t = np.arange(int(L))
        pg, sl = wl.block_table[b, t // 64], t % 64
        kf[pg, sl, 0, 512:] *= (1.0 + 30.0 * t / L)[:, None].astype(np.float32)
    wl.k_pages[:] = W.bf16_bits_from_f32(kf)
    got = run_step(wl, to_device(wl))
    ref = oracle.decode_step(wl)
    assert np.array_equal(got["indices"], np.stack(ref["indices"]))
    assert_out_close(got["out"], ref["out"], "rescale h128")
    np.testing.assert_allclose(got["lse"], ref["lse"], rtol=1e-4, atol=2e-3)
