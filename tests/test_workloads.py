"""The seeded input generator: determinism, layout, poison and planted clusters."""
import numpy as np

from top_sparse_decode_paged_b200 import workloads as W


def test_same_seed_same_batch():
    a = W.make(W.spec("b4_l4096_mla", B=2))
    b = W.make(W.spec("b4_l4096_mla", B=2))
    for f in ("seqlens", "block_table", "qi", "w", "ki_pages", "q", "k_pages"):
        assert np.array_equal(getattr(a, f), getattr(b, f)), f


def test_block_table_is_a_permutation_and_pads_with_minus_one():
    wl = W.make(W.spec("ragged_b64_mla", B=6, ragged=(100, 900), spare_pages=3))
    P = wl.spec.page_size
    used = []
    for b, L in enumerate(wl.seqlens):
        n = (int(L) + P - 1) // P
        assert (wl.block_table[b, n:] == -1).all()
        used.extend(wl.block_table[b, :n].tolist())
    assert len(set(used)) == len(used)
    assert set(used) <= set(range(wl.num_pages))
    assert wl.num_pages == len(used) + 3


def test_poison_sits_only_past_seqlen():
    wl = W.make(W.spec("tiny", seqlens=(250,)))
    P = wl.spec.page_size
    last = wl.block_table[0, 249 // P]
    assert (wl.ki_pages[last, 250 % P:] == W.INT8_POISON).all()
    assert (wl.k_pages[last, 250 % P:] == W.BF16_NAN).all()
    assert not (wl.k_pages[last, :250 % P] == W.BF16_NAN).any()


def test_value_ranges():
    wl = W.make(W.spec("b4_l4096_mla", B=1))
    assert wl.qi.min() >= -64 and wl.qi.max() <= 64
    assert wl.w.min() >= 1 and wl.w.max() <= 8
    live = wl.ki_pages[wl.block_table[0, :4096 // 64]]
    assert live.min() >= -64 and live.max() <= 64


def test_planted_clusters_cover_five_percent_in_page_runs():
    wl = W.make(W.spec("perhead_b16_gqa", B=2, seqlen=4096))
    for toks in wl.cluster_tokens:
        assert abs(len(toks) / 4096 - 0.05) < 0.01
        assert len(toks) % wl.spec.page_size == 0
        assert (toks[::wl.spec.page_size] % wl.spec.page_size == 0).all()


def test_bf16_rounding_is_nearest_even():
    x = np.array([1.0, 1.00390625, 1.01171875, -2.5, 3.0e38], dtype=np.float32)
    bits = W.bf16_bits_from_f32(x)
    # 1 + 2^-8 is a tie between 1 and 1+2^-7 -> even (1.0); 1+3*2^-8 -> 1+2^-6
    assert bits.tolist() == [0x3F80, 0x3F80, 0x3F82, 0xC020, 0x7F62]


def test_algorithmic_bytes_formula_matches_definition():
    s = W.spec("b32_l65536_mla")
    n = W.algorithmic_bytes(s, np.full(32, 65536))
    assert n == 32 * (65536 * 128 + 2048 * 1152)
