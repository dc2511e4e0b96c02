"""The selection in CSR offsets / block-sized form (sd_sparse_attn_csr)
against the oracle: a CSR copy of a top-k selection (bit-identical to the
padded call), ragged block lists with empty rows and blocks past the seqlen
(tensor-core path), per-KV-head rows (GQA path), and the error flag for an
entry whose whole block lies past the seqlen."""
import numpy as np
import pytest

from oracle import sd_oracle as oracle
from top_sparse_decode_paged_b200 import workloads as W
from helpers import assert_out_close, to_device

pytestmark = pytest.mark.gpu


def _run_csr(wl, flat, offs, bs, max_sel, expect_err=0):
    import torch
    import top_sparse_decode_paged_b200 as sd
    s = wl.spec
    d = to_device(wl)
    idx = torch.from_numpy(np.asarray(flat, dtype=np.int32)).cuda() if len(flat) else None
    off = torch.from_numpy(np.asarray(offs, dtype=np.int32)).cuda()
    lse = torch.empty((wl.seqlens.shape[0], s.H), dtype=torch.float32, device="cuda")
    out = sd.sd_sparse_attn_csr(d["q"], d["k_pages"], d["v_pages"], d["block_table"], d["seqlens"], idx, off, bs,
                                max_sel, s.scale, s.Dv, lse=lse)
    torch.cuda.synchronize()
    assert sd.device_errors() == expect_err
    o, ls = oracle.sparse_attention_csr(wl.q, wl.k_pages, wl.v_pages, s.Dv, wl.block_table, wl.seqlens,
                                        np.asarray(flat, dtype=np.int64), np.asarray(offs), bs, max_sel, s.scale)
    got = out.float().cpu().numpy()
    assert_out_close(got, o, "csr")
    lse_np = lse.cpu().numpy()
    fin = np.isfinite(ls)
    assert (np.isneginf(lse_np) == ~fin).all()
    np.testing.assert_allclose(lse_np[fin], ls[fin], rtol=1e-4, atol=2e-3)
    return out, d


def test_csr_copy_of_topk_matches_padded_call():
    import torch
    import top_sparse_decode_paged_b200 as sd
    wl = W.make(W.spec("b32_l65536_mla", seqlens=(3000, 1500, 700, 4096), seed=71))
    ref = oracle.decode_step(wl)
    flat, offs = [], [0]
    for b in range(4):
        row = [int(t) for t in ref["indices"][b][0] if t >= 0]
        flat += row
        offs.append(offs[-1] + len(row))
    out, d = _run_csr(wl, flat, offs, 1, wl.spec.k)
    idx = torch.from_numpy(np.stack(ref["indices"]).astype(np.int32)).cuda()
    padded = sd.sd_sparse_attn(d["q"], d["k_pages"], None, d["block_table"], d["seqlens"], idx, wl.spec.scale,
                               wl.spec.Dv)
    torch.cuda.synchronize()
    assert torch.equal(out, padded)


def test_csr_blocks_ragged_rows():
    """Blocks of 16 tokens: a long row, an empty row, a row whose last block is
    cut by the seqlen plus a negative entry, and a row of duplicates."""
    wl = W.make(W.spec("b32_l65536_mla", seqlens=(3000, 500, 1000, 800), seed=72))
    rng = np.random.default_rng(7)
    rows = [
        list(rng.choice(3000 // 16, size=100, replace=False)),
        [],
        [1000 // 16, -1, 3, 17, 40],          # block 62 covers 992..1007: 992..999 kept
        [5, 5, 9, 5],
    ]
    flat, offs = [], [0]
    for r in rows:
        flat += [int(x) for x in r]
        offs.append(offs[-1] + len(r))
    _run_csr(wl, flat, offs, 16, 2048)


def test_csr_per_kv_head_rows_gqa():
    wl = W.make(W.spec("perhead_b16_gqa", B=2, seqlen=2000, seed=73))
    rng = np.random.default_rng(8)
    flat, offs = [], [0]
    for b in range(2):
        for g in range(8):
            n = int(rng.integers(0, 200))
            flat += [int(x) for x in np.sort(rng.choice(2000, size=n, replace=False))]
            offs.append(offs[-1] + n)
    _run_csr(wl, flat, offs, 1, 256)


def test_csr_block_past_seqlen_is_flagged_and_skipped():
    import top_sparse_decode_paged_b200 as sd
    wl = W.make(W.spec("b32_l65536_mla", seqlens=(640, 300), seed=74))
    offs = [0, 3, 6]
    flat = [0, 3, 50, 7, 2, 1]           # blocks of 8: request 0 (L 640) reads 400..407, request 1 (L 300) 56..63
    _run_csr(wl, flat, offs, 8, 512)     # no error: every block starts below its seqlen
    flat = [0, 3, 90, 7, 2, 1]           # block 90 = 720..727 is past request 0's seqlen 640
    _run_csr(wl, flat, offs, 8, 512, expect_err=sd.SD_DEVERR_INDEX)
