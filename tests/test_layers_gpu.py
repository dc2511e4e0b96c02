"""Several layers sharing one selection (sd_sparse_attn_layers) against the
oracle, layer by layer: the tensor-core path (up to 16 layers per launch and
the split into launches of 16), and the layer-by-layer general path (MLA with
16 heads, GQA with separate value pools)."""
import dataclasses

import numpy as np
import pytest

from oracle import sd_oracle as oracle
from top_sparse_decode_paged_b200 import workloads as W
from helpers import assert_out_close, to_device

pytestmark = pytest.mark.gpu


def _layer_pools(wl, n_layers):
    """Per-layer queries and caches on the base workload's pages: layer l
    rolls the query heads by l and scales the cache by 1 + (l mod 4)/4 (so poisoned
    slots stay poisoned exactly where the block table never reads)."""
    def scaled(bits, f):
        if bits is None:
            return None
        x = (bits.astype(np.uint32) << 16).view(np.float32) * np.float32(f)
        return W.bf16_bits_from_f32(x)
    layers = [wl]
    for l in range(1, n_layers):
        layers.append(dataclasses.replace(wl, q=np.roll(wl.q, l, axis=1), k_pages=scaled(wl.k_pages, 1 + (l % 4) / 4),
                                          v_pages=scaled(wl.v_pages, 1 + (l % 4) / 4)))
    return layers


def _run_layers(wl, n_layers, lse=True):
    import torch
    import top_sparse_decode_paged_b200 as sd
    s = wl.spec
    layers = _layer_pools(wl, n_layers)
    ref = oracle.decode_step(wl)
    idx_np = np.stack(ref["indices"]).astype(np.int32)
    devs = [to_device(x) for x in layers]
    d0 = devs[0]
    q = torch.stack([d["q"] for d in devs])
    idx = torch.from_numpy(idx_np).cuda()
    lse_t = torch.empty((n_layers, wl.seqlens.shape[0], s.H), dtype=torch.float32, device="cuda") if lse else None
    out = sd.sd_sparse_attn_layers(q, [d["k_pages"] for d in devs],
                                   None if d0["v_pages"] is None else [d["v_pages"] for d in devs],
                                   d0["block_table"], d0["seqlens"], idx, s.scale, s.Dv, lse=lse_t)
    torch.cuda.synchronize()
    assert sd.device_errors() == 0
    got = out.float().cpu().numpy().astype(np.float64)
    for l, x in enumerate(layers):
        o, ls = oracle.sparse_attention(x.q, x.k_pages, x.v_pages, s.Dv, x.block_table, x.seqlens,
                                        ref["indices"], s.scale)
        assert_out_close(got[l], o, f"layer {l}")
        if lse:
            live = x.seqlens > 0
            np.testing.assert_allclose(lse_t[l].cpu().numpy()[live], ls[live], rtol=1e-4, atol=2e-3)


def test_mla_layers_one_launch():
    wl = W.make(W.spec("b32_l65536_mla", seqlens=(3000, 0, 700, 2048, 5000), seed=61))
    _run_layers(wl, 3)


def test_mla_layers_split_into_launches_of_16():
    wl = W.make(W.spec("b32_l65536_mla", seqlens=(900, 130), seed=62))
    _run_layers(wl, 18, lse=False)


def test_mla_16_heads_layer_by_layer():
    wl = W.make(W.spec("b4_l4096_mla", seqlens=(4096, 1500, 3000), seed=63))
    _run_layers(wl, 2)


def test_gqa_separate_values_layer_by_layer():
    wl = W.make(W.spec("perhead_b16_gqa", B=2, seqlen=3000, seed=64))
    _run_layers(wl, 2)
