"""GPU path vs the CPU oracle, through the C ABI.

Scores and indices must match bit for bit; the bf16 output must be within
max-abs 2e-2 and relative L2 5e-3 of the fp64 oracle. Small variants of every
workload are compared element by element (several tiles and a ragged tail);
the full-size workloads are compared on sampled requests, which the oracle
computes one by one, in the same launch configuration the benchmark times.
"""
import numpy as np
import pytest

import oracle
from top_sparse_decode_paged_b200 import workloads as W

from helpers import assert_out_close, run_step, to_device

pytestmark = pytest.mark.gpu

SMALL = {
    "tiny": W.spec("tiny"),
    "tiny_ragged": W.spec("tiny", seqlens=(203,)),
    "b4_l4096_mla": W.spec("b4_l4096_mla"),
    "b4_mla_ragged_tail": W.spec("b4_l4096_mla", seqlens=(4059, 3001, 2049, 2047)),
    "h128_small": W.spec("b32_l65536_mla", seqlens=(9000, 5003, 1500), seed=12),
    "ragged_small": W.spec("ragged_b64_mla", B=6, ragged=(1024, 8192), seed=13),
    "perhead_small": W.spec("perhead_b16_gqa", seqlens=(4096, 3001, 700), seed=14),
    "mla_page16": W.spec("b4_l4096_mla", seqlens=(3000, 1234, 129), page_size=16, seed=15),
    "mla_page32": W.spec("b4_l4096_mla", seqlens=(2500, 4097), page_size=32, seed=16),
    "mla_page48_fallback": W.spec("b4_l4096_mla", seqlens=(2100, 777), page_size=48, seed=17),
}


def _compare(wl, got, requests):
    ref = oracle.decode_step(wl, requests=requests)
    for i, b in enumerate(requests):
        L = int(wl.seqlens[b])
        if got["scores"] is not None:
            assert np.array_equal(got["scores"][b][:, :L], ref["scores"][i]), f"scores b={b}"
        assert np.array_equal(got["indices"][b], ref["indices"][i]), f"indices b={b}"
    assert_out_close(got["out"][requests], ref["out"], "out")
    fin = np.isfinite(ref["lse"])
    np.testing.assert_allclose(got["lse"][requests][fin], ref["lse"][fin], rtol=0, atol=2e-3)


@pytest.mark.parametrize("name", list(SMALL))
def test_small_workload_elementwise(name):
    wl = W.make(SMALL[name])
    got = run_step(wl, to_device(wl))
    _compare(wl, got, list(range(wl.seqlens.shape[0])))


@pytest.mark.parametrize("name,sample", [
    ("b32_l65536_mla", (0, 17, 31)),
    ("ragged_b64_mla", "extremes"),
    ("perhead_b16_gqa", (0, 15)),
])
def test_full_size_sampled(name, sample):
    wl = W.make(W.spec(name))
    got = run_step(wl, to_device(wl))
    if sample == "extremes":
        order = np.argsort(wl.seqlens)
        sample = (int(order[0]), int(order[len(order) // 2]), int(order[-1]))
    _compare(wl, got, list(sample))
