"""Seeded synthetic inputs for top-k sparse decode over a paged KV cache.

This module draws the inputs that both the CUDA path and the CPU oracle consume.
It holds none of the method's arithmetic: it only draws random values, lays them
out in paged pools and writes poison into slots that no valid read may touch.

Workloads (decode, one query per request):

* ``tiny``            B=1, seqlen 256, page 16; indexer Hi=4, Di=32; top-k 32;
                      MQA H=4, D=64 with V = the K row; scale 1/8; seed 0.
* ``b4_l4096_mla``    B=4, seqlen 4096, page 64; indexer Hi=64, Di=128; top-k 2048;
                      MLA latent rows of 576 (V = first 512) shared by H=16 heads.
* ``b32_l65536_mla``  B=32, seqlen 65536, page 64, shuffled pool; as above with H=128.
* ``ragged_b64_mla``  B=64, seqlens log-uniform in [1024, 131072]; MLA H=128.
* ``perhead_b16_gqa`` B=16, seqlen 32768, page 32; 8 KV heads, each with its own
                      int8 indexer (Hi=4, Di=64) and its own top-k 1024; GQA 32/8,
                      D=128 with separate K and V pools; 5% of tokens planted as
                      clusters whose indexer keys are shifted by +32.

Value distributions: int8 indexer queries and keys are uniform integers in
[-64, 64]; indexer head weights are uniform integers in [1, 8]; bf16 queries
and cache rows are N(0, 1) drawn in fp32 and rounded to bf16 (nearest even).

Layout: every pool is NHD, ``[num_pages, page_size, kv_heads, dim]``. Physical
page ids are a seeded permutation over all requests' pages (plus a few spare
pages nobody references). Block-table entries past a request's last page are -1.
Slots past ``seqlen`` in a request's last page and all spare pages hold poison:
int8 127 in the indexer pool, bf16 NaN in the K/V pools.
"""

from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np

BF16_NAN = np.uint16(0x7FC0)
INT8_POISON = np.int8(127)


@dataclasses.dataclass
class Spec:
    """Shape and seed of one synthetic decode batch."""

    name: str
    B: int
    page_size: int
    G: int          # KV heads (1 for MLA)
    Hi: int         # indexer heads per KV head
    Di: int         # indexer dim
    k: int          # top-k per (request, KV head)
    H: int          # query heads (all KV heads together)
    Dk: int         # key width
    Dv: int         # value width
    v_in_k: bool    # V is the first Dv columns of the K row (MLA / MQA with V=K)
    scale: float
    seed: int
    seqlen: Optional[int] = None              # fixed length for every request
    ragged: Optional[tuple] = None            # (lo, hi): log-uniform lengths
    seqlens: Optional[tuple] = None           # explicit lengths (tests)
    clusters: float = 0.0                     # fraction of tokens in planted runs
    cluster_shift: int = 32
    spare_pages: int = 2

    @property
    def qpk(self) -> int:
        """Query heads per KV head."""
        return self.H // self.G


def _spec_table():
    mla = dict(G=1, Hi=64, Di=128, k=2048, Dk=576, Dv=512, v_in_k=True,
               scale=1.0 / math.sqrt(576.0), page_size=64)
    return {
        "tiny": Spec("tiny", B=1, seqlen=256, page_size=16, G=1, Hi=4, Di=32, k=32,
                     H=4, Dk=64, Dv=64, v_in_k=True, scale=1.0 / 8.0, seed=0),
        "b4_l4096_mla": Spec("b4_l4096_mla", B=4, seqlen=4096, H=16, seed=1, **mla),
        "b32_l65536_mla": Spec("b32_l65536_mla", B=32, seqlen=65536, H=128, seed=2, **mla),
        "ragged_b64_mla": Spec("ragged_b64_mla", B=64, ragged=(1024, 131072), H=128,
                               seed=3, **mla),
        "perhead_b16_gqa": Spec("perhead_b16_gqa", B=16, seqlen=32768, page_size=32, G=8,
                                Hi=4, Di=64, k=1024, H=32, Dk=128, Dv=128, v_in_k=False,
                                scale=1.0 / math.sqrt(128.0), seed=4, clusters=0.05),
    }


SPECS = _spec_table()
CONFIG_ORDER = ["tiny", "b4_l4096_mla", "b32_l65536_mla", "ragged_b64_mla", "perhead_b16_gqa"]


def spec(name: str, **overrides) -> Spec:
    """A named spec, optionally with fields replaced (smaller B, other seqlens...)."""
    base = SPECS[name]
    return dataclasses.replace(base, **overrides) if overrides else base


@dataclasses.dataclass
class Workload:
    """One decode batch in host memory (numpy). bf16 arrays hold raw uint16 bits."""

    spec: Spec
    seqlens: np.ndarray       # int32 [B]
    block_table: np.ndarray   # int32 [B, max_pages_per_req]
    qi: np.ndarray            # int8  [B, G, Hi, Di]
    w: np.ndarray             # int32 [B, G, Hi]
    ki_pages: np.ndarray      # int8  [num_pages, P, G, Di]
    q: np.ndarray             # bf16 bits uint16 [B, H, Dk]
    k_pages: np.ndarray       # bf16 bits uint16 [num_pages, P, G, Dk]
    v_pages: Optional[np.ndarray]  # bf16 bits [num_pages, P, G, Dv] or None (V in K)
    cluster_tokens: Optional[list] = None  # per request: sorted planted token ids

    @property
    def num_pages(self) -> int:
        return int(self.ki_pages.shape[0])

    @property
    def max_seqlen(self) -> int:
        return int(self.seqlens.max()) if self.seqlens.size else 0

    @property
    def max_pages(self) -> int:
        return int(self.block_table.shape[1])


def _draw_seqlens(s: Spec, rng: np.random.Generator) -> np.ndarray:
    if s.seqlens is not None:
        return np.asarray(s.seqlens, dtype=np.int32)
    if s.ragged is not None:
        lo, hi = s.ragged
        u = rng.uniform(math.log(lo), math.log(hi), size=s.B)
        return np.clip(np.rint(np.exp(u)), lo, hi).astype(np.int32)
    return np.full(s.B, s.seqlen, dtype=np.int32)


def bf16_bits_from_f32(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (nearest, ties to even); returns the uint16 bits."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounded = b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))
    out = (rounded >> np.uint32(16)).astype(np.uint16)
    nan = np.isnan(x)
    if nan.any():
        out[nan] = BF16_NAN
    return out


def _normal_bf16(rng: np.random.Generator, shape, chunk: int = 1 << 24) -> np.ndarray:
    """N(0,1) in fp32, rounded to bf16 bits, drawn in chunks to bound host memory."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)
    for i in range(0, n, chunk):
        m = min(chunk, n - i)
        out[i:i + m] = bf16_bits_from_f32(rng.standard_normal(m, dtype=np.float32))
    return out.reshape(shape)


def _uniform_int8(rng: np.random.Generator, shape, chunk: int = 1 << 26) -> np.ndarray:
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.int8)
    for i in range(0, n, chunk):
        m = min(chunk, n - i)
        out[i:i + m] = rng.integers(-64, 65, size=m, dtype=np.int8)
    return out.reshape(shape)


def make(s: Spec) -> Workload:
    """Draw one batch. The draw order is fixed: seqlens, page permutation, qi, w,
    indexer pool, cluster runs, q, K pool, V pool; then poison is written."""
    rng = np.random.default_rng(s.seed)
    P, G = s.page_size, s.G
    seqlens = _draw_seqlens(s, rng)
    B = int(seqlens.shape[0])
    pages_per_req = [(int(L) + P - 1) // P for L in seqlens]
    used = int(sum(pages_per_req))
    num_pages = used + s.spare_pages
    max_pages = max(1, max(pages_per_req) if pages_per_req else 1)

    perm = rng.permutation(num_pages).astype(np.int32)
    block_table = np.full((B, max_pages), -1, dtype=np.int32)
    cursor = 0
    for b, n in enumerate(pages_per_req):
        block_table[b, :n] = perm[cursor:cursor + n]
        cursor += n
    spare = perm[cursor:]

    qi = rng.integers(-64, 65, size=(B, G, s.Hi, s.Di), dtype=np.int8)
    w = rng.integers(1, 9, size=(B, G, s.Hi), dtype=np.int32)
    ki_pages = _uniform_int8(rng, (num_pages, P, G, s.Di))

    cluster_tokens = None
    if s.clusters > 0.0:
        cluster_tokens = []
        for b in range(B):
            L = int(seqlens[b])
            n_full_pages = L // P
            n_runs = min(n_full_pages, int(round(s.clusters * L / P)))
            runs = np.sort(rng.choice(n_full_pages, size=n_runs, replace=False))
            toks = []
            for r in runs:
                phys = block_table[b, r]
                # shift every indexer-key element of the run's tokens, all KV heads
                ki_pages[phys] = (ki_pages[phys].astype(np.int16) + s.cluster_shift).astype(np.int8)
                toks.extend(range(int(r) * P, int(r) * P + P))
            cluster_tokens.append(np.asarray(toks, dtype=np.int64))

    q = _normal_bf16(rng, (B, s.H, s.Dk))
    k_pages = _normal_bf16(rng, (num_pages, P, G, s.Dk))
    v_pages = None if s.v_in_k else _normal_bf16(rng, (num_pages, P, G, s.Dv))

    # poison: slack slots of each last page, and every spare page
    for b in range(B):
        L, n = int(seqlens[b]), pages_per_req[b]
        if n and L % P:
            phys = block_table[b, n - 1]
            ki_pages[phys, L % P:] = INT8_POISON
            k_pages[phys, L % P:] = BF16_NAN
            if v_pages is not None:
                v_pages[phys, L % P:] = BF16_NAN
    for phys in spare:
        ki_pages[phys] = INT8_POISON
        k_pages[phys] = BF16_NAN
        if v_pages is not None:
            v_pages[phys] = BF16_NAN

    return Workload(spec=s, seqlens=seqlens, block_table=block_table, qi=qi, w=w,
                    ki_pages=ki_pages, q=q, k_pages=k_pages, v_pages=v_pages,
                    cluster_tokens=cluster_tokens)


@dataclasses.dataclass
class TriSpec:
    """Shape and seed of one layer's eviction batch (calibrated queries plus a
    paged K/V cache). Lengths: ``n_sink`` protected prefix tokens (the prompt)
    + ``region`` evictable decode tokens + ``n_recent`` protected tail tokens,
    or explicit ``seqlens``."""

    name: str
    B: int
    page_size: int
    G: int
    H: int
    D: int
    n_sink: int
    n_recent: int
    budget: int
    seed: int
    region: int = 0
    seqlens: Optional[tuple] = None
    ragged: Optional[tuple] = None   # (lo, hi) evictable region, uniform integers
    with_v: bool = True
    spare_pages: int = 2


def _tri_spec_table():
    # Qwen3-8B attention shape (32 query heads over 8 KV heads, head dim 128),
    # budget 2048, compaction every 2048 decode tokens: the region holds
    # budget + 2048 tokens when an eviction runs.
    q3 = dict(G=8, H=32, D=128, page_size=32, n_sink=1024, n_recent=16, budget=2048)
    return {
        "tri_tiny": TriSpec("tri_tiny", B=3, page_size=16, G=2, H=4, D=64, n_sink=4, n_recent=8, budget=24,
                            seqlens=(100, 20, 37), seed=10),
        "tri_b32_qwen3_8b": TriSpec("tri_b32_qwen3_8b", B=32, region=4096, seed=11, **q3),
        # the same kernels on a quarter of the batch (pools still larger than L2), for detailed profiles
        "tri_b8_qwen3_8b": TriSpec("tri_b8_qwen3_8b", B=8, region=4096, seed=13, **q3),
        "tri_ragged_b16": TriSpec("tri_ragged_b16", B=16, ragged=(0, 8192), seed=12, **q3),
    }


TRI_SPECS = _tri_spec_table()


def tri_spec(name: str, **overrides) -> TriSpec:
    base = TRI_SPECS[name]
    return dataclasses.replace(base, **overrides) if overrides else base


@dataclasses.dataclass
class TriWorkload:
    """One eviction batch in host memory; bf16 arrays hold raw uint16 bits."""

    spec: TriSpec
    seqlens: np.ndarray       # int32 [B]
    block_table: np.ndarray   # int32 [B, max_pages_per_req]
    q_cal: np.ndarray         # bf16 bits [H, D]
    k_pages: np.ndarray       # bf16 bits [num_pages, P, G, D]
    v_pages: Optional[np.ndarray]

    @property
    def max_seqlen(self) -> int:
        return int(self.seqlens.max()) if self.seqlens.size else 0


def make_tri(s: TriSpec) -> TriWorkload:
    """Draw order: seqlens, page permutation, q_cal, K pool, V pool; then poison
    (bf16 NaN) in the slack of each last page and in the spare pages."""
    rng = np.random.default_rng(s.seed)
    P = s.page_size
    if s.seqlens is not None:
        seqlens = np.asarray(s.seqlens, dtype=np.int32)
    elif s.ragged is not None:
        region = rng.integers(s.ragged[0], s.ragged[1] + 1, size=s.B)
        seqlens = (s.n_sink + region + s.n_recent).astype(np.int32)
    else:
        seqlens = np.full(s.B, s.n_sink + s.region + s.n_recent, dtype=np.int32)
    B = int(seqlens.shape[0])
    pages_per_req = [(int(L) + P - 1) // P for L in seqlens]
    num_pages = int(sum(pages_per_req)) + s.spare_pages
    max_pages = max(1, max(pages_per_req) if pages_per_req else 1)
    perm = rng.permutation(num_pages).astype(np.int32)
    block_table = np.full((B, max_pages), -1, dtype=np.int32)
    cursor = 0
    for b, n in enumerate(pages_per_req):
        block_table[b, :n] = perm[cursor:cursor + n]
        cursor += n
    spare = perm[cursor:]
    q_cal = bf16_bits_from_f32(rng.standard_normal((s.H, s.D), dtype=np.float32))
    k_pages = _normal_bf16(rng, (num_pages, P, s.G, s.D))
    v_pages = _normal_bf16(rng, (num_pages, P, s.G, s.D)) if s.with_v else None
    for b in range(B):
        L, n = int(seqlens[b]), pages_per_req[b]
        if n and L % P:
            for pool in (k_pages, v_pages):
                if pool is not None:
                    pool[block_table[b, n - 1], L % P:] = BF16_NAN
    for phys in spare:
        for pool in (k_pages, v_pages):
            if pool is not None:
                pool[phys] = BF16_NAN
    return TriWorkload(spec=s, seqlens=seqlens, block_table=block_table, q_cal=q_cal, k_pages=k_pages,
                       v_pages=v_pages)


def make_tri_layers(s: TriSpec, n_layers: int):
    """n_layers layers of one eviction batch: layer 0 is make_tri(s); each later
    layer draws its own q_cal, K pool and V pool (in that order, from one
    generator seeded seed + 7919) with the same lengths, block table and
    poison."""
    base = make_tri(s)
    out = [base]
    rng = np.random.default_rng(s.seed + 7919)
    shape = base.k_pages.shape
    for _ in range(1, n_layers):
        q_cal = bf16_bits_from_f32(rng.standard_normal((s.H, s.D), dtype=np.float32))
        k = _normal_bf16(rng, shape)
        v = _normal_bf16(rng, shape) if s.with_v else None
        nan = base.k_pages == BF16_NAN  # the base layer's poisoned slots
        k[nan] = BF16_NAN
        if v is not None:
            v[nan] = BF16_NAN
        out.append(TriWorkload(spec=s, seqlens=base.seqlens, block_table=base.block_table, q_cal=q_cal, k_pages=k,
                               v_pages=v))
    return out


def tri_algorithmic_bytes(s: TriSpec, seqlens: np.ndarray, mode: int = 0) -> int:
    """Bytes one eviction must move at minimum: every evictable token's K row
    read once for scoring, plus, for each request that evicts, every moved
    row (K and V) read once and written once."""
    row = s.G * s.D * 2
    total = 0
    for L in np.asarray(seqlens):
        E = max(0, int(L) - s.n_sink - s.n_recent)
        total += E * row
        if E > s.budget:
            total += (s.budget + s.n_recent) * row * (2 if s.with_v else 1) * 2
    return total


def algorithmic_bytes(s: Spec, seqlens: np.ndarray) -> int:
    """Bytes a decode step must move at minimum: every cached token's indexer key
    (G*Di int8) plus each selected row (K, and V when it is a separate row)."""
    row = s.Dk * 2 if s.v_in_k else (s.Dk + s.Dv) * 2
    total = 0
    for L in np.asarray(seqlens, dtype=np.int64):
        total += int(L) * s.G * s.Di + min(s.k, int(L)) * s.G * row
    return total
