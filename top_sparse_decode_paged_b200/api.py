"""Thin Python binding over the C ABI in ``include/sd_api.h`` (ctypes).

Argument marshalling only: each function takes torch tensors that already live
on the GPU, checks dtypes and shapes, passes raw device pointers and the
current CUDA stream to ``libsd.so`` and raises on a non-OK status. Every step of
the computation runs in the library's kernels. There is no CPU fallback: if
``libsd.so`` is missing the first call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libsd.so")

SD_DEVERR_SEQLEN = 0x1
SD_DEVERR_PAGE = 0x2
SD_DEVERR_INDEX = 0x4
SD_DEVERR_TIMEOUT = 0x8

EXPORTED = ("sd_workspace_size", "sd_indexer_topk", "sd_indexer_topk_noalloc", "sd_sparse_attn",
            "sd_attn_layers_workspace_size", "sd_sparse_attn_layers", "sd_csr_workspace_size",
            "sd_sparse_attn_csr", "sd_indexer_topk_hinted", "sd_decode_step_hinted", "sd_decode_step",
            "sd_tri_workspace_size", "sd_tri_compact", "sd_tri_layers_workspace_size", "sd_tri_compact_layers",
            "sd_set_stage_events", "sd_set_wait_limit", "sd_get_device_errors", "sd_status_str", "sd_last_cuda_error",
            "sd_last_launch_count", "sd_version")


class PagedDesc(ctypes.Structure):
    _fields_ = [("num_pages", ctypes.c_int32), ("page_size", ctypes.c_int32),
                ("max_pages_per_req", ctypes.c_int32), ("kv_heads", ctypes.c_int32)]


class SdError(RuntimeError):
    """A non-OK status returned by the library."""

    def __init__(self, status: int, name: str, cuda_error: int = 0):
        super().__init__(f"{name} (status {status}" + (f", cudaError {cuda_error})" if cuda_error else ")"))
        self.status = status
        self.name = name


_lib = None


def load_library(path: Optional[str] = None):
    """Loads libsd.so once and declares the exported signatures. The path is
    ``path``, else the ``SD_LIBRARY`` environment variable, else the in-tree
    build."""
    global _lib
    if _lib is not None:
        return _lib
    path = path or os.environ.get("SD_LIBRARY") or LIB_PATH
    if not os.path.exists(path):
        raise RuntimeError(f"libsd.so not built ({path}); run `python -m top_sparse_decode_paged_b200.build`")
    lib = ctypes.CDLL(path)
    p, i32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    lib.sd_workspace_size.restype = sz
    lib.sd_workspace_size.argtypes = [i32] * 6
    lib.sd_indexer_topk.restype = i32
    lib.sd_indexer_topk.argtypes = [p, p, p, p, p, PagedDesc, i32, i32, i32, i32, i32, p, p, p, sz, p]
    lib.sd_indexer_topk_noalloc.restype = i32
    lib.sd_indexer_topk_noalloc.argtypes = [p, p, p, p, p, PagedDesc, i32, i32, i32, i32, i32, p, p]
    lib.sd_sparse_attn.restype = i32
    lib.sd_sparse_attn.argtypes = [p, p, p, p, p, p, PagedDesc, i32, i32, i32, i32, i32,
                                   ctypes.c_float, p, p, p, sz, p]
    lib.sd_attn_layers_workspace_size.restype = sz
    lib.sd_attn_layers_workspace_size.argtypes = [i32] * 6
    lib.sd_sparse_attn_layers.restype = i32
    lib.sd_sparse_attn_layers.argtypes = [p, p, p, i32, p, p, p, PagedDesc, i32, i32, i32, i32, i32,
                                          ctypes.c_float, p, p, p, sz, p]
    lib.sd_csr_workspace_size.restype = sz
    lib.sd_csr_workspace_size.argtypes = [i32] * 5
    lib.sd_sparse_attn_csr.restype = i32
    lib.sd_sparse_attn_csr.argtypes = [p, p, p, p, p, p, p, i32, i32, PagedDesc, i32, i32, i32, i32,
                                       ctypes.c_float, p, p, p, sz, p]
    lib.sd_indexer_topk_hinted.restype = i32
    lib.sd_indexer_topk_hinted.argtypes = [p, p, p, p, p, PagedDesc, i32, i32, i32, i32, i32, p, p, p, p, sz, p]
    lib.sd_decode_step_hinted.restype = i32
    lib.sd_decode_step_hinted.argtypes = [p, p, p, p, p, p, p, p, PagedDesc, i32, i32, i32, i32, i32, i32,
                                          i32, i32, ctypes.c_float, p, p, p, p, p, p, sz, p]
    lib.sd_decode_step.restype = i32
    lib.sd_decode_step.argtypes = [p, p, p, p, p, p, p, p, PagedDesc, i32, i32, i32, i32, i32, i32,
                                   i32, i32, ctypes.c_float, p, p, p, p, p, sz, p]
    lib.sd_tri_workspace_size.restype = sz
    lib.sd_tri_workspace_size.argtypes = [i32] * 10
    lib.sd_tri_compact.restype = i32
    lib.sd_tri_compact.argtypes = [p, p, p, p, p, PagedDesc, i32, i32, i32, i32, i32, i32, i32, i32, p, p, sz, p]
    lib.sd_tri_layers_workspace_size.restype = sz
    lib.sd_tri_layers_workspace_size.argtypes = [i32] * 11
    lib.sd_tri_compact_layers.restype = i32
    lib.sd_tri_compact_layers.argtypes = [p, p, p, i32, p, p, PagedDesc, i32, i32, i32, i32, i32, i32, i32, i32, p, p,
                                          sz, p]
    lib.sd_set_stage_events.restype = i32
    lib.sd_set_stage_events.argtypes = [ctypes.POINTER(ctypes.c_void_p), i32]
    lib.sd_set_wait_limit.restype = i32
    lib.sd_set_wait_limit.argtypes = [i32]
    lib.sd_get_device_errors.restype = i32
    lib.sd_get_device_errors.argtypes = [ctypes.POINTER(ctypes.c_uint32), i32]
    lib.sd_status_str.restype = ctypes.c_char_p
    lib.sd_status_str.argtypes = [i32]
    lib.sd_last_cuda_error.restype = i32
    lib.sd_last_launch_count.restype = i32
    lib.sd_version.restype = i32
    _lib = lib
    return lib


def _check(status: int):
    if status != 0:
        lib = load_library()
        raise SdError(status, lib.sd_status_str(status).decode(), lib.sd_last_cuda_error())


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors passed to the library must be on the GPU")
    if not t.is_contiguous():
        raise ValueError("tensors passed to the library must be contiguous")
    return t.data_ptr()


def _stream(stream) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _desc(pool: torch.Tensor, block_table: torch.Tensor) -> PagedDesc:
    return PagedDesc(pool.shape[0], pool.shape[1], block_table.shape[1], pool.shape[2])


def _bits(t: torch.Tensor) -> torch.Tensor:
    if t.dtype == torch.bfloat16:
        return t
    if t.dtype in (torch.uint16, torch.int16):
        return t.view(torch.bfloat16)
    raise TypeError(f"expected bf16 (or its uint16 bits), got {t.dtype}")


def workspace_size(B: int, G: int, max_seqlen: int, k: int, H: int, Dv: int) -> int:
    return int(load_library().sd_workspace_size(B, G, max_seqlen, k, H, Dv))


def alloc_workspace(B: int, G: int, max_seqlen: int, k: int, H: int, Dv: int, device=None) -> torch.Tensor:
    """A workspace tensor of the size the library asks for (torch's allocator
    returns 256-byte aligned blocks)."""
    n = max(workspace_size(B, G, max_seqlen, k, H, Dv), 1)
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")


def sd_indexer_topk(qi, w, ki_pages, block_table, seqlens, k: int, max_seqlen: int,
                    indices=None, scores=None, workspace=None, stream=None):
    """Indexer scores + per-(request, KV head) top-k. Returns ``indices`` [B, G, k] int32."""
    lib = load_library()
    B, G, Hi, Di = qi.shape
    assert qi.dtype == torch.int8 and ki_pages.dtype == torch.int8 and w.dtype == torch.int32
    assert ki_pages.shape[2] == G and ki_pages.shape[3] == Di
    if indices is None:
        indices = torch.empty((B, G, k), dtype=torch.int32, device=qi.device)
    if workspace is None and scores is None:
        workspace = alloc_workspace(B, G, max_seqlen, k, G, 1, qi.device)
    ws_bytes = workspace.numel() if workspace is not None else 0
    _check(lib.sd_indexer_topk(_ptr(qi), _ptr(w), _ptr(ki_pages), _ptr(block_table), _ptr(seqlens),
                               _desc(ki_pages, block_table), B, Hi, Di, max_seqlen, k, _ptr(indices),
                               _ptr(scores), _ptr(workspace), ws_bytes, _stream(stream)))
    return indices


def sd_indexer_topk_hinted(qi, w, ki_pages, block_table, seqlens, k: int, max_seqlen: int, hint,
                           indices=None, scores=None, workspace=None, stream=None):
    """``sd_indexer_topk`` with the previous selection ``hint`` [B, G, k] (not
    the output buffer); the result is the same for any hint."""
    lib = load_library()
    B, G, Hi, Di = qi.shape
    if indices is None:
        indices = torch.empty((B, G, k), dtype=torch.int32, device=qi.device)
    if workspace is None and scores is None:
        workspace = alloc_workspace(B, G, max_seqlen, k, G, 1, qi.device)
    ws_bytes = workspace.numel() if workspace is not None else 0
    _check(lib.sd_indexer_topk_hinted(_ptr(qi), _ptr(w), _ptr(ki_pages), _ptr(block_table), _ptr(seqlens),
                                      _desc(ki_pages, block_table), B, Hi, Di, max_seqlen, k, _ptr(hint),
                                      _ptr(indices), _ptr(scores), _ptr(workspace), ws_bytes, _stream(stream)))
    return indices


NOALLOC_MAX_SCORES = 4 << 20


def sd_indexer_topk_noalloc(qi, w, ki_pages, block_table, seqlens, k: int, max_seqlen: int, indices,
                            stream=None):
    """Indexer + top-k for callers that cannot allocate device memory.

    The library keeps the scores in its own fixed scratch array (16 MiB per
    device; B * G * max_seqlen <= NOALLOC_MAX_SCORES), so this call takes no
    workspace. ``indices`` [B, G, k] int32 must be provided by the caller.
    Calls on one device share the scratch array: do not let them overlap on
    the GPU. Make the first call on a device before any CUDA-graph capture."""
    lib = load_library()
    B, G, Hi, Di = qi.shape
    assert qi.dtype == torch.int8 and ki_pages.dtype == torch.int8 and w.dtype == torch.int32
    assert tuple(indices.shape) == (B, G, k) and indices.dtype == torch.int32
    _check(lib.sd_indexer_topk_noalloc(_ptr(qi), _ptr(w), _ptr(ki_pages), _ptr(block_table),
                                       _ptr(seqlens), _desc(ki_pages, block_table), B, Hi, Di,
                                       max_seqlen, k, _ptr(indices), _stream(stream)))
    return indices


def sd_sparse_attn(q, k_pages, v_pages, block_table, seqlens, indices, scale: float, Dv: int,
                   out=None, lse=None, workspace=None, stream=None):
    """Attention over the selected rows + split combine. Returns ``out`` [B, H, Dv] bf16."""
    lib = load_library()
    q, k_pages = _bits(q), _bits(k_pages)
    v_pages = _bits(v_pages) if v_pages is not None else None
    B, H, Dk = q.shape
    G = k_pages.shape[2]
    k = indices.shape[-1]
    if out is None:
        out = torch.empty((B, H, Dv), dtype=torch.bfloat16, device=q.device)
    if workspace is None:
        workspace = alloc_workspace(B, G, 0, k, H, Dv, q.device)
    _check(lib.sd_sparse_attn(_ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(block_table), _ptr(seqlens),
                              _ptr(indices), _desc(k_pages, block_table), B, H, Dk, Dv, k, float(scale),
                              _ptr(out), _ptr(lse), _ptr(workspace), workspace.numel(), _stream(stream)))
    return out


def sd_decode_step_hinted(qi, w, ki_pages, q, k_pages, v_pages, block_table, seqlens, k: int, max_seqlen: int,
                          scale: float, Dv: int, hint, indices=None, scores=None, out=None, lse=None,
                          workspace=None, stream=None):
    """``sd_decode_step`` with the previous selection ``hint`` [B, G, k] (not
    the ``indices`` buffer). Returns (indices, out)."""
    lib = load_library()
    q, k_pages = _bits(q), _bits(k_pages)
    v_pages = _bits(v_pages) if v_pages is not None else None
    B, G, Hi, Di = qi.shape
    H, Dk = q.shape[1], q.shape[2]
    if indices is None:
        indices = torch.empty((B, G, k), dtype=torch.int32, device=q.device)
    if out is None:
        out = torch.empty((B, H, Dv), dtype=torch.bfloat16, device=q.device)
    if workspace is None:
        workspace = alloc_workspace(B, G, max_seqlen, k, H, Dv, q.device)
    _check(lib.sd_decode_step_hinted(_ptr(qi), _ptr(w), _ptr(ki_pages), _ptr(q), _ptr(k_pages), _ptr(v_pages),
                                     _ptr(block_table), _ptr(seqlens), _desc(k_pages, block_table), B, Hi, Di,
                                     H, Dk, Dv, max_seqlen, k, float(scale), _ptr(hint), _ptr(indices),
                                     _ptr(scores), _ptr(out), _ptr(lse), _ptr(workspace), workspace.numel(),
                                     _stream(stream)))
    return indices, out


def sd_sparse_attn_layers(q, k_pages, v_pages, block_table, seqlens, indices, scale: float, Dv: int,
                          out=None, lse=None, workspace=None, stream=None):
    """Attention + combine for several layers sharing one selection.

    ``q`` is [n_layers, B, H, Dk]; ``k_pages`` (and ``v_pages``, or None) are
    sequences of one pool per layer. Returns ``out`` [n_layers, B, H, Dv] bf16.
    """
    lib = load_library()
    q = _bits(q)
    kps = [_bits(t) for t in k_pages]
    vps = None if v_pages is None else [_bits(t) for t in v_pages]
    L, B, H, Dk = q.shape
    G = kps[0].shape[2]
    k = indices.shape[-1]
    if out is None:
        out = torch.empty((L, B, H, Dv), dtype=torch.bfloat16, device=q.device)
    if workspace is None:
        nbytes = int(lib.sd_attn_layers_workspace_size(L, B, G, k, H, Dv))
        workspace = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=q.device)
    karr = (ctypes.c_void_p * L)(*[t.data_ptr() for t in kps])
    varr = None if vps is None else (ctypes.c_void_p * L)(*[t.data_ptr() for t in vps])
    _check(lib.sd_sparse_attn_layers(_ptr(q), ctypes.cast(karr, ctypes.c_void_p),
                                     None if varr is None else ctypes.cast(varr, ctypes.c_void_p), L,
                                     _ptr(block_table), _ptr(seqlens), _ptr(indices), _desc(kps[0], block_table),
                                     B, H, Dk, Dv, k, float(scale), _ptr(out), _ptr(lse), _ptr(workspace),
                                     workspace.numel(), _stream(stream)))
    return out


def sd_sparse_attn_csr(q, k_pages, v_pages, block_table, seqlens, indices, offsets, block_size: int,
                       max_selected: int, scale: float, Dv: int, out=None, lse=None, workspace=None, stream=None):
    """Attention + combine with the selection in CSR form (``offsets`` [B*G+1],
    ``indices`` packed, each entry a block of ``block_size`` tokens when > 1).
    Returns ``out`` [B, H, Dv] bf16."""
    lib = load_library()
    q, k_pages = _bits(q), _bits(k_pages)
    v_pages = _bits(v_pages) if v_pages is not None else None
    B, H, Dk = q.shape
    G = k_pages.shape[2]
    if out is None:
        out = torch.empty((B, H, Dv), dtype=torch.bfloat16, device=q.device)
    if workspace is None:
        nbytes = int(lib.sd_csr_workspace_size(B, G, max_selected, H, Dv))
        workspace = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=q.device)
    idx = indices if indices is not None and indices.numel() > 0 else None
    _check(lib.sd_sparse_attn_csr(_ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(block_table), _ptr(seqlens),
                                  _ptr(idx), _ptr(offsets), int(block_size), int(max_selected),
                                  _desc(k_pages, block_table), B, H, Dk, Dv, float(scale), _ptr(out), _ptr(lse),
                                  _ptr(workspace), workspace.numel(), _stream(stream)))
    return out


def sd_decode_step(qi, w, ki_pages, q, k_pages, v_pages, block_table, seqlens, k: int, max_seqlen: int,
                   scale: float, Dv: int, indices=None, scores=None, out=None, lse=None, workspace=None,
                   stream=None):
    """The whole decode step. Returns (indices [B, G, k] int32, out [B, H, Dv] bf16)."""
    lib = load_library()
    q, k_pages = _bits(q), _bits(k_pages)
    v_pages = _bits(v_pages) if v_pages is not None else None
    B, G, Hi, Di = qi.shape
    H, Dk = q.shape[1], q.shape[2]
    if indices is None:
        indices = torch.empty((B, G, k), dtype=torch.int32, device=q.device)
    if out is None:
        out = torch.empty((B, H, Dv), dtype=torch.bfloat16, device=q.device)
    if workspace is None:
        workspace = alloc_workspace(B, G, max_seqlen, k, H, Dv, q.device)
    _check(lib.sd_decode_step(_ptr(qi), _ptr(w), _ptr(ki_pages), _ptr(q), _ptr(k_pages), _ptr(v_pages),
                              _ptr(block_table), _ptr(seqlens), _desc(k_pages, block_table), B, Hi, Di,
                              H, Dk, Dv, max_seqlen, k, float(scale), _ptr(indices), _ptr(scores),
                              _ptr(out), _ptr(lse), _ptr(workspace), workspace.numel(), _stream(stream)))
    return indices, out


TRI_UNION = 0
TRI_PER_HEAD = 1
TRI_PER_LAYER_PER_HEAD = 2


def sd_tri_compact(q_cal, k_pages, v_pages, block_table, seqlens, max_seqlen: int, n_sink: int, n_recent: int,
                   budget: int, mode: int = TRI_UNION, new_seqlens=None, workspace=None, stream=None):
    """TriAttention-style eviction of one layer: scores the evictable region of
    every request with ``q_cal``, keeps ``budget`` tokens and
    compacts ``k_pages`` (and ``v_pages``; bf16 [num_pages, P, G, D]) in place.
    ``q_cal`` is bf16 [H, D]. Returns ``new_seqlens`` [B] int32."""
    lib = load_library()
    q_cal, k_pages = _bits(q_cal), _bits(k_pages)
    v_pages = _bits(v_pages) if v_pages is not None else None
    H, D = q_cal.shape
    G = k_pages.shape[2]
    B = seqlens.shape[0]
    if new_seqlens is None:
        new_seqlens = torch.empty((B,), dtype=torch.int32, device=k_pages.device)
    if workspace is None:
        nbytes = int(lib.sd_tri_workspace_size(B, G, H, D, max_seqlen, n_sink, n_recent, budget, mode,
                                               1 if v_pages is not None else 0))
        workspace = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=k_pages.device)
    _check(lib.sd_tri_compact(_ptr(q_cal), _ptr(k_pages), _ptr(v_pages), _ptr(block_table), _ptr(seqlens),
                              _desc(k_pages, block_table), B, H, D, int(max_seqlen), int(n_sink), int(n_recent),
                              int(budget), int(mode), _ptr(new_seqlens), _ptr(workspace), workspace.numel(),
                              _stream(stream)))
    return new_seqlens


def sd_tri_compact_layers(q_cals, k_pools, v_pools, block_table, seqlens, max_seqlen: int, n_sink: int,
                          n_recent: int, budget: int, mode: int = TRI_UNION, new_seqlens=None, workspace=None,
                          stream=None):
    """Eviction over several layers sharing the block table: ``q_cals``,
    ``k_pools`` (and ``v_pools``) are per-layer lists; ``mode`` is TRI_UNION,
    TRI_PER_HEAD (one selection for all layers) or TRI_PER_LAYER_PER_HEAD.
    Compacts every layer in place; returns ``new_seqlens`` [B] int32."""
    lib = load_library()
    qs = [_bits(q) for q in q_cals]
    ks = [_bits(k) for k in k_pools]
    vs = None if v_pools is None else [_bits(v) for v in v_pools]
    L = len(ks)
    if len(qs) != L or (vs is not None and len(vs) != L):
        raise ValueError("q_cals, k_pools and v_pools need one entry per layer")
    H, D = qs[0].shape
    G = ks[0].shape[2]
    B = seqlens.shape[0]
    if new_seqlens is None:
        new_seqlens = torch.empty((B,), dtype=torch.int32, device=ks[0].device)
    if workspace is None:
        nbytes = int(lib.sd_tri_layers_workspace_size(L, B, G, H, D, max_seqlen, n_sink, n_recent, budget, mode,
                                                      1 if vs is not None else 0))
        workspace = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=ks[0].device)
    qarr = (ctypes.c_void_p * L)(*[_ptr(t) for t in qs])
    karr = (ctypes.c_void_p * L)(*[_ptr(t) for t in ks])
    varr = None if vs is None else (ctypes.c_void_p * L)(*[_ptr(t) for t in vs])
    _check(lib.sd_tri_compact_layers(ctypes.cast(qarr, ctypes.c_void_p), ctypes.cast(karr, ctypes.c_void_p),
                                     None if varr is None else ctypes.cast(varr, ctypes.c_void_p), L,
                                     _ptr(block_table), _ptr(seqlens), _desc(ks[0], block_table), B, H, D,
                                     int(max_seqlen), int(n_sink), int(n_recent), int(budget), int(mode),
                                     _ptr(new_seqlens), _ptr(workspace), workspace.numel(), _stream(stream)))
    return new_seqlens


def set_wait_limit(polls: int) -> None:
    """Polls the eviction compaction's cross-CTA waits make before giving up
    (a test hook; < 0 restores the default)."""
    _check(load_library().sd_set_wait_limit(int(polls)))


def device_errors(clear: bool = True) -> int:
    """Sticky device error bits (SD_DEVERR_*); synchronises the device."""
    bits = ctypes.c_uint32(0)
    _check(load_library().sd_get_device_errors(ctypes.byref(bits), 1 if clear else 0))
    return int(bits.value)


class StageTimer:
    """Records CUDA events around each stage (indexer, top-k, attention, combine)
    of every library call made by this thread while active; ``totals_ms()``
    sums the per-stage durations over the recorded calls."""

    STAGES = ("indexer", "topk", "attn", "combine")

    def __init__(self):
        self._pairs = []

    def arm(self):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(8)]
        for e in ev:
            e.record()  # torch creates the CUDA event lazily, on its first record
        arr = (ctypes.c_void_p * 8)(*[e.cuda_event for e in ev])
        _check(load_library().sd_set_stage_events(arr, 4))
        self._pairs.append(ev)

    @staticmethod
    def disarm():
        _check(load_library().sd_set_stage_events(None, 0))

    def totals_ms(self):
        torch.cuda.synchronize()
        tot = dict.fromkeys(self.STAGES, 0.0)
        for ev in self._pairs:
            for i, name in enumerate(self.STAGES):
                try:
                    tot[name] += ev[2 * i].elapsed_time(ev[2 * i + 1])
                except RuntimeError:  # stage not run by that call
                    pass
        return tot, len(self._pairs)


def last_launch_count() -> int:
    return int(load_library().sd_last_launch_count())
