"""The C ABI library without a GPU: it loads, exports every symbol the header
declares, sizes workspaces deterministically and rejects bad arguments before
any CUDA call."""
import ctypes
import os
import re

import pytest

import top_sparse_decode_paged_b200 as sd
from top_sparse_decode_paged_b200 import api

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    text = open(os.path.join(ROOT, "include", "sd_api.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sd_[a-z_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from top_sparse_decode_paged_b200 import build
    build.build()
    return sd.load_library()


def test_every_declared_symbol_is_exported(lib):
    names = _declared_functions()
    assert len(names) >= 9
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(api.EXPORTED)


def test_version_and_status_strings(lib):
    assert lib.sd_version() >= 1
    assert lib.sd_status_str(0) == b"SD_OK"
    assert lib.sd_status_str(3) == b"SD_ERR_WORKSPACE"
    assert lib.sd_status_str(99) == b"SD_ERR_UNKNOWN"


def test_workspace_size_is_deterministic_and_rejects_bad_shapes(lib):
    a = sd.workspace_size(32, 1, 65536, 2048, 128, 512)
    assert a == sd.workspace_size(32, 1, 65536, 2048, 128, 512)
    assert a >= 32 * 65536 * 4 and a % 256 == 0
    assert sd.workspace_size(-1, 1, 10, 4, 4, 64) == 0
    assert sd.workspace_size(1, 3, 10, 4, 4, 64) == 0     # H % G != 0


def _call_indexer(lib, **over):
    args = dict(qi=256, w=256, ki=256, bt=256, sl=256, B=1, Hi=4, Di=32, L=64, k=8, idx=256)
    args.update(over)
    desc = api.PagedDesc(4, 16, 4, 1)
    return lib.sd_indexer_topk(args["qi"], args["w"], args["ki"], args["bt"], args["sl"], desc,
                               args["B"], args["Hi"], args["Di"], args["L"], args["k"], args["idx"],
                               None, None, 0, None)


def test_argument_errors_return_before_any_launch(lib):
    assert _call_indexer(lib, qi=None) == 1                  # SD_ERR_INVALID_ARG
    assert _call_indexer(lib, k=0) == 1
    assert _call_indexer(lib, Di=48) == 2                    # SD_ERR_UNSUPPORTED
    assert _call_indexer(lib, k=4096) == 2
    assert _call_indexer(lib, Hi=65) == 2
    assert _call_indexer(lib) == 3                           # no scores, no workspace
    assert lib.sd_last_launch_count() == 0


def test_attention_argument_errors(lib):
    desc = api.PagedDesc(4, 16, 4, 1)
    f = lib.sd_sparse_attn
    # Dv > Dk with V taken from the K row
    assert f(256, 256, None, 256, 256, 256, desc, 1, 4, 64, 128, 8, ctypes.c_float(0.1), 256, None,
             None, 0, None) == 1
    # unsupported head width
    assert f(256, 256, None, 256, 256, 256, desc, 1, 4, 96, 96, 8, ctypes.c_float(0.1), 256, None,
             None, 0, None) == 2
    # non-finite scale
    assert f(256, 256, None, 256, 256, 256, desc, 1, 4, 64, 64, 8, ctypes.c_float(float("nan")), 256,
             None, None, 0, None) == 1


def test_layers_argument_errors(lib):
    desc = api.PagedDesc(4, 16, 4, 1)
    f = lib.sd_sparse_attn_layers
    pools = (ctypes.c_void_p * 2)(256, 256)
    holes = (ctypes.c_void_p * 2)(256, None)
    args = lambda kp, n, Dk=64, Dv=64: (256, ctypes.cast(kp, ctypes.c_void_p), None, n, 256, 256, 256, desc,  # noqa: E731
                                         1, 4, Dk, Dv, 8, ctypes.c_float(0.1), 256, None, None, 0, None)
    assert f(*args(pools, 0)) == 1          # no layers
    assert f(*args(holes, 2)) == 1          # a NULL pool
    assert f(*args(pools, 2, 96, 96)) == 2  # unsupported head width
    assert f(*args(pools, 2)) == 3          # no workspace
    assert lib.sd_attn_layers_workspace_size(0, 1, 1, 8, 4, 64) == 0
    one = lib.sd_attn_layers_workspace_size(1, 32, 1, 2048, 128, 512)
    assert lib.sd_attn_layers_workspace_size(4, 32, 1, 2048, 128, 512) > one > 0
    # layers beyond the 16 of one launch reuse the workspace of 16
    assert lib.sd_attn_layers_workspace_size(40, 32, 1, 2048, 128, 512) == \
        lib.sd_attn_layers_workspace_size(16, 32, 1, 2048, 128, 512)
    assert lib.sd_last_launch_count() == 0


def test_tri_compact_argument_errors(lib):
    """sd_tri_compact: 1 = invalid, 2 = unsupported, 3 = workspace, all before
    any launch; the workspace grows with the budget."""
    desc = api.PagedDesc(64, 16, 8, 2)
    f = lib.sd_tri_compact
    ws = lambda *a: lib.sd_tri_workspace_size(*a)  # noqa: E731
    args = lambda H=4, D=64, budget=8, mode=0, nws=0, B=2: (256, 256, None, 256, 256, desc, B, H, D, 100, 4,  # noqa: E731
                                                              8, budget, mode, 256, 256 if nws else None, nws, None)
    assert f(*args(H=5)) == 1            # H not a multiple of G
    assert f(*args(budget=0)) == 1       # empty budget
    assert f(*args(mode=3)) == 1         # unknown mode
    assert f(*args(D=96)) == 2           # head width
    assert f(*args(H=32)) == 2           # 16 query heads per KV head
    assert f(*args(budget=4096)) == 2    # above the top-k limit
    assert f(*args()) == 3               # no workspace
    assert f(*args(nws=16)) == 3         # too small
    assert ws(2, 2, 4, 64, 100, 4, 8, 0, 0, 1) == 0
    a = ws(2, 2, 4, 64, 100, 4, 8, 24, 0, 0)
    assert ws(2, 2, 4, 64, 100, 4, 8, 24, 0, 1) >= a > 0
    assert ws(2, 2, 4, 64, 100, 4, 8, 48, 0, 0) > a
    assert lib.sd_last_launch_count() == 0


def test_tri_layers_argument_errors(lib):
    desc = api.PagedDesc(64, 16, 8, 2)
    f = lib.sd_tri_compact_layers
    ptrs = (ctypes.c_void_p * 2)(256, 256)
    holes = (ctypes.c_void_p * 2)(256, None)
    arr = lambda a: ctypes.cast(a, ctypes.c_void_p)  # noqa: E731
    args = lambda q, k, n, mode=0: (arr(q), arr(k), None, n, 256, 256, desc, 2, 4, 64, 100, 4, 8, 24, mode,  # noqa: E731
                                    256, None, 0, None)
    assert f(*args(ptrs, ptrs, 0)) == 1          # no layers
    assert f(*args(ptrs, holes, 2)) == 1         # a NULL pool
    assert f(*args(ptrs, ptrs, 2, mode=3)) == 1  # unknown mode
    assert f(*args(ptrs, ptrs, 2)) == 3          # no workspace
    one = lib.sd_tri_layers_workspace_size(1, 2, 2, 4, 64, 100, 4, 8, 24, 0, 1)
    assert one == lib.sd_tri_workspace_size(2, 2, 4, 64, 100, 4, 8, 24, 0, 1)
    assert lib.sd_tri_layers_workspace_size(4, 64, 2, 4, 64, 5000, 4, 8, 2048, 0, 1) > \
        lib.sd_tri_layers_workspace_size(1, 64, 2, 4, 64, 5000, 4, 8, 2048, 0, 1)  # a flag set per layer
    assert lib.sd_last_launch_count() == 0


def test_indexer_rejects_a_misaligned_key_pool(lib):
    desc = api.PagedDesc(4, 16, 4, 1)
    # qi, w, ki_pages, block_table, seqlens, pd, B, Hi, Di, max_seqlen, k, indices, scores, ws, ws_bytes, stream
    assert lib.sd_indexer_topk(256, 256, 264, 256, 256, desc, 1, 4, 32, 64, 8, 256, None, None, 0, None) == 1


def test_tri_rejects_misaligned_pools(lib):
    desc = api.PagedDesc(64, 16, 8, 2)
    f = lib.sd_tri_compact
    # q_cal, k_pages, v_pages, block_table, seqlens, pd, B, H, D, max_seqlen, n_sink, n_recent, budget, mode,
    # new_seqlens, workspace, workspace_bytes, stream
    assert f(256, 264, None, 256, 256, desc, 2, 4, 64, 100, 4, 8, 24, 0, 256, None, 0, None) == 1
    assert f(256, 256, 264, 256, 256, desc, 2, 4, 64, 100, 4, 8, 24, 0, 256, None, 0, None) == 1
    assert f(256, 256, 256, 256, 256, desc, 2, 4, 64, 100, 4, 8, 24, 0, 256, None, 0, None) == 3  # aligned: workspace


def test_wait_limit_hook_checks_its_argument_without_cuda(lib):
    """sd_set_wait_limit makes no CUDA call: it accepts 0 .. 2^22 and < 0
    (the default) and rejects a limit above the default."""
    assert lib.sd_set_wait_limit(0) == 0
    assert lib.sd_set_wait_limit(1 << 22) == 0
    assert lib.sd_set_wait_limit((1 << 22) + 1) == 1
    assert lib.sd_set_wait_limit(-1) == 0


def test_noalloc_argument_errors_return_before_any_cuda_call(lib):
    """sd_indexer_topk_noalloc rejects bad arguments before it looks up its
    scratch array or launches anything."""
    desc = api.PagedDesc(4, 16, 4, 1)

    def call(qi=256, idx=256, Di=32, B=1, L=64):
        return lib.sd_indexer_topk_noalloc(qi, 256, 256, 256, 256, desc, B, 4, Di, L, 8, idx, None)

    assert call(qi=None) == 1                                   # SD_ERR_INVALID_ARG
    assert call(idx=None) == 1
    assert call(Di=48) == 2                                     # SD_ERR_UNSUPPORTED
    assert call(B=8, L=(api.NOALLOC_MAX_SCORES // 8) + 1) == 3  # SD_ERR_WORKSPACE
    assert lib.sd_last_launch_count() == 0
