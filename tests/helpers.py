"""Test helpers: move a generated workload to the GPU, run the library, and
compare against the oracle with the tolerances the parity bar fixes."""
import numpy as np

TOL_MAX_ABS = 2e-2   # bf16 output vs fp64 oracle: max |diff|
TOL_REL_L2 = 5e-3    # ||diff||_2 / ||ref||_2


def to_device(wl):
    import torch
    dev = "cuda"
    t = lambda a, dt=None: torch.from_numpy(np.ascontiguousarray(a)).to(dev)  # noqa: E731
    d = dict(
        qi=t(wl.qi), w=t(wl.w), ki_pages=t(wl.ki_pages), block_table=t(wl.block_table),
        seqlens=t(wl.seqlens),
        q=t(wl.q.view(np.int16)).view(torch.bfloat16),
        k_pages=t(wl.k_pages.view(np.int16)).view(torch.bfloat16),
        v_pages=None if wl.v_pages is None else t(wl.v_pages.view(np.int16)).view(torch.bfloat16),
    )
    return d


def run_step(wl, d, with_scores=True, lse=True):
    import torch
    import top_sparse_decode_paged_b200 as sd
    s = wl.spec
    B, G = wl.seqlens.shape[0], s.G
    Lmax = max(wl.max_seqlen, 1)
    scores = torch.empty((B, G, Lmax), dtype=torch.int32, device="cuda") if with_scores else None
    lse_t = torch.empty((B, s.H), dtype=torch.float32, device="cuda") if lse else None
    idx, out = sd.sd_decode_step(d["qi"], d["w"], d["ki_pages"], d["q"], d["k_pages"], d["v_pages"],
                                 d["block_table"], d["seqlens"], s.k, wl.max_seqlen, s.scale, s.Dv,
                                 scores=scores, lse=lse_t)
    torch.cuda.synchronize()
    return dict(indices=idx.cpu().numpy(), out=out.float().cpu().numpy().astype(np.float64),
                scores=None if scores is None else scores.cpu().numpy(),
                lse=None if lse_t is None else lse_t.cpu().numpy().astype(np.float64))


def assert_out_close(got, ref, what=""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    diff = got - ref
    max_abs = float(np.abs(diff).max()) if diff.size else 0.0
    nref = float(np.linalg.norm(ref))
    rel = float(np.linalg.norm(diff)) / nref if nref > 0 else float(np.linalg.norm(diff))
    assert max_abs <= TOL_MAX_ABS, f"{what}: max_abs {max_abs:.3e}"
    assert rel <= TOL_REL_L2, f"{what}: rel_l2 {rel:.3e}"
    return max_abs, rel
