"""Benchmark of one sparse decode step (indexer -> top-k -> sparse attention).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]

Prints ONE JSON line (rank 0). A step is ``sd_decode_step`` over one synthetic
batch of the named workload (default: 32 requests x 65536 cached tokens, MLA
latent rows shared by 128 heads, top-k 2048). Inputs are resident in HBM; L2 is
flushed before every step, outside the timed events: a 256 MiB write evicts
everything, then a 256 MiB read replaces the dirty lines with clean ones, so
that the timed step pays no write-back of the flush itself. With
N > 1 (torchrun) each rank runs its own batch (different seed): the path shards
by request with no collective, so the scaling is weak and the value is the
total queries/s of all ranks over the slowest rank's time.

``--impl reference`` times the CPU oracle (the only reference this path has)
on a bounded sample of the same workload, on rank 0 only.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from top_sparse_decode_paged_b200 import workloads as W  # noqa: E402

METRIC = "decode queries/s and achieved HBM GB/s (indexer+top-k+sparse attn), 1 B200"
DEFAULT_CONFIG = "b32_l65536_mla"
L2_FLUSH_BYTES = 256 << 20

# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of one launch,
# from the ncu captures summarised in profiles/, keyed by (workload, stage).
# Valid only for the library version they were taken on; any other version
# reports traffic as null.
NCU_TRAFFIC = {
    # captured at --batch 16 (half the workload's 32 requests) and scaled by 2:
    # both kernels' traffic grows with the requests they process
    ("b32_l65536_mla", "indexer"): (0x00000007, 2 * (134.464000e6 + 4.018176e6)),
    ("b32_l65536_mla", "attn"): (0x00000007, 2 * (40.339456e6 + 1.273856e6)),
}


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def _dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


BATCH_OVERRIDE = None  # --batch: requests per rank (profiling a reduced batch of the same workload)


def rank_spec(name: str, rank: int) -> W.Spec:
    """Each rank draws its own batch of the same shape (weak scaling)."""
    over = {} if BATCH_OVERRIDE is None else {"B": BATCH_OVERRIDE}
    base = W.spec(name, **over)
    return W.spec(name, seed=base.seed + 1000 * rank, **over) if rank else base


def max_over_ranks(value: float, world: int) -> float:
    """Slowest rank's time (all ranks take this collective in the same order)."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


class ClockSampler:
    """Samples nvidia-smi clocks and throttle reasons while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.rows = []
        self._stop = threading.Event()
        self._t = None

    def _run(self):
        while not self._stop.is_set():
            try:
                out = subprocess.run(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                      "--format=csv,noheader,nounits"], capture_output=True, text=True,
                                     timeout=5).stdout.strip()
                if out:
                    self.rows.append([x.strip() for x in out.split(",")])
            except Exception:
                pass
            self._stop.wait(0.1)

    def __enter__(self):
        self._t = threading.Thread(target=self._run, daemon=True)
        self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        self._t.join(timeout=10)

    def summary(self):
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        sm = [float(r[0]) for r in self.rows if r[0].replace(".", "").isdigit()]
        mx = [float(r[1]) for r in self.rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in self.rows for i in range(4) if r[3 + i] == "Active"})
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(self.rows)}


def run_oracle_sample(wl, n_req: int):
    """Times the CPU oracle on the first n_req requests of the batch."""
    import oracle
    t0 = time.perf_counter()
    oracle.decode_step(wl, requests=list(range(n_req)))
    return time.perf_counter() - t0


def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info()]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def _host():
    """The host the oracle ran on: logical CPUs and the CPU model."""
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    model = ln.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"nproc": os.cpu_count(), "cpu_model": model}


def cpu_baseline(name: str, budget_s: float = 15.0):
    """The oracle as it stands on a bounded sample: requests are added until the
    sample has taken about budget_s seconds of host time."""
    wl = W.make(W.spec(name))
    done, spent = 0, 0.0
    while done < wl.seqlens.shape[0] and spent < budget_s:
        t0 = time.perf_counter()
        import oracle
        oracle.decode_step(wl, requests=[done])
        spent += time.perf_counter() - t0
        done += 1
    return {"value": done / spent, "unit": "queries/s", "cores": _blas_threads(), "kind": "oracle",
            "sample": f"{done} of {wl.seqlens.shape[0]} requests of {name}, {spent:.1f} s host time",
            "threads": "the int and fp64 matmuls use `cores` BLAS threads; the lexsort top-k and the attention "
                       "loops run on one thread", **_host()}


def bench_reference(args, rank, world):
    """The oracle, unchanged, on the host cores. A step is the oracle's decode
    step over a fixed sample of the batch's requests (the full batch would take
    minutes per step); ms_per_step is the time of that sample, and the value
    is the requests it decoded per second."""
    if rank != 0:
        return
    n_steps = args.steps
    wl = W.make(rank_spec(args.config, 0))
    times = []
    per_step = max(1, min(wl.seqlens.shape[0], 2))
    for i in range(args.warmup + n_steps):
        t = run_oracle_sample(wl, per_step)
        if i >= args.warmup:
            times.append(t)
    ms = 1e3 * float(np.mean(times))
    value = per_step / float(np.mean(times))
    sample = f"the first {per_step} of {wl.seqlens.shape[0]} requests of {args.config} per step"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "queries/s", "n_gpus": world,
        "steps": n_steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "int64/f64", "data": "synthetic",
        "config": _config(wl.spec),
        "l2": "host memory (CPU oracle)",
        "queries_per_step": per_step,
        "cpu_baseline": {"value": value, "unit": "queries/s", "cores": _blas_threads(), "kind": "oracle",
                         "sample": sample,
                         "threads": "the int and fp64 matmuls use `cores` BLAS threads; the lexsort top-k and the "
                                    "attention loops run on one thread", **_host()},
        "e2e": {"value": value, "unit": "queries/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def _config(s: W.Spec):
    cfg = {"workload": s.name, "B": s.B, "page": s.page_size, "kv_heads": s.G, "Hi": s.Hi, "Di": s.Di,
           "k": s.k, "H": s.H, "Dk": s.Dk, "Dv": s.Dv}
    if s.seqlen is not None:
        cfg["seqlen"] = s.seqlen
    if s.ragged is not None:
        cfg["seqlen_loguniform"] = list(s.ragged)
    return cfg


def bench_ours(args, rank, world, local):
    import torch
    import top_sparse_decode_paged_b200 as sd
    from top_sparse_decode_paged_b200.api import StageTimer

    torch.cuda.set_device(local)
    spec = rank_spec(args.config, rank)
    wl = W.make(spec)
    s = wl.spec
    dev = "cuda"
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)  # noqa: E731
    qi, w, ki = t(wl.qi), t(wl.w), t(wl.ki_pages)
    bt, sl = t(wl.block_table), t(wl.seqlens)
    q = t(wl.q.view(np.int16)).view(torch.bfloat16)
    kp = t(wl.k_pages.view(np.int16)).view(torch.bfloat16)
    vp = None if wl.v_pages is None else t(wl.v_pages.view(np.int16)).view(torch.bfloat16)
    B, G = wl.seqlens.shape[0], s.G
    Lmax = wl.max_seqlen
    idx = torch.empty((B, G, s.k), dtype=torch.int32, device=dev)
    out = torch.empty((B, s.H, s.Dv), dtype=torch.bfloat16, device=dev)
    ws = sd.alloc_workspace(B, G, Lmax, s.k, s.H, s.Dv)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    clean = torch.zeros(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def flush_l2():
        # a write larger than L2 evicts everything; a read larger than L2 then
        # leaves only clean lines behind, so no write-back lands in the step
        flush.zero_()
        clean.max()

    def step():
        sd.sd_decode_step(qi, w, ki, q, kp, vp, bt, sl, s.k, Lmax, s.scale, s.Dv,
                          indices=idx, out=out, workspace=ws)

    for _ in range(args.warmup):
        flush_l2()
        step()
    launches_per_step = sd.last_launch_count()
    torch.cuda.synchronize()

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    stage_tot = dict.fromkeys(StageTimer.STAGES, 0.0)
    graph = None
    if not args.no_graph:
        # capture one step, with the stage events inside it; replays re-record them
        timer = StageTimer()
        side = torch.cuda.Stream()
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            step()
        torch.cuda.synchronize()
        # the timed graph has no events inside; a second graph with the stage
        # events gives the per-kernel split (its replays are timed separately)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=side):
            step()
        stage_graph = torch.cuda.CUDAGraph()
        timer.arm()
        with torch.cuda.graph(stage_graph, stream=side):
            step()
        StageTimer.disarm()
        stage_events = timer._pairs[0]
        for _ in range(args.warmup):
            flush_l2()
            graph.replay()
            flush_l2()
            stage_graph.replay()
        torch.cuda.synchronize()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local if "CUDA_VISIBLE_DEVICES" not in os.environ else int(
            os.environ["CUDA_VISIBLE_DEVICES"].split(",")[local])) as clocks:
        if graph is not None:
            for i in range(args.steps):
                flush_l2()
                starts[i].record(stream)
                graph.replay()
                ends[i].record(stream)
            torch.cuda.synchronize()
            for i in range(args.steps):
                flush_l2()
                stage_graph.replay()
                torch.cuda.synchronize()  # the stage events inside the graph are read before the next replay
                for j, name in enumerate(StageTimer.STAGES):
                    stage_tot[name] += stage_events[2 * j].elapsed_time(stage_events[2 * j + 1])
        else:
            timer = StageTimer()
            for i in range(args.steps):
                flush_l2()
                timer.arm()
                starts[i].record(stream)
                step()
                ends[i].record(stream)
            torch.cuda.synchronize()
            StageTimer.disarm()
            stage_tot, _ = timer.totals_ms()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
    step_ms = sum(a.elapsed_time(b) for a, b in zip(starts, ends)) / args.steps
    stage_ms = {k_: v / args.steps for k_, v in stage_tot.items()}
    step_ms = max_over_ranks(step_ms, world)
    if graph is not None:
        del graph, stage_graph

    # end to end through the public call: every step uploads its query-side
    # inputs (qi, w, q, block table, seqlens) from pinned host memory and
    # downloads its results (indices, output). As a serving loop would, each
    # step's inputs sit packed in one pinned buffer (one upload) and its
    # results in one device buffer (one download).
    def packed(parts, device, pin=False):
        """One uint8 buffer holding the given (shape, dtype) parts at 256-byte
        aligned offsets; returns (buffer, views)."""
        offs, total = [], 0
        for shape, dt in parts:
            offs.append(total)
            nbytes = int(np.prod(shape)) * torch.empty((), dtype=dt).element_size()
            total += (nbytes + 255) // 256 * 256
        buf = torch.empty(total, dtype=torch.uint8, device=device)
        if pin:
            buf = buf.pin_memory()
        views = []
        for (shape, dt), o in zip(parts, offs):
            n = int(np.prod(shape)) * torch.empty((), dtype=dt).element_size()
            views.append(buf[o:o + n].view(dt).view(shape))
        return buf, views

    in_parts = [(tuple(qi.shape), torch.int8), (tuple(w.shape), torch.int32), (tuple(q.shape), torch.int16),
                (tuple(bt.shape), torch.int32), (tuple(sl.shape), torch.int32)]
    out_parts = [(tuple(idx.shape), torch.int32), (tuple(out.shape), torch.int16)]
    h_in, h_in_v = packed(in_parts, "cpu", pin=True)
    for v_, a_ in zip(h_in_v, (wl.qi, wl.w, wl.q.view(np.int16), wl.block_table, wl.seqlens)):
        v_.copy_(torch.from_numpy(np.ascontiguousarray(a_)))
    h2d = h_in.numel()  # the packed buffers are what moves (each part padded to 256 bytes)
    e_steps = max(3, min(args.steps, 50))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def make_set():
        d_in, (dqi, dw, dq, dbt, dsl) = packed(in_parts, dev)
        d_out, (didx, dout) = packed(out_parts, dev)
        h_out, _ = packed(out_parts, "cpu", pin=True)
        return dict(d_in=d_in, qi=dqi, w=dw, q=dq.view(torch.bfloat16), bt=dbt, sl=dsl, d_out=d_out, idx=didx,
                    out=dout.view(torch.bfloat16), h_out=h_out, up=torch.cuda.Event(), done=torch.cuda.Event(),
                    down=torch.cuda.Event())

    def run_set(bb):
        sd.sd_decode_step(bb["qi"], bb["w"], ki, bb["q"], kp, vp, bb["bt"], bb["sl"], s.k, Lmax, s.scale, s.Dv,
                          indices=bb["idx"], out=bb["out"], workspace=ws)

    def graph_of(bb, st):
        """The public call for buffer set bb, captured once and replayed every
        step (a serving loop keeps the host out of the per-step launches)."""
        if args.no_graph:
            return None
        with torch.cuda.stream(st):
            run_set(bb)  # loads every kernel and settles the launch attributes
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=st):
            run_set(bb)
        torch.cuda.synchronize()
        return g

    torch.cuda.synchronize()
    # (a) one step at a time: upload, step, download, then wait
    one = make_set()
    d2h = one["h_out"].numel()
    side_e2e = torch.cuda.Stream()
    g_one = graph_of(one, side_e2e)
    e_ms_serial = 0.0
    for i in range(e_steps):
        flush_l2()
        e0.record(stream)
        one["d_in"].copy_(h_in, non_blocking=True)
        if g_one is not None:
            g_one.replay()
        else:
            run_set(one)
        one["h_out"].copy_(one["d_out"], non_blocking=True)
        e1.record(stream)
        e1.synchronize()
        e_ms_serial += e0.elapsed_time(e1)
    e_ms_serial = max_over_ranks(e_ms_serial / e_steps, world)
    # (b) as a serving loop runs it: step i's inputs go up while step i-1
    # computes and step i-2's results come down (two buffer sets, three
    # streams); every step still pays both copies. No flush: the inputs
    # (indexer keys and latent cache) are larger than L2.
    bufs = [make_set() for _ in range(2)]
    s_up, s_comp, s_down = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    for bb in bufs:
        bb["graph"] = graph_of(bb, s_comp)

    def pipelined(n):
        for i in range(n):
            bb = bufs[i % 2]
            with torch.cuda.stream(s_up):
                if i >= 2:
                    s_up.wait_event(bb["done"])  # step i-2 has consumed this buffer set
                bb["d_in"].copy_(h_in, non_blocking=True)
                bb["up"].record(s_up)
            with torch.cuda.stream(s_comp):
                s_comp.wait_event(bb["up"])
                if i >= 2:
                    s_comp.wait_event(bb["down"])  # step i-2's results are out of this buffer set
                if bb["graph"] is not None:
                    bb["graph"].replay()
                else:
                    run_set(bb)
                bb["done"].record(s_comp)
            with torch.cuda.stream(s_down):
                s_down.wait_event(bb["done"])
                bb["h_out"].copy_(bb["d_out"], non_blocking=True)
                bb["down"].record(s_down)

    pipelined(4)
    torch.cuda.synchronize()
    p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    p0.record(s_up)
    pipelined(e_steps)
    for st_ in (s_up, s_comp):
        s_down.wait_stream(st_)
    p1.record(s_down)
    p1.synchronize()
    e_ms = max_over_ranks(p0.elapsed_time(p1) / e_steps, world)

    alg = W.algorithmic_bytes(s, wl.seqlens)
    lens = wl.seqlens.astype(np.int64)
    idx_bytes = int(lens.sum()) * s.G * s.Di
    row_bytes = s.Dk * 2 if s.v_in_k else (s.Dk + s.Dv) * 2
    attn_bytes = int(np.minimum(lens, s.k).sum()) * s.G * row_bytes
    peak, peak_kind = _peaks()
    lib_version = int(sd.load_library().sd_version())

    def roofline(stage, nbytes):
        ms = stage_ms[stage]
        achieved = nbytes / (ms * 1e-3) / 1e9 if ms > 0 else None
        tv = NCU_TRAFFIC.get((s.name, stage))
        traffic = (tv[1] if tv and tv[0] == lib_version and rank_spec(args.config, 0).seed == s.seed
                   and BATCH_OVERRIDE is None else None)
        return {"kernel": stage, "bound": "hbm", "achieved": achieved, "peak": peak, "peak_kind": peak_kind,
                "unit": "GB/s", "frac": (achieved / peak) if achieved else None, "traffic": traffic,
                "algorithmic_bytes_per_launch": nbytes, "ms_per_launch": ms}

    rooflines = {"indexer": roofline("indexer", idx_bytes), "attn": roofline("attn", attn_bytes)}
    dominant = max(rooflines, key=lambda k_: stage_ms[k_])
    line = {
        "metric": METRIC,
        "value": world * B / (step_ms * 1e-3),
        "unit": "queries/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": step_ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int8/bf16", "data": "synthetic",
        "config": _config(s),
        "l2": "flushed before every step (256 MiB write, then 256 MiB read so the lines left are clean; outside the "
              "timed events)",
        "timing": ("CUDA graph of one sd_decode_step, replayed; the per-kernel split comes from a second graph with "
                   "stage events inside") if not args.no_graph else "eager sd_decode_step calls",
        "hbm_gbs_step": alg / (step_ms * 1e-3) / 1e9,
        "hbm_frac_step": alg / (step_ms * 1e-3) / 1e9 / peak,
        "algorithmic_bytes_per_step": alg,
        "stage_ms": stage_ms,
        "roofline": rooflines[dominant],
        "rooflines": rooflines,
        "e2e": {"value": world * B / (min(e_ms, e_ms_serial) * 1e-3), "unit": "queries/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "mode": "pipelined" if e_ms <= e_ms_serial else "serial",
                "pipelined_value": world * B / (e_ms * 1e-3),
                "serial_value": world * B / (e_ms_serial * 1e-3),
                "step_launch": ("sd_decode_step captured once per buffer set and replayed each step"
                                if not args.no_graph else "eager sd_decode_step calls")},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks.summary(),
        "library_version": lib_version,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args.config)
    if rank == 0:
        print(json.dumps(line), flush=True)


def bench_layers(args, rank, world, local):
    """Attention-only decode over args.layers layers that share one selection
    (sd_sparse_attn_layers), against the same layers as separate
    sd_sparse_attn calls. Layer l uses the workload's queries with the heads
    rolled by l and its cache scaled by 1 + (l mod 4)/4 (one pool per layer in
    HBM). L2 is flushed before every timed replay, as in the decode-step bench."""
    import torch
    import top_sparse_decode_paged_b200 as sd

    torch.cuda.set_device(local)
    wl = W.make(rank_spec(args.config, rank))
    s = wl.spec
    n = args.layers
    dev = "cuda"
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)  # noqa: E731
    qi, w, ki = t(wl.qi), t(wl.w), t(wl.ki_pages)
    bt, sl = t(wl.block_table), t(wl.seqlens)
    q0 = t(wl.q.view(np.int16)).view(torch.bfloat16)
    kp0 = t(wl.k_pages.view(np.int16)).view(torch.bfloat16)
    vp0 = None if wl.v_pages is None else t(wl.v_pages.view(np.int16)).view(torch.bfloat16)
    B = wl.seqlens.shape[0]
    idx = sd.sd_indexer_topk(qi, w, ki, bt, sl, s.k, wl.max_seqlen)
    del ki
    q = torch.stack([torch.roll(q0, l, dims=1) for l in range(n)]).contiguous()
    kps = [kp0] + [(kp0.float() * (1 + (l % 4) / 4)).to(torch.bfloat16) for l in range(1, n)]
    vps = None if vp0 is None else [vp0] + [(vp0.float() * (1 + (l % 4) / 4)).to(torch.bfloat16) for l in range(1, n)]
    out = torch.empty((n, B, s.H, s.Dv), dtype=torch.bfloat16, device=dev)
    lib = sd.load_library()
    ws_l = torch.empty(int(lib.sd_attn_layers_workspace_size(n, B, s.G, s.k, s.H, s.Dv)), dtype=torch.uint8, device=dev)
    ws_1 = sd.alloc_workspace(B, s.G, 0, s.k, s.H, s.Dv)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    clean = torch.zeros(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def flush_l2():
        flush.zero_()
        clean.max()

    def together():
        sd.sd_sparse_attn_layers(q, kps, vps, bt, sl, idx, s.scale, s.Dv, out=out, workspace=ws_l)

    def apart():
        for l in range(n):
            sd.sd_sparse_attn(q[l], kps[l], None if vps is None else vps[l], bt, sl, idx, s.scale, s.Dv,
                              out=out[l], workspace=ws_1)

    def timed(fn):
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            fn()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=side):
            fn()
        for _ in range(args.warmup):
            flush_l2()
            g.replay()
        torch.cuda.synchronize()
        stream = torch.cuda.current_stream()
        tot = 0.0
        for _ in range(args.steps):
            flush_l2()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            g.replay()
            b.record(stream)
            b.synchronize()
            tot += a.elapsed_time(b)
        del g
        return max_over_ranks(tot / args.steps, world)

    ms_together = timed(together)
    ms_apart = timed(apart)
    lens = wl.seqlens.astype(np.int64)
    row_bytes = s.Dk * 2 if s.v_in_k else (s.Dk + s.Dv) * 2
    nbytes = n * int(np.minimum(lens, s.k).sum()) * s.G * row_bytes
    peak, peak_kind = _peaks()
    achieved = nbytes / (ms_together * 1e-3) / 1e9
    line = {
        "metric": "attention-only decode layer-queries/s (layers sharing one selection), 1 B200",
        "value": world * n * B / (ms_together * 1e-3), "unit": "layer-queries/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "layers": n,
        "ms_per_step": ms_together, "ms_per_step_separate_calls": ms_apart,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": _config(s),
        "l2": "flushed before every step (256 MiB write, then 256 MiB read; outside the timed events)",
        "roofline": {"kernel": "attn (all layers, with combine)", "bound": "hbm", "achieved": achieved, "peak": peak,
                     "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / peak, "traffic": None,
                     "algorithmic_bytes_per_launch": nbytes, "ms_per_launch": ms_together},
    }
    if rank == 0:
        print(json.dumps(line), flush=True)


def bench_csr(args, rank, world, local):
    """Attention with the selection in CSR form (sd_sparse_attn_csr): the
    decode step's top-k selection packed per request (block size 1), or, with
    --csr-block bs > 1, the blocks of bs tokens that hold the first 2048 / bs
    selected tokens' blocks. Timed like the decode step (graph replay, L2
    flushed), beside sd_sparse_attn on the padded top-k selection."""
    import torch
    import top_sparse_decode_paged_b200 as sd

    torch.cuda.set_device(local)
    wl = W.make(rank_spec(args.config, rank))
    s = wl.spec
    dev = "cuda"
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)  # noqa: E731
    qi, w, ki = t(wl.qi), t(wl.w), t(wl.ki_pages)
    bt, sl = t(wl.block_table), t(wl.seqlens)
    q = t(wl.q.view(np.int16)).view(torch.bfloat16)
    kp = t(wl.k_pages.view(np.int16)).view(torch.bfloat16)
    vp = None if wl.v_pages is None else t(wl.v_pages.view(np.int16)).view(torch.bfloat16)
    B = wl.seqlens.shape[0]
    idx = sd.sd_indexer_topk(qi, w, ki, bt, sl, s.k, wl.max_seqlen)
    del ki
    bs = max(args.csr_block, 1)
    ix = idx.cpu().numpy().reshape(B * s.G, s.k)
    flat, offs = [], [0]
    for r in range(B * s.G):
        row = ix[r][ix[r] >= 0]
        if bs > 1:
            row = np.unique(row // bs)[: max(s.k // bs, 1)]
        flat.append(row.astype(np.int32))
        offs.append(offs[-1] + len(row))
    flat_t = t(np.concatenate(flat))
    offs_t = t(np.asarray(offs, dtype=np.int32))
    max_sel = s.k
    out = torch.empty((B, s.H, s.Dv), dtype=torch.bfloat16, device=dev)
    lib = sd.load_library()
    ws_c = torch.empty(int(lib.sd_csr_workspace_size(B, s.G, max_sel, s.H, s.Dv)), dtype=torch.uint8, device=dev)
    ws_p = sd.alloc_workspace(B, s.G, 0, s.k, s.H, s.Dv)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    clean = torch.zeros(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def flush_l2():
        flush.zero_()
        clean.max()

    def csr():
        sd.sd_sparse_attn_csr(q, kp, vp, bt, sl, flat_t, offs_t, bs, max_sel, s.scale, s.Dv, out=out, workspace=ws_c)

    def padded():
        sd.sd_sparse_attn(q, kp, vp, bt, sl, idx, s.scale, s.Dv, out=out, workspace=ws_p)

    def timed(fn):
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            fn()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=side):
            fn()
        for _ in range(args.warmup):
            flush_l2()
            g.replay()
        torch.cuda.synchronize()
        stream = torch.cuda.current_stream()
        tot = 0.0
        for _ in range(args.steps):
            flush_l2()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            g.replay()
            b.record(stream)
            b.synchronize()
            tot += a.elapsed_time(b)
        del g
        return max_over_ranks(tot / args.steps, world)

    ms_csr = timed(csr)
    ms_pad = timed(padded)
    sel_tokens = int(sum(min(len(f) * bs, int(wl.seqlens[r // s.G]), max_sel) for r, f in enumerate(flat)))
    row_bytes = s.Dk * 2 if s.v_in_k else (s.Dk + s.Dv) * 2
    nbytes = sel_tokens * row_bytes
    peak, peak_kind = _peaks()
    achieved = nbytes / (ms_csr * 1e-3) / 1e9
    line = {
        "metric": "attention-only decode queries/s, selection as CSR offsets / block-sized indices, 1 B200",
        "value": world * B / (ms_csr * 1e-3), "unit": "queries/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "block_size": bs, "selected_tokens": sel_tokens,
        "ms_per_step": ms_csr, "ms_per_step_padded_topk_selection": ms_pad,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": _config(s),
        "l2": "flushed before every step (256 MiB write, then 256 MiB read; outside the timed events)",
        "roofline": {"kernel": "csr expansion + attn + combine", "bound": "hbm", "achieved": achieved, "peak": peak,
                     "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / peak, "traffic": None,
                     "algorithmic_bytes_per_launch": nbytes, "ms_per_launch": ms_csr},
    }
    if rank == 0:
        print(json.dumps(line), flush=True)


def bench_hint(args, rank, world, local):
    """The decode step with the previous selection as the top-k hint, against
    the same step without it. The hint is the selection of a slightly
    different indexer query (10% of qi entries moved by up to 3), as between
    consecutive decode steps; the exact hint (the selection itself) is timed
    too. Each variant is a CUDA graph with stage events, so the top-k time is
    read directly."""
    import torch
    import top_sparse_decode_paged_b200 as sd
    from top_sparse_decode_paged_b200.api import StageTimer

    torch.cuda.set_device(local)
    wl = W.make(rank_spec(args.config, rank))
    s = wl.spec
    dev = "cuda"
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)  # noqa: E731
    rng = np.random.default_rng(1234)
    qi_p = wl.qi.astype(np.int16)
    m = rng.random(qi_p.shape) < 0.1
    qi_p[m] += rng.integers(-3, 4, size=int(m.sum())).astype(np.int16)
    qi_p = np.clip(qi_p, -64, 64).astype(np.int8)
    qi, qip, w, ki = t(wl.qi), t(qi_p), t(wl.w), t(wl.ki_pages)
    bt, sl = t(wl.block_table), t(wl.seqlens)
    q = t(wl.q.view(np.int16)).view(torch.bfloat16)
    kp = t(wl.k_pages.view(np.int16)).view(torch.bfloat16)
    vp = None if wl.v_pages is None else t(wl.v_pages.view(np.int16)).view(torch.bfloat16)
    B = wl.seqlens.shape[0]
    Lmax = wl.max_seqlen
    exact = sd.sd_indexer_topk(qi, w, ki, bt, sl, s.k, Lmax)
    perturbed = sd.sd_indexer_topk(qip, w, ki, bt, sl, s.k, Lmax)
    torch.cuda.synchronize()
    same = float((exact == perturbed).float().mean().item())
    idx = torch.empty_like(exact)
    out = torch.empty((B, s.H, s.Dv), dtype=torch.bfloat16, device=dev)
    ws = sd.alloc_workspace(B, s.G, Lmax, s.k, s.H, s.Dv)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    clean = torch.zeros(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def run(hint):
        if hint is None:
            sd.sd_decode_step(qi, w, ki, q, kp, vp, bt, sl, s.k, Lmax, s.scale, s.Dv, indices=idx, out=out,
                              workspace=ws)
        else:
            sd.sd_decode_step_hinted(qi, w, ki, q, kp, vp, bt, sl, s.k, Lmax, s.scale, s.Dv, hint, indices=idx,
                                     out=out, workspace=ws)

    res = {}
    for name, hint in (("none", None), ("perturbed", perturbed), ("exact", exact)):
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            run(hint)
        torch.cuda.synchronize()
        timer = StageTimer()
        g = torch.cuda.CUDAGraph()
        timer.arm()
        with torch.cuda.graph(g, stream=side):
            run(hint)
        StageTimer.disarm()
        ev = timer._pairs[0]
        for _ in range(args.warmup):
            flush.zero_()
            clean.max()
            g.replay()
        torch.cuda.synchronize()
        tot = dict.fromkeys(StageTimer.STAGES, 0.0)
        for _ in range(args.steps):
            flush.zero_()
            clean.max()
            g.replay()
            torch.cuda.synchronize()
            for j, nm in enumerate(StageTimer.STAGES):
                tot[nm] += ev[2 * j].elapsed_time(ev[2 * j + 1])
        res[name] = {k_: v / args.steps for k_, v in tot.items()}
        del g
        assert torch.equal(idx, exact), "hinted selection differs"
    line = {
        "metric": "top-k stage time of the decode step with and without the previous-selection hint, 1 B200",
        "value": res["perturbed"]["topk"], "unit": "ms", "higher_is_better": False, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "hint_overlap_with_selection": same,
        "stage_ms": res, "data": "synthetic",
        "config": _config(s),
        "l2": "flushed before every step (256 MiB write, then 256 MiB read; outside the timed events)",
    }
    if rank == 0:
        print(json.dumps(line), flush=True)


def bench_tri(args, rank, world, local):
    """TriAttention-style eviction of one layer (sd_tri_compact): score the
    evictable region with calibrated queries, select the budget, compact K and
    V in place. The pools are restored from pristine copies and L2 is flushed
    before every step, outside the timed events; the call is replayed from a
    CUDA graph."""
    import torch
    import top_sparse_decode_paged_b200 as sd

    torch.cuda.set_device(local)
    base = W.tri_spec(args.tri)
    s = W.tri_spec(args.tri, seed=base.seed + 1000 * rank) if rank else base
    n_layers = max(args.tri_layers, 1)
    wls = W.make_tri_layers(s, n_layers)
    w = wls[0]
    mode = {"union": sd.TRI_UNION, "per_head": sd.TRI_PER_HEAD,
            "per_layer_per_head": sd.TRI_PER_LAYER_PER_HEAD}[args.tri_mode]
    dev = "cuda"
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)  # noqa: E731
    bf = lambda a: t(a.view(np.int16)).view(torch.bfloat16)  # noqa: E731
    kp0 = [bf(x.k_pages) for x in wls]
    vp0 = [bf(x.v_pages) for x in wls]
    kp, vp = [x.clone() for x in kp0], [x.clone() for x in vp0]
    q_cals = [bf(x.q_cal) for x in wls]
    bt, sl = t(w.block_table), t(w.seqlens)
    B = int(w.seqlens.shape[0])
    lib = sd.load_library()
    ws = torch.empty(int(lib.sd_tri_layers_workspace_size(n_layers, B, s.G, s.H, s.D, w.max_seqlen, s.n_sink,
                                                            s.n_recent, s.budget, mode, 1)),
                     dtype=torch.uint8, device=dev)
    nl = torch.empty((B,), dtype=torch.int32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    clean = torch.zeros(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def prepare():
        for a, b in zip(kp + vp, kp0 + vp0):
            a.copy_(b)
        flush.zero_()
        clean.max()

    def call():
        if n_layers == 1:
            sd.sd_tri_compact(q_cals[0], kp[0], vp[0], bt, sl, w.max_seqlen, s.n_sink, s.n_recent, s.budget, mode,
                              new_seqlens=nl, workspace=ws)
        else:
            sd.sd_tri_compact_layers(q_cals, kp, vp, bt, sl, w.max_seqlen, s.n_sink, s.n_recent, s.budget, mode,
                                     new_seqlens=nl, workspace=ws)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        call()
    torch.cuda.synchronize()
    launches = sd.last_launch_count()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        call()
    for _ in range(args.warmup):
        prepare()
        g.replay()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    tot = 0.0
    with ClockSampler(local) as clk:
        for _ in range(args.steps):
            prepare()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            g.replay()
            b.record(stream)
            b.synchronize()
            tot += a.elapsed_time(b)
    del g
    ms = max_over_ranks(tot / args.steps, world)
    nbytes = n_layers * W.tri_algorithmic_bytes(s, w.seqlens, mode)
    peak, peak_kind = _peaks()
    achieved = nbytes / (ms * 1e-3) / 1e9
    line = {
        "metric": "KV-cache eviction (score, select, compact every layer) requests/s, 1 B200",
        "value": world * B / (ms * 1e-3), "unit": "requests/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32 scores, bf16 rows", "data": "synthetic",
        "config": {"workload": s.name, "B": B, "H": s.H, "kv_heads": s.G, "D": s.D, "page_size": s.page_size,
                   "n_sink": s.n_sink, "n_recent": s.n_recent, "budget": s.budget,
                   "mode": args.tri_mode, "layers": n_layers, "max_seqlen": w.max_seqlen,
                   "l2": "pools restored, then flushed (256 MiB write, 256 MiB read) before every step, "
                         "outside the timed events"},
        "gpu_launches": launches,
        "clocks": clk.summary(),
        "roofline": {"kernel": "score + reduce + top-k + gather + scatter", "bound": "hbm", "achieved": achieved,
                     "peak": peak, "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": None, "algorithmic_bytes_per_launch": nbytes, "ms_per_launch": ms},
    }
    if rank == 0 and not args.no_cpu_baseline:
        sys.path.insert(0, ROOT)
        from oracle import tri_oracle as T
        # the host pools are not used again: the oracle compacts them in place
        t0 = time.perf_counter()
        n = 0
        while n < B and (n == 0 or time.perf_counter() - t0 < 15.0):
            if n_layers == 1:
                T.tri_evict(w.q_cal, w.k_pages, w.v_pages, w.block_table[n:n + 1], w.seqlens[n:n + 1], s.n_sink,
                            s.n_recent, s.budget, mode, inplace=True)
            else:
                T.tri_evict_layers([x.q_cal for x in wls], [x.k_pages for x in wls], [x.v_pages for x in wls],
                                   w.block_table[n:n + 1], w.seqlens[n:n + 1], s.n_sink, s.n_recent, s.budget, mode)
            n += 1
        el = time.perf_counter() - t0
        line["cpu_baseline"] = {"value": n / el, "unit": "requests/s", "cores": 1, "kind": "oracle",
                                "sample": f"{n} of the {B} requests, one at a time"}
    if rank == 0:
        print(json.dumps(line), flush=True)


def _spawned_rank(rank: int, world: int, port: int, argv):
    """One rank started by _launch_ranks (torchrun's environment, set by hand)."""
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    sys.argv = [sys.argv[0]] + list(argv)
    main()


def _launch_ranks(n: int, argv) -> int:
    """`--gpus N` without torchrun: starts N ranks (spawned processes, one per
    GPU) with the same arguments and returns the first non-zero exit code."""
    import multiprocessing as mp
    import socket
    with socket.socket() as so:
        so.bind(("127.0.0.1", 0))
        port = so.getsockname()[1]
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_spawned_rank, args=(r, n, port, argv)) for r in range(n)]
    for p in procs:
        p.start()
    rc = 0
    for p in procs:
        p.join()
        rc = rc or (p.exitcode or 0)
    return rc


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", default=DEFAULT_CONFIG, choices=list(W.SPECS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="time eager calls instead of a CUDA graph replay")
    ap.add_argument("--hint", action="store_true",
                    help="time the decode step with the previous selection as the top-k hint instead")
    ap.add_argument("--csr-block", type=int, default=0,
                    help="time attention with the selection as CSR offsets, blocks of this many tokens (1: tokens)")
    ap.add_argument("--layers", type=int, default=0,
                    help="time attention-only decode over this many layers sharing one selection instead")
    ap.add_argument("--tri", default="", choices=[""] + list(W.TRI_SPECS),
                    help="time one layer's KV-cache eviction (score, select, compact) on this workload instead")
    ap.add_argument("--tri-mode", default="union", choices=["union", "per_head", "per_layer_per_head"],
                    help="with --tri: one selection per request, per KV head, or per (layer, KV head)")
    ap.add_argument("--tri-layers", type=int, default=1, help="with --tri: layers sharing the block table")
    ap.add_argument("--batch", type=int, default=0,
                    help="requests per rank instead of the workload's (a reduced batch for profiling)")
    args = ap.parse_args()
    global BATCH_OVERRIDE
    BATCH_OVERRIDE = args.batch if args.batch > 0 else None
    args.warmup = max(args.warmup, 3)
    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        sys.exit(_launch_ranks(args.gpus, sys.argv[1:]))
    rank, world, local = _dist_env()
    if world != args.gpus:
        sys.exit(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={world}")
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        if args.impl == "ours":
            torch.cuda.set_device(local)
        dist.init_process_group("nccl" if args.impl == "ours" else "gloo",
                                timeout=datetime.timedelta(seconds=300))
    try:
        if args.impl == "reference":
            bench_reference(args, rank, world)
        elif args.tri:
            bench_tri(args, rank, world, local)
        elif args.layers > 0:
            bench_layers(args, rank, world, local)
        elif args.csr_block > 0:
            bench_csr(args, rank, world, local)
        elif args.hint:
            bench_hint(args, rank, world, local)
        else:
            bench_ours(args, rank, world, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
