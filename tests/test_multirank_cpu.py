"""The N > 1 bench path on CPU: two gloo ranks draw different batches of the
same shape (weak scaling) and agree on the slowest rank's time (MAX)."""
import os
import socket

import numpy as np
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    import datetime
    import sys
    import torch.distributed as dist
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    from top_sparse_decode_paged_b200 import workloads as W
    s = bench.rank_spec("tiny", rank)
    wl = W.make(s)
    t = bench.max_over_ranks(1.0 + rank, world)
    np.savez(os.path.join(out_dir, f"r{rank}.npz"), qi=wl.qi, seed=s.seed, t=t, shape=np.array(wl.qi.shape))
    dist.destroy_process_group()


def test_two_gloo_ranks_shard_and_take_max(tmp_path):
    port = _free_port()
    mp.start_processes(_worker, args=(2, port, str(tmp_path)), nprocs=2, join=True, start_method="spawn")
    r0 = np.load(tmp_path / "r0.npz")
    r1 = np.load(tmp_path / "r1.npz")
    assert int(r0["seed"]) != int(r1["seed"])              # each rank its own batch
    assert (r0["shape"] == r1["shape"]).all()              # of the same shape
    assert not np.array_equal(r0["qi"], r1["qi"])
    assert float(r0["t"]) == float(r1["t"]) == 2.0         # MAX over ranks


def test_gpus_flag_starts_that_many_ranks():
    """`bench.py --gpus 2` without torchrun starts two ranks itself: the
    reference arm (CPU, gloo) prints one line from rank 0 with n_gpus 2, and
    the other rank exits 0 without output. A --gpus that contradicts
    WORLD_SIZE is refused."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK")}
    r = subprocess.run([sys.executable, "bench.py", "--gpus", "2", "--impl", "reference", "--config", "tiny",
                        "--steps", "1", "--warmup", "3"], cwd=root, env=env, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["ms_per_step"] * line["steps"] < 600e3
    env2 = dict(env, WORLD_SIZE="1", RANK="0", LOCAL_RANK="0")
    r2 = subprocess.run([sys.executable, "bench.py", "--gpus", "2", "--impl", "reference", "--config", "tiny",
                         "--steps", "1", "--warmup", "3"], cwd=root, env=env2, capture_output=True, text=True,
                        timeout=600)
    assert r2.returncode != 0 and "WORLD_SIZE" in r2.stderr
