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
