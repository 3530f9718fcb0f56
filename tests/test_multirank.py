"""The multi-process (N > 1) logic of bench.py on CPU: two gloo ranks on 127.0.0.1.

Each rank runs its own batch with replicated weights (weak scaling, no collective on the data
path); the time is the max over ranks and the throughput counts every rank's tokens.  The
reference arm runs on rank 0 only."""
import os
import socket
import subprocess
import sys

import numpy as np
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    import datetime

    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import bench
    import synth

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms = 10.0 + 5.0 * rank  # rank 1 is slower
        mx = bench.max_over_ranks(ms, "cpu")
        wl = synth.WORKLOADS["tiny"]
        x = synth.gen_x(bench.synth_replace(wl, seed=bench.rank_seed(wl, rank)))
        w = synth.gen_expert(wl, "w1", 0)
        out[rank] = (mx, bench.aggregate_tokens_per_s(world, wl.T, 7, mx), int(x[0, :4].astype(np.int64).sum()),
                     int(w[0, :4].astype(np.int64).sum()))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world, port = 2, free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
    (m0, v0, x0, w0), (m1, v1, x1, w1) = out[0], out[1]
    assert m0 == m1 == 15.0                      # max over ranks, agreed by both
    assert v0 == v1 == 2 * 64 * 7 / 0.015        # all ranks' tokens over the slowest rank's time
    assert x0 != x1                              # each rank has its own batch
    assert w0 == w1                              # weights are replicated


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, RANK="1", LOCAL_RANK="1", WORLD_SIZE="2")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "0", "--workload", "tiny"], env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == ""
