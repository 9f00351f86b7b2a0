"""The benchmark's N>1 path on the CPU: two gloo ranks, as torchrun would
start them. Each rank draws its own microbatch against the same weights (no
collective on the data path), the slowest rank's time is what counts, and
only rank 0 reports."""
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import bench
    from grouped_expert_ffn_top_b200 import workloads
    R = bench.Ranks("gloo", device=torch.device("cpu"))
    w = workloads.custom("mr", 64, 64, 4, 2, 64)
    params = workloads.make_params(w, seed=0)
    batch = workloads.make_batch(w, seed=R.batch_seed)
    R.barrier()
    t = R.max_over_ranks(10.0 * (rank + 1))
    out.put((rank, R.prints, t, float(params["Wg"].float().sum()), float(batch["x"].float().sum())))
    R.close()


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, p0, t0, w0, x0), (r1, p1, t1, w1, x1) = res
    assert (p0, p1) == (True, False)       # only rank 0 prints the JSON line
    assert t0 == t1 == 20.0                 # max over ranks
    assert w0 == w1                         # replicated weights
    assert x0 != x1                         # each rank has its own microbatch


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    env = {k: os.environ.pop(k) for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK") if k in os.environ}
    try:
        R = bench.Ranks("gloo", device=torch.device("cpu"))
        assert R.world == 1 and R.prints and R.max_over_ranks(3.5) == 3.5
        R.barrier()
        R.close()
    finally:
        os.environ.update(env)
