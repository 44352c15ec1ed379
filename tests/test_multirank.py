"""The multi-GPU host logic of bench.py with two `gloo` ranks on CPU: every
GPU rank draws its own batch (distinct seeds, no data exchange), timings are
taken as the maximum over ranks, and the whole-job value sums the GPUs."""
import os
import socket
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    try:
        mine = 10.0 + 5.0 * rank                       # rank 1 is the slow one
        slowest = bench.max_over_ranks(mine)
        seeds = [bench.gpu_seed(r, rank) for r in range(bench.NRANKS)]
        q.put((rank, slowest, seeds))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    got.sort()
    assert [g[1] for g in got] == [15.0, 15.0]                  # max over ranks, on every rank
    s0, s1 = set(got[0][2]), set(got[1][2])
    assert len(s0) == len(s1) == 8 and not (s0 & s1)             # independent batches


def test_whole_job_value_and_single_process():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5) == 3.5                      # no process group
    # 2 GPUs x 1 GB per step x 10 steps in 5 ms = 4000 GB/s
    assert abs(bench.whole_job_gbs(2, 10 ** 9, 10, 5.0) - 4000.0) < 1e-9
