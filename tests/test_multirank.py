"""The N > 1 plumbing of bench.py on CPU: two gloo ranks rendezvous on
127.0.0.1, take the barrier, agree on the max of their timings and compute the
whole-job rate from it (replicas: no data-path collective exists to test)."""
import os
import socket

import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    import bench
    import torch.distributed as dist
    w, r, local = bench.dist_setup("gloo")
    assert (w, r, local) == (world, rank, rank)
    bench.barrier(w, cuda=False)
    ms = [10.0, 12.5][rank]  # per-rank timed region of 5 steps
    m = bench.max_over_ranks(ms, w, device="cpu")
    out[rank] = (m, bench.job_throughput(w, 100.0, m, 5))
    bench.barrier(w, cuda=False)
    dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_max_time_and_job_rate():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=_rank, args=(r, 2, port, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        res = dict(out)
    assert res[0] == res[1]
    m, rate = res[0]
    assert m == 12.5
    # 2 ranks x 100 units per step, 5 steps in the slowest rank's 12.5 ms
    assert abs(rate - 2 * 100.0 / (12.5e-3 / 5)) < 1e-6
