"""Multi-rank host logic of the benchmark on CPU (gloo, world size 2): each rank gets an
independent problem of the same shape, device times are reduced with a max over ranks,
and the whole-job rate counts every rank's work over the slowest rank's time. The
operator itself has no collective: ranks never exchange data."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch.distributed as dist

    import bench
    from block_sparse_online_b200 import synth
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cfg = bench.rank_config(synth.CONFIGS["video480"], rank)
        ms = 10.0 + 5.0 * rank  # a per-rank device time
        t = bench.max_over_ranks(ms, world)
        rate = bench.whole_job_rate(world, cfg.dense_flops(), t)
        out.put((rank, cfg.seed, cfg.shape(), t, rate))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=90) for _ in procs)
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    (r0, s0, sh0, t0, v0), (r1, s1, sh1, t1, v1) = res
    assert s0 != s1 and sh0 == sh1          # independent problems of one shape
    assert t0 == t1 == 15.0                 # the slowest rank's time on every rank
    from block_sparse_online_b200 import synth
    flops = synth.CONFIGS["video480"].dense_flops()
    assert abs(v0 - 2 * flops / 15e-3 / 1e12) < 1e-6 and v0 == v1
