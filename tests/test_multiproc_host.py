"""The N>1 path of bench.py on CPU: world_size-2 gloo ranks (127.0.0.1).

The layer does not shard, so N GPUs run N independent replicas; the only
cross-rank step is the timing aggregation: a barrier, then the max of the
per-rank device times, and whole-job throughput = N x steps x flops / max.
"""

import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import datetime
    import torch.distributed as tdist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    tdist.init_process_group("gloo", rank=rank, world_size=world,
                             timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        per_rank_ms = [12.5, 20.0][rank]
        tdist.barrier()
        m = bench.max_over_ranks(per_rank_ms, "cpu")
        v = bench.whole_job_tflops(world, 10, 1e12, m)
        q.put((rank, m, v))
    finally:
        tdist.destroy_process_group()


def test_two_rank_timing_aggregation():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    out = sorted(q.get(timeout=10) for _ in range(2))
    for rank, m, v in out:
        assert m == 20.0                      # both ranks see the slowest rank's time
        assert v == pytest.approx(2 * 10 * 1e12 / 0.020 / 1e12)


def test_single_process_is_identity():
    import bench
    assert bench.max_over_ranks(3.5, "cpu") == 3.5
    assert bench.whole_job_tflops(1, 4, 2e12, 8.0) == pytest.approx(4 * 2e12 / 0.008 / 1e12)
