"""The N>1 paths on CPU: world_size-2 gloo ranks (127.0.0.1).

- bench.py runs N independent replicas of the layer; the only cross-rank
  step is the timing aggregation: a barrier, then the max of the per-rank
  device times, and whole-job throughput = N x steps x flops / max.
- A layer split by rows (tokens) across ranks stays the one-GPU layer when
  the ranks exchange one number, the activation's amax, by an all-reduce
  (MAX) before the NVFP4 quantisation (mxq_amax on the local rows, the
  all-reduce, then mxq_quantize_nvfp4 with that external amax and the GEMM).
  The test runs that protocol with the oracle on each rank and checks the
  gathered codes, scales and outputs against one process; with each rank's
  own amax instead, the codes differ.
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


M_SPLIT = (96, 128, 40)  # rows, K, N of the layer split across the two ranks


def _msplit_layer():
    import numpy as np
    import workloads
    M, K, N = M_SPLIT
    c = workloads.random_case(M, K, N, "nvfp4", seed=21)
    A = c.A.float()
    A[M // 2:] *= 4.0  # the second rank's rows hold the tensor's maximum
    return A.to(c.A.dtype), c.W, c.bias


def _msplit_worker(rank, world, port, q, exchange):
    import datetime
    import numpy as np
    import torch
    import torch.distributed as tdist
    from oracle import gemm as G
    from oracle import quant as Q
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    tdist.init_process_group("gloo", rank=rank, world_size=world,
                             timeout=datetime.timedelta(seconds=60))
    try:
        A, W, bias = _msplit_layer()
        M = A.shape[0]
        local = A[rank * M // world:(rank + 1) * M // world]
        amax = torch.tensor([float(Q.amax(local))], dtype=torch.float32)
        if exchange:
            tdist.all_reduce(amax, op=tdist.ReduceOp.MAX)
        qa = Q.quantize_nvfp4(local, global_amax=np.float32(amax.item()))
        qw = Q.quantize_nvfp4(W)
        Y, _ = G.linear_ref(Q.dequant_nvfp4(qa["codes"], qa["sf"], qa["g"]),
                            Q.dequant_nvfp4(qw["codes"], qw["sf"], qw["g"]), bias)
        q.put((rank, qa["codes"], qa["sf"], float(qa["g"]), Y))
    finally:
        tdist.destroy_process_group()


def _run_msplit(exchange):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_msplit_worker, args=(r, 2, port, q, exchange)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted((q.get(timeout=120) for _ in range(2)), key=lambda t: t[0])
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    return out


def test_row_split_with_amax_all_reduce_equals_one_process():
    import numpy as np
    from oracle import gemm as G
    from oracle import quant as Q
    A, W, bias = _msplit_layer()
    one = Q.quantize_nvfp4(A)
    qw = Q.quantize_nvfp4(W)
    Y_one, _ = G.linear_ref(Q.dequant_nvfp4(one["codes"], one["sf"], one["g"]),
                            Q.dequant_nvfp4(qw["codes"], qw["sf"], qw["g"]), bias)
    out = _run_msplit(exchange=True)
    assert all(g == float(one["g"]) for _, _, _, g, _ in out)
    assert np.array_equal(np.concatenate([c for _, c, _, _, _ in out]), one["codes"])
    assert np.array_equal(np.concatenate([s for _, _, s, _, _ in out]), one["sf"])
    assert np.array_equal(np.concatenate([y for _, _, _, _, y in out]), Y_one)


def test_row_split_without_the_exchange_differs():
    import numpy as np
    from oracle import quant as Q
    A, _, _ = _msplit_layer()
    one = Q.quantize_nvfp4(A)
    out = _run_msplit(exchange=False)
    # the first rank's own amax is 4x smaller: another g, so other scales
    assert out[0][3] != float(one["g"]) and out[1][3] == float(one["g"])
    M = A.shape[0]
    assert not np.array_equal(out[0][2], one["sf"][: M // 2])
