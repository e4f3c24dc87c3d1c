"""The N > 1 path of bench.py on CPU: two gloo ranks.  Rows are independent
problems, so ranks shard the rows of one layer with no data-path collective;
the only collective is the max-over-ranks reduction of the timed region."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as tmp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    import bench
    import torch.distributed as dist
    w, r, _ = bench.dist_init(world, backend="gloo")
    try:
        p = bench.workload("tiny", rank=r)
        local_ms = 10.0 * (r + 1)           # rank 1 is the slow one
        value, ms = bench.job_throughput(local_ms, 2, p.m_out, p.n, w)
        q.put((r, w, value, ms, p.W[0, :4].tolist(), p.X[0, :4].tolist()))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_weak_scaling_and_max_time():
    ctx = tmp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for pr in procs:
        pr.start()
    res = sorted(q.get(timeout=120) for _ in range(2))
    for pr in procs:
        pr.join(timeout=60)
        assert pr.exitcode == 0
    (r0, w0, v0, ms0, w0row, x0), (r1, w1, v1, ms1, w1row, x1) = res
    assert w0 == w1 == 2
    # both ranks report the job value from the slowest rank's time
    assert ms0 == ms1 == pytest.approx(20.0 / 2)
    assert v0 == v1 == pytest.approx(2 * 16 * 64 / (10.0 / 1e3))
    # same layer (same calibration X), different rows per rank
    assert np.allclose(x0, x1)
    assert not np.allclose(w0row, w1row)
