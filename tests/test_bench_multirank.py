"""bench.py's multi-rank timing on CPU: two gloo ranks with different device
times; the whole-job value uses the slowest rank's time and every rank's
tokens (replicas, no data-path collective)."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    my_ms = 10.0 + 5.0 * rank                  # rank 1 is slower
    mx = bench.reduce_max_ms(my_ms)
    v = bench.whole_job_tokens_per_s(world, 100, 4096, mx)
    q.put((rank, mx, v))
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_max_reduction():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [15.0, 15.0]
    assert res[0][2] == pytest.approx(2 * 100 * 4096 / 0.015)


def test_single_rank_identity():
    import bench
    assert bench.reduce_max_ms(3.5) == 3.5
