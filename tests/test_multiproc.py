"""Multi-process host logic of bench.py on CPU: two gloo ranks.

The decode path shards over independent batch rows with no data exchange;
the only cross-rank operations are the barrier around the timed region and
the MAX reduction of the per-rank times.  These run here on CPU, with
world size 2, over 127.0.0.1.
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

    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        r, w, lr = bench.dist_env()
        bench.barrier(w)
        t = bench.reduce_max(1.5 + rank, w)  # rank 1 is the slow one
        # the reference leg does no work off rank 0
        rc = bench.run_reference(type("A", (), {"config": 0, "steps": 1, "warmup": 3})()) \
            if rank == 1 else 0
        q.put((rank, r, w, lr, t, rc))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(180)
def test_two_gloo_ranks_barrier_and_max_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(150)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(2))
    for rank, r, w, lr, t, rc in got:
        assert r == rank and w == 2 and lr == rank
        assert t == 2.5  # max over ranks
        assert rc == 0


def test_single_process_helpers():
    import bench
    assert bench.reduce_max(3.25, 1) == 3.25
    b, f = bench.algorithmic_work(128, 2048)
    assert b == 347_078_656 and f == 77_309_411_328  # config-3 figures of the measurement plan
    cb, cf = bench.core_kernel_work(128, 2048)
    assert cb == 128 * 2048 * 1156 and cf == 128 * 2048 * 278_528
    peaks = bench.load_peaks()
    assert peaks["hbm_gbs"] > 1000 and peaks["bf16_tflops"] > 100
