"""The multi-rank path of bench.py on CPU: two gloo ranks (one process each) reduce their
device times with MAX and report the whole job's throughput, as `bench.py --gpus 2`
does over NCCL.  No GPU."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        # rank r took (r + 1) * 100 ms for its 10 steps and 20 + r ms of scan time
        tot_ms, scan_ms = bench.max_over_ranks([(rank + 1) * 100.0, 20.0 + rank], world, "cpu")
        value = bench.job_gbs(1e9, world, 10, tot_ms)
        q.put((rank, tot_ms, scan_ms, value))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_rank_and_count_every_rank_bytes():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, tot_ms, scan_ms, value in res:
        assert tot_ms == 200.0 and scan_ms == 21.0          # MAX over the ranks
        assert value == pytest.approx(1e9 * 2 * 10 / 0.2 / 1e9)  # all ranks' bytes / slowest time
