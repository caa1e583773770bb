"""The multi-rank host path of bench.py on CPU: two gloo ranks, each timing its
own replica; the reported time is the max over ranks and the value counts the
work of every rank (weak scaling).  The decode path itself has no exchange."""
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
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    import bench
    ws, r, local = bench.dist_env()
    local_ms = 100.0 + 50.0 * rank          # rank 1 is the slow one
    mx = bench.max_over_ranks(local_ms)
    val = bench.whole_job_value(ws, kv_bytes_per_call=1_000_000, steps=10, max_total_ms=mx)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, ws, r, mx, val))


@pytest.mark.timeout(120)
def test_two_rank_max_and_weak_scaling_value():
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
    for rank, ws, r, mx, val in res:
        assert ws == 2 and r == rank
        assert mx == 150.0                   # max over ranks, not the local time
        # 2 ranks x 10 calls x 1 MB in 150 ms
        assert abs(val - 2 * 10 * 1e6 / 0.150 / 1e9) < 1e-12


def test_reference_arm_other_ranks_exit(monkeypatch):
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")

    class A:
        steps, warmup, config, gpus, json_out = 3, 3, "tiny", 2, None
    assert bench.run_reference(A()) == 0
