"""The N>1 path of bench.py on CPU: two gloo ranks, each timing its own
replica; the job time is the slowest rank's and the value counts the tokens
of both ranks."""
import os
import socket

import pytest
import torch.multiprocessing as mp

from lora_fine_tuning_mlp_b200 import replicas


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), LOCAL_RANK=str(rank),
                      WORLD_SIZE=str(world))
    try:
        r, lr, w = replicas.world()
        replicas.init("gloo", timeout_s=60)
        replicas.barrier()
        my_ms = 100.0 + 50.0 * r          # rank 1 is the slow one
        ms_max = replicas.max_over_ranks(my_ms)
        value = replicas.job_throughput(4096, 10, ms_max, w)
        replicas.barrier()
        q.put((r, lr, w, ms_max, value))
    finally:
        import torch.distributed as dist
        if dist.is_initialized():
            dist.destroy_process_group()


def test_two_gloo_ranks_time_as_the_slowest_and_count_both():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(i, 2, port, q)) for i in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=5) for _ in range(2))
    for r, lr, w, ms_max, value in res:
        assert w == 2 and lr == r
        assert ms_max == 150.0
        assert value == pytest.approx(2 * 4096 * 10 / 0.150)


def test_single_process_needs_no_process_group():
    assert replicas.max_over_ranks(12.5) == 12.5
    assert replicas.job_throughput(100, 2, 1000.0, 1) == pytest.approx(200.0)
