"""The benchmark's multi-rank logic on the CPU: two gloo ranks (127.0.0.1).

bench.py --gpus N runs N independent replicas of the per-GPU work (the path
has no exchange step between GPUs), times on the device, and reports the
slowest rank; these tests check the barrier, the max over ranks and the
whole-job aggregate with the gloo backend instead of NCCL."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime

    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    bench.barrier(world)
    local_ms = 10.0 + 5.0 * rank                 # rank 1 is the slow one
    slowest = bench.max_over_ranks(local_ms, world, device="cpu")
    value = bench.replica_value(2 * 4096 * 4096, world, slowest)
    out.put((rank, slowest, value))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_two_gloo_ranks_report_the_slowest(world):
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    results = sorted(out.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    slowest = {r[1] for r in results}
    assert slowest == {15.0}                     # every rank sees the maximum
    expected = world * 2 * 4096 * 4096 / (15.0e-3) / 1e9
    assert all(abs(r[2] - expected) < 1e-9 * expected for r in results)


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert abs(bench.replica_value(1e9, 1, 1.0) - 1000.0) < 1e-9
