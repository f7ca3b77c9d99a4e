"""Row-sharded matrices on the CPU: the row split, and two gloo ranks
(127.0.0.1) whose shards' results are gathered into the whole y.  The local
products stand in for the GPU GEMV with the oracle, so what is checked here is
the split and the exchange; the GPU test runs the library on one shard."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from lossless_bf16_weight_nwc_b200 import sharded


@pytest.mark.parametrize("rows,world", [(1, 1), (8, 2), (9, 2), (77, 3), (4096, 8), (16, 5),
                                        (100003, 7)])
def test_row_ranges(rows, world):
    r = sharded.row_ranges(rows, world)
    assert len(r) == world and r[0][0] == 0 and r[-1][1] == rows
    assert all(a[1] == b[0] for a, b in zip(r, r[1:]))                     # contiguous
    assert all(s % 8 == 0 for s, _ in r)                                    # whole tile blocks
    sizes = [e - s for s, e in r]
    full = [n for n, (s, e) in zip(sizes, r) if e != rows]
    assert not full or max(full) - min(full) <= 8                           # balanced
    assert sizes == sorted(sizes, reverse=True) or rows % 8                 # extra blocks first
    with pytest.raises(ValueError):
        sharded.row_ranges(0, 2)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime

    import torch
    import torch.distributed as dist

    import oracle
    from lossless_bf16_weight_nwc_b200 import synth
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        w = synth.matrix(synth.MatrixSpec("w", 77, 300, "normal", 0.02, 0), 5)
        x = synth.activations(5, 3, 300)

        class Shard:
            def __init__(self, part, device=None):
                self.part = part

            def close(self):
                pass

        m = sharded.ShardedMatrix.compress(w, compress=lambda part, device=None: Shard(part),
                                           device="cpu")
        s, e = m.ranges[rank]
        assert m.local.part.shape == (e - s, 300)
        xt = torch.zeros((3, 300))
        y = m.gemv(xt, local_gemv=lambda _: torch.from_numpy(oracle.gemv(m.local.part, x)).float())
        full = oracle.gemv(w, x).astype(np.float32)
        # One row of x over equal shards (80 rows: 5 tile blocks each): the
        # gathered buffer is y itself.
        w1 = synth.matrix(synth.MatrixSpec("w1", 80, 300, "normal", 0.02, 0), 6)
        x1 = synth.activations(6, 1, 300)
        m1 = sharded.ShardedMatrix.compress(w1, compress=lambda part, device=None: Shard(part),
                                            device="cpu")
        y1 = m1.gemv(torch.zeros((1, 300)),
                     local_gemv=lambda _: torch.from_numpy(oracle.gemv(m1.local.part, x1)).float())
        full1 = oracle.gemv(w1, x1).astype(np.float32)
        out.put((rank, bool(np.array_equal(y.numpy(), full)), tuple(y.shape),
                 bool(np.array_equal(y1.numpy(), full1)), tuple(y1.shape)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_gather_the_whole_y():
    world = 2
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    results = sorted(out.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert results == [(0, True, (3, 77), True, (1, 80)), (1, True, (3, 77), True, (1, 80))]


def test_single_process_needs_no_collective():
    import torch
    m = sharded.ShardedMatrix(object(), [(0, 10)], 0)
    y = m.gemv(torch.zeros((2, 4)), local_gemv=lambda x: torch.ones((2, 10)))
    assert y.shape == (2, 10) and bool((y == 1).all())
