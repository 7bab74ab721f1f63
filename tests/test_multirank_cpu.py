"""The N > 1 plumbing of bench.py on CPU: world-size-2 gloo ranks.

Each rank runs its own batch (weak scaling, no collective on the data path);
the only collectives are the barrier around the timed region and the
reduction of the per-rank results: bytes and tokens summed, elapsed time
taken as the max over ranks.  Checked here with fake per-rank numbers.
"""

import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, results):
    import datetime

    import torch.distributed as dist

    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier()
        # rank r processed (r + 1) GB in (10 + r) ms
        rank_bytes = (rank + 1) * 1e9
        rank_ms = 10.0 + rank
        tot_bytes, max_ms, tot_tokens = bench.reduce_over_ranks(
            [rank_bytes, rank_ms, 1000 * (rank + 1)], ["sum", "max", "sum"])
        bench.barrier()
        results[rank] = (tot_bytes, max_ms, tot_tokens)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_aggregate_like_the_bench():
    world = 2
    port = _free_port()
    manager = mp.Manager()
    results = manager.dict()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, results)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    for p in procs:
        if p.is_alive():
            p.kill()
            pytest.fail("a gloo rank did not finish")
        assert p.exitcode == 0
    for r in range(world):
        tot_bytes, max_ms, tot_tokens = results[r]
        assert tot_bytes == 3e9            # 1 GB + 2 GB: bytes of all ranks
        assert max_ms == 11.0              # the slowest rank sets the time
        assert tot_tokens == 3000
    # whole-job throughput as the bench reports it: all ranks' bytes over the max time
    tot_bytes, max_ms, _ = results[0]
    assert abs(tot_bytes / (max_ms * 1e-3) / 1e9 - 3e9 / 11e-3 / 1e9) < 1e-9


def test_single_process_reduction_is_identity():
    import bench

    assert bench.reduce_over_ranks([5.0, 7.0], ["sum", "max"]) == [5.0, 7.0]
