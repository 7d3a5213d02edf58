"""The benchmark's multi-GPU host logic with two gloo ranks on the CPU: each rank is an
independent replica; the job's throughput is all ranks' tokens over the slowest rank's
time, and every rank takes the same collective steps."""
import os
import socket

import pytest


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    bench._init_dist(world)
    # rank r: 10 * (r + 1) ms for 16 * (r + 1) tokens
    value, ms_max, tokens = bench.combine_ranks(10.0 * (rank + 1), 16 * (rank + 1), world)
    bench._barrier(world)
    out[rank] = (value, ms_max, tokens)
    bench._PG.destroy_process_group()


def test_two_rank_aggregation_takes_max_time_and_total_tokens():
    import torch.multiprocessing as mp
    world = 2
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert set(res) == {0, 1}
    for rank in range(world):
        value, ms_max, tokens = res[rank]
        assert ms_max == pytest.approx(20.0)
        assert tokens == pytest.approx(48)
        assert value == pytest.approx(48 / 0.020)


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.combine_ranks(4.0, 8, 1) == (2000.0, 4.0, 8)
