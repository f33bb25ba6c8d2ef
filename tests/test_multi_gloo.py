"""Multi-rank host logic on CPU: two gloo ranks, as the benchmark runs them
(one replica per rank, barrier, max-over-ranks timing, whole-job value)."""
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


def _worker(rank, world, port, results):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    from ring_ulysses_sequence_b200 import multi
    r, w = multi.init("gloo", timeout_s=60)
    assert (r, w) == (rank, world)
    multi.barrier()
    ms = 10.0 + 5.0 * rank                   # per-rank step time
    slowest = multi.max_over_ranks(ms)
    units = multi.sum_over_ranks(1.0)        # one replica per rank
    results[rank] = (slowest, units)
    multi.shutdown()


def test_two_gloo_ranks_aggregate_like_the_benchmark():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=_worker, args=(r, 2, port, results)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        assert dict(results) == {0: (15.0, 2.0), 1: (15.0, 2.0)}


def test_single_process_needs_no_group():
    from ring_ulysses_sequence_b200 import multi
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        os.environ.pop(k, None)
    assert multi.env_ranks() == (0, 1, 0)
    assert multi.init("gloo") == (0, 1)
    assert multi.max_over_ranks(3.5) == 3.5
