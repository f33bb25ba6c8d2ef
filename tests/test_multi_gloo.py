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


# ---------------------------------------------------------------- p2p ring across processes

def _ring_worker(rank, world, port, order, causal, results):
    """One rank of a real ring over gloo: the block exchange and the schedule
    of ring_attn_fwd_p2p, with the oracle's step partial and merge standing in
    for the CUDA calls (this runs on CPU)."""
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import numpy as np
    import torch
    import oracle
    from ring_ulysses_sequence_b200 import multi, ring
    multi.init("gloo", timeout_s=60)
    B, H, Hkv, D = 1, 4, 2, 8
    S = 16 * world
    L = S // world
    rng = np.random.default_rng(5)
    q, k, v = (rng.standard_normal(s) for s in [(B, H, S, D), (B, Hkv, S, D), (B, Hkv, S, D)])
    pos = oracle.rank_major_positions(S, world, order)
    mine = pos[rank * L:(rank + 1) * L]
    ql, kl, vl = (torch.from_numpy(np.ascontiguousarray(x[:, :, mine])) for x in (q, k, v))
    seen = []

    def step(q_, k_, v_, P, r, owner, causal_, order_, scale):
        seen.append(owner)
        # the block held must be the owner's: compare with the global keys
        assert np.array_equal(k_.numpy(), k[:, :, pos[owner * L:(owner + 1) * L]])
        o, l = oracle.step_partial(q_, k_, v_, S, P, order_, r, owner, causal_, scale)
        return torch.from_numpy(o), torch.from_numpy(l)

    def merge(o_acc, l_acc, o_p, l_p):
        n = o_acc.numel() // D
        o, l = oracle.lse_merge(o_acc.reshape(n, D), l_acc.reshape(n), o_p.reshape(n, D),
                                l_p.reshape(n))
        o_acc.copy_(torch.from_numpy(o).reshape(o_acc.shape))
        l_acc.copy_(torch.from_numpy(l).reshape(l_acc.shape))

    o, lse = ring.ring_attn_fwd_p2p(ql, kl, vl, causal, order, step=step, merge=merge)
    o_ref, l_ref = oracle.attn_fwd(q, k, v, causal, rows=mine)
    results[rank] = (seen, float(np.abs(o.numpy() - o_ref).max()),
                     float(np.abs(lse.numpy() - l_ref).max()))
    multi.shutdown()


@pytest.mark.parametrize("world,order,causal", [(2, 1, True), (3, 0, True), (3, 1, False),
                                                (4, 1, True)])
def test_p2p_ring_over_gloo_matches_oracle(world, order, causal):
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=_ring_worker, args=(r, world, port, order, causal, results))
                 for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(180)
            assert p.exitcode == 0
        for r in range(world):
            seen, err_o, err_l = results[r]
            assert seen == [(r - t) % world for t in range(world)]   # owner (r - t) mod P
            assert err_o < 1e-5 and err_l < 1e-5, (r, err_o, err_l)


def test_ring_schedule_matches_the_oracle_owner():
    import oracle
    from ring_ulysses_sequence_b200 import ring
    for P in (1, 2, 3, 8):
        for i in range(P):
            assert ring.ring_schedule(P, i) == [(t, oracle.ring_owner(P, i, t)) for t in range(P)]


def test_p2p_ring_single_process_is_one_step():
    # without a process group the ring has one rank and one step
    import numpy as np
    import torch
    import oracle
    from ring_ulysses_sequence_b200 import ring
    q, k, v = (torch.from_numpy(np.random.default_rng(s).standard_normal((1, 2, 16, 4)))
               for s in (1, 2, 3))
    calls = []

    def step(q_, k_, v_, P, r, owner, causal, order, scale):
        calls.append((P, r, owner))
        o, l = oracle.step_partial(q_, k_, v_, 16, P, order, r, owner, causal, scale)
        return torch.from_numpy(o), torch.from_numpy(l)

    def merge(o_acc, l_acc, o_p, l_p):
        o_acc.copy_(o_p)
        l_acc.copy_(l_p)

    o, l = ring.ring_attn_fwd_p2p(q, k, v, True, 1, step=step, merge=merge)
    assert calls == [(1, 0, 0)]
    o_ref, l_ref = oracle.attn_fwd(q, k, v, True)
    assert np.abs(o.numpy() - o_ref).max() < 1e-6
