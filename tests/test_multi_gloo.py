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

    k_before, v_before = kl.clone(), vl.clone()
    o, lse = ring.ring_attn_fwd_p2p(ql, kl, vl, causal, order, step=step, merge=merge)
    # the caller's blocks are only sent, never received into
    unchanged = torch.equal(kl, k_before) and torch.equal(vl, v_before)
    o_ref, l_ref = oracle.attn_fwd(q, k, v, causal, rows=mine)
    results[rank] = (seen, float(np.abs(o.numpy() - o_ref).max()),
                     float(np.abs(lse.numpy() - l_ref).max()), unchanged)
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
            seen, err_o, err_l, unchanged = results[r]
            assert seen == [(r - t) % world for t in range(world)]   # owner (r - t) mod P
            assert err_o < 1e-5 and err_l < 1e-5, (r, err_o, err_l)
            assert unchanged, f"rank {r}: the caller's k/v were overwritten"


def _spawn(target, world, *args, timeout=180):
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=target, args=(r, world, port, *args, results))
                 for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout)
            assert p.exitcode == 0
        return dict(results)


def _oracle_fold(S, D):
    """fold() for ring_attn_fwd_p2p with the oracle's step partial and merge."""
    import numpy as np
    import torch
    import oracle

    def fold(q_, k_, v_, P, r, owner, causal_, order_, scale, o_acc, l_acc):
        o, l = oracle.step_partial(q_, k_, v_, S, P, order_, r, owner, causal_, scale)
        n = o_acc.numel() // D
        o2, l2 = oracle.lse_merge(o_acc.reshape(n, D), l_acc.reshape(n), o.reshape(n, D),
                                  l.reshape(n))
        o_acc.copy_(torch.from_numpy(o2).reshape(o_acc.shape))
        l_acc.copy_(torch.from_numpy(l2).reshape(l_acc.shape))
    return fold


def _oracle_bwd_step(S):
    import torch
    import oracle

    def bwd_step(q_, k_, v_, lse_, delta_, do_, dq, dk, dv, P, r, owner, causal_, order_, scale):
        a, b, c = oracle.step_bwd_partial(q_, k_, v_, do_, lse_, delta_, S, P, order_, r, owner,
                                          causal_, scale)
        dq += torch.from_numpy(a)
        dk += torch.from_numpy(b)
        dv += torch.from_numpy(c)
    return bwd_step


def _delta(o, do):
    return (o.double() * do.double()).sum(-1)


def _ring_fwd_bwd_worker(rank, world, port, order, causal, results):
    """Forward (fold) and reverse-ring backward of ring.py over gloo, with the
    oracle's arithmetic standing in for the CUDA calls."""
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import numpy as np
    import torch
    import oracle
    from ring_ulysses_sequence_b200 import multi, ring
    multi.init("gloo", timeout_s=60)
    B, H, Hkv, D = 1, 4, 2, 8
    S = 8 * world
    L = S // world
    rng = np.random.default_rng(7)
    q, k, v, do = (rng.standard_normal(sh) for sh in
                   [(B, H, S, D), (B, Hkv, S, D), (B, Hkv, S, D), (B, H, S, D)])
    pos = oracle.rank_major_positions(S, world, order)
    mine = pos[rank * L:(rank + 1) * L]
    ql, kl, vl, dol = (torch.from_numpy(np.ascontiguousarray(x[:, :, mine])) for x in (q, k, v, do))
    before = [t.clone() for t in (ql, kl, vl, dol)]
    o, lse = ring.ring_attn_fwd_p2p(ql, kl, vl, causal, order, fold=_oracle_fold(S, D))
    dq, dk, dv = ring.ring_attn_bwd_p2p(ql, kl, vl, o, lse, dol, causal, order,
                                        bwd_step=_oracle_bwd_step(S), delta=_delta)
    o_ref, l_ref = oracle.attn_fwd(q, k, v, causal, rows=mine)
    rdq, rdkv = oracle.attn_bwd(q, k, v, do, causal, qrows=mine, krows=mine)
    err = max(float(np.abs(o.numpy() - o_ref).max()), float(np.abs(lse.numpy() - l_ref).max()))
    gerr = 0.0
    for h in range(H):
        gerr = max(gerr, float(np.abs(dq[0, h].numpy() - rdq[(0, h)]).max()))
    for g in range(Hkv):
        gerr = max(gerr, float(np.abs(dk[0, g].numpy() - rdkv[(0, g)][0]).max()),
                   float(np.abs(dv[0, g].numpy() - rdkv[(0, g)][1]).max()))
    unchanged = all(torch.equal(a, b) for a, b in zip((ql, kl, vl, dol), before))
    results[rank] = (err, gerr, unchanged)
    multi.shutdown()


@pytest.mark.parametrize("world,order,causal", [(1, 1, True), (2, 1, True), (3, 0, True),
                                                (3, 1, False), (4, 1, True)])
def test_p2p_ring_forward_and_backward_over_gloo_match_oracle(world, order, causal):
    res = _spawn(_ring_fwd_bwd_worker, world, order, causal)
    for r in range(world):
        err, gerr, unchanged = res[r]
        # the running pair and the gradient sums are float32 by design
        assert err < 1e-5 and gerr < 1e-5, (r, err, gerr)
        assert unchanged, f"rank {r}: an input was modified"


# ---------------------------------------------------------------- Ulysses x ring (USP)

def _cpu_pack(tensors, U, direction):
    """Send buffer of the Ulysses exchange, written from the layout rm.h
    states: U chunks, in each the tensors one after another as [B, s, h/U, D]
    (sequence shards [B, s, h, D]; head shards [B, h/U, U*s, D])."""
    import torch
    parts = []
    for u in range(U):
        for x in tensors:
            if direction == "seq_to_head":
                hU = x.shape[2] // U
                parts.append(x[:, :, u * hU:(u + 1) * hU].reshape(-1))
            else:
                s = x.shape[2] // U
                parts.append(x[:, :, u * s:(u + 1) * s].transpose(1, 2).reshape(-1))
    return torch.cat(parts)


def _cpu_unpack(buf, U, heads, B, s, D, direction):
    import torch
    sizes = [B * s * (h // U) * D for h in heads]
    chunk = sum(sizes)
    outs = []
    off = 0
    for h, n in zip(heads, sizes):
        hU = h // U
        pieces = [buf[u * chunk + off:u * chunk + off + n].reshape(B, s, hU, D) for u in range(U)]
        off += n
        if direction == "seq_to_head":   # from device u: its s tokens of my heads
            outs.append(torch.cat(pieces, dim=1).transpose(1, 2).contiguous())
        else:                            # from device u: my tokens of its heads
            outs.append(torch.cat(pieces, dim=2).contiguous())
    return tuple(outs)


def _usp_worker(rank, world, port, U, R, results):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import numpy as np
    import torch
    import oracle
    from ring_ulysses_sequence_b200 import multi, ring, ulysses
    multi.init("gloo", timeout_s=60)
    ug, rg = ulysses.usp_groups(U, R)
    B, H, Hkv, D, s = 1, 8, 4, 8, 4
    S = U * R * s
    order = oracle.ZIGZAG
    rng = np.random.default_rng(11)
    q, k, v, do = (rng.standard_normal(sh) for sh in
                   [(B, H, S, D), (B, Hkv, S, D), (B, Hkv, S, D), (B, H, S, D)])
    pos = oracle.rank_major_positions(S, R, order)   # the ring's rank-major sequence
    mine = pos[rank * s:(rank + 1) * s]               # shard n = r*U + u = this rank
    ql, kl, vl, dol = (torch.from_numpy(np.ascontiguousarray(x[:, :, mine].transpose(0, 2, 1, 3)))
                       for x in (q, k, v, do))        # [B, s, heads, D]

    def ring_fwd(q_, k_, v_, c, o_, s_, g):
        return ring.ring_attn_fwd_p2p(q_, k_, v_, c, o_, s_, group=g, fold=_oracle_fold(S, D))

    def ring_bwd(q_, k_, v_, o_, l_, do_, c, or_, s_, g):
        return ring.ring_attn_bwd_p2p(q_, k_, v_, o_, l_, do_, c, or_, s_, group=g,
                                      bwd_step=_oracle_bwd_step(S), delta=_delta)

    o, ctx = ulysses.usp_attn_fwd(ql, kl, vl, ug, rg, True, order, pack=_cpu_pack,
                                  unpack=_cpu_unpack, ring_fwd=ring_fwd)
    dq, dk, dv = ulysses.usp_attn_bwd(dol, ctx, ug, rg, True, order, pack=_cpu_pack,
                                      unpack=_cpu_unpack, ring_bwd=ring_bwd)
    o_ref, _ = oracle.attn_fwd(q, k, v, True, rows=mine)
    rdq, rdkv = oracle.attn_bwd(q, k, v, do, True, qrows=mine, krows=mine)
    err = float(np.abs(o.numpy().transpose(0, 2, 1, 3) - o_ref).max())
    gerr = 0.0
    for h in range(H):
        gerr = max(gerr, float(np.abs(dq[0, :, h].numpy() - rdq[(0, h)]).max()))
    for g in range(Hkv):
        gerr = max(gerr, float(np.abs(dk[0, :, g].numpy() - rdkv[(0, g)][0]).max()),
                   float(np.abs(dv[0, :, g].numpy() - rdkv[(0, g)][1]).max()))
    results[rank] = (err, gerr, tuple(ctx.q.shape))
    multi.shutdown()


@pytest.mark.parametrize("U,R", [(2, 2), (4, 1), (1, 2), (2, 1)])
def test_usp_over_gloo_matches_oracle(U, R):
    res = _spawn(_usp_worker, U * R, U, R)
    for r in range(U * R):
        err, gerr, qshape = res[r]
        assert qshape == (1, 8 // U, U * 4 * R // R, 8)   # head shard [B, H/U, S/R, D]
        assert err < 1e-5 and gerr < 1e-5, (r, err, gerr)


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
