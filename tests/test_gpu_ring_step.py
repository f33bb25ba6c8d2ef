"""One ring step on the GPU (rm_ring_attn_fwd_step) against the fp64 oracle.

A rank of a ring spread over devices runs P of these steps, one per owner
block, and folds the partials with rm_lse_merge ("DeDLOC Guide", Step 3 and
section 3). Checked here:
* each partial against oracle.step_partial, including rows and whole tiles that
  see nothing of the block, which must come out as exactly (0, -inf);
* the P steps of every rank, merged on the GPU, against the one-launch ring
  forward and against the oracle's attention;
* the fused step + merge (rm_ring_attn_fwd_step_merge) against the oracle and
  against the step and merge run as two calls;
* the one-step backward (rm_ring_attn_bwd_step): every rank's P steps against
  the oracle's gradients and the one-launch backward, and single (rank, owner)
  steps against the oracle's step share, with untouched tiles left as they were;
* the p2p ring drivers with one process (P = 1: one step), which must leave
  the caller's K and V as they were.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import BF16_MAX_ABS, BF16_MEAN_ABS, LSE_MAX_ABS, ORDER, assert_close, to_natural
from ring_ulysses_sequence_b200.synth import WORKLOADS, make_inputs, make_tensor, sample_rows

pytestmark = pytest.mark.gpu


def _qkv(B, H, Hkv, S, D, seed, scale=0.5):
    return (make_tensor((B, H, S, D), seed, torch.bfloat16, scale),
            make_tensor((B, Hkv, S, D), seed + 1, torch.bfloat16, scale),
            make_tensor((B, Hkv, S, D), seed + 2, torch.bfloat16, scale))


def _shards(x, P, order):
    """Natural-order CPU tensor -> list of the P ranks' local slices (CPU),
    by the oracle's position map."""
    S = x.shape[2]
    L = S // P
    pos = oracle.rank_major_positions(S, P, ORDER[order])
    return [x[:, :, torch.from_numpy(pos[r * L:(r + 1) * L])].contiguous() for r in range(P)]


def _check_partial(o, lse, o_ref, lse_ref, what):
    lse, o = lse.cpu().numpy(), o.cpu().numpy()
    empty = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse), empty), f"{what}: empty rows differ"
    assert np.all(o[empty] == 0.0), f"{what}: empty rows must have O = 0"
    if (~empty).any():
        assert_close(lse[~empty], lse_ref[~empty], LSE_MAX_ABS, what=f"{what} LSE")
        assert_close(o[~empty], o_ref[~empty], BF16_MAX_ABS, BF16_MEAN_ABS, what=f"{what} O")


@pytest.mark.parametrize("B,H,Hkv,S,D,P,order,causal", [
    (1, 4, 2, 1024, 128, 4, "zigzag", True),      # GQA: head-paired tiles
    (1, 2, 2, 1024, 128, 2, "contiguous", True),
    (2, 3, 1, 1024, 64, 2, "zigzag", True),       # odd group, D = 64, B = 2
    (1, 4, 1, 2048, 128, 8, "zigzag", True),      # chunks of one tile
    (1, 2, 1, 1024, 128, 4, "contiguous", False),
    (1, 3, 3, 2048, 128, 8, "zigzag", True),      # odd group with one-tile chunks
])
def test_step_partials_match_oracle(B, H, Hkv, S, D, P, order, causal):
    import ring_ulysses_sequence_b200 as rm
    q, k, v = _qkv(B, H, Hkv, S, D, 1100 + S + H)
    qs, ks, vs = (_shards(x, P, order) for x in (q, k, v))
    ranks = sorted({0, P // 2, P - 1})
    for rank in ranks:
        ql = qs[rank].cuda()
        for owner in range(P):
            o, lse = rm.ring_attn_fwd_step(ql, ks[owner].cuda(), vs[owner].cuda(), P, rank,
                                           owner, causal, order)
            torch.cuda.synchronize()
            assert rm.native.rm_check_device_status() == 0
            o_ref, lse_ref = oracle.step_partial(qs[rank].float(), ks[owner].float(),
                                                 vs[owner].float(), S, P, ORDER[order], rank,
                                                 owner, causal)
            _check_partial(o, lse, o_ref, lse_ref, f"rank {rank} owner {owner}")


@pytest.mark.parametrize("H,Hkv,S,D,P,order,causal", [
    (4, 2, 2048, 128, 4, "zigzag", True),
    (8, 2, 4096, 128, 8, "zigzag", True),
    (2, 2, 2048, 64, 2, "contiguous", False),
    (3, 1, 2048, 128, 4, "contiguous", True),
])
def test_steps_merged_equal_the_ring(H, Hkv, S, D, P, order, causal):
    """Every rank's P steps, merged on the GPU in ring order, give that rank's
    slice of the one-launch ring forward, and the oracle's attention."""
    import ring_ulysses_sequence_b200 as rm
    q, k, v = _qkv(1, H, Hkv, S, D, 1200 + S + P)
    qs, ks, vs = (_shards(x, P, order) for x in (q, k, v))
    qr, kr, vr = (torch.cat(sh, dim=2).cuda() for sh in (qs, ks, vs))
    o_ring, lse_ring = rm.ring_attn_fwd(qr, kr, vr, P, causal, order)
    L = S // P
    outs, lses = [], []
    for rank in range(P):
        ql = qs[rank].cuda()
        o_acc = torch.zeros((1, H, L, D), dtype=torch.float32, device="cuda")
        l_acc = torch.full((1, H, L), float("-inf"), dtype=torch.float32, device="cuda")
        for t in range(P):
            owner = (rank - t) % P
            o_p, l_p = rm.ring_attn_fwd_step(ql, ks[owner].cuda(), vs[owner].cuda(), P, rank,
                                             owner, causal, order)
            rm.lse_merge_(o_acc, l_acc, o_p, l_p)
        outs.append(o_acc)
        lses.append(l_acc)
    torch.cuda.synchronize()
    assert rm.native.rm_check_device_status() == 0
    o_steps, lse_steps = torch.cat(outs, dim=2).cpu(), torch.cat(lses, dim=2).cpu()
    assert_close(o_steps.numpy(), o_ring.float().cpu().numpy(), BF16_MAX_ABS, BF16_MEAN_ABS,
                 what="O steps vs ring")
    assert_close(lse_steps.numpy(), lse_ring.cpu().numpy(), LSE_MAX_ABS, what="LSE")
    o_ref, lse_ref = oracle.attn_fwd(q.float(), k.float(), v.float(), causal)
    assert_close(to_natural(o_steps, P, order).numpy(), o_ref, BF16_MAX_ABS, BF16_MEAN_ABS,
                 what="O vs oracle")
    assert_close(to_natural(lse_steps.unsqueeze(-1), P, order).squeeze(-1).numpy(), lse_ref,
                 LSE_MAX_ABS, what="LSE vs oracle")


@pytest.mark.parametrize("H,Hkv,S,D,P,order,causal", [
    (4, 2, 2048, 128, 4, "zigzag", True),
    (8, 2, 4096, 128, 8, "zigzag", True),
    (2, 2, 2048, 64, 2, "contiguous", False),
    (3, 1, 2048, 128, 4, "contiguous", True),
    (3, 3, 2048, 128, 8, "zigzag", True),
])
def test_fused_step_merge_matches_oracle_and_the_two_calls(H, Hkv, S, D, P, order, causal):
    """rm_ring_attn_fwd_step_merge over every rank's P steps: the oracle's
    attention, and the same as rm_ring_attn_fwd_step + rm_lse_merge."""
    import ring_ulysses_sequence_b200 as rm
    q, k, v = _qkv(1, H, Hkv, S, D, 1250 + S + P)
    qs, ks, vs = (_shards(x, P, order) for x in (q, k, v))
    L = S // P
    fused, fused_l, split, split_l = [], [], [], []
    for rank in range(P):
        ql = qs[rank].cuda()
        o_f = torch.zeros((1, H, L, D), dtype=torch.float32, device="cuda")
        l_f = torch.full((1, H, L), float("-inf"), dtype=torch.float32, device="cuda")
        o_s, l_s = o_f.clone(), l_f.clone()
        for t in range(P):
            owner = (rank - t) % P
            kb, vb = ks[owner].cuda(), vs[owner].cuda()
            rm.ring_attn_fwd_step_merge(ql, kb, vb, o_f, l_f, P, rank, owner, causal, order)
            o_p, l_p = rm.ring_attn_fwd_step(ql, kb, vb, P, rank, owner, causal, order)
            rm.lse_merge_(o_s, l_s, o_p, l_p)
        fused.append(o_f)
        fused_l.append(l_f)
        split.append(o_s)
        split_l.append(l_s)
    torch.cuda.synchronize()
    assert rm.native.rm_check_device_status() == 0
    o_f, l_f = torch.cat(fused, dim=2).cpu(), torch.cat(fused_l, dim=2).cpu()
    o_s, l_s = torch.cat(split, dim=2).cpu(), torch.cat(split_l, dim=2).cpu()
    # the same algebra in two orders of fp32 rounding
    assert_close(o_f.numpy(), o_s.numpy(), 1e-5, what="fused vs two calls: O")
    assert_close(l_f.numpy(), l_s.numpy(), 1e-5, what="fused vs two calls: LSE")
    o_ref, lse_ref = oracle.attn_fwd(q.float(), k.float(), v.float(), causal)
    assert_close(to_natural(o_f, P, order).numpy(), o_ref, BF16_MAX_ABS, BF16_MEAN_ABS,
                 what="O vs oracle")
    assert_close(to_natural(l_f.unsqueeze(-1), P, order).squeeze(-1).numpy(), lse_ref,
                 LSE_MAX_ABS, what="LSE vs oracle")


def test_fused_step_merge_leaves_rows_that_see_nothing():
    """Contiguous causal: rank 0's queries see no key of owner 3, so the
    running pair must come back bit for bit."""
    import ring_ulysses_sequence_b200 as rm
    q, k, v = _qkv(1, 2, 2, 1024, 128, 1260)
    qs, ks, vs = (_shards(x, 4, "contiguous") for x in (q, k, v))
    o = torch.randn((1, 2, 256, 128), device="cuda")
    l = torch.randn((1, 2, 256), device="cuda")
    o0, l0 = o.clone(), l.clone()
    rm.ring_attn_fwd_step_merge(qs[0].cuda(), ks[3].cuda(), vs[3].cuda(), o, l, 4, 0, 3, True,
                                "contiguous")
    torch.cuda.synchronize()
    assert torch.equal(o, o0) and torch.equal(l, l0)


def _bwd_inputs(B, H, Hkv, S, D, P, order, causal, seed):
    """Natural-order CPU inputs and their GPU rank-major forward (O, LSE)."""
    import ring_ulysses_sequence_b200 as rm
    from gpu_util import to_rank_major
    q, k, v = _qkv(B, H, Hkv, S, D, seed)
    do = make_tensor((B, H, S, D), seed + 3, torch.bfloat16, 0.5)
    qr, kr, vr, dor = (to_rank_major(t, P, order).cuda() for t in (q, k, v, do))
    o, lse = rm.ring_attn_fwd(qr, kr, vr, P, causal, order)
    return (q, k, v, do), (qr, kr, vr, dor, o, lse)


@pytest.mark.parametrize("B,H,Hkv,S,D,P,order,causal", [
    (1, 4, 2, 2048, 128, 4, "zigzag", True),
    (1, 2, 2, 1024, 128, 2, "contiguous", True),
    (2, 3, 1, 1024, 64, 2, "zigzag", True),
    (1, 4, 1, 2048, 128, 8, "zigzag", True),
    (1, 2, 2, 1024, 128, 4, "contiguous", False),
])
def test_bwd_steps_sum_to_the_backward(B, H, Hkv, S, D, P, order, causal):
    """P ranks x P steps of rm_ring_attn_bwd_step, in the reverse ring's
    schedule: the oracle's gradients and the one-launch backward."""
    _bwd_steps_sum(B, H, Hkv, S, D, P, order, causal)


@pytest.mark.parametrize("B,H,Hkv,S,D,P,order,causal", [
    (1, 4, 2, 2048, 128, 4, "zigzag", True),
    (2, 3, 1, 1024, 64, 2, "zigzag", True),
])
def test_bwd_steps_with_the_fused_kernel(B, H, Hkv, S, D, P, order, causal):
    """The same with the fused backward kernel (dQ added by reductions)."""
    from ring_ulysses_sequence_b200 import native
    before = native.rm_get_bwd_deterministic()
    native.rm_set_bwd_deterministic(0)
    try:
        _bwd_steps_sum(B, H, Hkv, S, D, P, order, causal)
    finally:
        native.rm_set_bwd_deterministic(before)


def _bwd_steps_sum(B, H, Hkv, S, D, P, order, causal):
    import ring_ulysses_sequence_b200 as rm
    (q, k, v, do), (qr, kr, vr, dor, o, lse) = _bwd_inputs(B, H, Hkv, S, D, P, order, causal,
                                                          1400 + S + H)
    L = S // P
    sl = [slice(r * L, (r + 1) * L) for r in range(P)]
    qs, ks, vs, dos, os_, ls = ([x[:, :, s_].contiguous() for s_ in sl] for x in (qr, kr, vr, dor, o, lse))
    deltas = [rm.ring_attn_bwd_delta(os_[r], dos[r]) for r in range(P)]
    dq = [torch.zeros(qs[r].shape, dtype=torch.float32, device="cuda") for r in range(P)]
    dk = [torch.zeros(ks[r].shape, dtype=torch.float32, device="cuda") for r in range(P)]
    dv = [torch.zeros(ks[r].shape, dtype=torch.float32, device="cuda") for r in range(P)]
    for t in range(P):
        for rank in range(P):
            owner = (rank - t) % P
            rm.ring_attn_bwd_step(qs[rank], ks[owner], vs[owner], ls[rank], deltas[rank],
                                  dos[rank], dq[rank], dk[owner], dv[owner], P, rank, owner,
                                  causal, order)
    torch.cuda.synchronize()
    assert rm.native.rm_check_device_status() == 0
    gq, gk, gv = (torch.cat(x, dim=2).cpu() for x in (dq, dk, dv))
    ref = rm.ring_attn_bwd(qr, kr, vr, o, lse, dor, P, causal, order)
    for got, want, name in zip((gq, gk, gv), ref, ("dQ", "dK", "dV")):
        assert_close(got.numpy(), want.cpu().numpy(), BF16_MAX_ABS, BF16_MEAN_ABS,
                     what=f"{name} steps vs one launch")
    rdq, rdkv = oracle.attn_bwd(q.float(), k.float(), v.float(), do.float(), causal)
    nq, nk, nv = (to_natural(x, P, order) for x in (gq, gk, gv))
    for b in range(B):
        for h in range(H):
            assert_close(nq[b, h].numpy(), rdq[(b, h)], BF16_MAX_ABS, BF16_MEAN_ABS, f"dQ[{b},{h}]")
        for g in range(Hkv):
            assert_close(nk[b, g].numpy(), rdkv[(b, g)][0], BF16_MAX_ABS, BF16_MEAN_ABS, f"dK[{b},{g}]")
            assert_close(nv[b, g].numpy(), rdkv[(b, g)][1], BF16_MAX_ABS, BF16_MEAN_ABS, f"dV[{b},{g}]")


@pytest.mark.parametrize("order,causal", [("zigzag", True), ("contiguous", True),
                                          ("contiguous", False)])
def test_bwd_step_shares_match_oracle_and_skip_untouched_tiles(order, causal):
    """Single (rank, owner) steps added onto non-zero arrays: the change is the
    oracle's share of that pair; arrays of a pair that sees nothing stay as
    they were bit for bit."""
    import ring_ulysses_sequence_b200 as rm
    B, H, Hkv, S, D, P = 1, 4, 2, 1024, 128, 4
    (q, k, v, do), (qr, kr, vr, dor, o, lse) = _bwd_inputs(B, H, Hkv, S, D, P, order, causal, 1500)
    L = S // P
    delta = rm.ring_attn_bwd_delta(o, dor)
    for rank, owner in ((0, 0), (P - 1, 0), (1, P - 1), (P - 1, 1)):
        qs, ds, ls, dls = (x[:, :, rank * L:(rank + 1) * L].contiguous() for x in (qr, dor, lse, delta))
        kb, vb = (x[:, :, owner * L:(owner + 1) * L].contiguous() for x in (kr, vr))
        base = [torch.randn((B, H, L, D), device="cuda"), torch.randn((B, Hkv, L, D), device="cuda"),
                torch.randn((B, Hkv, L, D), device="cuda")]
        got = [x.clone() for x in base]
        rm.ring_attn_bwd_step(qs, kb, vb, ls, dls, ds, *got, P, rank, owner, causal, order)
        torch.cuda.synchronize()
        assert rm.native.rm_check_device_status() == 0
        ref = oracle.step_bwd_partial(qs.float().cpu(), kb.float().cpu(), vb.float().cpu(),
                                      ds.float().cpu(), ls.cpu(), dls.cpu(), S, P, ORDER[order],
                                      rank, owner, causal)
        for g_, b_, r_, name in zip(got, base, ref, ("dQ", "dK", "dV")):
            diff = (g_ - b_).cpu().numpy()
            assert_close(diff, r_, BF16_MAX_ABS, BF16_MEAN_ABS, f"{name} rank {rank} owner {owner}")
            # rows whose oracle share is exactly zero belong to skipped tiles or
            # to rows no pair reaches: those must be untouched
            zero = np.all(r_ == 0.0, axis=-1)
            assert np.array_equal(g_.cpu().numpy()[zero], b_.cpu().numpy()[zero]) or not zero.any()


def test_bwd_delta_matches_rowsum():
    import ring_ulysses_sequence_b200 as rm
    for D, odt in ((128, torch.bfloat16), (64, torch.float32), (128, torch.float32)):
        o = make_tensor((2, 3, 256, D), 1600 + D, odt, 0.5).cuda()
        do = make_tensor((2, 3, 256, D), 1601 + D, torch.bfloat16, 0.5).cuda()
        got = rm.ring_attn_bwd_delta(o, do).cpu().double()
        want = (o.double() * do.double()).sum(-1).cpu()
        assert float((got - want).abs().max()) < 1e-4


def test_steps_on_the_32k_workload_sampled_rows():
    """The S = 32768 GQA causal zigzag workload (P = 8) as eight ranks would
    run it: 64 step launches and merges; sampled rows against the oracle."""
    import ring_ulysses_sequence_b200 as rm
    w = WORKLOADS["ring_fwd_bf16_S32k_gqa_causal_zigzag"]
    q, k, v = make_inputs(w)
    qs, ks, vs = (_shards(x, w.P, w.order) for x in (q, k, v))
    ks, vs = [x.cuda() for x in ks], [x.cuda() for x in vs]
    L = w.S // w.P
    outs, lses = [], []
    for rank in range(w.P):
        ql = qs[rank].cuda()
        o_acc = torch.zeros((w.B, w.H, L, w.D), dtype=torch.float32, device="cuda")
        l_acc = torch.full((w.B, w.H, L), float("-inf"), dtype=torch.float32, device="cuda")
        for t in range(w.P):
            owner = (rank - t) % w.P
            o_p, l_p = rm.ring_attn_fwd_step(ql, ks[owner], vs[owner], w.P, rank, owner,
                                             w.causal, w.order)
            rm.lse_merge_(o_acc, l_acc, o_p, l_p)
        outs.append(o_acc.cpu())
        lses.append(l_acc.cpu())
    assert rm.native.rm_check_device_status() == 0
    o = to_natural(torch.cat(outs, dim=2), w.P, w.order)
    lse = to_natural(torch.cat(lses, dim=2).unsqueeze(-1), w.P, w.order).squeeze(-1)
    rows = sample_rows(w.S, 256, w.seed + 1000, w.chunk)
    o_ref, lse_ref = oracle.attn_fwd(q.float(), k.float(), v.float(), w.causal, rows=rows)
    assert_close(o[:, :, rows].numpy(), o_ref, BF16_MAX_ABS, BF16_MEAN_ABS, what="O")
    assert_close(lse[:, :, rows].numpy(), lse_ref, LSE_MAX_ABS, what="LSE")


def test_p2p_driver_with_one_process():
    import ring_ulysses_sequence_b200 as rm
    from ring_ulysses_sequence_b200 import ring
    q, k, v = (x.cuda() for x in _qkv(1, 4, 2, 1024, 128, 1300))
    do = make_tensor((1, 4, 1024, 128), 1303, torch.bfloat16, 0.5).cuda()
    k0, v0 = k.clone(), v.clone()
    o, lse = ring.ring_attn_fwd_p2p(q, k, v, True, "zigzag")
    o_ref, lse_ref = rm.ring_attn_fwd(q, k, v, 1, True, "zigzag")
    torch.cuda.synchronize()
    assert torch.equal(k, k0) and torch.equal(v, v0)    # the caller's blocks are untouched
    assert_close(o.cpu().numpy(), o_ref.float().cpu().numpy(), BF16_MAX_ABS, BF16_MEAN_ABS,
                 what="O")
    assert_close(lse.cpu().numpy(), lse_ref.cpu().numpy(), LSE_MAX_ABS, what="LSE")
    dq, dk, dv = ring.ring_attn_bwd_p2p(q, k, v, o, lse, do, True, "zigzag")
    ref = rm.ring_attn_bwd(q, k, v, o_ref, lse_ref, do, 1, True, "zigzag")
    torch.cuda.synchronize()
    assert rm.native.rm_check_device_status() == 0
    assert torch.equal(k, k0) and torch.equal(v, v0)
    for got, want, name in zip((dq, dk, dv), ref, ("dQ", "dK", "dV")):
        assert_close(got.cpu().numpy(), want.cpu().numpy(), BF16_MAX_ABS, BF16_MEAN_ABS,
                     what=name)


def test_step_rejects_bad_arguments():
    import ring_ulysses_sequence_b200 as rm
    q = torch.zeros((1, 2, 256, 128), dtype=torch.bfloat16, device="cuda")
    for rank, owner in ((4, 0), (0, 4), (-1, 0)):
        with pytest.raises(rm.RMError):
            rm.ring_attn_fwd_step(q, q, q, 4, rank, owner)
    with pytest.raises(rm.RMError):                      # fp32: no step variant
        qf = q.float()
        rm.ring_attn_fwd_step(qf, qf, qf, 4, 0, 0)


def test_usp_driver_with_one_process_uses_the_library():
    """ulysses.usp_attn_fwd / usp_attn_bwd with one process (U = R = 1) run the
    library's pack, unpack, fused step and step-backward kernels end to end:
    the result is the one-launch forward and backward on the same tokens."""
    import ring_ulysses_sequence_b200 as rm
    from ring_ulysses_sequence_b200 import ulysses
    B, H, Hkv, S, D = 1, 8, 2, 1024, 128
    q, k, v = (x.cuda() for x in _qkv(B, H, Hkv, S, D, 1700))
    do = make_tensor((B, H, S, D), 1703, torch.bfloat16, 0.5).cuda()
    seq = lambda x: x.transpose(1, 2).contiguous()            # [B, S, heads, D]
    o, ctx = ulysses.usp_attn_fwd(seq(q), seq(k), seq(v), None, None, True, "zigzag")
    dq, dk, dv = ulysses.usp_attn_bwd(seq(do), ctx, None, None, True, "zigzag")
    o_ref, lse_ref = rm.ring_attn_fwd(q, k, v, 1, True, "zigzag")
    g_ref = rm.ring_attn_bwd(q, k, v, o_ref, lse_ref, do, 1, True, "zigzag")
    torch.cuda.synchronize()
    assert rm.native.rm_check_device_status() == 0
    assert o.shape == (B, S, H, D) and o.dtype == torch.float32
    assert_close(o.transpose(1, 2).cpu().numpy(), o_ref.float().cpu().numpy(), BF16_MAX_ABS,
                 BF16_MEAN_ABS, what="O")
    assert_close(ctx.lse.cpu().numpy(), lse_ref.cpu().numpy(), LSE_MAX_ABS, what="LSE")
    for got, want, name in zip((dq, dk, dv), g_ref, ("dQ", "dK", "dV")):
        assert_close(got.transpose(1, 2).cpu().numpy(), want.cpu().numpy(), BF16_MAX_ABS,
                     BF16_MEAN_ABS, what=name)
