"""One ring step on the GPU (rm_ring_attn_fwd_step) against the fp64 oracle.

A rank of a ring spread over devices runs P of these steps, one per owner
block, and folds the partials with rm_lse_merge ("DeDLOC Guide", Step 3 and
section 3). Checked here:
* each partial against oracle.step_partial, including rows and whole tiles that
  see nothing of the block, which must come out as exactly (0, -inf);
* the P steps of every rank, merged on the GPU, against the one-launch ring
  forward and against the oracle's attention;
* the p2p ring driver with one process (P = 1: one step).
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
    o, lse = ring.ring_attn_fwd_p2p(q, k, v, True, "zigzag")
    o_ref, lse_ref = rm.ring_attn_fwd(q, k, v, 1, True, "zigzag")
    torch.cuda.synchronize()
    assert_close(o.cpu().numpy(), o_ref.float().cpu().numpy(), BF16_MAX_ABS, BF16_MEAN_ABS,
                 what="O")
    assert_close(lse.cpu().numpy(), lse_ref.cpu().numpy(), LSE_MAX_ABS, what="LSE")


def test_step_rejects_bad_arguments():
    import ring_ulysses_sequence_b200 as rm
    q = torch.zeros((1, 2, 256, 128), dtype=torch.bfloat16, device="cuda")
    for rank, owner in ((4, 0), (0, 4), (-1, 0)):
        with pytest.raises(rm.RMError):
            rm.ring_attn_fwd_step(q, q, q, 4, rank, owner)
    with pytest.raises(rm.RMError):                      # fp32: no step variant
        qf = q.float()
        rm.ring_attn_fwd_step(qf, qf, qf, 4, 0, 0)
