"""All-gather attention forward on the GPU against the fp64 oracle.

The axolotl-ringmaster README (Benchmark section) names two ways of bringing
every rank's keys to its queries: the p2p ring and an all-gather of the keys
before one attention pass. Both compute the same attention, so the oracle is
the plain definition here too. The gathered keys are given in natural order,
either straight from the natural-order inputs (independent of the library's
reorder) or formed on the device by allgather_kv from the rank-major shards.
"""
import pytest
import torch

import oracle
from gpu_util import (BF16_MAX_ABS, BF16_MEAN_ABS, LSE_MAX_ABS, assert_close, to_natural,
                      to_rank_major)
from ring_ulysses_sequence_b200.synth import WORKLOADS, make_inputs, make_tensor, sample_rows

pytestmark = pytest.mark.gpu


def _qkv(B, H, Hkv, S, D, seed, scale=0.5):
    return (make_tensor((B, H, S, D), seed, torch.bfloat16, scale),
            make_tensor((B, Hkv, S, D), seed + 1, torch.bfloat16, scale),
            make_tensor((B, Hkv, S, D), seed + 2, torch.bfloat16, scale))


def _run(qn, kn, vn, P, order, causal):
    """Natural-order CPU inputs -> all-gather forward (q rank-major, k/v
    natural) -> natural-order CPU (O, LSE)."""
    import ring_ulysses_sequence_b200 as rm
    q = to_rank_major(qn, P, order).cuda()
    o, lse = rm.allgather_attn_fwd(q, kn.cuda(), vn.cuda(), P, causal=causal, order=order)
    torch.cuda.synchronize()
    assert rm.native.rm_check_device_status() == 0
    return (to_natural(o.float().cpu(), P, order),
            to_natural(lse.cpu().unsqueeze(-1), P, order).squeeze(-1))


@pytest.mark.parametrize("B,H,Hkv,S,D,P,order,causal", [
    (1, 4, 2, 1024, 128, 4, "zigzag", True),      # GQA: head-paired tiles
    (1, 2, 2, 1024, 128, 4, "zigzag", False),     # MHA, full attention
    (2, 3, 1, 1024, 64, 2, "zigzag", True),       # odd group, D = 64, B = 2
    (1, 8, 2, 2048, 128, 2, "contiguous", True),
    (1, 4, 1, 2048, 128, 8, "zigzag", True),      # chunks of one tile
    (1, 2, 1, 512, 128, 1, "zigzag", True),       # P = 1
    (1, 3, 3, 2048, 128, 8, "zigzag", True),      # odd group with one-tile chunks
    (1, 4, 4, 1024, 128, 4, "contiguous", False),
])
def test_allgather_forward_matches_oracle(B, H, Hkv, S, D, P, order, causal):
    q, k, v = _qkv(B, H, Hkv, S, D, 900 + S + H)
    o, lse = _run(q, k, v, P, order, causal)
    o_ref, lse_ref = oracle.attn_fwd(q.float(), k.float(), v.float(), causal)
    assert_close(o.numpy(), o_ref, BF16_MAX_ABS, BF16_MEAN_ABS, what="O")
    assert_close(lse.numpy(), lse_ref, LSE_MAX_ABS, what="LSE")


def test_allgather_kv_is_the_natural_order():
    """allgather_kv of the rank-major shards gives back the natural-order keys,
    bit for bit (a pure permutation)."""
    import ring_ulysses_sequence_b200 as rm
    _, k, v = _qkv(1, 4, 2, 2048, 128, 77)
    for P, order in ((4, "zigzag"), (8, "zigzag"), (2, "contiguous")):
        kr, vr = (to_rank_major(t, P, order).cuda() for t in (k, v))
        k_all, v_all = rm.allgather_kv(kr, vr, P, order)
        torch.cuda.synchronize()
        assert torch.equal(k_all.cpu(), k) and torch.equal(v_all.cpu(), v)


@pytest.mark.parametrize("P,order", [(4, "zigzag"), (8, "zigzag"), (4, "contiguous")])
def test_allgather_agrees_with_the_ring(P, order):
    """The two ways to distribute the keys give the same attention: the ring and
    the all-gather outputs agree within the bf16 tolerance, and each matches
    the oracle on the rows of every chunk edge."""
    import ring_ulysses_sequence_b200 as rm
    q, k, v = _qkv(1, 8, 2, 4096, 128, 321 + P)
    qr, kr, vr = (to_rank_major(t, P, order).cuda() for t in (q, k, v))
    o_ring, lse_ring = rm.ring_attn_fwd(qr, kr, vr, P, True, order)
    k_all, v_all = rm.allgather_kv(kr, vr, P, order)
    o_ag, lse_ag = rm.allgather_attn_fwd(qr, k_all, v_all, P, True, order)
    torch.cuda.synchronize()
    assert rm.native.rm_check_device_status() == 0
    assert_close(o_ag.float().cpu().numpy(), o_ring.float().cpu().numpy(), BF16_MAX_ABS,
                 BF16_MEAN_ABS, what="O all-gather vs ring")
    assert_close(lse_ag.cpu().numpy(), lse_ring.cpu().numpy(), LSE_MAX_ABS, what="LSE")
    chunk = 4096 // (2 * P if order == "zigzag" else P)
    rows = sample_rows(4096, 64, 17, chunk)
    o_ref, lse_ref = oracle.attn_fwd(q.float(), k.float(), v.float(), True, rows=rows)
    o_n = to_natural(o_ag.float().cpu(), P, order)[:, :, rows]
    lse_n = to_natural(lse_ag.cpu().unsqueeze(-1), P, order).squeeze(-1)[:, :, rows]
    assert_close(o_n.numpy(), o_ref, BF16_MAX_ABS, BF16_MEAN_ABS, what="O rows")
    assert_close(lse_n.numpy(), lse_ref, LSE_MAX_ABS, what="LSE rows")


def test_allgather_workload_sampled_rows():
    """The S = 32768 GQA causal zigzag workload (P = 8) through the all-gather
    path, in the launch configuration the benchmark times, on sampled rows."""
    import ring_ulysses_sequence_b200 as rm
    w = WORKLOADS["ring_fwd_bf16_S32k_gqa_causal_zigzag"]
    q, k, v = make_inputs(w)
    qr = to_rank_major(q, w.P, w.order).cuda()
    kr, vr = (to_rank_major(t, w.P, w.order).cuda() for t in (k, v))
    k_all, v_all = rm.allgather_kv(kr, vr, w.P, w.order)
    o, lse = rm.allgather_attn_fwd(qr, k_all, v_all, w.P, w.causal, w.order)
    torch.cuda.synchronize()
    assert rm.native.rm_check_device_status() == 0
    rows = sample_rows(w.S, 256, w.seed + 1000, w.chunk)
    o_ref, lse_ref = oracle.attn_fwd(q.float(), k.float(), v.float(), w.causal, rows=rows)
    o_n = to_natural(o.float().cpu(), w.P, w.order)[:, :, rows]
    lse_n = to_natural(lse.cpu().unsqueeze(-1), w.P, w.order).squeeze(-1)[:, :, rows]
    assert_close(o_n.numpy(), o_ref, BF16_MAX_ABS, BF16_MEAN_ABS, what="O")
    assert_close(lse_n.numpy(), lse_ref, LSE_MAX_ABS, what="LSE")


def test_allgather_rejects_fp32_and_bad_shapes():
    import ring_ulysses_sequence_b200 as rm
    q = torch.zeros((1, 2, 1024, 128), dtype=torch.float32, device="cuda")
    with pytest.raises(rm.RMError):
        rm.allgather_attn_fwd(q, q, q, 4)
    q = torch.zeros((1, 2, 1000, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(rm.RMError):
        rm.allgather_attn_fwd(q, q, q, 4)
    e = torch.zeros((1, 2, 0, 128), dtype=torch.bfloat16, device="cuda")
    o, lse = rm.allgather_attn_fwd(e, e, e, 4)     # empty sequence: nothing to do
    assert o.shape == e.shape and lse.shape == (1, 2, 0)
