"""Causal sliding-window ring attention on the GPU against the fp64 oracle.

Query i sees keys i - W < j <= i (axolotl-ringmaster README, Status table,
phase 4: sliding-window attention). Windows are chosen around the 128-token
tile edges (1, 127, 128, 129, ...) so that tiles of every class occur: skipped
left of the window, full inside it, and masked on both of its edges, as well
as rows that see no key of a masked tile. Tolerances as for plain attention.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import (BF16_MAX_ABS, BF16_MEAN_ABS, FP32_MAX_ABS, LSE_MAX_ABS, assert_close,
                      run_fwd, to_natural, to_rank_major)
from ring_ulysses_sequence_b200.synth import WORKLOADS, make_inputs, make_tensor, sample_rows

pytestmark = pytest.mark.gpu


def _qkv(B, H, Hkv, S, D, seed, dtype, scale=0.5):
    return (make_tensor((B, H, S, D), seed, dtype, scale),
            make_tensor((B, Hkv, S, D), seed + 1, dtype, scale),
            make_tensor((B, Hkv, S, D), seed + 2, dtype, scale))


def _check_fwd(q, k, v, P, order, W, fp32=False, rows=None):
    o, lse = run_fwd(q, k, v, P, order, True, window=W)
    o_ref, lse_ref = oracle.attn_fwd(q.float(), k.float(), v.float(), True, rows=rows, window=W)
    if rows is not None:
        o, lse = o[:, :, rows], lse[:, :, rows]
    if fp32:
        assert_close(o.numpy(), o_ref, FP32_MAX_ABS, what=f"O (W={W})")
    else:
        assert_close(o.numpy(), o_ref, BF16_MAX_ABS, BF16_MEAN_ABS, what=f"O (W={W})")
    assert_close(lse.numpy(), lse_ref, LSE_MAX_ABS, what=f"LSE (W={W})")
    return o, lse


@pytest.mark.parametrize("W", [1, 64, 127, 128, 129, 255, 256, 300, 700, 1023])
def test_window_bf16_forward_zigzag_gqa(W):
    q, k, v = _qkv(1, 4, 2, 1024, 128, 500 + W, torch.bfloat16)
    _check_fwd(q, k, v, 4, "zigzag", W)


@pytest.mark.parametrize("B,H,Hkv,S,D,P,order,W", [
    (1, 2, 2, 1024, 128, 4, "zigzag", 200),      # MHA: position-paired tiles
    (2, 3, 1, 1024, 64, 2, "zigzag", 384),       # odd group, D = 64, B = 2
    (1, 8, 2, 2048, 128, 2, "contiguous", 512),
    (1, 4, 1, 2048, 128, 8, "zigzag", 129),      # chunks of one tile: tiles far apart
    (1, 2, 1, 512, 128, 1, "zigzag", 100),       # P = 1
    (1, 3, 3, 2048, 128, 8, "zigzag", 333),      # odd group with one-tile chunks
])
def test_window_bf16_forward_shapes(B, H, Hkv, S, D, P, order, W):
    q, k, v = _qkv(B, H, Hkv, S, D, 600 + S + W, torch.bfloat16)
    _check_fwd(q, k, v, P, order, W)


@pytest.mark.parametrize("H,Hkv,S,D,P,order,W", [
    (4, 2, 512, 64, 2, "zigzag", 1),
    (2, 1, 512, 128, 4, "zigzag", 90),
    (2, 2, 768, 64, 3, "contiguous", 200),
])
def test_window_fp32_forward(H, Hkv, S, D, P, order, W):
    q, k, v = _qkv(1, H, Hkv, S, D, 700 + W, torch.float32, 1.0)
    _check_fwd(q, k, v, P, order, W, fp32=True)


def test_window_one_is_the_identity_on_v():
    # W = 1: every query sees only its own key, so O_i = v_i exactly (the
    # softmax weight is 1) and LSE_i = scale * q_i . k_i
    q, k, v = _qkv(1, 4, 2, 1024, 128, 801, torch.bfloat16)
    o, lse = run_fwd(q, k, v, 4, "zigzag", True, window=1)
    vv = v.float().repeat_interleave(2, dim=1)
    assert torch.equal(o, vv)
    s = (q.float() * k.float().repeat_interleave(2, dim=1)).sum(-1) * 128 ** -0.5
    assert_close(lse.numpy(), s.numpy(), LSE_MAX_ABS, what="LSE")


def test_window_covering_the_sequence_is_causal_bitwise():
    import ring_ulysses_sequence_b200 as rm
    q, k, v = (to_rank_major(t, 4, "zigzag").cuda() for t in _qkv(1, 4, 2, 1024, 128, 802, torch.bfloat16))
    o_c, l_c = rm.ring_attn_fwd(q, k, v, 4, True, "zigzag")
    for W in (1024, 5000):
        o_w, l_w = rm.ring_attn_fwd(q, k, v, 4, True, "zigzag", window=W)
        assert torch.equal(o_w, o_c) and torch.equal(l_w, l_c)
    # and a window one short of it is a different computation, still exact
    _check_fwd(*_qkv(1, 4, 2, 1024, 128, 802, torch.bfloat16), 4, "zigzag", 1023)


def test_window_result_independent_of_P_and_order():
    q, k, v = _qkv(1, 4, 2, 2048, 128, 803, torch.bfloat16)
    ref, _ = run_fwd(q, k, v, 1, "zigzag", True, window=300)
    for P, order in ((2, "contiguous"), (4, "zigzag"), (8, "zigzag"), (4, "contiguous")):
        o, _ = run_fwd(q, k, v, P, order, True, window=300)
        assert_close(o.numpy(), ref.numpy(), BF16_MAX_ABS, BF16_MEAN_ABS, f"P={P} {order}")


def gpu_grads(qn, kn, vn, don, P, order, W):
    import ring_ulysses_sequence_b200 as rm
    q, k, v, do = (to_rank_major(t, P, order).cuda() for t in (qn, kn, vn, don))
    o, lse = rm.ring_attn_fwd(q, k, v, P, True, order, window=W)
    dq, dk, dv = rm.ring_attn_bwd(q, k, v, o, lse, do, P, True, order, window=W)
    torch.cuda.synchronize()
    assert rm.native.rm_check_device_status() == 0
    return tuple(to_natural(t.cpu(), P, order) for t in (dq, dk, dv))


@pytest.mark.parametrize("B,H,Hkv,S,D,P,order,W", [
    (1, 2, 2, 1024, 128, 4, "zigzag", 1),
    (1, 4, 2, 1024, 128, 4, "zigzag", 129),
    (1, 4, 2, 1024, 128, 2, "contiguous", 300),
    (2, 3, 1, 512, 64, 2, "zigzag", 128),
    (1, 2, 1, 2048, 128, 8, "zigzag", 700),
])
def test_window_backward(B, H, Hkv, S, D, P, order, W, bwd_kernels):
    q, k, v = _qkv(B, H, Hkv, S, D, 900 + W, torch.bfloat16)
    do = make_tensor((B, H, S, D), 950 + W, torch.bfloat16, 0.5)
    dq, dk, dv = gpu_grads(q, k, v, do, P, order, W)
    rdq, rdkv = oracle.attn_bwd(q.float(), k.float(), v.float(), do.float(), True, window=W)
    for b in range(B):
        for h in range(H):
            assert_close(dq[b, h].numpy(), rdq[(b, h)], BF16_MAX_ABS, BF16_MEAN_ABS, f"dQ[{b},{h}]")
        for g in range(Hkv):
            assert_close(dk[b, g].numpy(), rdkv[(b, g)][0], BF16_MAX_ABS, BF16_MEAN_ABS, f"dK[{b},{g}]")
            assert_close(dv[b, g].numpy(), rdkv[(b, g)][1], BF16_MAX_ABS, BF16_MEAN_ABS, f"dV[{b},{g}]")
    if W == 1:
        # O_i = v_i: no gradient reaches q or k (only rounding residue of
        # dP - Delta, both dO_i . v_i summed in different orders); dV_i sums
        # dO_i over the group
        assert float(dq.abs().max()) < 1e-5 and float(dk.abs().max()) < 1e-5
        G = H // Hkv
        ref = do.float().reshape(B, Hkv, G, S, D).sum(dim=2)
        assert_close(dv.numpy(), ref.numpy(), 1e-6)


def test_window_workload_sampled_rows():
    """The windowed benchmark workload, in its launch configuration, on seeded rows."""
    w = WORKLOADS["ring_fwd_bf16_S32k_gqa_causal_zigzag_window4k"]
    q, k, v = make_inputs(w)
    rows = sample_rows(w.S, 256, w.seed + 1000, w.chunk)
    _check_fwd(q, k, v, w.P, w.order, w.window, rows=rows)


@pytest.mark.parametrize("W", [1, 100, 257])
def test_window_d64_forward_and_backward(W, bwd_kernels):
    B, H, Hkv, S, D, P, order = 1, 4, 2, 1024, 64, 4, "zigzag"
    q, k, v = _qkv(B, H, Hkv, S, D, 1900 + W, torch.bfloat16)
    _check_fwd(q, k, v, P, order, W)
    do = make_tensor((B, H, S, D), 1950 + W, torch.bfloat16, 0.5)
    dq, dk, dv = gpu_grads(q, k, v, do, P, order, W)
    rdq, rdkv = oracle.attn_bwd(q.float(), k.float(), v.float(), do.float(), True, window=W)
    for h in range(H):
        assert_close(dq[0, h].numpy(), rdq[(0, h)], BF16_MAX_ABS, BF16_MEAN_ABS, f"dQ[{h}]")
    for g in range(Hkv):
        assert_close(dk[0, g].numpy(), rdkv[(0, g)][0], BF16_MAX_ABS, BF16_MEAN_ABS, f"dK[{g}]")
        assert_close(dv[0, g].numpy(), rdkv[(0, g)][1], BF16_MAX_ABS, BF16_MEAN_ABS, f"dV[{g}]")
