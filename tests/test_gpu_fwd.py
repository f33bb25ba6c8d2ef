"""Ring attention forward on the GPU against the fp64 oracle.

Small shapes are compared element by element on every row; the full-size
workloads on seeded query rows (plus every chunk's first and last row), in the
launch configuration the benchmark times. Tolerances: bf16 inputs with fp32
accumulation, O max-abs 2e-2 and mean-abs 2e-3; fp32 path O max-abs 1e-4;
LSE max-abs 1e-3.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from gpu_util import (BF16_MAX_ABS, BF16_MEAN_ABS, FP32_MAX_ABS, LSE_MAX_ABS, ORDER,
                      assert_close, run_fwd, to_natural, to_rank_major)
from ring_ulysses_sequence_b200.synth import WORKLOADS, make_inputs, make_tensor, sample_rows

pytestmark = pytest.mark.gpu


def _qkv(B, H, Hkv, S, D, seed, dtype, scale=0.5):
    q = make_tensor((B, H, S, D), seed, dtype, scale)
    k = make_tensor((B, Hkv, S, D), seed + 1, dtype, scale)
    v = make_tensor((B, Hkv, S, D), seed + 2, dtype, scale)
    return q, k, v


def _check(qn, kn, vn, P, order, causal, dtype, rows=None, scale=None):
    o, lse = run_fwd(qn, kn, vn, P, order, causal, scale)
    o_ref, lse_ref = oracle.attn_fwd(qn.float(), kn.float(), vn.float(), causal, scale, rows=rows)
    if rows is not None:
        o, lse = o[:, :, rows], lse[:, :, rows]
    if dtype == torch.float32:
        assert_close(o.numpy(), o_ref, FP32_MAX_ABS, what="O")
    else:
        assert_close(o.numpy(), o_ref, BF16_MAX_ABS, BF16_MEAN_ABS, what="O")
    assert_close(lse.numpy(), lse_ref, LSE_MAX_ABS, what="LSE")
    return o, lse


# ---------------------------------------------------------------- fp32 path

def test_fp32_workload_S1k_full():
    w = WORKLOADS["ring_fwd_fp32_S1k"]
    q, k, v = make_inputs(w)
    _check(q, k, v, w.P, w.order, w.causal, torch.float32)


@pytest.mark.parametrize("H,Hkv,S,D,P,order,causal", [
    (4, 2, 512, 64, 2, "zigzag", True),
    (2, 1, 256, 128, 1, "contiguous", True),
    (3, 3, 768, 64, 3, "contiguous", False),
])
def test_fp32_shapes(H, Hkv, S, D, P, order, causal):
    q, k, v = _qkv(1, H, Hkv, S, D, 10 + S, torch.float32, 1.0)
    _check(q, k, v, P, order, causal, torch.float32)


# ---------------------------------------------------------------- bf16 tensor-core path

@pytest.mark.parametrize("B,H,Hkv,S,D,P,order,causal", [
    (1, 2, 2, 1024, 128, 4, "zigzag", True),       # MHA: position-paired tiles
    (1, 4, 2, 1024, 128, 4, "zigzag", True),       # GQA group 2: head-paired tiles
    (1, 8, 2, 1024, 128, 4, "contiguous", True),   # group 4
    (2, 3, 1, 1024, 64, 2, "zigzag", True),        # group 3 (odd), D = 64, B = 2
    (1, 4, 4, 1024, 128, 4, "zigzag", False),
    (1, 2, 1, 512, 128, 1, "zigzag", True),        # P = 1: no ring at all
    (1, 4, 1, 2048, 128, 8, "zigzag", True),       # MQA, chunk of one tile
    (1, 2, 2, 4096, 64, 2, "contiguous", False),
])
def test_bf16_shapes_full(B, H, Hkv, S, D, P, order, causal):
    q, k, v = _qkv(B, H, Hkv, S, D, 100 + S + H, torch.bfloat16)
    _check(q, k, v, P, order, causal, torch.bfloat16)


def test_bf16_hard_softmax():
    """Large logits (queries and keys x4, with planted near-duplicate keys) make
    the row maximum jump between tiles and ring steps, exercising the O
    rescale. Values stay at the workloads' scale (0.5), so the O tolerance of
    the workloads applies unchanged."""
    B, H, Hkv, S, D, P = 1, 4, 2, 2048, 128, 4
    q, k, _ = _qkv(B, H, Hkv, S, D, 7, torch.float32, 4.0)
    v = make_tensor((B, Hkv, S, D), 9, torch.float32, 0.5)
    g = torch.Generator().manual_seed(8)
    idx = torch.randint(0, S, (64,), generator=g)
    for j, i in enumerate(idx.tolist()):   # key i ~ a scaled copy of query row j
        k[0, :, i] = q[0, ::2, j] * 1.5
    q, k, v = q.bfloat16(), k.bfloat16(), v.bfloat16()
    for causal in (True, False):
        _check(q, k, v, P, "zigzag", causal, torch.bfloat16)


def test_result_independent_of_P_and_order():
    """Ring = dense for every P and both chunk orders (after un-permuting)."""
    B, H, Hkv, S, D = 1, 4, 2, 4096, 128
    q, k, v = _qkv(B, H, Hkv, S, D, 21, torch.bfloat16)
    o_ref, l_ref = oracle.attn_fwd(q.float(), k.float(), v.float(), True)
    outs = []
    for P, order in ((1, "zigzag"), (2, "zigzag"), (4, "zigzag"), (8, "zigzag"),
                     (2, "contiguous"), (8, "contiguous")):
        o, lse = run_fwd(q, k, v, P, order, True)
        assert_close(o.numpy(), o_ref, BF16_MAX_ABS, BF16_MEAN_ABS, what=f"O P={P} {order}")
        assert_close(lse.numpy(), l_ref, LSE_MAX_ABS, what=f"LSE P={P} {order}")
        outs.append(o)
    for o in outs[1:]:
        assert_close(o.numpy(), outs[0].numpy(), 2 * BF16_MAX_ABS, 2 * BF16_MEAN_ABS)


def test_deterministic_and_custom_scale():
    import ring_ulysses_sequence_b200 as rm
    q, k, v = _qkv(1, 4, 2, 2048, 128, 31, torch.bfloat16)
    P, order = 4, "zigzag"
    qg, kg, vg = (to_rank_major(t, P, order).cuda() for t in (q, k, v))
    o1, l1 = rm.ring_attn_fwd(qg, kg, vg, P, True, order, scale=0.05)
    o2, l2 = rm.ring_attn_fwd(qg, kg, vg, P, True, order, scale=0.05)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    _check(q, k, v, P, order, True, torch.bfloat16, scale=0.05)


def test_gpu_reorder_feeds_forward():
    """End to end with the library's own reorder kernel on both sides."""
    import ring_ulysses_sequence_b200 as rm
    q, k, v = _qkv(1, 4, 4, 2048, 128, 41, torch.bfloat16)
    P, order = 4, "zigzag"
    qg, kg, vg = (rm.seq_reorder(t.cuda(), P, order, "to_rank_major") for t in (q, k, v))
    o, lse = rm.ring_attn_fwd(qg, kg, vg, P, True, order)
    o_nat = rm.seq_reorder(o, P, order, "to_natural").float().cpu()
    l_nat = rm.seq_reorder(lse, P, order, "to_natural").cpu()
    o_ref, l_ref = oracle.attn_fwd(q.float(), k.float(), v.float(), True)
    assert_close(o_nat.numpy(), o_ref, BF16_MAX_ABS, BF16_MEAN_ABS)
    assert_close(l_nat.numpy(), l_ref, LSE_MAX_ABS)


def test_empty_and_unsupported():
    import ring_ulysses_sequence_b200 as rm
    e = torch.empty((0, 2, 1024, 128), dtype=torch.bfloat16, device="cuda")
    rm.ring_attn_fwd(e, e, e, 4)                       # empty batch: a no-op
    q = torch.zeros((1, 2, 1000, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(rm.RMError):                    # ragged length: rejected
        rm.ring_attn_fwd(q, q, q, 4)
    q = torch.zeros((1, 2, 1024, 96), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(rm.RMError):                    # unsupported head dim
        rm.ring_attn_fwd(q, q, q, 4)


# ---------------------------------------------------------------- full-size workloads

@pytest.mark.parametrize("name,nrows", [("ring_fwd_bf16_S8k_causal_zigzag", 1024),
                                        ("ring_fwd_bf16_S32k_gqa_causal_zigzag", 256)])
def test_workload_sampled_rows(name, nrows):
    w = WORKLOADS[name]
    q, k, v = make_inputs(w)
    rows = sample_rows(w.S, nrows, w.seed + 1000, w.chunk)
    _check(q, k, v, w.P, w.order, w.causal, torch.bfloat16, rows=rows)


def test_usp_workload_permute_ring_permute():
    """Ulysses x Ring on the 131072-token workload: sequence-sharded input ->
    head-sharded (fused Q/K/V permute) -> ring attention over R ranks ->
    sequence-sharded output. Permutes bit-exact; attention on sampled rows."""
    import ring_ulysses_sequence_b200 as rm
    w = WORKLOADS["usp_fwd_bf16_S128k_u4r4"]
    U, R = w.ulysses, w.P
    qn, kn, vn = make_inputs(w)
    # sequence-sharded rank-major [B, S, heads, D]: shard n = r*U + u holds tokens [n*T, (n+1)*T)
    seq = [to_rank_major(t, R, w.order).transpose(1, 2).contiguous() for t in (qn, kn, vn)]
    qh, kh, vh = rm.ulysses_permute_qkv(*(t.cuda() for t in seq), U, R, "seq_to_head")
    for got, t in zip((qh, kh, vh), seq):
        assert torch.equal(got.cpu(), t.transpose(1, 2).contiguous())
    o, lse = rm.ring_attn_fwd(qh, kh, vh, R, causal=True, order=w.order)
    o_seq = rm.ulysses_permute(o, U, R, "head_to_seq")
    torch.cuda.synchronize()
    assert rm.native.rm_check_device_status() == 0
    o_nat = to_natural(o_seq.cpu().transpose(1, 2), R, w.order)
    l_nat = to_natural(lse.cpu().unsqueeze(-1), R, w.order).squeeze(-1)
    rows = sample_rows(w.S, 256, w.seed + 1000, w.chunk)
    o_ref, l_ref = oracle.attn_fwd(qn.float(), kn.float(), vn.float(), True, rows=rows)
    assert_close(o_nat[:, :, rows].float().numpy(), o_ref, BF16_MAX_ABS, BF16_MEAN_ABS, what="O")
    assert_close(l_nat[:, :, rows].numpy(), l_ref, LSE_MAX_ABS, what="LSE")


def test_watchdog_reports_timeout_without_hanging():
    import ring_ulysses_sequence_b200 as rm
    assert rm.native.rm_check_device_status() == 0
    rm.native.rm_watchdog_selftest(2_000_000)          # 2 ms on a barrier nobody completes
    assert rm.native.rm_check_device_status() == rm.native.RM_ERR_TIMEOUT
    assert rm.native.rm_check_device_status() == 0     # the word is cleared by the read
    q, k, v = _qkv(1, 2, 2, 1024, 128, 51, torch.bfloat16)
    _check(q, k, v, 4, "zigzag", True, torch.bfloat16)  # the context is still usable
