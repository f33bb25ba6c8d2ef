"""Packed variable-length documents on the GPU against the fp64 oracle.

A query sees keys of its own document only (axolotl-ringmaster README, Status
table: packing / varlen), causal or not, optionally with a sliding window.
Document boundaries are chosen to fall inside tiles, on tile and chunk edges,
to make one-token and empty documents, and documents that span ranks, so that
every tile class and per-row mask occurs. Tolerances as for plain attention.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import (BF16_MAX_ABS, BF16_MEAN_ABS, FP32_MAX_ABS, LSE_MAX_ABS, assert_close,
                      to_natural, to_rank_major)
from ring_ulysses_sequence_b200.synth import WORKLOADS, make_inputs, make_tensor, sample_rows

pytestmark = pytest.mark.gpu

DOCS_1K = {
    "mixed": [0, 3, 130, 131, 512, 700, 1024],
    "tile_edges": [0, 128, 256, 640, 1024],
    "one_token_and_empty": [0, 1, 1, 2, 300, 300, 1023, 1024],
    "single": [0, 1024],
    "many": list(range(0, 1024, 37)) + [1024],
}


def _qkv(B, H, Hkv, S, D, seed, dtype, scale=0.5):
    return (make_tensor((B, H, S, D), seed, dtype, scale),
            make_tensor((B, Hkv, S, D), seed + 1, dtype, scale),
            make_tensor((B, Hkv, S, D), seed + 2, dtype, scale))


def _fwd(qn, kn, vn, P, order, cu, causal, window=0):
    import ring_ulysses_sequence_b200 as rm
    q, k, v = (to_rank_major(t, P, order).cuda() for t in (qn, kn, vn))
    table = rm.varlen_bounds(cu, qn.shape[2], causal, window)
    o, lse = rm.ring_attn_fwd(q, k, v, P, causal, order, bounds=table)
    torch.cuda.synchronize()
    assert rm.native.rm_check_device_status() == 0
    return (to_natural(o.float().cpu(), P, order),
            to_natural(lse.cpu().unsqueeze(-1), P, order).squeeze(-1))


def _check(q, k, v, P, order, cu, causal, window=0, fp32=False, rows=None):
    o, lse = _fwd(q, k, v, P, order, cu, causal, window)
    o_ref, lse_ref = oracle.attn_fwd(q.float(), k.float(), v.float(), causal, rows=rows,
                                     window=window, cu_seqlens=cu)
    if rows is not None:
        o, lse = o[:, :, rows], lse[:, :, rows]
    what = f"docs {len(cu) - 1} causal={causal} W={window}"
    if fp32:
        assert_close(o.numpy(), o_ref, FP32_MAX_ABS, what="O " + what)
    else:
        assert_close(o.numpy(), o_ref, BF16_MAX_ABS, BF16_MEAN_ABS, what="O " + what)
    assert_close(lse.numpy(), lse_ref, LSE_MAX_ABS, what="LSE " + what)


@pytest.mark.parametrize("docs", sorted(DOCS_1K))
@pytest.mark.parametrize("causal,window", [(True, 0), (False, 0), (True, 200)])
def test_varlen_bf16_forward(docs, causal, window):
    q, k, v = _qkv(1, 4, 2, 1024, 128, 1100 + len(docs), torch.bfloat16)
    _check(q, k, v, 4, "zigzag", DOCS_1K[docs], causal, window)


@pytest.mark.parametrize("B,H,Hkv,S,D,P,order,causal", [
    (1, 2, 2, 1024, 128, 4, "zigzag", True),      # MHA: position-paired tiles
    (2, 3, 1, 1024, 64, 2, "zigzag", True),       # odd group, D = 64, B = 2
    (1, 8, 2, 2048, 128, 2, "contiguous", False),
    (1, 4, 1, 2048, 128, 8, "zigzag", True),      # chunks of one tile
])
def test_varlen_bf16_forward_shapes(B, H, Hkv, S, D, P, order, causal):
    cu = [0, 77, 500, 1300, 1301, S] if S == 2048 else [0, 77, 500, 501, 900, S]
    q, k, v = _qkv(B, H, Hkv, S, D, 1200 + S + H, torch.bfloat16)
    _check(q, k, v, P, order, cu, causal)


@pytest.mark.parametrize("causal", [True, False])
def test_varlen_fp32_forward(causal):
    q, k, v = _qkv(1, 2, 1, 512, 64, 1300, torch.float32, 1.0)
    _check(q, k, v, 2, "zigzag", [0, 10, 200, 201, 512], causal, fp32=True)


def test_varlen_one_document_is_plain_attention_bitwise():
    import ring_ulysses_sequence_b200 as rm
    qn, kn, vn = _qkv(1, 4, 2, 1024, 128, 1400, torch.bfloat16)
    q, k, v = (to_rank_major(t, 4, "zigzag").cuda() for t in (qn, kn, vn))
    for causal in (True, False):
        o1, l1 = rm.ring_attn_fwd(q, k, v, 4, causal, "zigzag")
        table = rm.varlen_bounds([0, 1024], 1024, causal)
        o2, l2 = rm.ring_attn_fwd(q, k, v, 4, causal, "zigzag", bounds=table)
        assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_varlen_result_independent_of_P_and_order():
    cu = [0, 300, 301, 1500, 2048]
    q, k, v = _qkv(1, 4, 2, 2048, 128, 1500, torch.bfloat16)
    ref, _ = _fwd(q, k, v, 1, "zigzag", cu, True)
    for P, order in ((2, "contiguous"), (4, "zigzag"), (8, "zigzag")):
        o, _ = _fwd(q, k, v, P, order, cu, True)
        assert_close(o.numpy(), ref.numpy(), BF16_MAX_ABS, BF16_MEAN_ABS, f"P={P} {order}")


@pytest.mark.parametrize("cu,causal,window", [
    ([0, 3, 130, 131, 512, 700, 1024], True, 0),
    ([0, 128, 256, 640, 1024], False, 0),
    ([0, 1, 1, 2, 300, 1023, 1024], True, 150),
])
def test_varlen_backward(cu, causal, window, bwd_kernels):
    import ring_ulysses_sequence_b200 as rm
    B, H, Hkv, S, D, P, order = 1, 4, 2, 1024, 128, 4, "zigzag"
    qn, kn, vn = _qkv(B, H, Hkv, S, D, 1600 + len(cu), torch.bfloat16)
    don = make_tensor((B, H, S, D), 1650 + len(cu), torch.bfloat16, 0.5)
    q, k, v, do = (to_rank_major(t, P, order).cuda() for t in (qn, kn, vn, don))
    table = rm.varlen_bounds(cu, S, causal, window)
    o, lse = rm.ring_attn_fwd(q, k, v, P, causal, order, bounds=table)
    dq, dk, dv = rm.ring_attn_bwd(q, k, v, o, lse, do, P, causal, order, bounds=table)
    torch.cuda.synchronize()
    assert rm.native.rm_check_device_status() == 0
    dq, dk, dv = (to_natural(t.cpu(), P, order) for t in (dq, dk, dv))
    rdq, rdkv = oracle.attn_bwd(qn.float(), kn.float(), vn.float(), don.float(), causal,
                                window=window, cu_seqlens=cu)
    for h in range(H):
        assert_close(dq[0, h].numpy(), rdq[(0, h)], BF16_MAX_ABS, BF16_MEAN_ABS, f"dQ[{h}]")
    for g in range(Hkv):
        assert_close(dk[0, g].numpy(), rdkv[(0, g)][0], BF16_MAX_ABS, BF16_MEAN_ABS, f"dK[{g}]")
        assert_close(dv[0, g].numpy(), rdkv[(0, g)][1], BF16_MAX_ABS, BF16_MEAN_ABS, f"dV[{g}]")


def test_varlen_workload_sampled_rows():
    """The packed-documents benchmark workload, in its launch configuration."""
    w = WORKLOADS["ring_fwd_bf16_S32k_gqa_causal_zigzag_packed"]
    q, k, v = make_inputs(w)
    rows = sample_rows(w.S, 256, w.seed + 1000, w.chunk)
    rows = np.unique(np.concatenate([rows, np.array(w.cu_seqlens[1:-1]), np.array(w.cu_seqlens[1:-1]) - 1]))
    _check(q, k, v, w.P, w.order, list(w.cu_seqlens), w.causal, rows=rows)


@pytest.mark.parametrize("B,H,Hkv,D,causal", [(2, 4, 4, 64, True), (3, 2, 1, 128, False)])
def test_varlen_batched_and_d64(B, H, Hkv, D, causal):
    # every batch row uses the same documents; D = 64 takes the other tile shape
    cu = [0, 200, 201, 700, 1024]
    q, k, v = _qkv(B, H, Hkv, 1024, D, 1700 + B + D, torch.bfloat16)
    _check(q, k, v, 4, "zigzag", cu, causal)


def test_varlen_backward_d64_batched(bwd_kernels):
    import ring_ulysses_sequence_b200 as rm
    B, H, Hkv, S, D, P, order, cu = 2, 2, 1, 512, 64, 2, "contiguous", [0, 100, 356, 512]
    qn, kn, vn = _qkv(B, H, Hkv, S, D, 1800, torch.bfloat16)
    don = make_tensor((B, H, S, D), 1804, torch.bfloat16, 0.5)
    q, k, v, do = (to_rank_major(t, P, order).cuda() for t in (qn, kn, vn, don))
    table = rm.varlen_bounds(cu, S, True)
    o, lse = rm.ring_attn_fwd(q, k, v, P, True, order, bounds=table)
    dq, dk, dv = rm.ring_attn_bwd(q, k, v, o, lse, do, P, True, order, bounds=table)
    torch.cuda.synchronize()
    dq, dk, dv = (to_natural(t.cpu(), P, order) for t in (dq, dk, dv))
    rdq, rdkv = oracle.attn_bwd(qn.float(), kn.float(), vn.float(), don.float(), True,
                                cu_seqlens=cu)
    for b in range(B):
        for h in range(H):
            assert_close(dq[b, h].numpy(), rdq[(b, h)], BF16_MAX_ABS, BF16_MEAN_ABS, f"dQ[{b},{h}]")
        assert_close(dk[b, 0].numpy(), rdkv[(b, 0)][0], BF16_MAX_ABS, BF16_MEAN_ABS, f"dK[{b}]")
        assert_close(dv[b, 0].numpy(), rdkv[(b, 0)][1], BF16_MAX_ABS, BF16_MEAN_ABS, f"dV[{b}]")
