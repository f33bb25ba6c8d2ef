"""Edge cases of the attention path on the GPU against the fp64 oracle.

* Ragged lengths. The kernels tile the sequence in 128-token tiles that never
  straddle a chunk, so a length that is not a multiple of 2P x 128 (zigzag)
  is padded to one, and the padding is masked off as a document of its own
  (the packed-documents mask, axolotl-ringmaster README: packing / varlen):
  real queries see real keys only. The oracle computes the unpadded attention
  of the real tokens alone, and the real rows of the GPU result must match it
  (forward, and the backward with zero upstream gradient on the padding).
* The largest sequence the kernels are meant for in one launch here,
  S = 2^20 tokens (row indices near the 32-bit limits of the tile
  addressing), checked on seeded sampled rows.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import (BF16_MAX_ABS, BF16_MEAN_ABS, LSE_MAX_ABS, assert_close, to_natural,
                      to_rank_major)
from ring_ulysses_sequence_b200.synth import make_tensor, sample_rows

pytestmark = pytest.mark.gpu


def _padded_len(S_real, P, order):
    unit = 2 * P * 128 if order == "zigzag" else P * 256
    return -(-S_real // unit) * unit


@pytest.mark.parametrize("S_real,P,order,causal", [
    (1000, 2, "zigzag", True),
    (777, 4, "zigzag", True),
    (129, 1, "zigzag", True),
    (1, 2, "zigzag", True),
    (1500, 2, "contiguous", False),
])
def test_ragged_length_padded_and_masked(S_real, P, order, causal, bwd_kernels):
    import ring_ulysses_sequence_b200 as rm
    B, H, Hkv, D = 1, 4, 2, 128
    S = _padded_len(S_real, P, order)
    seed = 3000 + S_real
    q = make_tensor((B, H, S, D), seed, torch.bfloat16, 0.5)
    k = make_tensor((B, Hkv, S, D), seed + 1, torch.bfloat16, 0.5)
    v = make_tensor((B, Hkv, S, D), seed + 2, torch.bfloat16, 0.5)
    do = make_tensor((B, H, S, D), seed + 3, torch.bfloat16, 0.5)
    do[:, :, S_real:] = 0  # the padding takes no part in the loss
    cu = [0, S_real, S] if S > S_real else [0, S]
    qr, kr, vr, dor = (to_rank_major(t, P, order).cuda() for t in (q, k, v, do))
    table = rm.varlen_bounds(cu, S, causal)
    o, lse = rm.ring_attn_fwd(qr, kr, vr, P, causal, order, bounds=table)
    dq, dk, dv = rm.ring_attn_bwd(qr, kr, vr, o, lse, dor, P, causal, order, bounds=table)
    torch.cuda.synchronize()
    assert rm.native.rm_check_device_status() == 0
    o, dq, dk, dv = (to_natural(t.float().cpu(), P, order)[:, :, :S_real] for t in (o, dq, dk, dv))
    lse = to_natural(lse.cpu().unsqueeze(-1), P, order).squeeze(-1)[:, :, :S_real]
    real = [t[:, :, :S_real].float() for t in (q, k, v, do)]
    o_ref, lse_ref = oracle.attn_fwd(*real[:3], causal)
    assert_close(o.numpy(), o_ref, BF16_MAX_ABS, BF16_MEAN_ABS, "O")
    assert_close(lse.numpy(), lse_ref, LSE_MAX_ABS, what="LSE")
    rdq, rdkv = oracle.attn_bwd(*real, causal)
    for h in range(H):
        assert_close(dq[0, h].numpy(), rdq[(0, h)], BF16_MAX_ABS, BF16_MEAN_ABS, f"dQ[{h}]")
    for g in range(Hkv):
        assert_close(dk[0, g].numpy(), rdkv[(0, g)][0], BF16_MAX_ABS, BF16_MEAN_ABS, f"dK[{g}]")
        assert_close(dv[0, g].numpy(), rdkv[(0, g)][1], BF16_MAX_ABS, BF16_MEAN_ABS, f"dV[{g}]")


def test_one_million_tokens_sampled_rows():
    """S = 2^20, two query heads over one KV head, P = 8 zigzag, causal:
    forward O/LSE and dQ on 256 seeded rows per head plus chunk edges."""
    import ring_ulysses_sequence_b200 as rm
    B, H, Hkv, S, D, P, order = 1, 2, 1, 1 << 20, 128, 8, "zigzag"
    q = make_tensor((B, H, S, D), 3100, torch.bfloat16, 0.5)
    k = make_tensor((B, Hkv, S, D), 3101, torch.bfloat16, 0.5)
    v = make_tensor((B, Hkv, S, D), 3102, torch.bfloat16, 0.5)
    do = make_tensor((B, H, S, D), 3103, torch.bfloat16, 0.5)
    qr, kr, vr, dor = (to_rank_major(t, P, order).cuda() for t in (q, k, v, do))
    o, lse = rm.ring_attn_fwd(qr, kr, vr, P, True, order)
    dq, _, _ = rm.ring_attn_bwd(qr, kr, vr, o, lse, dor, P, True, order)
    torch.cuda.synchronize()
    assert rm.native.rm_check_device_status() == 0
    rows = sample_rows(S, 256, 3104, S // (2 * P))
    o = to_natural(o.float().cpu(), P, order)[:, :, rows]
    lse = to_natural(lse.cpu().unsqueeze(-1), P, order).squeeze(-1)[:, :, rows]
    dq = to_natural(dq.cpu(), P, order)[:, :, rows]
    o_ref, lse_ref = oracle.attn_fwd(q.float(), k.float(), v.float(), True, rows=rows)
    assert_close(o.numpy(), o_ref, BF16_MAX_ABS, BF16_MEAN_ABS, "O")
    assert_close(lse.numpy(), lse_ref, LSE_MAX_ABS, what="LSE")
    rdq, _ = oracle.attn_bwd(q.float(), k.float(), v.float(), do.float(), True, qrows=rows,
                             krows=np.zeros(0, dtype=np.int64),
                             heads=([(0, h) for h in range(H)], []))
    for h in range(H):
        assert_close(dq[0, h].numpy(), rdq[(0, h)], BF16_MAX_ABS, BF16_MEAN_ABS, f"dQ[{h}]")
