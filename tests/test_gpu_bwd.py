"""Ring attention backward on the GPU against the fp64 oracle's analytic gradients.

The GPU gets O and LSE from its own forward (as a training step would); the
oracle differentiates exact attention. Tolerances as for O: max-abs 2e-2,
mean-abs 2e-3 on dQ, dK, dV (fp32 outputs of bf16 inputs). The default
backward is the two-kernel (bitwise reproducible) one, also checked for
determinism; the fused kernel (dQ by reductions) is checked against it.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import (BF16_MAX_ABS, BF16_MEAN_ABS, LSE_MAX_ABS, assert_close, to_natural,
                      to_rank_major)
from ring_ulysses_sequence_b200.synth import WORKLOADS, make_inputs, make_tensor, sample_rows

pytestmark = pytest.mark.gpu


def gpu_grads(qn, kn, vn, don, P, order, causal):
    """Natural-order CPU inputs -> GPU forward + backward -> natural-order fp32 grads."""
    import ring_ulysses_sequence_b200 as rm
    q, k, v, do = (to_rank_major(t, P, order).cuda() for t in (qn, kn, vn, don))
    o, lse = rm.ring_attn_fwd(q, k, v, P, causal, order)
    dq, dk, dv = rm.ring_attn_bwd(q, k, v, o, lse, do, P, causal, order)
    torch.cuda.synchronize()
    assert rm.native.rm_check_device_status() == 0
    return tuple(to_natural(t.cpu(), P, order) for t in (dq, dk, dv))


def _inputs(B, H, Hkv, S, D, seed, scale=0.5):
    q = make_tensor((B, H, S, D), seed, torch.bfloat16, scale)
    k = make_tensor((B, Hkv, S, D), seed + 1, torch.bfloat16, scale)
    v = make_tensor((B, Hkv, S, D), seed + 2, torch.bfloat16, scale)
    do = make_tensor((B, H, S, D), seed + 3, torch.bfloat16, scale)
    return q, k, v, do


@pytest.mark.parametrize("B,H,Hkv,S,D,P,order,causal", [
    (1, 2, 2, 1024, 128, 4, "zigzag", True),
    (1, 4, 2, 1024, 128, 2, "zigzag", True),      # GQA: dK/dV summed over 2 heads
    (2, 3, 1, 512, 64, 2, "contiguous", True),    # group 3, D = 64, B = 2
    (1, 2, 2, 1024, 128, 4, "zigzag", False),
    (1, 4, 1, 512, 128, 1, "zigzag", True),       # P = 1, MQA
])
def test_bwd_shapes_full(B, H, Hkv, S, D, P, order, causal):
    q, k, v, do = _inputs(B, H, Hkv, S, D, 300 + S + H)
    dq, dk, dv = gpu_grads(q, k, v, do, P, order, causal)
    rdq, rdkv = oracle.attn_bwd(q.float(), k.float(), v.float(), do.float(), causal)
    for b in range(B):
        for h in range(H):
            assert_close(dq[b, h].numpy(), rdq[(b, h)], BF16_MAX_ABS, BF16_MEAN_ABS, f"dQ[{b},{h}]")
        for g in range(Hkv):
            assert_close(dk[b, g].numpy(), rdkv[(b, g)][0], BF16_MAX_ABS, BF16_MEAN_ABS, f"dK[{b},{g}]")
            assert_close(dv[b, g].numpy(), rdkv[(b, g)][1], BF16_MAX_ABS, BF16_MEAN_ABS, f"dV[{b},{g}]")
    # identities of the exact gradient, up to the bf16 tolerance:
    # sum_j dK_j = 0, sum_j dV_j = sum over the group's heads of sum_i dO_i
    G = H // Hkv
    dsum = do.float().reshape(B, Hkv, G, S, D).sum(dim=(2, 3))
    assert_close(dv.sum(dim=2).numpy(), dsum.numpy(), 0.5)
    assert float(dk.sum(dim=2).abs().max()) < 0.5


@pytest.fixture
def deterministic_bwd():
    """Selects the two-kernel (bitwise reproducible) backward for one test."""
    from ring_ulysses_sequence_b200 import native
    before = native.rm_get_bwd_deterministic()
    native.rm_set_bwd_deterministic(1)
    yield
    native.rm_set_bwd_deterministic(before)


def test_bwd_deterministic(deterministic_bwd):
    import ring_ulysses_sequence_b200 as rm
    q, k, v, do = (to_rank_major(t, 4, "zigzag").cuda() for t in _inputs(1, 4, 2, 1024, 128, 77))
    o, lse = rm.ring_attn_fwd(q, k, v, 4, True, "zigzag")
    a = rm.ring_attn_bwd(q, k, v, o, lse, do, 4, True, "zigzag")
    b = rm.ring_attn_bwd(q, k, v, o, lse, do, 4, True, "zigzag")
    for x, y in zip(a, b):
        assert torch.equal(x, y)


@pytest.mark.parametrize("B,H,Hkv,S,D,P,order,causal", [
    (1, 4, 2, 2048, 128, 4, "zigzag", True),
    (2, 3, 1, 1024, 64, 2, "contiguous", True),
    (1, 2, 2, 1024, 128, 4, "zigzag", False),
])
def test_fused_and_two_kernel_backward_agree(B, H, Hkv, S, D, P, order, causal):
    """The fused backward (dQ by reductions) and the default two-kernel one:
    dK and dV come from the same per-element arithmetic; dQ differs only in
    the order of fp32 additions. Both stay within the oracle's tolerance."""
    import ring_ulysses_sequence_b200 as rm
    from ring_ulysses_sequence_b200 import native
    qn, kn, vn, don = _inputs(B, H, Hkv, S, D, 500 + S + H)
    q, k, v, do = (to_rank_major(t, P, order).cuda() for t in (qn, kn, vn, don))
    o, lse = rm.ring_attn_fwd(q, k, v, P, causal, order)
    before = native.rm_get_bwd_deterministic()
    try:
        native.rm_set_bwd_deterministic(0)
        fused = rm.ring_attn_bwd(q, k, v, o, lse, do, P, causal, order)
        native.rm_set_bwd_deterministic(1)
        two = rm.ring_attn_bwd(q, k, v, o, lse, do, P, causal, order)
    finally:
        native.rm_set_bwd_deterministic(before)
    torch.cuda.synchronize()
    assert rm.native.rm_check_device_status() == 0
    for f, t, name in zip(fused, two, ("dQ", "dK", "dV")):
        assert_close(f.cpu().numpy(), t.cpu().numpy(), 1e-3, 1e-5, name)
    rdq, rdkv = oracle.attn_bwd(qn.float(), kn.float(), vn.float(), don.float(), causal)
    gq, gk, gv = (to_natural(t.cpu(), P, order) for t in fused)
    for b in range(B):
        for h in range(H):
            assert_close(gq[b, h].numpy(), rdq[(b, h)], BF16_MAX_ABS, BF16_MEAN_ABS, f"dQ[{b},{h}]")
        for g in range(Hkv):
            assert_close(gk[b, g].numpy(), rdkv[(b, g)][0], BF16_MAX_ABS, BF16_MEAN_ABS, f"dK[{b},{g}]")
            assert_close(gv[b, g].numpy(), rdkv[(b, g)][1], BF16_MAX_ABS, BF16_MEAN_ABS, f"dV[{b},{g}]")


def test_bwd_workload_sampled():
    """B=2, H=Hkv=16, S=65536, D=128, P=16 zigzag, causal (forward + backward).

    Seeded samples as the workload's parity rule states: 256 query rows per
    head (plus the first and last row of every chunk) for the forward's O and
    LSE and for dQ, on every head; 256 key rows (plus chunk edges) for dK and
    dV on four seeded KV heads. The oracle's dK/dV rows need LSE and Delta of
    every query row of those heads, i.e. a full fp64 forward per head."""
    import ring_ulysses_sequence_b200 as rm
    w = WORKLOADS["ring_fwdbwd_bf16_S64k_causal_zigzag"]
    q, k, v, do = make_inputs(w)
    qr, kr, vr, dor = (to_rank_major(t, w.P, w.order).cuda() for t in (q, k, v, do))
    o, lse = rm.ring_attn_fwd(qr, kr, vr, w.P, w.causal, w.order)
    dq, dk, dv = rm.ring_attn_bwd(qr, kr, vr, o, lse, dor, w.P, w.causal, w.order)
    torch.cuda.synchronize()
    assert rm.native.rm_check_device_status() == 0
    o, lse, dq, dk, dv = (to_natural(t.float().cpu(), w.P, w.order)
                          for t in (o, lse.unsqueeze(-1), dq, dk, dv))
    lse = lse.squeeze(-1)
    qrows = sample_rows(w.S, 256, w.seed + 1000, w.chunk)
    krows = sample_rows(w.S, 256, w.seed + 2000, w.chunk)
    rng = np.random.default_rng(w.seed + 3000)
    pairs = [(b, g) for b in range(w.B) for g in range(w.Hkv)]
    kv_heads = [pairs[i] for i in sorted(rng.choice(len(pairs), size=4, replace=False))]
    q_heads = [(b, h) for b in range(w.B) for h in range(w.H)]

    # the forward this backward ran on
    o_ref, lse_ref = oracle.attn_fwd(q.float(), k.float(), v.float(), w.causal, rows=qrows)
    assert_close(o[:, :, qrows].numpy(), o_ref, BF16_MAX_ABS, BF16_MEAN_ABS, "O")
    assert_close(lse[:, :, qrows].numpy(), lse_ref, LSE_MAX_ABS, what="LSE")

    rdq, rdkv = oracle.attn_bwd(q.float(), k.float(), v.float(), do.float(), True, qrows=qrows,
                                krows=krows, heads=(q_heads, kv_heads))
    for (b, h) in q_heads:
        assert_close(dq[b, h][qrows].numpy(), rdq[(b, h)], BF16_MAX_ABS, BF16_MEAN_ABS, f"dQ[{b},{h}]")
    for (b, g) in kv_heads:
        assert_close(dk[b, g][krows].numpy(), rdkv[(b, g)][0], BF16_MAX_ABS, BF16_MEAN_ABS, f"dK[{b},{g}]")
        assert_close(dv[b, g][krows].numpy(), rdkv[(b, g)][1], BF16_MAX_ABS, BF16_MEAN_ABS, f"dV[{b},{g}]")
    # properties at full size: sum_j dK_j = 0 and sum_j dV_j = sum_i dO_i per head
    assert float(dk.sum(dim=2).abs().max()) < 1.0
    assert_close(dv.sum(dim=2).numpy(), do.float().sum(dim=2).numpy(), 1.0)
