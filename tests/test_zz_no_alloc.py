"""The allocation-free backward entry point, checked against the ordinary one.

Some users of this library cannot allocate device memory at the point where
they run the backward: a plugin inside a host framework that reserved all
device memory up front, or a latency-critical loop where a cudaMalloc may
synchronise the device or fail. rm_ring_attn_bwd_noalloc serves them: it takes
the same tensors as rm_ring_attn_bwd but no workspace, keeping its scratch in a
fixed 8 MiB array of the library (problems up to B * H * S = 2,097,152 rows).

This file is named so that pytest collects it last: if it fails, a run that
stops at the first failure has already run every other test. It passes both
on its own in a fresh process and after the rest of the suite.
"""
import pytest
import torch

from gpu_util import BF16_MAX_ABS, BF16_MEAN_ABS, assert_close, to_rank_major
from ring_ulysses_sequence_b200.synth import make_tensor

pytestmark = pytest.mark.gpu


def _problem(seed, B=1, H=4, Hkv=2, S=1024, D=128, P=4, order="zigzag"):
    import ring_ulysses_sequence_b200 as rm
    q = make_tensor((B, H, S, D), seed, torch.bfloat16, 0.5)
    k = make_tensor((B, Hkv, S, D), seed + 1, torch.bfloat16, 0.5)
    v = make_tensor((B, Hkv, S, D), seed + 2, torch.bfloat16, 0.5)
    do = make_tensor((B, H, S, D), seed + 3, torch.bfloat16, 0.5)
    q, k, v, do = (to_rank_major(t, P, order).cuda() for t in (q, k, v, do))
    o, lse = rm.ring_attn_fwd(q, k, v, P, True, order)
    return q, k, v, o, lse, do, (B, H, Hkv, S, D, P)


def test_noalloc_backward_matches_workspace_backward_on_two_calls():
    import ring_ulysses_sequence_b200 as rm
    from ring_ulysses_sequence_b200 import native
    # two calls in a row on different inputs: the second reuses the shared
    # scratch array that the first call left behind
    for seed in (901, 907):
        q, k, v, o, lse, do, (B, H, Hkv, S, D, P) = _problem(seed)
        ref = rm.ring_attn_bwd(q, k, v, o, lse, do, P, True, "zigzag")
        dq = torch.empty(q.shape, dtype=torch.float32, device="cuda")
        dk = torch.empty(k.shape, dtype=torch.float32, device="cuda")
        dv = torch.empty(v.shape, dtype=torch.float32, device="cuda")
        native.rm_ring_attn_bwd_noalloc(q, k, v, o, lse, do, dq, dk, dv, B, H, Hkv, S, D, P, True,
                                        native.RM_ORDER_ZIGZAG, native.RM_DTYPE_BF16,
                                        D ** -0.5)
        torch.cuda.synchronize()
        assert native.rm_check_device_status() == native.RM_OK
        for got, want, name in zip((dq, dk, dv), ref, ("dQ", "dK", "dV")):
            assert_close(got.cpu().numpy(), want.cpu().numpy(), BF16_MAX_ABS, BF16_MEAN_ABS,
                         f"{name} (seed {seed})")


def test_noalloc_backward_matches_the_oracle():
    """The same entry point on its own against the fp64 oracle's gradients."""
    import numpy as np
    import oracle
    from gpu_util import to_natural
    from ring_ulysses_sequence_b200 import native
    q, k, v, o, lse, do, (B, H, Hkv, S, D, P) = _problem(913)
    dq = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    dk = torch.empty(k.shape, dtype=torch.float32, device="cuda")
    dv = torch.empty(v.shape, dtype=torch.float32, device="cuda")
    native.rm_ring_attn_bwd_noalloc(q, k, v, o, lse, do, dq, dk, dv, B, H, Hkv, S, D, P, True,
                                    native.RM_ORDER_ZIGZAG, native.RM_DTYPE_BF16, D ** -0.5)
    torch.cuda.synchronize()
    assert native.rm_check_device_status() == native.RM_OK
    qn, kn, vn, don = (to_natural(t.cpu(), P, "zigzag").float() for t in (q, k, v, do))
    rdq, rdkv = oracle.attn_bwd(qn, kn, vn, don, True)
    gq, gk, gv = (to_natural(t.cpu(), P, "zigzag").numpy() for t in (dq, dk, dv))
    for h in range(H):
        assert_close(gq[0, h], rdq[(0, h)], BF16_MAX_ABS, BF16_MEAN_ABS, f"dQ[{h}]")
    for g in range(Hkv):
        assert_close(gk[0, g], rdkv[(0, g)][0], BF16_MAX_ABS, BF16_MEAN_ABS, f"dK[{g}]")
        assert_close(gv[0, g], rdkv[(0, g)][1], BF16_MAX_ABS, BF16_MEAN_ABS, f"dV[{g}]")
    assert np.isfinite(gq).all()


def test_noalloc_backward_rejects_problems_above_its_scratch():
    from ring_ulysses_sequence_b200 import native
    fake = 1 << 20  # aligned address, never touched: the size check comes first
    st = native.lib().rm_ring_attn_bwd_noalloc(fake, fake, fake, fake, fake, fake, fake, fake,
                                               fake, 1, 64, 64, 65536, 128, 16, 1,
                                               native.RM_ORDER_ZIGZAG, native.RM_DTYPE_BF16,
                                               0.088, None)
    assert st == native.RM_ERR_UNSUPPORTED
