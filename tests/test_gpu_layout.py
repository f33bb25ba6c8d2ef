"""GPU layout kernels against the oracle's maps: bit-exact reorder and Ulysses
permute (one tensor and fused Q/K/V), and the standalone LSE merge."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import ORDER

pytestmark = pytest.mark.gpu


def _bits(shape, dtype, seed):
    """Seeded values of the given dtype (no NaNs, so torch.equal is exact)."""
    g = torch.Generator().manual_seed(seed)
    if dtype.is_floating_point:
        return torch.randn(shape, generator=g).to(dtype)
    info = torch.iinfo(dtype)
    return torch.randint(max(info.min, -2**31), min(info.max, 2**31 - 1), shape, generator=g,
                         dtype=torch.int64).to(dtype)


def _np(t):
    """numpy view of a CPU tensor (bf16 as its int16 bit pattern)."""
    return (t.view(torch.int16) if t.dtype == torch.bfloat16 else t).numpy()


def _from_np(a, dtype):
    t = torch.from_numpy(np.ascontiguousarray(a))
    return t.view(torch.bfloat16) if dtype == torch.bfloat16 else t


@pytest.mark.parametrize("S,P,order", [(1024, 4, "zigzag"), (1024, 4, "contiguous"),
                                       (96, 3, "zigzag"), (8192, 8, "zigzag"), (64, 1, "zigzag")])
@pytest.mark.parametrize("D,dtype", [(128, torch.bfloat16), (1, torch.float32), (3, torch.int16),
                                     (5, torch.uint8), (2, torch.int64)])
def test_seq_reorder_bit_exact(S, P, order, D, dtype):
    import ring_ulysses_sequence_b200 as rm
    B, H = 2, 3
    x = _bits((B, H, S, D), dtype, S + D)
    xg = x.cuda()
    if D == 1 and dtype == torch.float32:
        xg = xg.view(B, H, S)  # the LSE shape
    y = rm.seq_reorder(xg, P, order, "to_rank_major")
    pos = torch.from_numpy(oracle.rank_major_positions(S, P, ORDER[order]))
    expect = x.index_select(2, pos)
    assert torch.equal(y.cpu().reshape(expect.shape), expect)
    back = rm.seq_reorder(y, P, order, "to_natural")
    assert torch.equal(back.cpu().reshape(x.shape), x)


@pytest.mark.parametrize("B,S,H,D,U,R,dtype", [
    (2, 256, 8, 128, 4, 2, torch.bfloat16),
    (1, 96, 6, 3, 3, 2, torch.int16),       # 6-byte rows: 2-byte vectors
    (1, 64, 4, 5, 2, 2, torch.uint8),       # 5-byte rows: 1-byte vectors
    (3, 40, 2, 2, 2, 4, torch.int64),       # 16-byte rows
    (1, 1024, 32, 128, 4, 4, torch.bfloat16),
])
def test_ulysses_permute_bit_exact(B, S, H, D, U, R, dtype):
    import ring_ulysses_sequence_b200 as rm
    x = _bits((B, S, H, D), dtype, B * S + H)
    y = rm.ulysses_permute(x.cuda(), U, R, "seq_to_head")
    expect = _from_np(oracle.ulysses_seq_to_head(_np(x)), dtype)
    assert torch.equal(y.cpu(), expect)
    z = rm.ulysses_permute(y, U, R, "head_to_seq")
    assert torch.equal(z.cpu(), x)


def test_ulysses_permute_qkv_fused():
    import ring_ulysses_sequence_b200 as rm
    B, S, H, Hkv, D, U, R = 1, 512, 16, 4, 128, 4, 2
    q = _bits((B, S, H, D), torch.bfloat16, 1)
    k = _bits((B, S, Hkv, D), torch.bfloat16, 2)
    v = _bits((B, S, Hkv, D), torch.bfloat16, 3)
    outs = rm.ulysses_permute_qkv(q.cuda(), k.cuda(), v.cuda(), U, R, "seq_to_head")
    for got, src in zip(outs, (q, k, v)):
        assert torch.equal(got.cpu(), _from_np(oracle.ulysses_seq_to_head(_np(src)), src.dtype))
    back = rm.ulysses_permute_qkv(*outs, U, R, "head_to_seq")
    for got, src in zip(back, (q, k, v)):
        assert torch.equal(got.cpu(), src)


def test_empty_layout_calls_are_noops():
    import ring_ulysses_sequence_b200 as rm
    x = torch.zeros((0, 8, 4, 16), dtype=torch.bfloat16, device="cuda")
    assert rm.ulysses_permute(x, 2, 2, "seq_to_head").shape == (0, 4, 8, 16)
    o = torch.zeros((0, 8), device="cuda")
    l = torch.zeros((0,), device="cuda")
    rm.lse_merge_(o, l, o.clone(), l.clone())


@pytest.mark.parametrize("rows,D", [(1000, 64), (33, 128), (7, 3), (4096, 1)])
def test_lse_merge(rows, D):
    import ring_ulysses_sequence_b200 as rm
    g = torch.Generator().manual_seed(rows + D)
    oa = torch.randn(rows, D, generator=g)
    ob = torch.randn(rows, D, generator=g)
    la = torch.randn(rows, generator=g) * 4
    lb = torch.randn(rows, generator=g) * 4
    # empty partials: one side, and both sides
    la[::7] = -float("inf")
    oa[::7] = 0
    lb[::11] = -float("inf")
    ob[::11] = 0
    oa_g, la_g = oa.cuda(), la.cuda()
    rm.lse_merge_(oa_g, la_g, ob.cuda(), lb.cuda())
    o_ref, l_ref = oracle.lse_merge(oa.numpy(), la.numpy(), ob.numpy(), lb.numpy())
    got_o, got_l = oa_g.cpu().double().numpy(), la_g.cpu().double().numpy()
    both_empty = np.isneginf(l_ref)
    assert np.array_equal(np.isneginf(got_l), both_empty)
    assert np.all(got_o[both_empty] == 0)
    np.testing.assert_allclose(got_o, o_ref, rtol=1e-5, atol=1e-5)
    np.testing.assert_allclose(got_l[~both_empty], l_ref[~both_empty], rtol=1e-6, atol=1e-5)


@pytest.mark.parametrize("B,s,H,Hkv,D,U,R,dtype", [
    (1, 64, 8, 4, 128, 4, 2, torch.bfloat16),
    (2, 48, 6, 3, 64, 3, 1, torch.bfloat16),
    (1, 40, 4, 2, 5, 2, 2, torch.uint8),     # 5-byte rows: 1-byte vectors
    (1, 32, 4, 4, 1, 2, 3, torch.float32),   # D = 1 (an LSE-like tensor)
    (1, 2048, 32, 8, 128, 4, 1, torch.bfloat16),
])
def test_ulysses_pack_unpack_is_the_all_to_all(B, s, H, Hkv, D, U, R, dtype):
    """U x R devices simulated on one GPU. Each packs its sequence shard of Q,
    K, V into one send buffer; chunk u2 of every sender, in sender order, is
    what device u2 receives (the all-to-all); unpacking it must give exactly
    the device's slab of the oracle's head-sharded tensors (bit-exact), and
    the way back must restore every shard."""
    import ring_ulysses_sequence_b200 as rm
    S = U * R * s
    full = [_bits((B, S, h, D), dtype, 10 * h + i) for i, h in enumerate((H, Hkv, Hkv))]
    heads = [H, Hkv, Hkv]
    n_chunk = sum(heads) // U * B * s * D
    shard = lambda x, n: x[:, n * s:(n + 1) * s].contiguous().cuda()
    sent = {(r, u): rm.ulysses_pack([shard(x, r * U + u) for x in full], U, "seq_to_head")
            for r in range(R) for u in range(U)}
    held = {}
    for r in range(R):
        for u2 in range(U):
            recv = torch.cat([sent[(r, u)][u2 * n_chunk:(u2 + 1) * n_chunk] for u in range(U)])
            held[(r, u2)] = rm.ulysses_unpack(recv, U, heads, B, s, D, "seq_to_head")
    L = S // R
    for (r, u), outs in held.items():
        for x, h, got in zip(full, heads, outs):
            hU = h // U
            want = _from_np(oracle.ulysses_seq_to_head(_np(x)), dtype)[:, u * hU:(u + 1) * hU,
                                                                       r * L:(r + 1) * L]
            assert torch.equal(got.cpu(), want), (r, u, h)
    # the inverse: head shards -> sequence shards
    sent_back = {key: rm.ulysses_pack(list(outs), U, "head_to_seq") for key, outs in held.items()}
    for r in range(R):
        for u in range(U):
            recv = torch.cat([sent_back[(r, u2)][u * n_chunk:(u + 1) * n_chunk]
                              for u2 in range(U)])
            back = rm.ulysses_unpack(recv, U, heads, B, s, D, "head_to_seq")
            for x, got in zip(full, back):
                assert torch.equal(got.cpu(), x[:, (r * U + u) * s:(r * U + u + 1) * s])


def test_ulysses_pack_rejects_bad_arguments():
    import ring_ulysses_sequence_b200 as rm
    from ring_ulysses_sequence_b200 import native
    x = torch.zeros((1, 8, 6, 16), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(rm.RMError):          # 6 heads do not split over U = 4
        rm.ulysses_pack([x], 4, "seq_to_head")
    buf = torch.empty(8 * 6 * 16, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(rm.RMError):          # the buffer may not be a tensor
        native.rm_ulysses_pack([buf], [6], buf, 1, 8, 16, 2, 2, native.RM_SEQ_TO_HEAD)
