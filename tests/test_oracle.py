"""Pins for the fp64 oracle, each against something other than the oracle itself.

* brute force with numpy/scipy library routines on tiny inputs,
* closed forms (equal keys, zero queries, a planted dominant logit, causal row 0),
* the two-chunk parity harness of "DeDLOC Guide", Step 4 (merge of two
  chunks' (O, LSE) equals dense attention over their union),
* ring == dense for many P and both chunk orders,
* merge order independence and the empty-partial (-inf) rule,
* gradients: central finite differences, torch fp64 autograd, and the
  identities sum_j dK_j = 0 and sum_j dV_j = sum_i dO_i,
* hand-derived rank-major maps and ring schedules from tests/golden/.
"""
import itertools
import math
import os

import numpy as np
import pytest
import torch
from scipy.special import logsumexp

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _np_attention(q, k, v, causal, scale):
    """Textbook dense attention with numpy/scipy (independent of the oracle)."""
    B, H, S, D = q.shape
    Hkv, Sk = k.shape[1], k.shape[2]
    G = H // Hkv
    o = np.zeros((B, H, S, D))
    lse = np.zeros((B, H, S))
    for b in range(B):
        for h in range(H):
            s = scale * q[b, h] @ k[b, h // G].T
            if causal:
                mask = np.arange(Sk)[None, :] > np.arange(S)[:, None]
                s = np.where(mask, -np.inf, s)
            lse[b, h] = logsumexp(s, axis=-1)
            w = np.exp(s - lse[b, h][:, None])
            o[b, h] = w @ v[b, h // G]
    return o, lse


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("H,Hkv", [(1, 1), (4, 2), (4, 1), (3, 3)])
@pytest.mark.parametrize("S,D", [(1, 1), (5, 3), (16, 8), (9, 4)])
def test_forward_matches_numpy_bruteforce(causal, H, Hkv, S, D):
    seed = hash((causal, H, Hkv, S, D)) % 2**31
    q, k, v = _rand((2, H, S, D), seed), _rand((2, Hkv, S, D), seed + 1), _rand((2, Hkv, S, D), seed + 2)
    scale = 1 / math.sqrt(D)
    o, lse = oracle.attn_fwd(q, k, v, causal, scale)
    o_ref, lse_ref = _np_attention(q, k, v, causal, scale)
    np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse, lse_ref, rtol=0, atol=1e-13)


def test_forward_row_subset_and_scale_argument():
    q, k, v = _rand((1, 2, 12, 4), 1), _rand((1, 2, 12, 4), 2), _rand((1, 2, 12, 4), 3)
    rows = np.array([0, 5, 11])
    o_all, lse_all = oracle.attn_fwd(q, k, v, True, 0.3)
    o, lse = oracle.attn_fwd(q, k, v, True, 0.3, rows=rows)
    np.testing.assert_array_equal(o, o_all[:, :, rows])
    np.testing.assert_array_equal(lse, lse_all[:, :, rows])
    o_ref, lse_ref = _np_attention(q, k, v, True, 0.3)
    np.testing.assert_allclose(lse_all, lse_ref, atol=1e-13, rtol=0)


def test_closed_form_equal_keys():
    # all keys equal: every visible score is s = scale <q_i, k>, so attention is
    # the mean of the visible values and LSE = s + ln |V(i)|.
    S, D = 10, 4
    q = _rand((1, 1, S, D), 5)
    kvec = _rand((D,), 6)
    k = np.broadcast_to(kvec, (1, 1, S, D)).copy()
    v = _rand((1, 1, S, D), 7)
    scale = 0.7
    for causal in (False, True):
        o, lse = oracle.attn_fwd(q, k, v, causal, scale)
        for i in range(S):
            n = i + 1 if causal else S
            s = scale * q[0, 0, i] @ kvec
            np.testing.assert_allclose(o[0, 0, i], v[0, 0, :n].mean(axis=0), atol=1e-14)
            assert abs(lse[0, 0, i] - (s + math.log(n))) < 1e-13


def test_closed_form_zero_queries_and_causal_row0():
    S, D = 8, 3
    q = np.zeros((1, 1, S, D))
    k, v = _rand((1, 1, S, D), 8), _rand((1, 1, S, D), 9)
    o, lse = oracle.attn_fwd(q, k, v, False, 1.0)
    np.testing.assert_allclose(o[0, 0], np.broadcast_to(v[0, 0].mean(0), (S, D)), atol=1e-14)
    np.testing.assert_allclose(lse[0, 0], math.log(S), atol=1e-14)
    # causal row 0 sees only key 0: O_0 = v_0, LSE_0 = s_00
    q = _rand((1, 1, S, D), 10)
    o, lse = oracle.attn_fwd(q, k, v, True, 0.5)
    np.testing.assert_allclose(o[0, 0, 0], v[0, 0, 0], atol=1e-15)
    assert abs(lse[0, 0, 0] - 0.5 * q[0, 0, 0] @ k[0, 0, 0]) < 1e-14


def test_closed_form_dominant_logit():
    # one key aligned with the query at a huge logit: softmax is one-hot.
    S, D = 6, 4
    q = np.zeros((1, 1, S, D)); q[0, 0, :, 0] = 1.0
    k = np.zeros((1, 1, S, D)); k[0, 0, 3, 0] = 1000.0
    v = _rand((1, 1, S, D), 11)
    o, lse = oracle.attn_fwd(q, k, v, False, 1.0)
    np.testing.assert_allclose(o[0, 0], np.broadcast_to(v[0, 0, 3], (S, D)), atol=1e-14)
    np.testing.assert_allclose(lse[0, 0], 1000.0, atol=1e-12)


def test_two_chunk_merge_harness():
    # "DeDLOC Guide", Step 4: attention over KV chunk 0 and chunk 1 separately,
    # merged, equals dense attention over both (B=1, H=8, 64 queries, 64+64 keys,
    # D=64, fp32 there with max-abs < 1e-5; fp64 here).
    B, H, S, D = 1, 8, 64, 64
    q = _rand((B, H, S, D), 12)
    k0, v0 = _rand((B, H, S, D), 13), _rand((B, H, S, D), 14)
    k1, v1 = _rand((B, H, S, D), 15), _rand((B, H, S, D), 16)
    scale = 1 / math.sqrt(D)
    o0, l0 = oracle.attn_fwd(q, k0, v0, False, scale)
    o1, l1 = oracle.attn_fwd(q, k1, v1, False, scale)
    om, lm = oracle.lse_merge(o0.reshape(-1, D), l0.reshape(-1), o1.reshape(-1, D), l1.reshape(-1))
    kf, vf = np.concatenate([k0, k1], axis=2), np.concatenate([v0, v1], axis=2)
    o_ref, lse_ref = _np_attention(q, kf, vf, False, scale)
    assert np.abs(om.reshape(o_ref.shape) - o_ref).max() < 1e-12
    assert np.abs(lm.reshape(lse_ref.shape) - lse_ref).max() < 1e-12
    # and the oracle's own dense path over the concatenation agrees too
    od, ld = oracle.attn_fwd(q, kf, vf, False, scale)
    assert np.abs(od - o_ref).max() < 1e-13


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("order", [oracle.CONTIGUOUS, oracle.ZIGZAG])
@pytest.mark.parametrize("P", [1, 2, 3, 4, 8])
def test_ring_equals_dense(causal, order, P):
    S = 48 if P == 3 else 32
    H, Hkv, D = 4, 2, 8
    q, k, v = _rand((1, H, S, D), 17 + P), _rand((1, Hkv, S, D), 18), _rand((1, Hkv, S, D), 19)
    o_d, l_d = oracle.attn_fwd(q, k, v, causal)
    o_r, l_r = oracle.ring_fwd(q, k, v, causal, P, order)
    assert np.abs(o_r - o_d).max() < 1e-12
    assert np.abs(l_r - l_d).max() < 1e-12


def test_ring_zigzag_equals_contiguous_after_unpermute():
    # The orders only move tokens between ranks; in natural order the results agree.
    S, D, P = 64, 4, 4
    q, k, v = _rand((1, 2, S, D), 20), _rand((1, 2, S, D), 21), _rand((1, 2, S, D), 22)
    oz, lz = oracle.ring_fwd(q, k, v, True, P, oracle.ZIGZAG)
    oc, lc = oracle.ring_fwd(q, k, v, True, P, oracle.CONTIGUOUS)
    assert np.abs(oz - oc).max() < 1e-12 and np.abs(lz - lc).max() < 1e-12


def test_merge_order_independence_and_empty_partials():
    rng = np.random.default_rng(23)
    n, rows, D = 6, 5, 7
    parts = [(rng.standard_normal((rows, D)), rng.standard_normal(rows) * 3) for _ in range(n)]
    # one partial is empty on some rows: (0, -inf) is the identity
    parts[2][1][1] = -np.inf
    parts[2][0][1] = 0.0

    def fold(order):
        o, l = parts[order[0]][0].copy(), parts[order[0]][1].copy()
        for idx in order[1:]:
            o, l = oracle.lse_merge(o, l, parts[idx][0], parts[idx][1])
        return o, l

    ref_o, ref_l = fold(list(range(n)))
    for perm in list(itertools.permutations(range(n)))[::37]:
        o, l = fold(list(perm))
        assert np.abs(o - ref_o).max() < 1e-12 and np.abs(l - ref_l).max() < 1e-12
    # tree-shaped merge
    a = oracle.lse_merge(*fold([0, 1]), *fold([2, 3]))
    t = oracle.lse_merge(*a, *fold([4, 5]))
    assert np.abs(t[0] - ref_o).max() < 1e-12 and np.abs(t[1] - ref_l).max() < 1e-12
    # closed form of the merge: partials over disjoint sets merge to softmax over the union
    w = np.exp(np.stack([p[1] for p in parts]))           # per-partial normaliser
    o_cf = sum(wi[:, None] * p[0] for wi, p in zip(w, parts)) / w.sum(0)[:, None]
    assert np.abs(ref_o - o_cf).max() < 1e-12
    assert np.abs(ref_l - np.log(w.sum(0))).max() < 1e-12
    # both empty -> (0, -inf), never NaN
    o, l = oracle.lse_merge(np.ones((1, D)), np.array([-np.inf]), np.ones((1, D)), np.array([-np.inf]))
    assert np.all(o == 0) and l[0] == -np.inf


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("order", [oracle.CONTIGUOUS, oracle.ZIGZAG])
@pytest.mark.parametrize("P", [1, 2, 3, 4])
def test_step_partials_fold_to_dense_attention(causal, order, P):
    # One rank's P step partials (one per owner block), merged in ring order,
    # are attention over all keys: compared with the textbook numpy attention.
    S = 24 if P == 3 else 32
    L, H, Hkv, D = S // P, 4, 2, 8
    q, k, v = _rand((1, H, S, D), 60 + P), _rand((1, Hkv, S, D), 61), _rand((1, Hkv, S, D), 62)
    o_ref, l_ref = _np_attention(q, k, v, causal, 1.0 / math.sqrt(D))
    pos = oracle.rank_major_positions(S, P, order)
    qr, kr, vr = (x[:, :, pos] for x in (q, k, v))   # rank-major by fancy indexing
    for rank in range(P):
        sl = slice(rank * L, (rank + 1) * L)
        o = np.zeros((H * L, D))
        l = np.full(H * L, -np.inf)
        for t in range(P):
            owner = (rank - t) % P
            blk = slice(owner * L, (owner + 1) * L)
            op, lp = oracle.step_partial(qr[:, :, sl], kr[:, :, blk], vr[:, :, blk], S, P, order,
                                         rank, owner, causal)
            o, l = oracle.lse_merge(o, l, op.reshape(H * L, D), lp.reshape(H * L))
        rows = pos[sl]
        assert np.abs(o.reshape(1, H, L, D) - o_ref[:, :, rows]).max() < 1e-12
        assert np.abs(l.reshape(1, H, L) - l_ref[:, :, rows]).max() < 1e-12


def test_step_partial_special_cases():
    S, P, D = 32, 4, 4
    L = S // P
    q, k, v = _rand((1, 2, L, D), 70), _rand((1, 1, L, D), 71), _rand((1, 1, L, D), 72)
    # contiguous causal: rank 0's queries precede every key of owner 3 -> all empty
    o, l = oracle.step_partial(q, k, v, S, P, oracle.CONTIGUOUS, 0, 3, True)
    assert np.all(o == 0) and np.all(l == -np.inf)
    # an earlier block is fully visible: plain softmax over its L keys
    o, l = oracle.step_partial(q, k, v, S, P, oracle.CONTIGUOUS, 3, 1, True)
    s = (q[0, 0] @ k[0, 0].T) / math.sqrt(D)
    assert np.abs(l[0, 0] - logsumexp(s, axis=1)).max() < 1e-12
    # P = 1: the step is the whole attention
    o1, l1 = oracle.step_partial(q, k, v, L, 1, oracle.ZIGZAG, 0, 0, True)
    o_ref, l_ref = _np_attention(q, k, v, True, 1.0 / math.sqrt(D))
    assert np.abs(o1 - o_ref).max() < 1e-12 and np.abs(l1 - l_ref).max() < 1e-12


def _loss(q, k, v, dout, causal, scale):
    o, _ = oracle.attn_fwd(q, k, v, causal, scale)
    return float((o * dout).sum())


@pytest.mark.parametrize("causal", [False, True])
def test_backward_finite_differences(causal):
    B, H, Hkv, S, D = 1, 4, 2, 12, 4
    q, k, v = _rand((B, H, S, D), 24), _rand((B, Hkv, S, D), 25), _rand((B, Hkv, S, D), 26)
    dout = _rand((B, H, S, D), 27)
    scale = 1 / math.sqrt(D)
    dq, dkv = oracle.attn_bwd(q, k, v, dout, causal, scale)
    h = 1e-6
    rng = np.random.default_rng(28)
    for name, x in (("q", q), ("k", k), ("v", v)):
        for _ in range(12):
            idx = tuple(rng.integers(0, n) for n in x.shape)
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args = {"q": q, "k": k, "v": v}
            args[name] = xp
            lp = _loss(args["q"], args["k"], args["v"], dout, causal, scale)
            args[name] = xm
            lm = _loss(args["q"], args["k"], args["v"], dout, causal, scale)
            fd = (lp - lm) / (2 * h)
            b, hh, s, d = idx
            if name == "q":
                an = dq[(b, hh)][s, d]
            elif name == "k":
                an = dkv[(b, hh)][0][s, d]
            else:
                an = dkv[(b, hh)][1][s, d]
            assert abs(fd - an) <= 1e-7 * max(1.0, abs(an)), (name, idx, fd, an)


@pytest.mark.parametrize("causal", [False, True])
def test_backward_matches_torch_autograd(causal):
    B, H, Hkv, S, D = 2, 4, 1, 10, 6
    q, k, v = _rand((B, H, S, D), 29), _rand((B, Hkv, S, D), 30), _rand((B, Hkv, S, D), 31)
    dout = _rand((B, H, S, D), 32)
    scale = 0.37
    tq, tk, tv = (torch.tensor(a, requires_grad=True) for a in (q, k, v))
    G = H // Hkv
    kk = tk.repeat_interleave(G, dim=1)
    vv = tv.repeat_interleave(G, dim=1)
    s = torch.matmul(tq, kk.transpose(-1, -2)) * scale
    if causal:
        s = s.masked_fill(torch.triu(torch.ones(S, S, dtype=torch.bool), 1), float("-inf"))
    o = torch.matmul(torch.softmax(s, -1), vv)
    (o * torch.tensor(dout)).sum().backward()
    dq, dkv = oracle.attn_bwd(q, k, v, dout, causal, scale)
    for b in range(B):
        for h in range(H):
            np.testing.assert_allclose(dq[(b, h)], tq.grad[b, h].numpy(), atol=1e-12, rtol=0)
        for g in range(Hkv):
            np.testing.assert_allclose(dkv[(b, g)][0], tk.grad[b, g].numpy(), atol=1e-12, rtol=0)
            np.testing.assert_allclose(dkv[(b, g)][1], tv.grad[b, g].numpy(), atol=1e-12, rtol=0)


def test_backward_identities_and_row_subsets():
    # sum_j dS_ij = 0 per query row, hence sum_j dK_j = 0; softmax rows sum to
    # one, hence sum_j dV_j = sum_i dO_i (per KV head, summed over its group).
    B, H, Hkv, S, D = 1, 2, 1, 20, 5
    q, k, v = _rand((B, H, S, D), 33), _rand((B, Hkv, S, D), 34), _rand((B, Hkv, S, D), 35)
    dout = _rand((B, H, S, D), 36)
    for causal in (False, True):
        dq, dkv = oracle.attn_bwd(q, k, v, dout, causal)
        dk, dv = dkv[(0, 0)]
        assert np.abs(dk.sum(0)).max() < 1e-12
        np.testing.assert_allclose(dv.sum(0), dout[0].sum(axis=(0, 1)), atol=1e-12)
        rows = np.array([3, 7, 19])
        dq_s, dkv_s = oracle.attn_bwd(q, k, v, dout, causal, qrows=rows, krows=rows,
                                      heads=([(0, 1)], [(0, 0)]))
        np.testing.assert_allclose(dq_s[(0, 1)], dq[(0, 1)][rows], atol=1e-13)
        np.testing.assert_allclose(dkv_s[(0, 0)][0], dk[rows], atol=1e-13)
        np.testing.assert_allclose(dkv_s[(0, 0)][1], dv[rows], atol=1e-13)


def _golden_lines(name):
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                lhs, rhs = line.split(":")
                yield lhs.split(), [int(x) for x in rhs.split()]


def test_rank_major_positions_golden():
    n = 0
    for (order, S, P), expect in _golden_lines("rank_major_positions.txt"):
        o = oracle.ZIGZAG if order == "zigzag" else oracle.CONTIGUOUS
        assert list(oracle.rank_major_positions(int(S), int(P), o)) == expect
        n += 1
    assert n >= 6


def test_ring_schedule_golden():
    n = 0
    for (P, i), expect in _golden_lines("ring_schedule.txt"):
        assert [oracle.ring_owner(int(P), int(i), t) for t in range(int(P))] == expect
        n += 1
    assert n >= 5


@pytest.mark.parametrize("S,P", [(64, 4), (96, 3), (1024, 8), (32, 16)])
def test_rank_major_positions_bijection_and_roundtrip(S, P):
    for order in (oracle.CONTIGUOUS, oracle.ZIGZAG):
        pos = oracle.rank_major_positions(S, P, order)
        assert sorted(pos.tolist()) == list(range(S))
        x = np.arange(S * 3).reshape(1, S, 3)
        assert np.array_equal(oracle.to_natural(oracle.to_rank_major(x, P, order, 1), P, order, 1), x)
    with pytest.raises(ValueError):
        oracle.rank_major_positions(S + 1, P, oracle.ZIGZAG)


def test_ulysses_layout_is_a_bijection():
    B, S, H, D = 2, 12, 4, 3
    src = np.arange(B * S * H * D).reshape(B, S, H, D)
    dst = oracle.ulysses_seq_to_head(src)
    assert dst.shape == (B, H, S, D)
    # every element lands exactly once, at [b, h, s, d] <- [b, s, h, d]
    assert sorted(dst.ravel().tolist()) == list(range(src.size))
    for b, s, h, d in [(0, 0, 0, 0), (1, 11, 3, 2), (0, 5, 2, 1)]:
        assert dst[b, h, s, d] == src[b, s, h, d]
    assert np.array_equal(oracle.ulysses_head_to_seq(dst), src)


def _literal_all_to_all(shards, U, R, H):
    """The Ulysses exchange done message by message ("Sequence Parallelism II:
    DeepSpeed Ulysses and All-to-All Attention": before it a device has all
    heads of some tokens, after it all tokens of some heads). shards[(r, u)]
    is device (r, u)'s [B, s, H, D] slice; inside ring group r, device u sends
    device u2 the heads [u2*H/U, (u2+1)*H/U) of its tokens, and u2 stacks what
    it receives in sender order. Returns {(r, u2): [B, H/U, U*s, D]}."""
    hU = H // U
    inbox = {(r, u2): {} for r in range(R) for u2 in range(U)}
    for (r, u), x in shards.items():
        for u2 in range(U):
            inbox[(r, u2)][u] = x[:, :, u2 * hU:(u2 + 1) * hU]      # message u -> u2
    out = {}
    for key, msgs in inbox.items():
        tokens = np.concatenate([msgs[u] for u in range(U)], axis=1)  # [B, U*s, hU, D]
        out[key] = np.ascontiguousarray(tokens.transpose(0, 2, 1, 3))
    return out


@pytest.mark.parametrize("U,R", [(2, 2), (4, 2), (2, 3), (1, 4), (4, 1)])
def test_ulysses_map_equals_a_literal_all_to_all(U, R):
    # U x R devices as separate arrays: device (r, u) starts with shard
    # n = r*U + u (its s tokens, all heads). After a literal all-to-all inside
    # each ring group it must hold exactly the slab [heads of u, tokens of
    # ring rank r] of the oracle's head-sharded tensor; the way back restores
    # every shard.
    B, H, D = 2, 8, 3
    s = 5
    S = U * R * s
    x = np.arange(B * S * H * D).reshape(B, S, H, D)
    shards = {(r, u): x[:, (r * U + u) * s:(r * U + u + 1) * s] for r in range(R)
              for u in range(U)}
    held = _literal_all_to_all(shards, U, R, H)
    full = oracle.ulysses_seq_to_head(x)
    hU, L = H // U, S // R
    for (r, u), got in held.items():
        want = full[:, u * hU:(u + 1) * hU, r * L:(r + 1) * L]
        assert np.array_equal(got, want), (r, u)
    # the inverse exchange: device (r, u2) sends device u its token rows u*s..
    back = {}
    for r in range(R):
        for u in range(U):
            parts = [held[(r, u2)][:, :, u * s:(u + 1) * s] for u2 in range(U)]  # [B, hU, s, D]
            back[(r, u)] = np.concatenate(parts, axis=1).transpose(0, 2, 1, 3)   # [B, s, H, D]
    seq = oracle.ulysses_head_to_seq(full)
    for (r, u), got in back.items():
        n = r * U + u
        assert np.array_equal(got, shards[(r, u)])
        assert np.array_equal(got, seq[:, n * s:(n + 1) * s])


def test_ulysses_literal_exchange_detects_a_planted_swap():
    # the literal exchange is sensitive enough: swapping two heads in the
    # oracle's map (a plausible indexing mistake) breaks the comparison
    B, H, D, U, R, s = 1, 4, 2, 2, 2, 3
    S = U * R * s
    x = np.arange(B * S * H * D).reshape(B, S, H, D)
    shards = {(r, u): x[:, (r * U + u) * s:(r * U + u + 1) * s] for r in range(R)
              for u in range(U)}
    held = _literal_all_to_all(shards, U, R, H)
    wrong = oracle.ulysses_seq_to_head(x)[:, [1, 0, 2, 3]]
    assert not np.array_equal(held[(0, 0)], wrong[:, 0:2, 0:S // R])


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("order", [oracle.CONTIGUOUS, oracle.ZIGZAG])
@pytest.mark.parametrize("P", [1, 2, 3])
def test_step_backward_partials_sum_to_the_full_gradients(causal, order, P):
    # The reverse ring: every (rank, owner) pair's share, summed over owners
    # for dQ and over ranks for dK/dV, equals the oracle's dense gradients
    # (which finite differences and torch autograd pin above).
    S = 24 if P == 3 else 16
    L, H, Hkv, D = S // P, 4, 2, 4
    q, k, v, do = (_rand(sh, 80 + i) for i, sh in
                   enumerate([(1, H, S, D), (1, Hkv, S, D), (1, Hkv, S, D), (1, H, S, D)]))
    o, lse = oracle.attn_fwd(q, k, v, causal)
    delta = (o * do).sum(axis=-1)
    rdq, rdkv = oracle.attn_bwd(q, k, v, do, causal)
    pos = oracle.rank_major_positions(S, P, order)
    qr, kr, vr, dor, lr, dr = (x[:, :, pos] for x in (q, k, v, do, lse, delta))
    dq = np.zeros_like(qr)
    dk = np.zeros_like(kr)
    dv = np.zeros_like(vr)
    for rank in range(P):
        sl = slice(rank * L, (rank + 1) * L)
        for t in range(P):
            owner = (rank - t) % P
            blk = slice(owner * L, (owner + 1) * L)
            a, b_, c = oracle.step_bwd_partial(qr[:, :, sl], kr[:, :, blk], vr[:, :, blk],
                                               dor[:, :, sl], lr[:, :, sl], dr[:, :, sl], S, P,
                                               order, rank, owner, causal)
            dq[:, :, sl] += a
            dk[:, :, blk] += b_
            dv[:, :, blk] += c
    inv = np.empty_like(pos)
    inv[pos] = np.arange(S)
    for h in range(H):
        assert np.abs(dq[0, h][inv] - rdq[(0, h)]).max() < 1e-12
    for g in range(Hkv):
        assert np.abs(dk[0, g][inv] - rdkv[(0, g)][0]).max() < 1e-12
        assert np.abs(dv[0, g][inv] - rdkv[(0, g)][1]).max() < 1e-12


def test_step_backward_partial_of_an_invisible_block_is_zero():
    # contiguous causal: rank 0's queries precede every key of owner 3
    S, P, D = 32, 4, 4
    L = S // P
    q, k, v, do = _rand((1, 2, L, D), 90), _rand((1, 1, L, D), 91), _rand((1, 1, L, D), 92), \
        _rand((1, 2, L, D), 93)
    lse, delta = _rand((1, 2, L), 94), _rand((1, 2, L), 95)
    for x in oracle.step_bwd_partial(q, k, v, do, lse, delta, S, P, oracle.CONTIGUOUS, 0, 3, True):
        assert np.all(x == 0)


# --- causal sliding window (axolotl-ringmaster README, Status: sliding-window
# attention via flash's `window`): query i sees keys i-W < j <= i ---

def _np_window_attention(q, k, v, W, scale):
    """Band-masked dense attention with numpy/scipy (independent of the oracle)."""
    B, H, S, D = q.shape
    G = H // k.shape[1]
    i = np.arange(S)[:, None]
    j = np.arange(S)[None, :]
    hidden = (j > i) | (j <= i - W)
    o = np.zeros((B, H, S, D))
    lse = np.zeros((B, H, S))
    for b in range(B):
        for h in range(H):
            s = np.where(hidden, -np.inf, scale * q[b, h] @ k[b, h // G].T)
            lse[b, h] = logsumexp(s, axis=-1)
            o[b, h] = np.exp(s - lse[b, h][:, None]) @ v[b, h // G]
    return o, lse


@pytest.mark.parametrize("W", [1, 2, 3, 7, 16, 40])
@pytest.mark.parametrize("H,Hkv,S,D", [(4, 2, 17, 5), (2, 2, 33, 8), (3, 1, 9, 3)])
def test_window_forward_matches_numpy_bruteforce(W, H, Hkv, S, D):
    seed = 7000 + W * 31 + S
    q, k, v = _rand((2, H, S, D), seed), _rand((2, Hkv, S, D), seed + 1), _rand((2, Hkv, S, D), seed + 2)
    scale = 1 / math.sqrt(D)
    o, lse = oracle.attn_fwd(q, k, v, True, scale, window=W)
    o_ref, lse_ref = _np_window_attention(q, k, v, W, scale)
    np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse, lse_ref, rtol=0, atol=1e-13)


def test_window_special_cases():
    B, H, Hkv, S, D = 1, 4, 2, 23, 6
    q, k, v = _rand((B, H, S, D), 71), _rand((B, Hkv, S, D), 72), _rand((B, Hkv, S, D), 73)
    scale = 0.41
    # W = 1: each query sees only its own key, so O_i = v_i and LSE_i = s_ii
    o, lse = oracle.attn_fwd(q, k, v, True, scale, window=1)
    kk = np.repeat(k, 2, axis=1)
    np.testing.assert_allclose(o, np.repeat(v, 2, axis=1), atol=1e-14, rtol=0)
    np.testing.assert_allclose(lse, scale * (q * kk).sum(-1), atol=1e-13, rtol=0)
    # W >= S and W = 0 are plain causal attention; non-causal ignores W
    o_c, lse_c = _np_attention(q, k, v, True, scale)
    for W in (0, S, S + 5):
        o_w, lse_w = oracle.attn_fwd(q, k, v, True, scale, window=W)
        np.testing.assert_allclose(o_w, o_c, atol=1e-13, rtol=0)
        np.testing.assert_allclose(lse_w, lse_c, atol=1e-13, rtol=0)
    o_n, _ = oracle.attn_fwd(q, k, v, False, scale, window=3)
    np.testing.assert_allclose(o_n, _np_attention(q, k, v, False, scale)[0], atol=1e-13, rtol=0)


@pytest.mark.parametrize("order", [oracle.CONTIGUOUS, oracle.ZIGZAG])
@pytest.mark.parametrize("P,W", [(2, 5), (3, 1), (4, 9), (4, 30), (5, 13)])
def test_window_ring_equals_dense(order, P, W):
    B, H, Hkv, D = 1, 2, 1, 4
    S = 2 * P * 4
    q, k, v = _rand((B, H, S, D), 80 + P), _rand((B, Hkv, S, D), 81 + P), _rand((B, Hkv, S, D), 82 + P)
    o_ref, lse_ref = _np_window_attention(q, k, v, W, 0.5)
    # natural order in and out; the ring layout decides each step's key subset
    o, lse = oracle.ring_fwd(q, k, v, True, P, order, 0.5, window=W)
    np.testing.assert_allclose(o, o_ref, atol=1e-13, rtol=0)
    np.testing.assert_allclose(lse, lse_ref, atol=1e-13, rtol=0)


@pytest.mark.parametrize("W", [1, 3, 8])
def test_window_backward_matches_torch_autograd(W):
    B, H, Hkv, S, D = 1, 4, 2, 14, 5
    q, k, v = _rand((B, H, S, D), 90 + W), _rand((B, Hkv, S, D), 91 + W), _rand((B, Hkv, S, D), 92 + W)
    dout = _rand((B, H, S, D), 93 + W)
    scale = 0.45
    tq, tk, tv = (torch.tensor(a, requires_grad=True) for a in (q, k, v))
    kk = tk.repeat_interleave(H // Hkv, dim=1)
    vv = tv.repeat_interleave(H // Hkv, dim=1)
    i = torch.arange(S)[:, None]
    j = torch.arange(S)[None, :]
    s = (torch.matmul(tq, kk.transpose(-1, -2)) * scale).masked_fill((j > i) | (j <= i - W),
                                                                     float("-inf"))
    (torch.matmul(torch.softmax(s, -1), vv) * torch.tensor(dout)).sum().backward()
    dq, dkv = oracle.attn_bwd(q, k, v, dout, True, scale, window=W)
    for h in range(H):
        np.testing.assert_allclose(dq[(0, h)], tq.grad[0, h].numpy(), atol=1e-12, rtol=0)
    for g in range(Hkv):
        np.testing.assert_allclose(dkv[(0, g)][0], tk.grad[0, g].numpy(), atol=1e-12, rtol=0)
        np.testing.assert_allclose(dkv[(0, g)][1], tv.grad[0, g].numpy(), atol=1e-12, rtol=0)
    if W == 1:
        # O_i = v_i does not depend on q or k: dQ = dK = 0, dV_i = sum over the group of dO_i
        assert max(np.abs(dq[(0, h)]).max() for h in range(H)) == 0
        np.testing.assert_allclose(dkv[(0, 0)][1], dout[0, 0] + dout[0, 1], atol=1e-14)


def test_window_backward_finite_differences_and_row_subsets():
    B, H, Hkv, S, D, W = 1, 2, 1, 11, 3, 4
    q, k, v = _rand((B, H, S, D), 95), _rand((B, Hkv, S, D), 96), _rand((B, Hkv, S, D), 97)
    dout = _rand((B, H, S, D), 98)
    dq, dkv = oracle.attn_bwd(q, k, v, dout, True, 0.6, window=W)

    def loss(qq, kk_):
        o, _ = oracle.attn_fwd(qq, kk_, v, True, 0.6, window=W)
        return float((o * dout).sum())
    h = 1e-6
    for (s_, d_) in ((0, 0), (5, 2), (10, 1)):
        qp, qm = q.copy(), q.copy()
        qp[0, 1, s_, d_] += h
        qm[0, 1, s_, d_] -= h
        fd = (loss(qp, k) - loss(qm, k)) / (2 * h)
        assert abs(fd - dq[(0, 1)][s_, d_]) <= 1e-7 * max(1.0, abs(fd))
        kp, km = k.copy(), k.copy()
        kp[0, 0, s_, d_] += h
        km[0, 0, s_, d_] -= h
        fd = (loss(q, kp) - loss(q, km)) / (2 * h)
        assert abs(fd - dkv[(0, 0)][0][s_, d_]) <= 1e-7 * max(1.0, abs(fd))
    rows = np.array([0, 4, 10])
    dq_s, dkv_s = oracle.attn_bwd(q, k, v, dout, True, 0.6, qrows=rows, krows=rows,
                                  heads=([(0, 0)], [(0, 0)]), window=W)
    np.testing.assert_allclose(dq_s[(0, 0)], dq[(0, 0)][rows], atol=1e-13)
    np.testing.assert_allclose(dkv_s[(0, 0)][0], dkv[(0, 0)][0][rows], atol=1e-13)


# --- packed variable-length documents (axolotl-ringmaster README, Status:
# packing / varlen): a query sees keys of its own document [cu[d], cu[d+1])
# only, with the causal and window rules applied inside it ---

def _doc_ids(cu, S):
    d = np.zeros(S, dtype=np.int64)
    for n in range(len(cu) - 1):
        d[cu[n]:cu[n + 1]] = n
    return d


def _np_doc_attention(q, k, v, cu, causal, W, scale):
    """Block-diagonal (optionally causal, windowed) attention with numpy/scipy."""
    B, H, S, D = q.shape
    G = H // k.shape[1]
    doc = _doc_ids(cu, S)
    i = np.arange(S)[:, None]
    j = np.arange(S)[None, :]
    hidden = doc[:, None] != doc[None, :]
    if causal:
        hidden |= j > i
        if W:
            hidden |= j <= i - W
    o = np.zeros((B, H, S, D))
    lse = np.zeros((B, H, S))
    for b in range(B):
        for h in range(H):
            s = np.where(hidden, -np.inf, scale * q[b, h] @ k[b, h // G].T)
            lse[b, h] = logsumexp(s, axis=-1)
            o[b, h] = np.exp(s - lse[b, h][:, None]) @ v[b, h // G]
    return o, lse


DOCS = [[0, 5, 6, 19, 32], [0, 1, 2, 3, 32], [0, 32], [0, 11, 11, 23, 32]]


@pytest.mark.parametrize("cu", DOCS)
@pytest.mark.parametrize("causal,W", [(True, 0), (False, 0), (True, 4)])
def test_varlen_forward_matches_numpy_bruteforce(cu, causal, W):
    S, D = 32, 5
    q, k, v = _rand((2, 4, S, D), 120), _rand((2, 2, S, D), 121), _rand((2, 2, S, D), 122)
    o, lse = oracle.attn_fwd(q, k, v, causal, 0.4, window=W, cu_seqlens=cu)
    o_ref, lse_ref = _np_doc_attention(q, k, v, cu, causal, W, 0.4)
    np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse, lse_ref, rtol=0, atol=1e-13)


@pytest.mark.parametrize("causal", [True, False])
def test_varlen_each_document_is_attention_over_itself(causal):
    # packing must not leak across documents: each document's rows equal the
    # plain attention of that document taken alone
    cu = [0, 7, 20, 21, 40]
    S, D = 40, 6
    q, k, v = _rand((1, 2, S, D), 130), _rand((1, 1, S, D), 131), _rand((1, 1, S, D), 132)
    o, lse = oracle.attn_fwd(q, k, v, causal, cu_seqlens=cu)
    for a, b in zip(cu[:-1], cu[1:]):
        o_d, lse_d = oracle.attn_fwd(q[:, :, a:b], k[:, :, a:b], v[:, :, a:b], causal)
        np.testing.assert_allclose(o[:, :, a:b], o_d, rtol=0, atol=1e-14)
        np.testing.assert_allclose(lse[:, :, a:b], lse_d, rtol=0, atol=1e-14)
    # a document of one token attends to itself only
    np.testing.assert_allclose(o[0, :, 20], np.repeat(v[0, :, 20], 2, axis=0), atol=1e-14)


def test_varlen_special_cases():
    S, D = 24, 4
    q, k, v = _rand((1, 2, S, D), 140), _rand((1, 2, S, D), 141), _rand((1, 2, S, D), 142)
    for causal in (True, False):
        # one document is the plain definition; empty documents change nothing
        a = oracle.attn_fwd(q, k, v, causal, cu_seqlens=[0, S])
        b = oracle.attn_fwd(q, k, v, causal)
        np.testing.assert_array_equal(a[0], b[0])
        c = oracle.attn_fwd(q, k, v, causal, cu_seqlens=[0, 0, 9, 9, 9, S, S])
        d = oracle.attn_fwd(q, k, v, causal, cu_seqlens=[0, 9, S])
        np.testing.assert_array_equal(c[0], d[0])
        # documents of one token: O_i = v_i
        e, _ = oracle.attn_fwd(q, k, v, causal, cu_seqlens=list(range(S + 1)))
        np.testing.assert_allclose(e, v, atol=1e-14)
    with pytest.raises(ValueError):
        oracle.attn_fwd(q, k, v, True, cu_seqlens=[0, 10, 9, S])
    with pytest.raises(ValueError):
        oracle.attn_fwd(q, k, v, True, cu_seqlens=[1, S])


@pytest.mark.parametrize("order", [oracle.CONTIGUOUS, oracle.ZIGZAG])
@pytest.mark.parametrize("P,causal,W", [(2, True, 0), (4, True, 0), (4, False, 0), (3, True, 5)])
def test_varlen_ring_equals_dense(order, P, causal, W):
    S, D = 2 * P * 6, 4
    cu = [0, 5, 17, S - 3, S]
    q, k, v = _rand((1, 2, S, D), 150 + P), _rand((1, 1, S, D), 151), _rand((1, 1, S, D), 152)
    o_r, l_r = oracle.ring_fwd(q, k, v, causal, P, order, 0.5, window=W, cu_seqlens=cu)
    o_d, l_d = _np_doc_attention(q, k, v, cu, causal, W, 0.5)
    np.testing.assert_allclose(o_r, o_d, atol=1e-13, rtol=0)
    np.testing.assert_allclose(l_r, l_d, atol=1e-13, rtol=0)


@pytest.mark.parametrize("causal,W", [(True, 0), (False, 0), (True, 3)])
def test_varlen_backward_matches_torch_autograd(causal, W):
    B, H, Hkv, S, D = 1, 2, 1, 18, 4
    cu = [0, 4, 5, 13, 18]
    q, k, v = _rand((B, H, S, D), 160), _rand((B, Hkv, S, D), 161), _rand((B, Hkv, S, D), 162)
    dout = _rand((B, H, S, D), 163)
    scale = 0.55
    tq, tk, tv = (torch.tensor(a, requires_grad=True) for a in (q, k, v))
    doc = torch.from_numpy(_doc_ids(cu, S))
    i = torch.arange(S)[:, None]
    j = torch.arange(S)[None, :]
    hidden = doc[:, None] != doc[None, :]
    if causal:
        hidden = hidden | (j > i)
        if W:
            hidden = hidden | (j <= i - W)
    s = (torch.matmul(tq, tk.repeat_interleave(H // Hkv, 1).transpose(-1, -2)) * scale)
    s = s.masked_fill(hidden, float("-inf"))
    o = torch.matmul(torch.softmax(s, -1), tv.repeat_interleave(H // Hkv, 1))
    (o * torch.tensor(dout)).sum().backward()
    dq, dkv = oracle.attn_bwd(q, k, v, dout, causal, scale, window=W, cu_seqlens=cu)
    for h in range(H):
        np.testing.assert_allclose(dq[(0, h)], tq.grad[0, h].numpy(), atol=1e-12, rtol=0)
    np.testing.assert_allclose(dkv[(0, 0)][0], tk.grad[0, 0].numpy(), atol=1e-12, rtol=0)
    np.testing.assert_allclose(dkv[(0, 0)][1], tv.grad[0, 0].numpy(), atol=1e-12, rtol=0)
    # per document, sum_j dK_j = 0 (softmax shift invariance inside each document)
    for a, b in zip(cu[:-1], cu[1:]):
        assert np.abs(dkv[(0, 0)][0][a:b].sum(0)).max() < 1e-12
