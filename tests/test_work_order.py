"""The persistent kernels' work-item orders, restated on the host (CPU only).

A launch numbers its work items w = 0 .. n_items-1 and the CTAs claim them in
that order, so the order decides which tiles run at the same time. Two orders
exist (see decode_item in fwd_tc.cu, decode_kv_item / decode_q_item in bwd.cu):
* head-major (whole-ring launches with plain causal or full masks): the items
  of one KV head (forward: the head units that read it; backward: one head)
  come together, positions inside, so the CTAs running at one time share one
  head's K/V (or Q/dO) in L2;
* position-major (windows, packed documents, one step): every head of one
  position adjacent.
Checked here: each order is a bijection onto the (batch, heads, position unit)
triples, the head-major groups are contiguous and read one KV head, and the
position order inside a group is the one the kernels rely on (latest query
first when causal; earliest key first).
"""
import itertools

import pytest


def fwd_decode(w, B, H, Hkv, n_units, causal, head_major):
    """(b, h0, h1, g, position unit) of forward item w."""
    G = H // Hkv
    head_pair = G % 2 == 0
    n_head_units = B * (H // 2 if head_pair else H)
    if head_major:
        gu = G // 2 if head_pair else G
        per_group = n_units * gu
        grp, rem = divmod(w, per_group)
        unit_rank, r = divmod(rem, gu)
        hu = grp * gu + r
    else:
        unit_rank, hu = divmod(w, n_head_units)
    heads_per_b = H // 2 if head_pair else H
    b, hh = divmod(hu, heads_per_b)
    h0 = 2 * hh if head_pair else hh
    h1 = h0 + 1 if head_pair else h0
    nu = n_units - 1 - unit_rank if causal else unit_rank
    return b, h0, h1, h0 // G, nu


def kv_decode(w, B, Hkv, nu, head_major):
    """(b, g, key unit) of dK/dV item w (key tiles earliest first)."""
    nhu = B * Hkv
    if head_major:
        hu, unit = divmod(w, nu)
    else:
        unit, hu = divmod(w, nhu)
    b, g = divmod(hu, Hkv)
    return b, g, unit


def q_decode(w, B, H, nq, causal, head_major):
    """(b, h, query unit) of dQ item w."""
    nhu = B * H
    if head_major:
        hu, unit = divmod(w, nq)
    else:
        unit, hu = divmod(w, nhu)
    b, h = divmod(hu, H)
    return b, h, (nq - 1 - unit if causal else unit)


SHAPES = [(1, 32, 8, 16), (2, 4, 4, 6), (2, 6, 2, 5), (1, 3, 1, 4), (3, 8, 2, 3)]


@pytest.mark.parametrize("B,H,Hkv,n_units", SHAPES)
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("head_major", [True, False])
def test_forward_order(B, H, Hkv, n_units, causal, head_major):
    G = H // Hkv
    head_pair = G % 2 == 0
    n_items = n_units * B * (H // 2 if head_pair else H)
    items = [fwd_decode(w, B, H, Hkv, n_units, causal, head_major) for w in range(n_items)]
    # a bijection onto (batch, head unit, position unit)
    heads = range(0, H, 2) if head_pair else range(H)
    want = {(b, h, u) for b in range(B) for h in heads for u in range(n_units)}
    assert {(b, h0, u) for b, h0, _, _, u in items} == want and len(items) == len(want)
    for b, h0, h1, g, _ in items:  # both query tiles read KV head g
        assert h0 // G == g and h1 // G == g
    if head_major:
        per_group = n_units * (G // 2 if head_pair else G)
        for grp in range(B * Hkv):
            block = items[grp * per_group:(grp + 1) * per_group]
            assert {(b, g) for b, _, _, g, _ in block} == {divmod(grp, Hkv)}
            units = [u for *_, u in block]
            # positions latest first when causal, each once per head unit
            assert units == sorted(units, reverse=causal)
    else:
        per_pos = B * (H // 2 if head_pair else H)
        for p in range(n_units):
            block = items[p * per_pos:(p + 1) * per_pos]
            assert len({u for *_, u in block}) == 1


@pytest.mark.parametrize("B,H,Hkv,n", SHAPES)
@pytest.mark.parametrize("head_major", [True, False])
def test_backward_key_tile_order(B, H, Hkv, n, head_major):
    items = [kv_decode(w, B, Hkv, n, head_major) for w in range(B * Hkv * n)]
    assert sorted(items) == list(itertools.product(range(B), range(Hkv), range(n)))
    if head_major:
        for i in range(B * Hkv):
            block = items[i * n:(i + 1) * n]
            assert {(b, g) for b, g, _ in block} == {divmod(i, Hkv)}
            assert [u for *_, u in block] == list(range(n))  # earliest key first
    else:
        for u in range(n):
            assert {x[2] for x in items[u * B * Hkv:(u + 1) * B * Hkv]} == {u}


@pytest.mark.parametrize("B,H,Hkv,n", SHAPES)
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("head_major", [True, False])
def test_backward_query_tile_order(B, H, Hkv, n, causal, head_major):
    items = [q_decode(w, B, H, n, causal, head_major) for w in range(B * H * n)]
    assert sorted(items) == list(itertools.product(range(B), range(H), range(n)))
    if head_major:
        for i in range(B * H):
            units = [u for b, h, u in items[i * n:(i + 1) * n]]
            assert {(b, h) for b, h, _ in items[i * n:(i + 1) * n]} == {divmod(i, H)}
            assert units == sorted(units, reverse=causal)  # latest query first when causal
