"""Ulysses x ring (USP) attention whose ranks are separate processes.

"Sequence Parallelism II: DeepSpeed Ulysses and All-to-All Attention"
(duoan.github.io): before the all-to-all a device has all heads of its
tokens, after it all tokens of its heads; attention then runs per head, and a
second all-to-all brings the output back to the token layout. The
axolotl-ringmaster README (Why; Benchmark) combines it with ring attention:
the Ulysses groups (consecutive ranks, inside a node) exchange heads, and the
ring groups pass key/value blocks; the Ulysses leg moves K and V together, and
its size U is capped by the number of KV heads.

Mesh: world = U * R processes, process g = r * U + u is device u of Ulysses
group r and rank r of ring group u. It holds sequence shard n = g: the s =
S / (U R) tokens [n s, (n + 1) s) of the ring's rank-major sequence (ring rank
r's L = S / R tokens are the shards of its Ulysses group, in order).

Forward, per device (2 collectives plus the ring's block exchange):
  1. pack Q, K, V into one send buffer (rm_ulysses_pack, SEQ_TO_HEAD);
  2. one all_to_all_single over the Ulysses group;
  3. unpack to head shards [B, H/U, L, D], [B, Hkv/U, L, D] (rm_ulysses_unpack);
  4. ring attention over the ring group (ring.ring_attn_fwd_p2p);
  5. pack O (HEAD_TO_SEQ), all_to_all_single, unpack to [B, s, H, D].
The README fuses K/V into one exchange besides Q and O (three collectives);
here Q travels in the same buffer as K and V, so the way in is one. LSE stays
in the head layout: only the backward needs it.

The backward reverses it: dO goes to the head layout, the ring backward runs
(ring.ring_attn_bwd_p2p), and dQ, dK, dV return in one buffer.

Only this module and ring.py exchange data between processes; the layout
transforms and the arithmetic are the library's. The pack/unpack/attention
callables are parameters so that the exchange can be exercised with other
implementations (the tests run it on CPU with gloo).
"""
from dataclasses import dataclass


def usp_groups(U: int, R: int):
    """Creates the process groups of a U x R mesh (every rank must call this,
    in the same order). Returns (ulysses_group, ring_group) of this rank."""
    import torch.distributed as dist
    world, rank = dist.get_world_size(), dist.get_rank()
    if U * R != world:
        raise ValueError(f"U * R = {U * R} is not the world size {world}")
    mine_u = mine_r = None
    for r in range(R):  # Ulysses groups: consecutive ranks
        g = dist.new_group([r * U + u for u in range(U)])
        if rank // U == r:
            mine_u = g
    for u in range(U):  # ring groups: one rank of every Ulysses group
        g = dist.new_group([r * U + u for r in range(R)])
        if rank % U == u:
            mine_r = g
    return mine_u, mine_r


def _group_size(group):
    import torch.distributed as dist
    return dist.get_world_size(group) if dist.is_initialized() else 1


def _all_to_all(buf, group):
    """Equal-split all-to-all of a flat buffer over `group` (chunk u goes to
    member u; chunk u of the result came from member u)."""
    import torch
    import torch.distributed as dist
    if _group_size(group) == 1:
        return buf
    out = torch.empty_like(buf)
    dist.all_to_all_single(out, buf, group=group)
    return out


def _default_pack(tensors, U, direction):
    import ring_ulysses_sequence_b200 as rm
    return rm.ulysses_pack(tensors, U, direction)


def _default_unpack(buf, U, heads, B, s, D, direction):
    import ring_ulysses_sequence_b200 as rm
    return rm.ulysses_unpack(buf, U, heads, B, s, D, direction)


@dataclass
class UspContext:
    """What the backward needs from the forward (head layout)."""
    q: object
    k: object
    v: object
    o: object
    lse: object
    U: int
    heads: tuple
    shape: tuple  # (B, s, D)


def usp_attn_fwd(q, k, v, ulysses_group=None, ring_group=None, causal=True, order="zigzag",
                 scale=None, pack=None, unpack=None, ring_fwd=None):
    """Forward of Ulysses x ring attention on this device's sequence shard.

    q [B, s, H, D], k/v [B, s, Hkv, D] (bf16): the device's s tokens. Returns
    (O [B, s, H, D] float32, ctx) where ctx holds the head-layout tensors the
    backward uses. H and Hkv must be multiples of U (the Ulysses group size).

    pack(tensors, U, direction) -> buf, unpack(buf, U, heads, B, s, D,
    direction) -> tensors and ring_fwd(q, k, v, causal, order, scale, group)
    -> (o, lse) default to the library's calls and ring.ring_attn_fwd_p2p.
    """
    from . import ring
    pack = _default_pack if pack is None else pack
    unpack = _default_unpack if unpack is None else unpack
    if ring_fwd is None:
        def ring_fwd(q_, k_, v_, c, o_, s_, g):
            return ring.ring_attn_fwd_p2p(q_, k_, v_, c, o_, s_, group=g)
    U = _group_size(ulysses_group)
    B, s, H, D = q.shape
    Hkv = k.shape[2]
    if H % U or Hkv % U:
        raise ValueError(f"H = {H} and Hkv = {Hkv} must be multiples of U = {U}")
    heads = (H, Hkv, Hkv)
    recv = _all_to_all(pack([q, k, v], U, "seq_to_head"), ulysses_group)
    qh, kh, vh = unpack(recv, U, list(heads), B, s, D, "seq_to_head")
    oh, lse = ring_fwd(qh, kh, vh, causal, order, scale, ring_group)
    back = _all_to_all(pack([oh], U, "head_to_seq"), ulysses_group)
    (o,) = unpack(back, U, [H], B, s, D, "head_to_seq")
    return o, UspContext(qh, kh, vh, oh, lse, U, heads, (B, s, D))


def usp_attn_bwd(dout, ctx: UspContext, ulysses_group=None, ring_group=None, causal=True,
                 order="zigzag", scale=None, pack=None, unpack=None, ring_bwd=None):
    """Backward of usp_attn_fwd: dout [B, s, H, D] (bf16) -> (dQ [B, s, H, D],
    dK [B, s, Hkv, D], dV [B, s, Hkv, D]) float32 on this device's tokens.

    ring_bwd(q, k, v, o, lse, dout, causal, order, scale, group) -> (dq, dk,
    dv) defaults to ring.ring_attn_bwd_p2p; pack/unpack as in the forward.
    """
    from . import ring
    pack = _default_pack if pack is None else pack
    unpack = _default_unpack if unpack is None else unpack
    if ring_bwd is None:
        def ring_bwd(q_, k_, v_, o_, l_, do_, c, or_, s_, g):
            return ring.ring_attn_bwd_p2p(q_, k_, v_, o_, l_, do_, c, or_, s_, group=g)
    U = ctx.U
    B, s, D = ctx.shape
    H, Hkv, _ = ctx.heads
    recv = _all_to_all(pack([dout], U, "seq_to_head"), ulysses_group)
    (doh,) = unpack(recv, U, [H], B, s, D, "seq_to_head")
    dqh, dkh, dvh = ring_bwd(ctx.q, ctx.k, ctx.v, ctx.o, ctx.lse, doh, causal, order, scale,
                             ring_group)
    back = _all_to_all(pack([dqh, dkh, dvh], U, "head_to_seq"), ulysses_group)
    return unpack(back, U, [H, Hkv, Hkv], B, s, D, "head_to_seq")
