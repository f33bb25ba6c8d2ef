"""Ring attention whose ranks are separate processes (one per device).

"Sequence Parallelism III: Ring Attention" (duoan.github.io) and "DeDLOC
Guide" (Step 3 and section 3): each rank keeps its L = S / P query rows; its
key/value block travels around the ring, so at step t the rank holds the block
of owner (rank - t) mod P. The rank folds that step's partial (O, LSE) into its
running pair, while the block it holds goes on to rank + 1 and the next
arrives from rank - 1 (the p2p rotater of the axolotl-ringmaster README: the
blocks in flight are the only K/V a rank holds besides its own). The backward
is the README's flash-style reverse ring: the block travels the same way,
carrying fp32 dK/dV accumulators that every rank adds its part to, and after
the last step the accumulators go one hop further, back to their owner.

Only this module exchanges data between processes; the arithmetic is the
library's (rm_ring_attn_fwd_step_merge, rm_ring_attn_bwd_delta,
rm_ring_attn_bwd_step).

The exchange of step t is posted before step t's kernel is launched, so the
transfer of the next block overlaps the compute on the current one. The
caller's k_local / v_local are only ever SENT: blocks are received into two
buffers of this module, used in turn, so the caller's tensors come back
unchanged (the backward needs them). A receive buffer last held the block of
step t - 1; the collective stream does not overwrite it before the compute
launched on it has finished (torch orders NCCL's stream after the work already
queued on the current stream).
"""


def _default_fold(q_local, k_block, v_block, P, rank, owner, causal, order, scale, o_acc,
                  lse_acc):
    import ring_ulysses_sequence_b200 as rm
    rm.ring_attn_fwd_step_merge(q_local, k_block, v_block, o_acc, lse_acc, P, rank, owner, causal,
                                order, scale)


def _default_delta(o_local, dout_local):
    import ring_ulysses_sequence_b200 as rm
    return rm.ring_attn_bwd_delta(o_local, dout_local)


def _default_bwd_step(q_local, k_block, v_block, lse_local, delta_local, dout_local, dq, dk, dv,
                      P, rank, owner, causal, order, scale):
    import ring_ulysses_sequence_b200 as rm
    rm.ring_attn_bwd_step(q_local, k_block, v_block, lse_local, delta_local, dout_local, dq, dk,
                          dv, P, rank, owner, causal, order, scale)


def ring_schedule(P: int, rank: int):
    """[(t, owner)] of the blocks rank `rank` holds at steps t = 0..P-1."""
    return [(t, (rank - t) % P) for t in range(P)]


def _ring_peers(group):
    import torch.distributed as dist
    if dist.is_initialized():
        P, rank = dist.get_world_size(group), dist.get_rank(group)
    else:
        P, rank = 1, 0
    to_rank, from_rank = (rank + 1) % P, (rank - 1) % P
    if group is not None and P > 1:
        to_rank = dist.get_global_rank(group, to_rank)
        from_rank = dist.get_global_rank(group, from_rank)
    return P, rank, to_rank, from_rank


def _exchange(send, recv, to_rank, from_rank, group):
    """Posts the sends of `send` to the next rank and the receives into `recv`
    from the previous one; returns the requests."""
    import torch.distributed as dist
    ops = [dist.P2POp(dist.isend, t, to_rank, group) for t in send]
    ops += [dist.P2POp(dist.irecv, t, from_rank, group) for t in recv]
    return dist.batch_isend_irecv(ops)


def ring_attn_fwd_p2p(q_local, k_local, v_local, causal=True, order="zigzag", scale=None,
                      group=None, step=None, merge=None, fold=None):
    """Forward of ring attention across the ranks of `group`.

    q_local [B,H,L,D], k_local/v_local [B,Hkv,L,D]: this rank's slice of the
    rank-major layout (zigzag: chunk rank then chunk 2P-1-rank). Returns this
    rank's (O [B,H,L,D] float32, LSE [B,H,L] float32). k_local and v_local
    are not modified.

    fold(q, k_blk, v_blk, P, rank, owner, causal, order, scale, o_acc, lse_acc)
    folds one step into the running pair in place; it defaults to the fused
    CUDA call (rm_ring_attn_fwd_step_merge). Alternatively step(q, k_blk,
    v_blk, P, rank, owner, causal, order, scale) -> (o, lse) and
    merge(o_acc, lse_acc, o_part, lse_part) give the same fold in two calls
    (rm_ring_attn_fwd_step + rm_lse_merge, or other arithmetic for tests).

    With NCCL, each process must have made its own device current
    (torch.cuda.set_device) before the first call, and every rank of the
    group must call this with blocks of the same shape.
    """
    import torch
    if step is not None or merge is not None:
        if step is None or merge is None:
            raise ValueError("step and merge go together")

        def fold(q, k_blk, v_blk, P_, r, owner, c, o_, s_, o_acc, lse_acc):
            o_part, lse_part = step(q, k_blk, v_blk, P_, r, owner, c, o_, s_)
            merge(o_acc, lse_acc, o_part, lse_part)
    elif fold is None:
        fold = _default_fold
    P, rank, to_rank, from_rank = _ring_peers(group)
    B, H, L, D = q_local.shape
    o_acc = torch.zeros((B, H, L, D), dtype=torch.float32, device=q_local.device)
    lse_acc = torch.full((B, H, L), float("-inf"), dtype=torch.float32, device=q_local.device)
    cur = (k_local.contiguous(), v_local.contiguous())
    bufs = [(torch.empty_like(cur[0]), torch.empty_like(cur[1])) for _ in range(min(P - 1, 2))]
    for t, owner in ring_schedule(P, rank):
        reqs = []
        nxt = None
        if t + 1 < P:  # pass the held block on and take the next one
            nxt = bufs[t % 2]
            reqs = _exchange(cur, nxt, to_rank, from_rank, group)
        fold(q_local, cur[0], cur[1], P, rank, owner, causal, order, scale, o_acc, lse_acc)
        for r in reqs:
            r.wait()
        if nxt is not None:
            cur = nxt
    return o_acc, lse_acc


def ring_attn_bwd_p2p(q_local, k_local, v_local, o_local, lse_local, dout_local, causal=True,
                      order="zigzag", scale=None, group=None, bwd_step=None, delta=None):
    """Backward of ring attention across the ranks of `group` (the reverse
    ring of the axolotl-ringmaster README's p2p rotater).

    q_local, dout_local [B,H,L,D] and k_local, v_local [B,Hkv,L,D] as in the
    forward; o_local [B,H,L,D] (bf16, or the forward's float32) and lse_local
    [B,H,L] float32 are this rank's forward results. Returns this rank's
    (dQ [B,H,L,D], dK [B,Hkv,L,D], dV [B,Hkv,L,D]), all float32. The inputs
    are not modified.

    Per step t the rank holds owner (rank - t) mod P's block together with the
    fp32 dK/dV sums that ranks owner .. rank - 1 have added to it. The next
    block's K/V arrive while this step computes; the sums, which this step
    updates, travel after it. After the last step every rank holds the block
    of rank + 1 with complete sums and sends them home.

    bwd_step(q, k_blk, v_blk, lse, delta, dout, dq, dk_blk, dv_blk, P, rank,
    owner, causal, order, scale) adds one step's part in place, and
    delta(o, dout) -> Delta; they default to the CUDA calls.
    """
    import torch
    bwd_step = _default_bwd_step if bwd_step is None else bwd_step
    delta = _default_delta if delta is None else delta
    P, rank, to_rank, from_rank = _ring_peers(group)
    dev = q_local.device
    delta_local = delta(o_local, dout_local)
    dq = torch.zeros(q_local.shape, dtype=torch.float32, device=dev)
    kv = (k_local.contiguous(), v_local.contiguous())
    kv_bufs = [(torch.empty_like(kv[0]), torch.empty_like(kv[1])) for _ in range(min(P - 1, 2))]
    acc_bufs = [(torch.zeros(k_local.shape, dtype=torch.float32, device=dev),
                 torch.zeros(k_local.shape, dtype=torch.float32, device=dev))
                for _ in range(2 if P > 1 else 1)]
    acc = acc_bufs[0]
    for t, owner in ring_schedule(P, rank):
        kv_reqs, kv_nxt = [], None
        if t + 1 < P:
            kv_nxt = kv_bufs[t % 2]
            kv_reqs = _exchange(kv, kv_nxt, to_rank, from_rank, group)
        bwd_step(q_local, kv[0], kv[1], lse_local, delta_local, dout_local, dq, acc[0], acc[1],
                 P, rank, owner, causal, order, scale)
        if P > 1:
            # the block's sums go on with it (after the last step: home to
            # their owner, rank + 1); the next block's sums arrive
            acc_nxt = acc_bufs[(t + 1) % 2]
            for r in _exchange(acc, acc_nxt, to_rank, from_rank, group):
                r.wait()
            acc = acc_nxt
        for r in kv_reqs:
            r.wait()
        if kv_nxt is not None:
            kv = kv_nxt
    return dq, acc[0], acc[1]
