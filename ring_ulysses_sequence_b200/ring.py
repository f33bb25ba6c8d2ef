"""Ring attention whose ranks are separate processes (one per device).

"Sequence Parallelism III: Ring Attention" (duoan.github.io) and "DeDLOC
Guide" (Step 3 and section 3): each rank keeps its L = S / P query rows; its
key/value block travels around the ring, so at step t the rank holds the block
of owner (rank - t) mod P. The rank computes that step's partial (O, LSE) and
folds it into its running pair, while the block it holds goes on to rank + 1
and the next arrives from rank - 1 (the p2p rotater of the axolotl-ringmaster
README: two blocks resident per rank). Only this module exchanges data between
processes; the arithmetic is the library's (rm_ring_attn_fwd_step for a step,
rm_lse_merge for the fold).

The exchange of step t is posted before step t's kernel is launched, so the
transfer of the next block overlaps the compute on the current one; the
receive buffer is the block of step t - 1, which the collective stream does
not overwrite before the compute launched on it has finished.
"""


def _default_step(q_local, k_block, v_block, P, rank, owner, causal, order, scale):
    import ring_ulysses_sequence_b200 as rm
    return rm.ring_attn_fwd_step(q_local, k_block, v_block, P, rank, owner, causal, order, scale)


def _default_merge(o_acc, lse_acc, o_part, lse_part):
    import ring_ulysses_sequence_b200 as rm
    rm.lse_merge_(o_acc, lse_acc, o_part, lse_part)


def ring_schedule(P: int, rank: int):
    """[(t, owner)] of the blocks rank `rank` holds at steps t = 0..P-1."""
    return [(t, (rank - t) % P) for t in range(P)]


def ring_attn_fwd_p2p(q_local, k_local, v_local, causal=True, order="zigzag", scale=None,
                      group=None, step=None, merge=None):
    """Forward of ring attention across the ranks of `group`.

    q_local [B,H,L,D], k_local/v_local [B,Hkv,L,D]: this rank's slice of the
    rank-major layout (zigzag: chunk rank then chunk 2P-1-rank). Returns this
    rank's (O [B,H,L,D] float32, LSE [B,H,L] float32).

    step(q, k_blk, v_blk, P, rank, owner, causal, order, scale) -> (o, lse) and
    merge(o_acc, lse_acc, o_part, lse_part) (in place) default to the CUDA
    calls; they are parameters so that the exchange can be exercised with
    other arithmetic.

    With NCCL, each process must have made its own device current
    (torch.cuda.set_device) before the first call, and every rank of the
    group must call this with blocks of the same shape.
    """
    import torch
    import torch.distributed as dist
    step = _default_step if step is None else step
    merge = _default_merge if merge is None else merge
    if dist.is_initialized():
        P, rank = dist.get_world_size(group), dist.get_rank(group)
    else:
        P, rank = 1, 0
    B, H, L, D = q_local.shape
    o_acc = torch.zeros((B, H, L, D), dtype=torch.float32, device=q_local.device)
    lse_acc = torch.full((B, H, L), float("-inf"), dtype=torch.float32, device=q_local.device)
    cur = (k_local.contiguous(), v_local.contiguous())
    nxt = (torch.empty_like(cur[0]), torch.empty_like(cur[1]))
    to_rank = (rank + 1) % P
    from_rank = (rank - 1) % P
    if group is not None:
        to_rank = dist.get_global_rank(group, to_rank)
        from_rank = dist.get_global_rank(group, from_rank)
    for t, owner in ring_schedule(P, rank):
        reqs = []
        if t + 1 < P:  # pass the held block on and take the next one
            ops = [dist.P2POp(dist.isend, cur[0], to_rank, group),
                   dist.P2POp(dist.isend, cur[1], to_rank, group),
                   dist.P2POp(dist.irecv, nxt[0], from_rank, group),
                   dist.P2POp(dist.irecv, nxt[1], from_rank, group)]
            reqs = dist.batch_isend_irecv(ops)
        o_part, lse_part = step(q_local, cur[0], cur[1], P, rank, owner, causal, order, scale)
        merge(o_acc, lse_acc, o_part, lse_part)
        for r in reqs:
            r.wait()
        cur, nxt = nxt, cur
    return o_acc, lse_acc
