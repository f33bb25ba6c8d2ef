"""Blockwise ring attention with Ulysses permutes on one B200 (sm_100a).

P virtual sequence-parallel ranks are simulated on one GPU; the ring's
key/value rotation is HBM block indexing. The computation lives in librm.so
(include/rm.h); this package is its ctypes binding (``native``) plus tensor
conveniences that allocate outputs with PyTorch and call the C ABI.

Layouts: attention tensors are [B, heads, S, D] with S in rank-major ring
order (rank 0's S/P tokens first); ``seq_reorder`` converts from/to natural
order. Sequence-sharded Ulysses tensors are [B, S, heads, D].
"""
import math

from . import native
from .native import (RM_DTYPE_BF16, RM_DTYPE_FP32, RM_HEAD_TO_SEQ,
                     RM_NATURAL_TO_RANK_MAJOR, RM_ORDER_CONTIGUOUS, RM_ORDER_ZIGZAG,
                     RM_RANK_MAJOR_TO_NATURAL, RM_SEQ_TO_HEAD, RMError)

__all__ = ["ring_attn_fwd", "ring_attn_bwd", "varlen_bounds", "lse_merge_", "ulysses_permute",
           "ulysses_permute_qkv", "seq_reorder", "native", "RMError"]

_ORDERS = {"contiguous": RM_ORDER_CONTIGUOUS, "zigzag": RM_ORDER_ZIGZAG}


def _order(order):
    return _ORDERS[order] if isinstance(order, str) else int(order)


def _dtype_code(t):
    import torch
    if t.dtype == torch.bfloat16:
        return RM_DTYPE_BF16
    if t.dtype == torch.float32:
        return RM_DTYPE_FP32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _need(t, name):
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA tensor")


def varlen_bounds(cu_seqlens, S, causal=True, window=0, device=None, stream=None):
    """Visibility table of packed documents (boundaries cu_seqlens, natural
    positions, from 0 to S) for the *_varlen calls: a uint8 device tensor."""
    import torch
    n_docs = len(cu_seqlens) - 1
    nbytes = native.rm_varlen_bounds_size(S, n_docs)
    table = torch.empty(max(nbytes, 256), dtype=torch.uint8,
                        device=device if device is not None else "cuda")
    native.rm_varlen_bounds(cu_seqlens, n_docs, S, causal, window, table, table.numel(), stream)
    return table


def ring_attn_fwd(q, k, v, P, causal=True, order="zigzag", scale=None, out=None, lse=None,
                  stream=None, window=0, bounds=None):
    """Ring attention forward. q [B,H,S,D], k/v [B,Hkv,S,D] (rank-major S).

    window > 0 (causal only): query i sees keys i - window < j <= i.
    bounds: a varlen_bounds() table (packed documents); it carries the mask,
    and causal/window are then ignored.
    Returns (O [B,H,S,D] in q's dtype, LSE [B,H,S] float32).
    """
    import torch
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n)
    B, H, S, D = q.shape
    Hkv = k.shape[1]
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, S), dtype=torch.float32, device=q.device)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    if bounds is not None:
        native.rm_ring_attn_fwd_varlen(q, k, v, out, lse, bounds, B, H, Hkv, S, D, P,
                                       _order(order), _dtype_code(q), scale, stream)
    elif window:
        if not causal:
            raise ValueError("a sliding window needs causal=True")
        native.rm_ring_attn_fwd_window(q, k, v, out, lse, B, H, Hkv, S, D, P, window,
                                       _order(order), _dtype_code(q), scale, stream)
    else:
        native.rm_ring_attn_fwd(q, k, v, out, lse, B, H, Hkv, S, D, P, causal, _order(order),
                                _dtype_code(q), scale, stream)
    return out, lse


def allgather_kv(k, v, P, order="zigzag", outs=None, stream=None):
    """The all-gather of the rank-major k, v [B,Hkv,S,D] on one device: both in
    natural token order, for allgather_attn_fwd."""
    k_all = seq_reorder(k, P, order, "to_natural", out=None if outs is None else outs[0],
                        stream=stream)
    v_all = seq_reorder(v, P, order, "to_natural", out=None if outs is None else outs[1],
                        stream=stream)
    return k_all, v_all


def allgather_attn_fwd(q, k_all, v_all, P, causal=True, order="zigzag", scale=None, out=None,
                       lse=None, stream=None):
    """All-gather attention forward: q [B,H,S,D] rank-major, k_all/v_all
    [B,Hkv,S,D] in natural order (allgather_kv). Returns rank-major (O, LSE),
    the same attention as ring_attn_fwd."""
    import torch
    for t, n in ((q, "q"), (k_all, "k_all"), (v_all, "v_all")):
        _need(t, n)
    B, H, S, D = q.shape
    Hkv = k_all.shape[1]
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, S), dtype=torch.float32, device=q.device)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    native.rm_allgather_attn_fwd(q, k_all, v_all, out, lse, B, H, Hkv, S, D, P, causal,
                                 _order(order), _dtype_code(q), scale, stream)
    return out, lse


def ring_attn_fwd_step(q_local, k_block, v_block, P, rank, owner, causal=True, order="zigzag",
                       scale=None, out=None, lse=None, stream=None):
    """One ring step of rank `rank`: its queries q_local [B,H,L,D] against the
    block k_block/v_block [B,Hkv,L,D] of rank `owner` (L = S / P, local order).
    Returns the step's partial (O [B,H,L,D] float32, LSE [B,H,L] float32); a row
    that sees none of the block gets (0, -inf). Fold partials with lse_merge_."""
    import torch
    for t, n in ((q_local, "q_local"), (k_block, "k_block"), (v_block, "v_block")):
        _need(t, n)
    B, H, L, D = q_local.shape
    Hkv = k_block.shape[1]
    if out is None:
        out = torch.empty(q_local.shape, dtype=torch.float32, device=q_local.device)
    if lse is None:
        lse = torch.empty((B, H, L), dtype=torch.float32, device=q_local.device)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    native.rm_ring_attn_fwd_step(q_local, k_block, v_block, out, lse, B, H, Hkv, L * P, D, P,
                                 rank, owner, causal, _order(order), _dtype_code(q_local), scale,
                                 stream)
    return out, lse


def ring_attn_bwd(q, k, v, o, lse, dout, P, causal=True, order="zigzag", scale=None,
                  workspace=None, stream=None, window=0, bounds=None):
    """Ring attention backward. Returns fp32 (dQ, dK, dV).

    window, bounds: as in ring_attn_fwd (o and lse must come from that mask).
    """
    import torch
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (lse, "lse"), (dout, "dout")):
        _need(t, n)
    B, H, S, D = q.shape
    Hkv = k.shape[1]
    dq = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    dk = torch.empty(k.shape, dtype=torch.float32, device=q.device)
    dv = torch.empty(v.shape, dtype=torch.float32, device=q.device)
    ws_bytes = native.rm_ring_attn_bwd_workspace_size(B, H, S)
    if workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    if bounds is not None:
        native.rm_ring_attn_bwd_varlen(q, k, v, o, lse, dout, dq, dk, dv, bounds, workspace,
                                       workspace.numel(), B, H, Hkv, S, D, P, _order(order),
                                       _dtype_code(q), scale, stream)
    elif window:
        if not causal:
            raise ValueError("a sliding window needs causal=True")
        native.rm_ring_attn_bwd_window(q, k, v, o, lse, dout, dq, dk, dv, workspace,
                                       workspace.numel(), B, H, Hkv, S, D, P, window,
                                       _order(order), _dtype_code(q), scale, stream)
    else:
        native.rm_ring_attn_bwd(q, k, v, o, lse, dout, dq, dk, dv, workspace, workspace.numel(),
                                B, H, Hkv, S, D, P, causal, _order(order), _dtype_code(q), scale,
                                stream)
    return dq, dk, dv


def lse_merge_(o_acc, lse_acc, o_part, lse_part, stream=None):
    """In-place merge of (o_part, lse_part) into (o_acc, lse_acc); fp32 [rows, D], [rows]."""
    for t, n in ((o_acc, "o_acc"), (lse_acc, "lse_acc"), (o_part, "o_part"), (lse_part, "lse_part")):
        _need(t, n)
    D = o_acc.shape[-1]
    rows = o_acc.numel() // D
    native.rm_lse_merge(o_acc, lse_acc, o_part, lse_part, rows, D, stream)
    return o_acc, lse_acc


def ulysses_permute(x, U, R, direction="seq_to_head", out=None, stream=None):
    """[B,S,Hx,D] <-> [B,Hx,S,D] (the Ulysses all-to-all on one device)."""
    import torch
    _need(x, "x")
    if direction == "seq_to_head":
        B, S, Hx, D = x.shape
        shape, d = (B, Hx, S, D), RM_SEQ_TO_HEAD
    else:
        B, Hx, S, D = x.shape
        shape, d = (B, S, Hx, D), RM_HEAD_TO_SEQ
    if out is None:
        out = torch.empty(shape, dtype=x.dtype, device=x.device)
    native.rm_ulysses_permute(x, out, B, S, Hx, D, U, R, x.element_size(), d, stream)
    return out


def ulysses_permute_qkv(q, k, v, U, R, direction="seq_to_head", outs=None, stream=None):
    """Fused Q/K/V Ulysses permute in one launch."""
    import torch
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n)
    if direction == "seq_to_head":
        B, S, H, D = q.shape
        Hkv = k.shape[2]
        shapes, d = [(B, H, S, D), (B, Hkv, S, D), (B, Hkv, S, D)], RM_SEQ_TO_HEAD
    else:
        B, H, S, D = q.shape
        Hkv = k.shape[1]
        shapes, d = [(B, S, H, D), (B, S, Hkv, D), (B, S, Hkv, D)], RM_HEAD_TO_SEQ
    if outs is None:
        outs = [torch.empty(s, dtype=q.dtype, device=q.device) for s in shapes]
    native.rm_ulysses_permute_qkv(q, k, v, outs[0], outs[1], outs[2], B, S, H, Hkv, D, U, R,
                                  q.element_size(), d, stream)
    return tuple(outs)


def seq_reorder(x, P, order="zigzag", direction="to_rank_major", out=None, stream=None):
    """Natural <-> rank-major token order along dim 2 of [B,H,S,D] (or [B,H,S])."""
    import torch
    _need(x, "x")
    if x.dim() == 3:
        B, H, S = x.shape
        D = 1
    else:
        B, H, S, D = x.shape
    if out is None:
        out = torch.empty_like(x)
    d = RM_NATURAL_TO_RANK_MAJOR if direction == "to_rank_major" else RM_RANK_MAJOR_TO_NATURAL
    native.rm_seq_reorder(x, out, B, H, S, D, P, _order(order), d, x.element_size(), stream)
    return out
