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

__all__ = ["ring_attn_fwd", "ring_attn_bwd", "ring_attn_fwd_step", "ring_attn_fwd_step_merge",
           "ring_attn_bwd_delta", "ring_attn_bwd_step", "allgather_kv", "allgather_attn_fwd",
           "varlen_bounds", "lse_merge_", "ulysses_permute", "ulysses_permute_qkv", "ulysses_pack",
           "ulysses_unpack", "seq_reorder", "native", "RMError"]

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


def _check(specs):
    """Host-side checks before any native call: specs is a list of
    (tensor, name, shape, dtype); shape/dtype None skip that check. Every tensor
    must be a contiguous CUDA tensor on the current device, with the stated
    shape and dtype (a mismatch would make the kernels read or write outside
    the allocation, or read the wrong element type)."""
    import torch
    dev = torch.cuda.current_device() if torch.cuda.is_available() else None
    for t, name, shape, dtype in specs:
        if not isinstance(t, torch.Tensor):
            raise TypeError(f"{name} must be a torch.Tensor")
        _need(t, name)
        if dev is not None and t.device.index != dev:
            raise ValueError(f"{name} is on {t.device}, the current device is cuda:{dev}")
        if shape is not None and tuple(t.shape) != tuple(shape):
            raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
        if dtype is not None and t.dtype != dtype:
            raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")


def _dims(t, name, n):
    if t.dim() != n:
        raise ValueError(f"{name} must have {n} dimensions, has {t.dim()}")
    return tuple(t.shape)


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
    B, H, S, D = _dims(q, "q", 4)
    Hkv = _dims(k, "k", 4)[1]
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, S), dtype=torch.float32, device=q.device)
    _check([(q, "q", None, None), (k, "k", (B, Hkv, S, D), q.dtype), (v, "v", (B, Hkv, S, D), q.dtype),
            (out, "out", (B, H, S, D), q.dtype), (lse, "lse", (B, H, S), torch.float32)]
           + ([(bounds, "bounds", None, torch.uint8)] if bounds is not None else []))
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
    B, H, S, D = _dims(q, "q", 4)
    Hkv = _dims(k_all, "k_all", 4)[1]
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, S), dtype=torch.float32, device=q.device)
    _check([(q, "q", None, None), (k_all, "k_all", (B, Hkv, S, D), q.dtype),
            (v_all, "v_all", (B, Hkv, S, D), q.dtype), (out, "out", (B, H, S, D), q.dtype),
            (lse, "lse", (B, H, S), torch.float32)])
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
    B, H, L, D = _dims(q_local, "q_local", 4)
    Hkv = _dims(k_block, "k_block", 4)[1]
    if out is None:
        out = torch.empty(q_local.shape, dtype=torch.float32, device=q_local.device)
    if lse is None:
        lse = torch.empty((B, H, L), dtype=torch.float32, device=q_local.device)
    _check([(q_local, "q_local", None, None), (k_block, "k_block", (B, Hkv, L, D), q_local.dtype),
            (v_block, "v_block", (B, Hkv, L, D), q_local.dtype),
            (out, "out", (B, H, L, D), torch.float32), (lse, "lse", (B, H, L), torch.float32)])
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    native.rm_ring_attn_fwd_step(q_local, k_block, v_block, out, lse, B, H, Hkv, L * P, D, P,
                                 rank, owner, causal, _order(order), _dtype_code(q_local), scale,
                                 stream)
    return out, lse


def ring_attn_fwd_step_merge(q_local, k_block, v_block, o_acc, lse_acc, P, rank, owner,
                             causal=True, order="zigzag", scale=None, stream=None):
    """One ring step of rank `rank` folded into its running pair, in place:
    (o_acc [B,H,L,D] float32, lse_acc [B,H,L] float32) <- merge with the
    step's partial over owner `owner`'s block (k_block/v_block [B,Hkv,L,D]).
    Start from o_acc = 0, lse_acc = -inf; rows that see nothing of the block
    are unchanged. Returns (o_acc, lse_acc)."""
    import torch
    B, H, L, D = _dims(q_local, "q_local", 4)
    Hkv = _dims(k_block, "k_block", 4)[1]
    _check([(q_local, "q_local", None, None), (k_block, "k_block", (B, Hkv, L, D), q_local.dtype),
            (v_block, "v_block", (B, Hkv, L, D), q_local.dtype),
            (o_acc, "o_acc", (B, H, L, D), torch.float32),
            (lse_acc, "lse_acc", (B, H, L), torch.float32)])
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    native.rm_ring_attn_fwd_step_merge(q_local, k_block, v_block, o_acc, lse_acc, B, H, Hkv, L * P,
                                       D, P, rank, owner, causal, _order(order),
                                       _dtype_code(q_local), scale, stream)
    return o_acc, lse_acc


def ring_attn_bwd_delta(o, dout, out=None, stream=None):
    """Delta = rowsum(dout * o) in float32: o [..., D] bf16 or float32, dout
    [..., D] bf16 of the same shape. Returns Delta [...]."""
    import torch
    D = o.shape[-1]
    if out is None:
        out = torch.empty(o.shape[:-1], dtype=torch.float32, device=o.device)
    _check([(o, "o", None, None), (dout, "dout", tuple(o.shape), torch.bfloat16),
            (out, "out", tuple(o.shape[:-1]), torch.float32)])
    native.rm_ring_attn_bwd_delta(o, dout, out, o.numel() // D if D else 0, D, _dtype_code(o),
                                  stream)
    return out


def ring_attn_bwd_step(q_local, k_block, v_block, lse_local, delta_local, dout_local, dq_local,
                       dk_block, dv_block, P, rank, owner, causal=True, order="zigzag",
                       scale=None, stream=None):
    """One step of the backward of a ring across devices, in place: adds rank
    `rank`'s part of the gradients over owner `owner`'s block to dq_local
    [B,H,L,D] and dk_block, dv_block [B,Hkv,L,D] (all float32). lse_local is
    the rank's final forward LSE, delta_local ring_attn_bwd_delta of its O and
    dO. Returns (dq_local, dk_block, dv_block)."""
    import torch
    B, H, L, D = _dims(q_local, "q_local", 4)
    Hkv = _dims(k_block, "k_block", 4)[1]
    dt = q_local.dtype
    _check([(q_local, "q_local", None, None), (k_block, "k_block", (B, Hkv, L, D), dt),
            (v_block, "v_block", (B, Hkv, L, D), dt),
            (lse_local, "lse_local", (B, H, L), torch.float32),
            (delta_local, "delta_local", (B, H, L), torch.float32),
            (dout_local, "dout_local", (B, H, L, D), dt),
            (dq_local, "dq_local", (B, H, L, D), torch.float32),
            (dk_block, "dk_block", (B, Hkv, L, D), torch.float32),
            (dv_block, "dv_block", (B, Hkv, L, D), torch.float32)])
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    native.rm_ring_attn_bwd_step(q_local, k_block, v_block, lse_local, delta_local, dout_local,
                                 dq_local, dk_block, dv_block, B, H, Hkv, L * P, D, P, rank, owner,
                                 causal, _order(order), _dtype_code(q_local), scale, stream)
    return dq_local, dk_block, dv_block


def ring_attn_bwd(q, k, v, o, lse, dout, P, causal=True, order="zigzag", scale=None,
                  workspace=None, stream=None, window=0, bounds=None):
    """Ring attention backward. Returns fp32 (dQ, dK, dV).

    window, bounds: as in ring_attn_fwd (o and lse must come from that mask).
    """
    import torch
    B, H, S, D = _dims(q, "q", 4)
    Hkv = _dims(k, "k", 4)[1]
    dq = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    dk = torch.empty(k.shape, dtype=torch.float32, device=q.device)
    dv = torch.empty(k.shape, dtype=torch.float32, device=q.device)
    ws_bytes = native.rm_ring_attn_bwd_workspace_size(B, H, S)
    if workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    _check([(q, "q", None, None), (k, "k", (B, Hkv, S, D), q.dtype), (v, "v", (B, Hkv, S, D), q.dtype),
            (o, "o", (B, H, S, D), q.dtype), (lse, "lse", (B, H, S), torch.float32),
            (dout, "dout", (B, H, S, D), q.dtype), (workspace, "workspace", None, None)]
           + ([(bounds, "bounds", None, torch.uint8)] if bounds is not None else []))
    if workspace.numel() * workspace.element_size() < ws_bytes:
        raise ValueError(f"workspace holds {workspace.numel() * workspace.element_size()} bytes, "
                         f"needs {ws_bytes}")
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    if bounds is not None:
        native.rm_ring_attn_bwd_varlen(q, k, v, o, lse, dout, dq, dk, dv, bounds, workspace,
                                       workspace.numel() * workspace.element_size(), B, H, Hkv, S, D, P, _order(order),
                                       _dtype_code(q), scale, stream)
    elif window:
        if not causal:
            raise ValueError("a sliding window needs causal=True")
        native.rm_ring_attn_bwd_window(q, k, v, o, lse, dout, dq, dk, dv, workspace,
                                       workspace.numel() * workspace.element_size(), B, H, Hkv, S, D, P, window,
                                       _order(order), _dtype_code(q), scale, stream)
    else:
        native.rm_ring_attn_bwd(q, k, v, o, lse, dout, dq, dk, dv, workspace,
                                workspace.numel() * workspace.element_size(),
                                B, H, Hkv, S, D, P, causal, _order(order), _dtype_code(q), scale,
                                stream)
    return dq, dk, dv


def lse_merge_(o_acc, lse_acc, o_part, lse_part, stream=None):
    """In-place merge of (o_part, lse_part) into (o_acc, lse_acc); fp32 [rows, D], [rows]."""
    import torch
    D = o_acc.shape[-1]
    _check([(o_acc, "o_acc", None, torch.float32),
            (lse_acc, "lse_acc", tuple(o_acc.shape[:-1]), torch.float32),
            (o_part, "o_part", tuple(o_acc.shape), torch.float32),
            (lse_part, "lse_part", tuple(o_acc.shape[:-1]), torch.float32)])
    rows = o_acc.numel() // D
    native.rm_lse_merge(o_acc, lse_acc, o_part, lse_part, rows, D, stream)
    return o_acc, lse_acc


def ulysses_permute(x, U, R, direction="seq_to_head", out=None, stream=None):
    """[B,S,Hx,D] <-> [B,Hx,S,D] (the Ulysses all-to-all on one device)."""
    import torch
    _dims(x, "x", 4)
    if direction == "seq_to_head":
        B, S, Hx, D = x.shape
        shape, d = (B, Hx, S, D), RM_SEQ_TO_HEAD
    else:
        B, Hx, S, D = x.shape
        shape, d = (B, S, Hx, D), RM_HEAD_TO_SEQ
    if out is None:
        out = torch.empty(shape, dtype=x.dtype, device=x.device)
    _check([(x, "x", None, None), (out, "out", shape, x.dtype)])
    native.rm_ulysses_permute(x, out, B, S, Hx, D, U, R, x.element_size(), d, stream)
    return out


def ulysses_permute_qkv(q, k, v, U, R, direction="seq_to_head", outs=None, stream=None):
    """Fused Q/K/V Ulysses permute in one launch."""
    import torch
    _dims(q, "q", 4)
    _dims(k, "k", 4)
    if direction == "seq_to_head":
        B, S, H, D = q.shape
        Hkv = k.shape[2]
        shapes, d = [(B, H, S, D), (B, Hkv, S, D), (B, Hkv, S, D)], RM_SEQ_TO_HEAD
        kshape = (B, S, Hkv, D)
    else:
        B, H, S, D = q.shape
        Hkv = k.shape[1]
        shapes, d = [(B, S, H, D), (B, S, Hkv, D), (B, S, Hkv, D)], RM_HEAD_TO_SEQ
        kshape = (B, Hkv, S, D)
    if outs is None:
        outs = [torch.empty(s, dtype=q.dtype, device=q.device) for s in shapes]
    _check([(q, "q", None, None), (k, "k", kshape, q.dtype), (v, "v", kshape, q.dtype)]
           + [(o, f"outs[{i}]", sh, q.dtype) for i, (o, sh) in enumerate(zip(outs, shapes))])
    native.rm_ulysses_permute_qkv(q, k, v, outs[0], outs[1], outs[2], B, S, H, Hkv, D, U, R,
                                  q.element_size(), d, stream)
    return tuple(outs)


def ulysses_pack(tensors, U, direction="seq_to_head", buf=None, stream=None):
    """One device's send buffer of the Ulysses all-to-all (rm_ulysses_pack).

    seq_to_head: tensors are this device's sequence shards [B, s, heads, D]
    (e.g. Q, K, V); head_to_seq: its head shards [B, heads/U, U*s, D] (e.g.
    O). Returns buf (U equal chunks, chunk u for device u of the group), a
    flat tensor of the tensors' dtype."""
    import torch
    if not 1 <= len(tensors) <= 3:
        raise ValueError("one to three tensors")
    x0 = tensors[0]
    shapes = [_dims(t, f"tensors[{i}]", 4) for i, t in enumerate(tensors)]
    if direction == "seq_to_head":
        B, s, _, D = shapes[0]
        heads = [sh[2] for sh in shapes]
        want = [(B, s, h, D) for h in heads]
        d = RM_SEQ_TO_HEAD
    else:
        B, hU0, Us, D = shapes[0]
        if Us % U:
            raise ValueError(f"the head shard's {Us} tokens do not split over U = {U}")
        s = Us // U
        heads = [sh[1] * U for sh in shapes]
        want = [(B, h // U, Us, D) for h in heads]
        d = RM_HEAD_TO_SEQ
    n = sum(heads) * B * s * D
    if buf is None:
        buf = torch.empty(n, dtype=x0.dtype, device=x0.device)
    _check([(t, f"tensors[{i}]", want[i], x0.dtype) for i, t in enumerate(tensors)]
           + [(buf, "buf", (n,), x0.dtype)])
    native.rm_ulysses_pack(list(tensors), heads, buf, B, s, D, U, x0.element_size(), d, stream)
    return buf


def ulysses_unpack(buf, U, heads, B, s, D, direction="seq_to_head", outs=None, stream=None):
    """The inverse side (rm_ulysses_unpack): the received buffer (chunk u from
    device u) -> this device's head shards [B, heads/U, U*s, D] (seq_to_head)
    or sequence shards [B, s, heads, D] (head_to_seq), one per entry of
    `heads`."""
    import torch
    if direction == "seq_to_head":
        shapes, d = [(B, h // U, U * s, D) for h in heads], RM_SEQ_TO_HEAD
    else:
        shapes, d = [(B, s, h, D) for h in heads], RM_HEAD_TO_SEQ
    if outs is None:
        outs = [torch.empty(sh, dtype=buf.dtype, device=buf.device) for sh in shapes]
    n = sum(heads) * B * s * D
    _check([(buf, "buf", (n,), None)]
           + [(o, f"outs[{i}]", sh, buf.dtype) for i, (o, sh) in enumerate(zip(outs, shapes))])
    native.rm_ulysses_unpack(buf, list(outs), heads, B, s, D, U, buf.element_size(), d, stream)
    return tuple(outs)


def seq_reorder(x, P, order="zigzag", direction="to_rank_major", out=None, stream=None):
    """Natural <-> rank-major token order along dim 2 of [B,H,S,D] (or [B,H,S])."""
    import torch
    if x.dim() == 3:
        B, H, S = x.shape
        D = 1
    else:
        B, H, S, D = _dims(x, "x", 4)
    if out is None:
        out = torch.empty_like(x)
    _check([(x, "x", None, None), (out, "out", tuple(x.shape), x.dtype)])
    d = RM_NATURAL_TO_RANK_MAJOR if direction == "to_rank_major" else RM_RANK_MAJOR_TO_NATURAL
    native.rm_seq_reorder(x, out, B, H, S, D, P, _order(order), d, x.element_size(), stream)
    return out
