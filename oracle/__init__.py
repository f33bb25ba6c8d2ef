"""fp64 CPU oracle for blockwise ring attention and its layout transforms.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference legs are the only callers. It shares no
code with the CUDA library and imports nothing from it.

Every array here is numpy. Attention tensors are [B, H, S, D] (keys/values
[B, Hkv, S, D]) in NATURAL token order; the functions widen their inputs to
float64 (exact for bf16 and fp32 values) and return float64.

Pages followed (cited by title and section):
  * "DeDLOC Guide: Decentralized Long-Context Attention", Step 3: local step
    returning (O, LSE) with scale 1/sqrt(D); section 3 "Online Softmax
    Rescaling Across Decentralized Ranks": the merge of partials; Best
    Practices table, "Causal Mask Handling".
  * "Sequence Parallelism III: Ring Attention ..." (duoan.github.io LLM tag
    index): fixed query block, key/value blocks circulating around the ring.
  * "Sequence Parallelism II: DeepSpeed Ulysses and All-to-All Attention"
    (same index): before the all-to-all every rank has all heads for a subset of
    tokens; after it, all tokens for a subset of heads.
  * "context parallelism" (Last Dictionary) and the axolotl-ringmaster README
    (Layout: balancers.py head_tail index generation): chunk reordering for
    causal load balance.
"""
import ctypes
import os

import numpy as np

from . import build as _build

CONTIGUOUS = 0
ZIGZAG = 1

_lib = None


def _L():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        i64, dp, ip, c_int, c_double = (ctypes.c_int64, ctypes.POINTER(ctypes.c_double),
                                        ctypes.POINTER(ctypes.c_int64), ctypes.c_int,
                                        ctypes.c_double)
        lib.orc_rank_major_position.restype = i64
        lib.orc_rank_major_position.argtypes = [i64, i64, c_int, i64]
        lib.orc_attn_fwd_head.restype = None
        lib.orc_attn_fwd_head.argtypes = [dp, dp, dp, i64, i64, c_int, i64, ip, i64, c_double, ip,
                                          i64, dp, dp]
        lib.orc_ring_fwd_head.restype = None
        lib.orc_ring_fwd_head.argtypes = [dp, dp, dp, i64, i64, c_int, i64, ip, i64, c_double, i64,
                                          c_int, ip, i64, dp, dp]
        lib.orc_lse_merge.restype = None
        lib.orc_lse_merge.argtypes = [dp, dp, dp, dp, i64, i64]
        lib.orc_attn_bwd_head.restype = None
        lib.orc_attn_bwd_head.argtypes = [dp, dp, dp, dp, i64, i64, c_int, i64, ip, i64, c_double,
                                          ip, i64, dp, ip, i64, dp, dp]
        lib.orc_ring_owner.restype = i64
        lib.orc_ring_owner.argtypes = [i64, i64, i64]
        lib.orc_num_threads.restype = c_int
        lib.orc_num_threads.argtypes = []
        _lib = lib
    return _lib


def _f64(a):
    """Exact widening to contiguous float64 (numpy or torch input)."""
    if hasattr(a, "detach"):  # torch tensor: bf16/fp32 -> fp64 exactly
        import torch
        a = a.detach().to("cpu", torch.float64).numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _i64(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.int64))


def _p(a, t=ctypes.c_double):
    return a.ctypes.data_as(ctypes.POINTER(t))


def _shape(a):
    return tuple(a.shape)


def _rows_of(x, r):
    """Rows r (int64 numpy) of a 2-D numpy array or torch tensor."""
    if hasattr(x, "index_select"):
        import torch
        return x.index_select(0, torch.from_numpy(r))
    return x[r]


def num_threads() -> int:
    return int(_L().orc_num_threads())


# ---------------------------------------------------------------------------
# Token order of the ring
# ---------------------------------------------------------------------------

def rank_major_positions(S: int, P: int, order: int) -> np.ndarray:
    """pos[s] = natural token position held by rank-major slot s.

    Rank i's L = S/P tokens occupy slots [i*L, (i+1)*L). Contiguous: rank i
    holds tokens [i*L, (i+1)*L). Zigzag: 2P chunks of c = S/(2P); rank i holds
    chunk i then chunk 2P-1-i.
    """
    lib = _L()
    pos = np.array([lib.orc_rank_major_position(S, P, order, s) for s in range(S)],
                   dtype=np.int64)
    if (pos < 0).any():
        raise ValueError(f"bad ring layout S={S} P={P} order={order}")
    return pos


def ring_owner(P: int, i: int, t: int) -> int:
    """Owner of the key/value block rank i holds at ring step t."""
    return int(_L().orc_ring_owner(P, i, t))


def to_rank_major(x: np.ndarray, P: int, order: int, axis: int = -2) -> np.ndarray:
    """Natural token order -> rank-major slots along `axis` (a gather)."""
    S = x.shape[axis]
    return np.take(x, rank_major_positions(S, P, order), axis=axis)


def to_natural(x: np.ndarray, P: int, order: int, axis: int = -2) -> np.ndarray:
    """Rank-major slots -> natural token order along `axis` (the inverse scatter)."""
    S = x.shape[axis]
    pos = rank_major_positions(S, P, order)
    inv = np.empty_like(pos)
    inv[pos] = np.arange(S, dtype=np.int64)
    return np.take(x, inv, axis=axis)


# ---------------------------------------------------------------------------
# Ulysses all-to-all as a layout map
# ---------------------------------------------------------------------------

def ulysses_seq_to_head(x: np.ndarray) -> np.ndarray:
    """Sequence-sharded [B, S, H, D] -> head-sharded [B, H, S, D].

    Device (r, u) of a U x R mesh holds the S/(U R) tokens of shard n = r*U+u
    and all H heads before the exchange; afterwards it holds all S/R tokens of
    ring rank r for heads [u*H/U, (u+1)*H/U). Laid out on one device, both
    sides are the same tensor in two index orders: [B, S, H, D] and
    [B, H, S, D] with S rank-major.
    """
    return np.ascontiguousarray(np.transpose(x, (0, 2, 1, 3)))


def ulysses_head_to_seq(x: np.ndarray) -> np.ndarray:
    """Head-sharded [B, H, S, D] -> sequence-sharded [B, S, H, D]."""
    return np.ascontiguousarray(np.transpose(x, (0, 2, 1, 3)))


# ---------------------------------------------------------------------------
# Attention
# ---------------------------------------------------------------------------

def _rows_arg(rows, S):
    return _i64(np.arange(S) if rows is None else rows)


def _cu_arg(cu_seqlens, S):
    """Document boundaries as an int64 array (cu[0] = 0, ..., cu[n] = S), or None."""
    if cu_seqlens is None:
        return None, 0
    cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
    if cu.ndim != 1 or len(cu) < 2 or cu[0] != 0 or cu[-1] != S or np.any(np.diff(cu) < 0):
        raise ValueError("cu_seqlens must rise from 0 to S")
    return cu, len(cu) - 1


def attn_fwd(q, k, v, causal: bool, scale: float = None, rows=None, window: int = 0,
             cu_seqlens=None):
    """Dense softmax attention in natural order.

    window: with causal, each query sees its last `window` keys (itself
    included); 0 = no window.
    cu_seqlens: packed documents [cu[d], cu[d+1]); a query sees keys of its
    own document only. None = one document.

    q [B,H,S,D], k/v [B,Hkv,Sk,D] (numpy or torch, any float dtype; widened to
    fp64 one head at a time); query head h reads KV head h // (H/Hkv).
    rows: natural query positions to evaluate (same for every head), or None
    for all. Returns O [B,H,n,D] and LSE [B,H,n] (natural log of the scaled
    scores), float64.
    """
    B, H, S, D = _shape(q)
    Hkv, Sk = _shape(k)[1], _shape(k)[2]
    G = H // Hkv
    scale = 1.0 / np.sqrt(D) if scale is None else float(scale)
    cu, ndoc = _cu_arg(cu_seqlens, Sk)
    r = _rows_arg(rows, S)
    o = np.zeros((B, H, len(r), D))
    lse = np.zeros((B, H, len(r)))
    lib = _L()
    for b in range(B):
        for g in range(Hkv):
            kh, vh = _f64(k[b, g]), _f64(v[b, g])
            for h in range(g * G, (g + 1) * G):
                qh = _f64(_rows_of(q[b, h], r) if rows is not None else q[b, h])
                ob = np.zeros((len(r), D))
                lb = np.zeros(len(r))
                lib.orc_attn_fwd_head(_p(qh), _p(kh), _p(vh), Sk, D, int(causal), int(window),
                                      _p(cu, ctypes.c_int64) if cu is not None else None, ndoc,
                                      scale, _p(r, ctypes.c_int64), len(r), _p(ob), _p(lb))
                o[b, h], lse[b, h] = ob, lb
    return o, lse


def ring_fwd(q, k, v, causal: bool, P: int, order: int, scale: float = None, rows=None,
             window: int = 0, cu_seqlens=None):
    """Ring-structured forward: per (rank, step) partials merged step by step.

    Same arguments and results as attn_fwd (natural order in and out); the
    ring layout only decides which keys each step's partial covers.
    """
    B, H, S, D = _shape(q)
    Hkv = _shape(k)[1]
    G = H // Hkv
    scale = 1.0 / np.sqrt(D) if scale is None else float(scale)
    cu, ndoc = _cu_arg(cu_seqlens, S)
    r = _rows_arg(rows, S)
    o = np.zeros((B, H, len(r), D))
    lse = np.zeros((B, H, len(r)))
    lib = _L()
    for b in range(B):
        for g in range(Hkv):
            kh, vh = _f64(k[b, g]), _f64(v[b, g])
            for h in range(g * G, (g + 1) * G):
                qh = _f64(_rows_of(q[b, h], r) if rows is not None else q[b, h])
                ob = np.zeros((len(r), D))
                lb = np.zeros(len(r))
                lib.orc_ring_fwd_head(_p(qh), _p(kh), _p(vh), S, D, int(causal), int(window),
                                      _p(cu, ctypes.c_int64) if cu is not None else None, ndoc,
                                      scale, P, order, _p(r, ctypes.c_int64), len(r), _p(ob),
                                      _p(lb))
                o[b, h], lse[b, h] = ob, lb
    return o, lse


def step_partial(q_local, k_block, v_block, S: int, P: int, order: int, rank: int, owner: int,
                 causal: bool, scale: float = None):
    """One ring step's partial ("DeDLOC Guide", Step 3, restricted to one
    owner's keys): softmax attention of rank `rank`'s queries over the keys of
    rank `owner`'s block only, causal on GLOBAL positions. A row that sees no
    key of the block gets (O, LSE) = (0, -inf), the identity of the merge.

    q_local [B,H,L,D], k_block/v_block [B,Hkv,L,D] in the ranks' local order
    (L = S/P). Plain dense fp64 numpy, written out from the definition; meant
    for small cases. Returns O [B,H,L,D], LSE [B,H,L] float64.
    """
    q, k, v = _f64(q_local), _f64(k_block), _f64(v_block)
    B, H, L, D = q.shape
    Hkv = k.shape[1]
    G = H // Hkv
    scale = 1.0 / np.sqrt(D) if scale is None else float(scale)
    pos = rank_major_positions(S, P, order)
    qpos = pos[rank * L:(rank + 1) * L]
    kpos = pos[owner * L:(owner + 1) * L]
    visible = kpos[None, :] <= qpos[:, None] if causal else np.ones((L, L), dtype=bool)
    o = np.zeros((B, H, L, D))
    lse = np.full((B, H, L), -np.inf)
    for b in range(B):
        for h in range(H):
            s = np.where(visible, (q[b, h] @ k[b, h // G].T) * scale, -np.inf)
            seen = visible.any(axis=1)
            if not seen.any():
                continue
            m = s[seen].max(axis=1, keepdims=True)
            e = np.exp(s[seen] - m)
            l = e.sum(axis=1, keepdims=True)
            o[b, h][seen] = (e / l) @ v[b, h // G]
            lse[b, h][seen] = (m + np.log(l))[:, 0]
    return o, lse


def step_bwd_partial(q_local, k_block, v_block, dout_local, lse_local, delta_local, S: int,
                     P: int, order: int, rank: int, owner: int, causal: bool,
                     scale: float = None):
    """One ring step's share of the gradients (the backward of L = sum(dO * O)
    restricted to the pairs (query of rank `rank`, key of owner `owner`'s
    block); axolotl-ringmaster README, Benchmark: the reverse-ring backward).
    With P_ij = exp(scale q_i.k_j - LSE_i) over the visible pairs and
    Delta_i = <dO_i, O_i> of the FULL attention (both inputs here):
      dV_j = sum_i P_ij dO_i,  dS_ij = P_ij (<dO_i, v_j> - Delta_i),
      dQ_i = scale sum_j dS_ij k_j,  dK_j = scale sum_i dS_ij q_i,
    KV gradients summed over the G heads that share a KV head.

    q_local, dout_local [B,H,L,D], k_block, v_block [B,Hkv,L,D] in local
    order; lse_local, delta_local [B,H,L]. Plain dense fp64 numpy, written
    out from the definition; meant for small cases. Returns (dQ [B,H,L,D],
    dK [B,Hkv,L,D], dV [B,Hkv,L,D]) float64.
    """
    q, k, v, do = _f64(q_local), _f64(k_block), _f64(v_block), _f64(dout_local)
    lse, delta = _f64(lse_local), _f64(delta_local)
    B, H, L, D = q.shape
    Hkv = k.shape[1]
    G = H // Hkv
    scale = 1.0 / np.sqrt(D) if scale is None else float(scale)
    pos = rank_major_positions(S, P, order)
    qpos = pos[rank * L:(rank + 1) * L]
    kpos = pos[owner * L:(owner + 1) * L]
    visible = kpos[None, :] <= qpos[:, None] if causal else np.ones((L, L), dtype=bool)
    dq = np.zeros((B, H, L, D))
    dk = np.zeros((B, Hkv, L, D))
    dv = np.zeros((B, Hkv, L, D))
    for b in range(B):
        for h in range(H):
            g = h // G
            s = (q[b, h] @ k[b, g].T) * scale
            p = np.where(visible, np.exp(s - lse[b, h][:, None]), 0.0)
            dp = do[b, h] @ v[b, g].T
            ds = p * (dp - delta[b, h][:, None])
            dq[b, h] = scale * (ds @ k[b, g])
            dk[b, g] += scale * (ds.T @ q[b, h])
            dv[b, g] += p.T @ do[b, h]
    return dq, dk, dv


def lse_merge(o_acc, lse_acc, o_part, lse_part):
    """Merge partial (O, LSE) pairs row by row; returns new (O, LSE).

    o_* [rows, D], lse_* [rows]. Empty partials are (0, -inf).
    """
    oa, la = _f64(o_acc).copy(), _f64(lse_acc).copy()
    op, lp = _f64(o_part), _f64(lse_part)
    rows, D = oa.shape
    _L().orc_lse_merge(_p(oa), _p(la), _p(op), _p(lp), rows, D)
    return oa, la


def attn_bwd(q, k, v, dout, causal: bool, scale: float = None, qrows=None,
             krows=None, heads=None, window: int = 0, cu_seqlens=None):
    """Gradients of L = sum(dout * O) for dense attention (natural order).

    qrows: natural query positions for dQ (None = all); krows: key positions
    for dK/dV (None = all). heads: iterable of (b, h) query heads for dQ and
    (b, g) KV heads for dK/dV to evaluate (None = all). Returns dicts keyed by
    (b, h) -> dQ [nq, D] and (b, g) -> (dK [nk, D], dV [nk, D]); the KV
    gradients are summed over the G query heads that share KV head g.
    """
    B, H, S, D = _shape(q)
    Hkv = _shape(k)[1]
    G = H // Hkv
    scale = 1.0 / np.sqrt(D) if scale is None else float(scale)
    cu, ndoc = _cu_arg(cu_seqlens, S)
    qr = _rows_arg(qrows, S)
    kr = _rows_arg(krows, S)
    lib = _L()
    dq_out, dkv_out = {}, {}
    qheads = [(b, h) for b in range(B) for h in range(H)] if heads is None else \
        [bh for bh in heads[0]]
    kvheads = [(b, g) for b in range(B) for g in range(Hkv)] if heads is None else \
        [bg for bg in heads[1]]
    need = {}
    for (b, h) in qheads:
        need.setdefault((b, h), [False, False])[0] = True
    for (b, g) in kvheads:
        for h in range(g * G, (g + 1) * G):
            need.setdefault((b, h), [False, False])[1] = True
    for (b, h), (want_q, want_kv) in sorted(need.items()):
        g = h // G
        qh, kh = _f64(q[b, h]), _f64(k[b, g])
        vh, doh = _f64(v[b, g]), _f64(dout[b, h])
        nq = len(qr) if want_q else 0
        nk = len(kr) if want_kv else 0
        dq = np.zeros((max(nq, 1), D))
        dk = np.zeros((max(nk, 1), D))
        dv = np.zeros((max(nk, 1), D))
        lib.orc_attn_bwd_head(_p(qh), _p(kh), _p(vh), _p(doh), S, D, int(causal), int(window),
                              _p(cu, ctypes.c_int64) if cu is not None else None, ndoc,
                              scale, _p(qr, ctypes.c_int64), nq, _p(dq),
                              _p(kr, ctypes.c_int64), nk, _p(dk), _p(dv))
        if want_q:
            dq_out[(b, h)] = dq[:nq]
        if want_kv and (b, g) in set(kvheads):
            acc = dkv_out.setdefault((b, g), [np.zeros((nk, D)), np.zeros((nk, D))])
            acc[0] += dk[:nk]
            acc[1] += dv[:nk]
    return dq_out, {key: (val[0], val[1]) for key, val in dkv_out.items()}
