"""ctypes binding of librm.so (include/rm.h), one Python function per C entry point.

Argument marshalling only: tensors go in as device pointers, the stream as the
CUDA stream handle. No computation happens here, and there is no fallback: if
the library is missing or a call fails, an exception is raised.
"""
import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "librm.so")

(RM_OK, RM_ERR_INVALID_ARG, RM_ERR_UNSUPPORTED, RM_ERR_CUDA, RM_ERR_TIMEOUT, RM_ERR_SLOT_REUSE,
 RM_ERR_SMEM_LAYOUT) = range(7)
RM_ORDER_CONTIGUOUS, RM_ORDER_ZIGZAG = 0, 1
RM_DTYPE_BF16, RM_DTYPE_FP32 = 0, 1
RM_SEQ_TO_HEAD, RM_HEAD_TO_SEQ = 0, 1
RM_NATURAL_TO_RANK_MAJOR, RM_RANK_MAJOR_TO_NATURAL = 0, 1

# name -> (restype, argtypes), in the order of include/rm.h
_vp, _i, _i64, _f, _sz, _u64 = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float,
                                 ctypes.c_size_t, ctypes.c_uint64)
SIGNATURES = {
    "rm_ring_attn_fwd": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _i, _f, _vp]),
    "rm_allgather_attn_fwd": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _i,
                                   _f, _vp]),
    "rm_ring_attn_fwd_step": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _i,
                                   _i, _i, _f, _vp]),
    "rm_ring_attn_fwd_step_merge": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i,
                                         _i, _i, _i, _i, _f, _vp]),
    "rm_ring_attn_fwd_window": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _i,
                                     _f, _vp]),
    "rm_varlen_bounds_size": (_sz, [_i, _i]),
    "rm_varlen_bounds": (_i, [_vp, _i, _i, _i, _i, _vp, _sz, _vp]),
    "rm_ring_attn_fwd_varlen": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i,
                                     _f, _vp]),
    "rm_ring_attn_bwd_workspace_size": (_sz, [_i, _i, _i]),
    "rm_ring_attn_bwd": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz,
                              _i, _i, _i, _i, _i, _i, _i, _i, _i, _f, _vp]),
    "rm_ring_attn_bwd_window": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz,
                                     _i, _i, _i, _i, _i, _i, _i, _i, _i, _f, _vp]),
    "rm_ring_attn_bwd_varlen": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz,
                                     _i, _i, _i, _i, _i, _i, _i, _i, _f, _vp]),
    "rm_ring_attn_bwd_noalloc": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                      _i, _i, _i, _i, _i, _i, _i, _i, _i, _f, _vp]),
    "rm_ring_attn_bwd_delta": (_i, [_vp, _vp, _vp, _i64, _i, _i, _vp]),
    "rm_ring_attn_bwd_step": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i,
                                   _i, _i, _i, _i, _i, _i, _i, _f, _vp]),
    "rm_lse_merge": (_i, [_vp, _vp, _vp, _vp, _i64, _i, _vp]),
    "rm_ulysses_permute": (_i, [_vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _vp]),
    "rm_ulysses_permute_qkv": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i,
                                    _i, _i, _vp]),
    "rm_ulysses_buffer_size": (_sz, [_vp, _i, _i, _i, _i, _i]),
    "rm_ulysses_pack": (_i, [_vp, _vp, _i, _vp, _i, _i, _i, _i, _i, _i, _vp]),
    "rm_ulysses_unpack": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _vp]),
    "rm_seq_reorder": (_i, [_vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _vp]),
    "rm_check_device_status": (_i, [_vp]),
    "rm_set_watchdog_ns": (None, [_u64]),
    "rm_set_bwd_deterministic": (None, [_i]),
    "rm_get_bwd_deterministic": (_i, []),
    "rm_watchdog_selftest": (_i, [_u64, _vp]),
    "rm_status_string": (ctypes.c_char_p, [_i]),
    "rm_last_cuda_error": (_i, []),
}

_lib = None


class RMError(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        msg = lib().rm_status_string(status).decode()
        if status == RM_ERR_CUDA:
            msg += f" (cudaError {lib().rm_last_cuda_error()})"
        super().__init__(f"{fn}: {msg}")


def lib():
    """The loaded librm.so; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m ring_ulysses_sequence_b200.build` (needs nvcc).")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def _call(name, *args):
    st = getattr(lib(), name)(*args)
    if st != RM_OK:
        raise RMError(name, st)
    return st


def _p(t):
    """Device pointer of a tensor (or an int address, or None)."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _s(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def rm_ring_attn_fwd(q, k, v, o, lse, B, H, Hkv, S, D, P, causal, order, dtype, scale,
                     stream=None):
    return _call("rm_ring_attn_fwd", _p(q), _p(k), _p(v), _p(o), _p(lse), B, H, Hkv, S, D, P,
                 int(causal), order, dtype, scale, _s(stream))


def rm_allgather_attn_fwd(q, k_all, v_all, o, lse, B, H, Hkv, S, D, P, causal, order, dtype,
                          scale, stream=None):
    return _call("rm_allgather_attn_fwd", _p(q), _p(k_all), _p(v_all), _p(o), _p(lse), B, H, Hkv,
                 S, D, P, int(causal), order, dtype, scale, _s(stream))


def rm_ring_attn_fwd_step(q_local, k_block, v_block, o_part, lse_part, B, H, Hkv, S, D, P, rank,
                          owner, causal, order, dtype, scale, stream=None):
    return _call("rm_ring_attn_fwd_step", _p(q_local), _p(k_block), _p(v_block), _p(o_part),
                 _p(lse_part), B, H, Hkv, S, D, P, rank, owner, int(causal), order, dtype, scale,
                 _s(stream))


def rm_ring_attn_fwd_step_merge(q_local, k_block, v_block, o_acc, lse_acc, B, H, Hkv, S, D, P,
                                rank, owner, causal, order, dtype, scale, stream=None):
    return _call("rm_ring_attn_fwd_step_merge", _p(q_local), _p(k_block), _p(v_block), _p(o_acc),
                 _p(lse_acc), B, H, Hkv, S, D, P, rank, owner, int(causal), order, dtype, scale,
                 _s(stream))


def rm_ring_attn_fwd_window(q, k, v, o, lse, B, H, Hkv, S, D, P, window, order, dtype, scale,
                            stream=None):
    return _call("rm_ring_attn_fwd_window", _p(q), _p(k), _p(v), _p(o), _p(lse), B, H, Hkv, S, D,
                 P, window, order, dtype, scale, _s(stream))


def rm_varlen_bounds_size(S, n_docs):
    return int(lib().rm_varlen_bounds_size(S, n_docs))


def rm_varlen_bounds(cu_seqlens, n_docs, S, causal, window, bounds, bounds_bytes, stream=None):
    """cu_seqlens: a sequence of n_docs + 1 host integers."""
    arr = (ctypes.c_int * (n_docs + 1))(*[int(x) for x in cu_seqlens])
    return _call("rm_varlen_bounds", ctypes.cast(arr, ctypes.c_void_p), n_docs, S, int(causal),
                 window, _p(bounds), bounds_bytes, _s(stream))


def rm_ring_attn_fwd_varlen(q, k, v, o, lse, bounds, B, H, Hkv, S, D, P, order, dtype, scale,
                            stream=None):
    return _call("rm_ring_attn_fwd_varlen", _p(q), _p(k), _p(v), _p(o), _p(lse), _p(bounds), B,
                 H, Hkv, S, D, P, order, dtype, scale, _s(stream))


def rm_ring_attn_bwd_workspace_size(B, H, S):
    return int(lib().rm_ring_attn_bwd_workspace_size(B, H, S))


def rm_ring_attn_bwd(q, k, v, o, lse, dout, dq, dk, dv, workspace, workspace_bytes, B, H, Hkv, S,
                     D, P, causal, order, dtype, scale, stream=None):
    return _call("rm_ring_attn_bwd", _p(q), _p(k), _p(v), _p(o), _p(lse), _p(dout), _p(dq),
                 _p(dk), _p(dv), _p(workspace), workspace_bytes, B, H, Hkv, S, D, P, int(causal),
                 order, dtype, scale, _s(stream))


def rm_ring_attn_bwd_window(q, k, v, o, lse, dout, dq, dk, dv, workspace, workspace_bytes, B, H,
                            Hkv, S, D, P, window, order, dtype, scale, stream=None):
    return _call("rm_ring_attn_bwd_window", _p(q), _p(k), _p(v), _p(o), _p(lse), _p(dout),
                 _p(dq), _p(dk), _p(dv), _p(workspace), workspace_bytes, B, H, Hkv, S, D, P,
                 window, order, dtype, scale, _s(stream))


def rm_ring_attn_bwd_varlen(q, k, v, o, lse, dout, dq, dk, dv, bounds, workspace, workspace_bytes,
                            B, H, Hkv, S, D, P, order, dtype, scale, stream=None):
    return _call("rm_ring_attn_bwd_varlen", _p(q), _p(k), _p(v), _p(o), _p(lse), _p(dout),
                 _p(dq), _p(dk), _p(dv), _p(bounds), _p(workspace), workspace_bytes, B, H, Hkv,
                 S, D, P, order, dtype, scale, _s(stream))


def rm_ring_attn_bwd_noalloc(q, k, v, o, lse, dout, dq, dk, dv, B, H, Hkv, S, D, P, causal,
                             order, dtype, scale, stream=None):
    return _call("rm_ring_attn_bwd_noalloc", _p(q), _p(k), _p(v), _p(o), _p(lse), _p(dout),
                 _p(dq), _p(dk), _p(dv), B, H, Hkv, S, D, P, int(causal), order, dtype, scale,
                 _s(stream))


def rm_ring_attn_bwd_delta(o, dout, delta, rows, D, o_dtype, stream=None):
    return _call("rm_ring_attn_bwd_delta", _p(o), _p(dout), _p(delta), rows, D, o_dtype,
                 _s(stream))


def rm_ring_attn_bwd_step(q_local, k_block, v_block, lse_local, delta_local, dout_local, dq_local,
                          dk_block, dv_block, B, H, Hkv, S, D, P, rank, owner, causal, order,
                          dtype, scale, stream=None):
    return _call("rm_ring_attn_bwd_step", _p(q_local), _p(k_block), _p(v_block), _p(lse_local),
                 _p(delta_local), _p(dout_local), _p(dq_local), _p(dk_block), _p(dv_block), B, H,
                 Hkv, S, D, P, rank, owner, int(causal), order, dtype, scale, _s(stream))


def rm_lse_merge(o_acc, lse_acc, o_part, lse_part, rows, D, stream=None):
    return _call("rm_lse_merge", _p(o_acc), _p(lse_acc), _p(o_part), _p(lse_part), rows, D,
                 _s(stream))


def rm_ulysses_permute(src, dst, B, S, Hx, D, U, R, elem_bytes, direction, stream=None):
    return _call("rm_ulysses_permute", _p(src), _p(dst), B, S, Hx, D, U, R, elem_bytes,
                 direction, _s(stream))


def rm_ulysses_permute_qkv(q_src, k_src, v_src, q_dst, k_dst, v_dst, B, S, H, Hkv, D, U, R,
                           elem_bytes, direction, stream=None):
    return _call("rm_ulysses_permute_qkv", _p(q_src), _p(k_src), _p(v_src), _p(q_dst),
                 _p(k_dst), _p(v_dst), B, S, H, Hkv, D, U, R, elem_bytes, direction, _s(stream))


def _host_arrays(tensors, heads):
    n = len(tensors)
    ptrs = (ctypes.c_void_p * n)(*[_p(t) for t in tensors])
    hs = (ctypes.c_int * n)(*[int(h) for h in heads])
    return n, ctypes.cast(ptrs, ctypes.c_void_p), ctypes.cast(hs, ctypes.c_void_p), (ptrs, hs)


def rm_ulysses_buffer_size(heads, B, s, D, elem_bytes):
    hs = (ctypes.c_int * len(heads))(*[int(h) for h in heads])
    return int(lib().rm_ulysses_buffer_size(ctypes.cast(hs, ctypes.c_void_p), len(heads), B, s,
                                            D, elem_bytes))


def rm_ulysses_pack(tensors, heads, send_buf, B, s, D, U, elem_bytes, direction, stream=None):
    n, ptrs, hs, keep = _host_arrays(tensors, heads)
    return _call("rm_ulysses_pack", ptrs, hs, n, _p(send_buf), B, s, D, U, elem_bytes, direction,
                 _s(stream))


def rm_ulysses_unpack(recv_buf, tensors, heads, B, s, D, U, elem_bytes, direction, stream=None):
    n, ptrs, hs, keep = _host_arrays(tensors, heads)
    return _call("rm_ulysses_unpack", _p(recv_buf), ptrs, hs, n, B, s, D, U, elem_bytes,
                 direction, _s(stream))


def rm_seq_reorder(src, dst, B, H, S, D, P, order, direction, elem_bytes, stream=None):
    return _call("rm_seq_reorder", _p(src), _p(dst), B, H, S, D, P, order, direction, elem_bytes,
                 _s(stream))


def rm_check_device_status(stream=None):
    """Returns the status code (does not raise on RM_ERR_TIMEOUT)."""
    return int(lib().rm_check_device_status(_s(stream)))


def rm_set_watchdog_ns(ns):
    lib().rm_set_watchdog_ns(int(ns))


def rm_set_bwd_deterministic(on):
    lib().rm_set_bwd_deterministic(int(bool(on)))


def rm_get_bwd_deterministic():
    return int(lib().rm_get_bwd_deterministic())


def rm_watchdog_selftest(timeout_ns, stream=None):
    return _call("rm_watchdog_selftest", int(timeout_ns), _s(stream))


def rm_status_string(status):
    return lib().rm_status_string(status).decode()


def rm_last_cuda_error():
    return int(lib().rm_last_cuda_error())
