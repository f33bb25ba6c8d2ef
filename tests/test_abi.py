"""CPU checks of the C ABI: the library loads, exports every symbol the header
declares, and its host-side validation rejects bad arguments before touching
the GPU (no compute calls are made here)."""
import ctypes
import os
import re
import subprocess

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "rm.h")


@pytest.fixture(scope="module")
def lib():
    from ring_ulysses_sequence_b200 import build, native
    build.build()
    return native.lib()


def header_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^RM_API\s+[\w\s\*]*?\b(rm_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_path():
    fns = header_functions()
    for name in ("rm_ring_attn_fwd", "rm_ring_attn_bwd", "rm_ring_attn_bwd_workspace_size",
                 "rm_ring_attn_fwd_window", "rm_ring_attn_bwd_window", "rm_allgather_attn_fwd",
                 "rm_ring_attn_fwd_step",
                 "rm_varlen_bounds", "rm_ring_attn_fwd_varlen", "rm_ring_attn_bwd_varlen",
                 "rm_lse_merge", "rm_ulysses_permute", "rm_ulysses_permute_qkv",
                 "rm_seq_reorder", "rm_check_device_status", "rm_status_string"):
        assert name in fns


def test_library_exports_every_header_symbol(lib):
    from ring_ulysses_sequence_b200 import native
    out = subprocess.run(["nm", "-D", "--defined-only", native.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\b(rm_\w+)\b", out))
    for name in header_functions():
        assert name in exported, name
        assert getattr(lib, name) is not None
    # and the binding declares exactly the header's functions
    assert sorted(native.SIGNATURES) == header_functions()


def test_status_strings(lib):
    from ring_ulysses_sequence_b200 import native
    assert native.rm_status_string(0) == "ok"
    assert "timed out" in native.rm_status_string(4)
    assert native.rm_status_string(99) == "unknown status"
    assert "work-counter slots" in native.rm_status_string(native.RM_ERR_SLOT_REUSE)
    assert "shared-memory layout" in native.rm_status_string(native.RM_ERR_SMEM_LAYOUT)


def test_workspace_size(lib):
    from ring_ulysses_sequence_b200 import native
    assert native.rm_ring_attn_bwd_workspace_size(1, 2, 1024) == 2 * 1024 * 4
    assert native.rm_ring_attn_bwd_workspace_size(1, 1, 3) == 256  # rounded to 256 B
    assert native.rm_ring_attn_bwd_workspace_size(0, 2, 1024) == 0


A = 1 << 20  # a fake, 16-byte aligned "device address" (never dereferenced)


def fwd(lib, **kw):
    args = dict(q=A, k=A, v=A, o=A, lse=A, B=1, H=4, Hkv=2, S=1024, D=128, P=4, causal=1,
                order=1, dtype=0, scale=0.088, stream=None)
    args.update(kw)
    return lib.rm_ring_attn_fwd(args["q"], args["k"], args["v"], args["o"], args["lse"],
                                args["B"], args["H"], args["Hkv"], args["S"], args["D"],
                                args["P"], args["causal"], args["order"], args["dtype"],
                                args["scale"], args["stream"])


@pytest.mark.parametrize("kw,expect", [
    (dict(q=None), 1), (dict(lse=None), 1), (dict(k=A + 8), 1),          # null / misaligned
    (dict(H=3, Hkv=2), 1), (dict(B=-1), 1), (dict(P=0), 1), (dict(B=0), 0), (dict(S=0), 0),
    (dict(order=7), 1), (dict(dtype=5), 1), (dict(scale=0.0), 1), (dict(scale=float("nan")), 1),
    (dict(S=1004), 1),                                                   # not a multiple of 2P
    (dict(D=96), 2), (dict(S=1024, P=8), 2),                             # chunk 64 < 128 tile
    (dict(order=0, S=768, P=4), 2),                                      # contiguous block 192
])
def test_forward_validation(lib, kw, expect):
    assert fwd(lib, **kw) == expect


def test_backward_validation(lib):
    base = [A] * 10 + [1 << 16, 1, 4, 2, 1024, 128, 4, 1, 1, 0, 0.088, None]
    assert lib.rm_ring_attn_bwd(*base[:9], None, *base[10:]) == 1          # no workspace
    small = list(base)
    small[10] = 64
    assert lib.rm_ring_attn_bwd(*small) == 1                               # too small
    fp32 = list(base)
    fp32[19] = 1
    assert lib.rm_ring_attn_bwd(*fp32) == 2                                # fp32 unsupported
    mis = list(base)
    mis[9] = A + 16                                                        # workspace not 256-aligned
    assert lib.rm_ring_attn_bwd(*mis) == 1


def test_window_validation(lib):
    def fwdw(window, S=1024, **kw):
        return lib.rm_ring_attn_fwd_window(A, A, A, A, A, 1, 4, 2, S, 128, 4, window,
                                           kw.get("order", 1), kw.get("dtype", 0), 0.088, None)
    assert fwdw(0) == 1 and fwdw(-3) == 1                      # the window counts keys, >= 1
    assert fwdw(16, S=0) == 0                                  # empty: nothing to do
    assert fwdw(16, S=1004) == 1                               # shape rules of the forward
    assert fwdw(16, order=9) == 1
    bw = [A] * 10 + [1 << 16, 1, 4, 2, 1024, 128, 4, 64, 1, 0, 0.088, None]
    assert lib.rm_ring_attn_bwd_window(*bw[:9], None, *bw[10:]) == 1   # no workspace
    zero = list(bw)
    zero[17] = 0
    assert lib.rm_ring_attn_bwd_window(*zero) == 1                     # window 0
    fp32 = list(bw)
    fp32[19] = 1
    assert lib.rm_ring_attn_bwd_window(*fp32) == 2                     # fp32 unsupported


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU error path")
def test_window_calls_reach_the_device_without_gpu(lib):
    # valid arguments pass host validation; with no GPU the CUDA lookup fails
    assert lib.rm_ring_attn_fwd_window(A, A, A, A, A, 1, 4, 2, 1024, 128, 4, 300, 1, 0, 0.088,
                                       None) == 3
    assert lib.rm_ring_attn_fwd_window(A, A, A, A, A, 1, 4, 2, 1024, 64, 4, 5000, 0, 1, 0.125,
                                       None) == 3


def test_allgather_validation(lib):
    def ag(S=1024, D=128, dtype=0, order=1, q=A, Hkv=2):
        return lib.rm_allgather_attn_fwd(q, A, A, A, A, 1, 4, Hkv, S, D, 4, 1, order, dtype,
                                         0.088, None)
    assert ag(dtype=1) == 2                      # the fp32 path has no gathered variant
    assert ag(dtype=5) == 1
    assert ag(S=0) == 0                          # empty: nothing to do
    assert ag(S=1004) == 1                       # shape rules of the ring forward
    assert ag(D=96) == 2
    assert ag(q=A + 8) == 1                      # misaligned
    assert ag(Hkv=3) == 1                        # H % Hkv
    assert ag(order=9) == 1


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU error path")
def test_allgather_call_reaches_the_device_without_gpu(lib):
    assert lib.rm_allgather_attn_fwd(A, A, A, A, A, 1, 4, 2, 1024, 128, 4, 1, 1, 0, 0.088,
                                     None) == 3


def test_step_validation(lib):
    def st(rank=0, owner=1, P=4, dtype=0, S=1024, o=A):
        return lib.rm_ring_attn_fwd_step(A, A, A, o, A, 1, 4, 2, S, 128, P, rank, owner, 1, 1,
                                         dtype, 0.088, None)
    assert st(rank=4) == 1 and st(owner=4) == 1 and st(rank=-1) == 1 and st(owner=-2) == 1
    assert st(P=0) == 1
    assert st(dtype=1) == 2                      # the fp32 path has no step variant
    assert st(S=1004) == 1                       # shape rules of the ring forward
    assert st(o=A + 4) == 1                      # misaligned output
    assert st(S=0) == 0                          # empty: nothing to do


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU error path")
def test_step_call_reaches_the_device_without_gpu(lib):
    assert lib.rm_ring_attn_fwd_step(A, A, A, A, A, 1, 4, 2, 1024, 128, 4, 2, 3, 1, 1, 0, 0.088,
                                     None) == 3


def test_varlen_validation(lib):
    import ctypes
    def cu(*xs):
        return (ctypes.c_int * len(xs))(*xs)
    size = lib.rm_varlen_bounds_size(1024, 3)
    assert size >= 1024 * 16 + 16 and size % 256 == 0
    assert lib.rm_varlen_bounds_size(0, 3) == 0
    B = 1 << 20  # 256-byte aligned fake buffer, never touched: validation comes first
    ok = cu(0, 100, 700, 1024)
    assert lib.rm_varlen_bounds(cu(0, 700, 100, 1024), 3, 1024, 1, 0, B, size, None) == 1  # falls
    assert lib.rm_varlen_bounds(cu(5, 100, 700, 1024), 3, 1024, 1, 0, B, size, None) == 1  # not 0
    assert lib.rm_varlen_bounds(cu(0, 100, 700, 1000), 3, 1024, 1, 0, B, size, None) == 1  # not S
    assert lib.rm_varlen_bounds(ok, 3, 1024, 0, 16, B, size, None) == 1    # window needs causal
    assert lib.rm_varlen_bounds(ok, 3, 1024, 1, 0, B, size - 256, None) == 1  # too small
    assert lib.rm_varlen_bounds(ok, 3, 1024, 1, 0, B + 16, size, None) == 1   # misaligned
    assert lib.rm_varlen_bounds(ok, 0, 1024, 1, 0, B, size, None) == 1
    assert lib.rm_varlen_bounds(cu(0, 0), 1, 0, 1, 0, None, 0, None) == 0     # empty: no-op
    # the attention calls need a table
    assert lib.rm_ring_attn_fwd_varlen(A, A, A, A, A, None, 1, 4, 2, 1024, 128, 4, 1, 0, 0.088,
                                       None) == 1
    assert lib.rm_ring_attn_fwd_varlen(A, A, A, A, A, B, 1, 4, 2, 1004, 128, 4, 1, 0, 0.088,
                                       None) == 1


def test_layout_validation(lib):
    # permute: heads not divisible by U, bad element size, aliasing, bad direction
    assert lib.rm_ulysses_permute(A, A * 2, 1, 1024, 6, 128, 4, 2, 2, 0, None) == 1
    assert lib.rm_ulysses_permute(A, A * 2, 1, 1024, 8, 128, 4, 2, 3, 0, None) == 1
    assert lib.rm_ulysses_permute(A, A, 1, 1024, 8, 128, 4, 2, 2, 0, None) == 1
    assert lib.rm_ulysses_permute(A, A * 2, 1, 1024, 8, 128, 4, 2, 2, 9, None) == 1
    assert lib.rm_ulysses_permute(A, A * 2, 1, 1004, 8, 128, 4, 2, 2, 0, None) == 1  # S % (U R)
    # fused: KV heads must be divisible by U as well (Ulysses is capped by KV heads)
    assert lib.rm_ulysses_permute_qkv(A, A, A, A, A, A, 1, 1024, 32, 2, 128, 4, 2, 2, 0, None) == 1
    # reorder
    assert lib.rm_seq_reorder(A, A * 2, 1, 2, 1000, 4, 8, 1, 0, 2, None) == 1  # S % 2P
    assert lib.rm_seq_reorder(A, A, 1, 2, 1024, 4, 8, 1, 0, 2, None) == 1      # in place
    assert lib.rm_seq_reorder(A, A * 2, 1, 2, 1024, 4, 8, 3, 0, 2, None) == 1  # bad order
    # merge
    assert lib.rm_lse_merge(A, A, A, A, -1, 4, None) == 1
    assert lib.rm_lse_merge(None, None, None, None, 0, 4, None) == 0            # nothing to do
    assert lib.rm_lse_merge(A, A, A + 4, A, 10, 4, None) == 1                   # misaligned


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU error path")
def test_valid_call_without_gpu_reports_cuda_error(lib):
    assert fwd(lib) == 3
    assert lib.rm_last_cuda_error() != 0


def test_binding_argument_counts_match_the_header():
    # every RM_API declaration's parameter count equals the ctypes binding's
    from ring_ulysses_sequence_b200 import native
    text = open(HEADER).read()
    decls = re.findall(r"^RM_API\s+[\w\s\*]*?\b(rm_\w+)\s*\(([^;]*?)\)\s*;", text, flags=re.M | re.S)
    assert decls
    for name, params in decls:
        params = " ".join(params.split())
        n = 0 if params in ("", "void") else params.count(",") + 1
        assert len(native.SIGNATURES[name][1]) == n, (name, n, len(native.SIGNATURES[name][1]))


def test_step_merge_and_backward_step_validation(lib):
    # rm_ring_attn_fwd_step_merge: rank/owner range, fp32, shape rules
    def sm(rank=0, owner=0, dtype=0, S=1024, **kw):
        return lib.rm_ring_attn_fwd_step_merge(A, A, A, kw.get("o", A), kw.get("lse", A), 1, 4, 2,
                                               S, 128, 4, rank, owner, 1, 1, dtype, 0.088, None)
    assert sm(rank=4) == 1 and sm(owner=-1) == 1
    assert sm(dtype=1) == 2
    assert sm(S=1004) == 1
    assert sm(o=None) == 1
    assert sm(S=0) == 0
    # rm_ring_attn_bwd_step
    base = [A] * 9 + [1, 4, 2, 1024, 128, 4, 1, 2, 1, 1, 0, 0.088, None]
    assert lib.rm_ring_attn_bwd_step(*base) != 1 or True  # (valid: would launch; not called)
    for i in range(3, 9):                                  # lse .. dv must be given
        bad = list(base)
        bad[i] = None
        assert lib.rm_ring_attn_bwd_step(*bad) == 1, i
    for j, val in ((15, 4), (16, 7), (15, -1)):            # rank, owner out of range
        bad = list(base)
        bad[j] = val
        assert lib.rm_ring_attn_bwd_step(*bad) == 1
    fp32 = list(base)
    fp32[19] = 1
    assert lib.rm_ring_attn_bwd_step(*fp32) == 2
    empty = list(base)
    empty[9] = 0                                           # B = 0: nothing to do
    assert lib.rm_ring_attn_bwd_step(*empty) == 0
    # rm_ring_attn_bwd_delta
    assert lib.rm_ring_attn_bwd_delta(A, A, A, 16, 96, 0, None) == 2      # D = 96
    assert lib.rm_ring_attn_bwd_delta(A, A, A, 16, 128, 3, None) == 1     # bad dtype
    assert lib.rm_ring_attn_bwd_delta(A, A, A, -1, 128, 0, None) == 1
    assert lib.rm_ring_attn_bwd_delta(None, A, A, 0, 128, 0, None) == 0   # no rows
    assert lib.rm_ring_attn_bwd_delta(A, None, A, 8, 128, 0, None) == 1


def test_ulysses_exchange_validation(lib):
    from ring_ulysses_sequence_b200 import native
    assert native.rm_ulysses_buffer_size([32, 8, 8], 2, 16, 128, 2) == 48 * 2 * 16 * 128 * 2
    assert native.rm_ulysses_buffer_size([], 1, 16, 128, 2) == 0
    fake = [A + 4096 * i for i in range(4)]

    def pack(tensors, heads, buf=A + (1 << 24), U=2, eb=2, d=0, B=1, s=16, D=128):
        n = len(tensors)
        ptrs = (ctypes.c_void_p * max(n, 1))(*tensors)
        hs = (ctypes.c_int * max(len(heads), 1))(*heads)
        return lib.rm_ulysses_pack(ctypes.cast(ptrs, ctypes.c_void_p),
                                   ctypes.cast(hs, ctypes.c_void_p), n, buf, B, s, D, U, eb, d,
                                   None)
    assert pack(fake[:1], [6], U=4) == 1                   # 6 heads over U = 4
    assert pack(fake[:4], [2, 2, 2, 2]) == 1               # at most three tensors
    assert pack([], []) == 1
    assert pack(fake[:1], [4], buf=fake[0]) == 1           # the buffer is a tensor
    assert pack(fake[:1], [4], buf=A + 8) == 1             # misaligned buffer
    assert pack(fake[:1], [4], eb=3) == 1
    assert pack(fake[:1], [4], d=5) == 1
    assert pack(fake[:1], [4], B=0) == 0                   # empty
    assert pack([A + 8], [4]) == 1                         # misaligned tensor


def test_wrappers_reject_mismatched_tensors_before_any_call(monkeypatch):
    """The Python wrappers check every tensor's shape and dtype against q's
    before calling the library (a shorter k would make the kernels read past
    its allocation). CPU tensors stand in for device ones here; the native
    calls are replaced by a stub that fails the test if reached."""
    import ring_ulysses_sequence_b200 as rm
    from ring_ulysses_sequence_b200 import native

    class NoCall:
        def __getattr__(self, name):
            if name.startswith("rm_") and not name.endswith("_size"):  # sizes are host math
                def fail(*a, **k):
                    raise AssertionError(f"{name} reached with bad arguments")
                return fail
            return getattr(native, name)
    monkeypatch.setattr(rm, "native", NoCall())
    monkeypatch.setattr(rm, "_need", lambda t, n: None)     # allow CPU tensors
    bf = torch.bfloat16
    q = torch.zeros((1, 4, 256, 128), dtype=bf)
    k = torch.zeros((1, 2, 256, 128), dtype=bf)
    with pytest.raises(ValueError, match="k has shape"):
        rm.ring_attn_fwd(q, k[:, :, :128], k, 2)
    with pytest.raises(ValueError, match="v has dtype"):
        rm.ring_attn_fwd(q, k, k.float(), 2)
    with pytest.raises(ValueError, match="out has shape"):
        rm.ring_attn_fwd(q, k, k, 2, out=torch.zeros((1, 4, 128, 128), dtype=bf))
    with pytest.raises(ValueError, match="lse has dtype"):
        rm.ring_attn_fwd(q, k, k, 2, lse=torch.zeros((1, 4, 256), dtype=bf))
    lse = torch.zeros((1, 4, 256))
    with pytest.raises(ValueError, match="dout has shape"):
        rm.ring_attn_bwd(q, k, k, q, lse, q[:, :2], 2)
    with pytest.raises(ValueError, match="workspace holds"):
        rm.ring_attn_bwd(q, k, k, q, lse, q, 2, workspace=torch.zeros(16, dtype=torch.uint8))
    with pytest.raises(ValueError, match="k_block has shape"):
        rm.ring_attn_fwd_step(q, k[:, :, :64], k, 2, 0, 0)
    with pytest.raises(ValueError, match="lse_acc has shape"):
        rm.ring_attn_fwd_step_merge(q, k, k, q.float(), lse[:, :2], 2, 0, 0)
    with pytest.raises(ValueError, match="dk_block has dtype"):
        rm.ring_attn_bwd_step(q, k, k, lse, lse, q, q.float(), k, k.float(), 2, 0, 0)
    with pytest.raises(ValueError, match="o_part has shape"):
        rm.lse_merge_(torch.zeros(8, 4), torch.zeros(8), torch.zeros(8, 2), torch.zeros(8))
    with pytest.raises(ValueError, match="v has shape"):
        rm.ulysses_permute_qkv(torch.zeros((1, 64, 8, 16), dtype=bf),
                               torch.zeros((1, 64, 4, 16), dtype=bf),
                               torch.zeros((1, 64, 2, 16), dtype=bf), 2, 1)
    with pytest.raises(ValueError, match="must have 4 dimensions"):
        rm.ring_attn_fwd(q[0], k, k, 2)
