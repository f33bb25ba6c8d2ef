"""Helpers shared by the GPU parity tests (no attention arithmetic here)."""
import numpy as np
import torch

import oracle

ORDER = {"contiguous": oracle.CONTIGUOUS, "zigzag": oracle.ZIGZAG}

# Tolerances: bf16 inputs with fp32 accumulation, and the fp32 path.
BF16_MAX_ABS, BF16_MEAN_ABS = 2e-2, 2e-3
FP32_MAX_ABS = 1e-4
LSE_MAX_ABS = 1e-3


def to_rank_major(x: torch.Tensor, P: int, order: str, dim: int = 2) -> torch.Tensor:
    """Natural -> rank-major along `dim`, with the oracle's position map."""
    pos = torch.from_numpy(oracle.rank_major_positions(x.shape[dim], P, ORDER[order]))
    return x.index_select(dim, pos).contiguous()


def to_natural(x: torch.Tensor, P: int, order: str, dim: int = 2) -> torch.Tensor:
    pos = oracle.rank_major_positions(x.shape[dim], P, ORDER[order])
    inv = np.empty_like(pos)
    inv[pos] = np.arange(len(pos))
    return x.index_select(dim, torch.from_numpy(inv)).contiguous()


def assert_close(got, ref, max_abs, mean_abs=None, what=""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite values"
    err = np.abs(got - ref)
    mx = float(err.max()) if err.size else 0.0
    assert mx <= max_abs, f"{what}: max-abs {mx:.3e} > {max_abs:.1e}"
    if mean_abs is not None and err.size:
        mn = float(err.mean())
        assert mn <= mean_abs, f"{what}: mean-abs {mn:.3e} > {mean_abs:.1e}"
    return mx


def run_fwd(qn, kn, vn, P, order, causal, scale=None, window=0):
    """Natural-order CPU inputs -> GPU ring forward -> natural-order CPU (O, LSE)."""
    import ring_ulysses_sequence_b200 as rm
    q = to_rank_major(qn, P, order).cuda()
    k = to_rank_major(kn, P, order).cuda()
    v = to_rank_major(vn, P, order).cuda()
    o, lse = rm.ring_attn_fwd(q, k, v, P, causal=causal, order=order, scale=scale, window=window)
    torch.cuda.synchronize()
    assert rm.native.rm_check_device_status() == 0
    return (to_natural(o.float().cpu(), P, order),
            to_natural(lse.cpu().unsqueeze(-1), P, order).squeeze(-1))
