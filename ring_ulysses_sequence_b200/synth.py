"""Seeded synthetic inputs and the workload table.

This module draws random numbers and names shapes; it holds none of the
attention arithmetic, so the CUDA path and the CPU oracle can both take their
inputs from it.

Recipe: a CPU ``torch.Generator`` seeded with the workload's seed draws
``randn`` float32 tensors in the order q, k, v, dO (natural token order,
[B, H, S, D] and [B, Hkv, S, D]); each is multiplied by the workload's input
scale and cast to its dtype. The oracle reads the cast values.
"""
from dataclasses import dataclass, field
from typing import Optional

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    Hkv: int
    S: int
    D: int
    P: int
    order: str            # "contiguous" | "zigzag"
    causal: bool
    dtype: torch.dtype
    seed: int
    input_scale: float = 1.0
    ulysses: int = 1      # U; the ring size is P
    backward: bool = False
    window: int = 0       # causal sliding window in keys (query i sees i-W < j <= i); 0 = none
    cu_seqlens: tuple = ()  # packed document boundaries (natural positions, 0 .. S); () = none
    notes: str = field(default="", compare=False)

    @property
    def G(self) -> int:
        return self.H // self.Hkv

    @property
    def chunk(self) -> int:
        """Tokens per contiguous run of natural positions held by one rank."""
        return self.S // (2 * self.P) if self.order == "zigzag" else self.S // self.P

    def fwd_flops(self) -> float:
        """Algorithmic forward FLOPs: 4 B H S^2 D, halved when causal; with a
        window or packed documents, 4 B H D times the number of visible
        (query, key) pairs."""
        if self.cu_seqlens:
            lens = np.diff(np.asarray(self.cu_seqlens, dtype=np.int64))
            pairs = int((lens * (lens + 1) // 2).sum()) if self.causal else int((lens * lens).sum())
            return 4.0 * self.B * self.H * self.D * pairs
        if self.causal and 0 < self.window < self.S:
            W, S = self.window, self.S
            pairs = W * (W + 1) // 2 + (S - W) * W
            return 4.0 * self.B * self.H * self.D * pairs
        f = 4.0 * self.B * self.H * self.S * self.S * self.D
        return f / 2 if self.causal else f

    def bwd_flops(self) -> float:
        """Algorithmic backward FLOPs: 2.5x the forward (five products vs two)."""
        return 2.5 * self.fwd_flops()


def packed_boundaries(S: int, seed: int, lo: int = 512, hi: int = 8192) -> list:
    """Document boundaries 0 = cu[0] < ... < cu[n] = S: lengths drawn uniformly
    from [lo, hi] with a seeded generator, the last document cut at S."""
    rng = np.random.default_rng(seed)
    cu = [0]
    while cu[-1] < S:
        cu.append(min(S, cu[-1] + int(rng.integers(lo, hi + 1))))
    return cu


WORKLOADS = {
    # fp32, non-causal, 4 virtual ranks in contiguous chunks of 256.
    "ring_fwd_fp32_S1k": Workload("ring_fwd_fp32_S1k", 1, 2, 2, 1024, 64, 4, "contiguous",
                                  False, torch.float32, 0, 1.0),
    # bf16, causal, zigzag over 8 ranks (16 chunks of 512).
    "ring_fwd_bf16_S8k_causal_zigzag": Workload("ring_fwd_bf16_S8k_causal_zigzag", 1, 8, 8,
                                                8192, 128, 8, "zigzag", True,
                                                torch.bfloat16, 1, 0.5),
    # bf16 GQA (32 query heads over 8 KV heads), causal zigzag over 8 ranks,
    # chunk 2048: a Llama-3-8B attention layer at 32k tokens.
    "ring_fwd_bf16_S32k_gqa_causal_zigzag": Workload("ring_fwd_bf16_S32k_gqa_causal_zigzag",
                                                     1, 32, 8, 32768, 128, 8, "zigzag", True,
                                                     torch.bfloat16, 2, 0.5),
    # The same layer with a 4096-token causal sliding window (Mistral-style
    # local attention): most key tiles of a query tile are skipped.
    "ring_fwd_bf16_S32k_gqa_causal_zigzag_window4k": Workload(
        "ring_fwd_bf16_S32k_gqa_causal_zigzag_window4k", 1, 32, 8, 32768, 128, 8, "zigzag", True,
        torch.bfloat16, 5, 0.5, window=4096),
    # The same layer over packed documents of seeded lengths (512 to 8192
    # tokens): attention stays inside each document.
    "ring_fwd_bf16_S32k_gqa_causal_zigzag_packed": Workload(
        "ring_fwd_bf16_S32k_gqa_causal_zigzag_packed", 1, 32, 8, 32768, 128, 8, "zigzag", True,
        torch.bfloat16, 6, 0.5, cu_seqlens=tuple(packed_boundaries(32768, 6))),
    # Ulysses x Ring: 4 x 4 mesh over 131072 tokens, sequence-sharded input
    # [16 shards, 8192 tokens, heads, 128].
    "usp_fwd_bf16_S128k_u4r4": Workload("usp_fwd_bf16_S128k_u4r4", 1, 32, 8, 131072, 128, 4,
                                        "zigzag", True, torch.bfloat16, 3, 0.5, ulysses=4),
    # bf16 forward + backward, causal zigzag over 16 ranks, chunk 2048.
    "ring_fwdbwd_bf16_S64k_causal_zigzag": Workload("ring_fwdbwd_bf16_S64k_causal_zigzag", 2,
                                                    16, 16, 65536, 128, 16, "zigzag", True,
                                                    torch.bfloat16, 4, 0.5, backward=True),
}

# The workload the benchmark times on one GPU.
BENCH_WORKLOAD = "ring_fwd_bf16_S32k_gqa_causal_zigzag"


def make_inputs(w: Workload, with_dout: Optional[bool] = None, seed: Optional[int] = None):
    """q [B,H,S,D], k/v [B,Hkv,S,D] (and dO [B,H,S,D]) in natural order, CPU."""
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed if seed is None else seed)
    with_dout = w.backward if with_dout is None else with_dout
    shapes = [(w.B, w.H, w.S, w.D), (w.B, w.Hkv, w.S, w.D), (w.B, w.Hkv, w.S, w.D)]
    if with_dout:
        shapes.append((w.B, w.H, w.S, w.D))
    out = []
    for shp in shapes:
        t = torch.randn(shp, generator=g, dtype=torch.float32)
        if w.input_scale != 1.0:
            t.mul_(w.input_scale)
        out.append(t.to(w.dtype))
    return tuple(out)


def make_tensor(shape, seed: int, dtype=torch.float32, scale: float = 1.0):
    """One seeded N(0, scale^2) tensor on the CPU."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    t = torch.randn(shape, generator=g, dtype=torch.float32)
    if scale != 1.0:
        t.mul_(scale)
    return t.to(dtype)


def sample_rows(S: int, n: int, seed: int, chunk: int) -> np.ndarray:
    """n seeded natural positions (uniform, no replacement) plus the first and
    last position of every chunk; sorted, unique."""
    rng = np.random.default_rng(seed)
    pick = rng.choice(S, size=min(n, S), replace=False)
    edges = []
    for c0 in range(0, S, chunk):
        edges += [c0, min(c0 + chunk, S) - 1]
    return np.unique(np.concatenate([pick, np.array(edges, dtype=np.int64)]))


def to_numpy_f64(t: torch.Tensor) -> np.ndarray:
    """Exact widening of a CPU tensor (bf16/fp32) to float64 numpy."""
    return t.detach().to(torch.float64).cpu().numpy()
